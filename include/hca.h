/*
 * hca.h -- C ABI of libhca.so, the hybrid CSA / HCA attention layer on B200.
 *
 * What the layer computes (DeepSeek-V4 write-ups; sections named per call):
 *   "DeepSeek V4 Architecture Tricks" (pinktalk.online)        -> [Tricks]
 *   QbitAI write-up of the V4 report (admirer.cn), "混合注意力機制" -> [QbitAI]
 *   "DeepSeek-V4 Technical Report: Hybrid Attention and Post-Training
 *    for Million-Token Contexts" (xutianle.me), sections 3-5   -> [Report]
 *
 * Conventions for every entry point
 *   - Tensor pointers are DEVICE pointers, owned by the caller; the library
 *     never frees or retains them.  Struct and config pointers (cfg, args)
 *     are HOST pointers, read during the call only.
 *   - Layouts are row-major with the strides stated; all strides are in
 *     elements.  bf16 tensors are passed as raw 16-bit patterns (hca_bf16).
 *     Every bf16/f32 row must start on a 16-byte boundary (base pointers
 *     16-byte aligned, row strides multiples of 8 bf16 / 4 f32 elements).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*,
 *     NULL = legacy default stream) and never synchronise the host.
 *   - The library does not allocate device memory.  Scratch space comes from
 *     the caller's `ws` (device pointer, 256-byte aligned) of at least
 *     hca_workspace_size(...) bytes; ws may be NULL when that size is 0.
 *   - Return value: HCA_OK, or a negative hca_status.  Arguments are checked
 *     on the host before anything is launched; on error nothing is launched
 *     and hca_last_error() describes the problem.  A failed launch returns
 *     HCA_ERR_CUDA.  Device-side errors of an earlier call may surface as
 *     HCA_ERR_CUDA from a later one (standard CUDA semantics).
 *   - Fault injection for tests: if the environment variable
 *     HCA_INJECT_FAULT names an entry point (or is "all"), that entry point
 *     returns HCA_ERR_INJECTED after argument checking, launching nothing.
 *   - Bounded device waits: every wait of a kernel on its own pipeline gives
 *     up after a poll budget, records an error, lets its own copies and MMAs
 *     drain, frees its tensor memory and returns; hca_check_device() then
 *     reports HCA_ERR_DEVICE_CHECK.  For tests of that path only,
 *     HCA_TEST_STALL=indexer makes the decode indexer's key producer issue
 *     nothing, with a budget of a few thousand polls, so that its waits run
 *     out (the call's top-k output is then meaningless).
 *   - Index check: with HCA_DEBUG=1 in the environment at call time, the
 *     attention kernels of sparse_mqa_attend, hybrid_attn_decode and
 *     hybrid_attn_prefill record every selected entry outside [-1, N), every
 *     entry e that its query at position t cannot see yet ((e+1)*rate - 1 > t)
 *     and every block-table entry outside the pool; hca_check_device() then
 *     reports HCA_ERR_DEVICE_CHECK naming the kinds found.  Out-of-range
 *     entries are skipped (as empty slots) with or without the check; the
 *     check changes no result.
 *   - Every entry point that launches work opens an NVTX range named after
 *     itself for the duration of the host call (no cost without a tool).
 *   - Supported shapes: c in {64, 512}, d_idx in {32, 128}; n_heads,
 *     n_idx_heads <= 64; topk <= 2048; n_win <= 256.  Other shapes return
 *     HCA_ERR_UNSUPPORTED.
 */
#ifndef HCA_H_
#define HCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t hca_bf16; /* raw bfloat16 bit pattern */

typedef enum {
  HCA_OK = 0,
  HCA_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, bad size, bad stride */
  HCA_ERR_UNSUPPORTED = -2,  /* valid but not a specialised shape */
  HCA_ERR_WORKSPACE = -3,    /* ws smaller than hca_workspace_size() */
  HCA_ERR_CUDA = -4,         /* a CUDA call or launch failed */
  HCA_ERR_DEVICE_CHECK = -5, /* a kernel's own bounds/wait check tripped */
  HCA_ERR_INJECTED = -6      /* HCA_INJECT_FAULT asked for a failure */
} hca_status;

/* Hyper-parameters of one layer.
 *   c            KV entry width = attention head dim (512 in V4-Pro, [QbitAI] CSA step four)
 *   m            CSA compression rate (4, [Tricks] CSA section)
 *   m_hca        HCA compression rate m' (128, [Tricks] HCA section)
 *   topk         CSA entries selected per query (1024, [Tricks] CSA section)
 *   n_idx_heads  lightning-indexer heads H_I (64), d_idx their dim (128)
 *   n_heads      query heads sharing the single KV head (MQA)
 *   n_win        sliding-window length (128, [Tricks] Sliding Window Branch)
 *   scale        attention logit scale (1/sqrt(c))
 * Q/KV normalisation and partial RoPE ([QbitAI] "混合注意力機制", the Q/KV
 * normalisation and partial-RoPE tricks; [Tricks] "Partial RoPE 和 Attention
 * Sink"); read only by calls that are given normalisation weights or asked to
 * rotate their output:
 *   rope_dims    rotated channels at the end of every row (64); pair j =
 *                channels (c - rope_dims + 2j, +1) turns by pos * rope_base^(-2j/rope_dims).
 *                0 = no rotation; else even, a multiple of 8 and <= min(c, 256)
 *   rope_base    frequency base (10000); > 0 when rope_dims > 0
 *   norm_eps     RMSNorm epsilon (1e-6), >= 0 */
typedef struct {
  int c, m, m_hca, topk, n_idx_heads, d_idx, n_heads, n_win;
  float scale;
  int rope_dims;
  float rope_base;
  float norm_eps;
} hca_layer_cfg;

/* Query modes of the indexer and attention calls. */
enum {
  HCA_MODE_PREFILL = 0, /* Tq queries of ONE sequence; window rows are that
                           sequence's raw token rows [T, c] (row r = token r) */
  HCA_MODE_DECODE = 1   /* query i belongs to request i; each request has its
                           own caches and its own window block [n_win, c] */
};

/* Operations, for hca_workspace_size().  The layer calls size their
 * workspace with hybrid_attn_decode_workspace / hybrid_attn_prefill_workspace. */
enum {
  HCA_OP_INDEXER_TOPK = 1,
  HCA_OP_SPARSE_MQA = 2
};

/* ---------------------------------------------------------------------------
 * csa_compress -- overlapped CSA KV compression ([Tricks] "压缩 KV 的具体 trick";
 * [QbitAI] CSA step one; [Report] section 3).
 *   out[i, j] = sum_{r in W(i)} softmax_r(logits[r, j] + pos_bias[r-(i-1)m, j]) * cand[r, j]
 *   W(i) = tokens [(i-1)m, (i+1)m) that exist; bias rows 0..m-1 weight the
 *   previous block, m..2m-1 the current one; entry 0 pools its own block only.
 *   Softmax and sum in f32; the result is rounded to bf16.
 *   cand   [T, c] bf16, row stride ld_cand;   logits [T, c] bf16, row stride ld_logits
 *   pos_bias [2m, c] f32, row stride ld_bias; out [floor(T/m), c] bf16, row stride ld_out
 *   A trailing incomplete block produces no entry.  T may be 0 (no-op).
 *   The same call compresses indexer keys: pass the key candidates as cand,
 *   the first d_idx channels of the logits/bias (same pointers, same strides)
 *   and c = d_idx.  c must be a multiple of 8; m in [1, 16].
 * ------------------------------------------------------------------------- */
int csa_compress(const hca_bf16* cand, int ld_cand, const hca_bf16* logits, int ld_logits,
                 const float* pos_bias, int ld_bias, int T, int c, int m,
                 hca_bf16* out, int ld_out, void* stream);

/* ---------------------------------------------------------------------------
 * hca_compress -- HCA KV compression, no overlap ([Tricks] HCA section;
 * [QbitAI] HCA paragraph; [Report] section 4).
 *   out[i, j] = sum_{r in [i m', (i+1) m')} softmax_r(logits[r, j] + pos_bias[r - i m', j]) * cand[r, j]
 *   for B independent sequences: sequence b reads cand + b*seq_stride_in,
 *   logits + b*seq_stride_in and writes out + b*seq_stride_out.
 *   cand/logits [T, c] bf16 (row strides ld_cand / ld_logits), pos_bias [m', c]
 *   f32 (row stride ld_bias, shared by all sequences), out [floor(T/m'), c] bf16.
 *   Decode use: compress the newest complete block by passing its m' raw
 *   rows (T = m') and out = the cache row it fills.  m' in [1, 1024].
 * ------------------------------------------------------------------------- */
int hca_compress(const hca_bf16* cand, int ld_cand, const hca_bf16* logits, int ld_logits,
                 const float* pos_bias, int ld_bias, int B, long long seq_stride_in, int T, int c,
                 int m_hca, hca_bf16* out, int ld_out, long long seq_stride_out, void* stream);

/* ---------------------------------------------------------------------------
 * rms_norm_rope -- Q/KV RMSNorm followed by partial RoPE, row by row
 * ([QbitAI] "混合注意力機制": queries and KV entries are RMS-normalised before
 * core attention, and only their last 64 channels carry a rotary position;
 * [Tricks] "Partial RoPE 和 Attention Sink").
 *   y = rms_norm(x) with weights gamma: x / sqrt(mean_j x_j^2 + cfg->norm_eps) * gamma,
 *   then pair j of the last cfg->rope_dims channels turns by pos * theta_j,
 *   theta_j = cfg->rope_base^(-2j / rope_dims):  (a, b) -> (a cos - b sin, a sin + b cos).
 *   f32 arithmetic (the angle is reduced in f64); y is rounded to bf16.
 *   Rows come in n_seq sequences of rows_per_seq rows: row r of sequence s is
 *     x + s*seq_stride_x + r*ld_x   ->   y + s*seq_stride_y + r*ld_y
 *   and sits at position max((pos ? pos[s] : 0) + pos_add, 0) + r*pos_step.
 *   Examples: queries [Tq, H, c] -> n_seq = Tq, rows_per_seq = H, pos = q_pos,
 *   pos_step = 0; compressed entries -> pos = NULL, pos_add = rate-1,
 *   pos_step = rate; a decode window block [n_win, c] ending at q_pos[s] ->
 *   pos = q_pos, pos_add = -(n_win-1), pos_step = 1.
 *   x: bf16 (x_is_f32 = 0) or f32 (x_is_f32 = 1), cfg->c channels per row;
 *   gamma [c] f32; pos [n_seq] int32 or NULL; y bf16.  Strides in elements
 *   (multiples of 8 for bf16, 4 for f32).  x and y may be the same rows
 *   (in place, bf16 only).  n_seq or rows_per_seq 0: no-op.
 * ------------------------------------------------------------------------- */
int rms_norm_rope(const void* x, int x_is_f32, long long ld_x, long long seq_stride_x, int n_seq,
                  int rows_per_seq, const int32_t* pos, int pos_add, int pos_step, const float* gamma,
                  const hca_layer_cfg* cfg, hca_bf16* y, long long ld_y, long long seq_stride_y,
                  void* stream);

/* ---------------------------------------------------------------------------
 * csa_indexer_topk -- lightning-indexer scores and per-query top-k
 * ([QbitAI] CSA step two; [Tricks] CSA section: 64 heads x 128, top-k 1024).
 *   I(t, s) = sum_j w_idx[t, j] * ReLU(q_idx[t, j, :] . k_idx[s, :])   (f32 accumulation)
 *   over the causally complete entries s, (s+1)*cfg->m - 1 <= q_pos[t], s < N.
 *   topk_idx[t, :] receives the cfg->topk entries with the largest scores
 *   (ties: lower index first), in no particular order, padded with -1 when
 *   fewer than topk entries are visible (then all visible ones are taken).
 *   q_idx  [Tq, H_I, d_I] bf16 (contiguous); w_idx [Tq, H_I] f32 (contiguous)
 *   k_idx  request r's keys at k_idx + r*k_seq_stride: [N, d_I] bf16 contiguous
 *   q_pos  [Tq] int32 device: position of each query (0-based)
 *   mode   HCA_MODE_PREFILL: all queries in request 0 (k_seq_stride ignored);
 *          HCA_MODE_DECODE: query i reads request i's keys.
 *   topk_idx [Tq, topk] int32 out.  ws: hca_workspace_size(HCA_OP_INDEXER_TOPK, cfg, Tq, N, mode).
 * ------------------------------------------------------------------------- */
int csa_indexer_topk(const hca_bf16* q_idx, const float* w_idx, const hca_bf16* k_idx,
                     long long k_seq_stride, int N, const int32_t* q_pos, int Tq, int mode,
                     const hca_layer_cfg* cfg, int32_t* topk_idx, void* ws, size_t ws_bytes,
                     void* stream);

/* ---------------------------------------------------------------------------
 * csa_indexer_topk_noalloc -- csa_indexer_topk for callers that cannot
 * allocate device memory.  (Not an operation of the method: the write-ups
 * have no counterpart; it is the same indexer + top-k with built-in scratch.)
 *
 * Some callers can't call cudaMalloc or hand the library a workspace: for
 * instance a plugin running inside another runtime that owns all device
 * memory and gives its plugins no allocator, or a serving loop that forbids
 * device allocation once it has started.  This entry point takes the same
 * arguments as csa_indexer_topk minus ws/ws_bytes, computes the same result
 * with the same kernels, and allocates nothing: its scratch is one static
 * device array of HCA_NOALLOC_SCRATCH_BYTES (16 MiB) inside libhca.so, which
 * every GPU that loads the library's device code holds until the process
 * exits.
 *   - Limit: calls whose scratch need (the same bytes
 *     hca_workspace_size(HCA_OP_INDEXER_TOPK, cfg, Tq, N, mode) reports)
 *     exceeds HCA_NOALLOC_SCRATCH_BYTES return HCA_ERR_WORKSPACE and launch
 *     nothing.  For the 64 x 128 indexer and top-1024 in decode mode: a
 *     request of up to 49,152 entries needs its f32 score row (4 B per
 *     entry), so 32 requests x 32,768 entries fit (4 MiB); a longer request
 *     also needs the histogram select's regions (about 12 B per entry in
 *     all), so 5 requests x 262,144 entries fit (about 15.5 MiB) and 6 do
 *     not.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.  It allocates nothing.
 *   - All calls share the one array and it keeps the last call's contents
 *     (nothing in it needs to start at zero: each call writes all it reads).
 *     Calls whose kernels may overlap on the GPU -- on different streams, or
 *     from several host threads -- race on the array; order them on one
 *     stream (or synchronise) instead.
 * ------------------------------------------------------------------------- */
#define HCA_NOALLOC_SCRATCH_BYTES (16u << 20)
int csa_indexer_topk_noalloc(const hca_bf16* q_idx, const float* w_idx, const hca_bf16* k_idx,
                             long long k_seq_stride, int N, const int32_t* q_pos, int Tq, int mode,
                             const hca_layer_cfg* cfg, int32_t* topk_idx, void* stream);

/* ---------------------------------------------------------------------------
 * FP4 indexer variant ([Tricks] "FP4 / FP8 Quantization-Aware Training": the
 * indexer's QK path is cached, loaded and multiplied in FP4; index scores are
 * kept in BF16; FP4 values dequantise losslessly because the wider format's
 * exponent absorbs the fine-grained scale).  The FP4 format is MXFP4: E2M1
 * elements (0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives; code bit 3 = sign), one
 * power-of-two scale 2^X per 32 consecutive elements of a row, X =
 * floor(log2 max|x|) - 2 clamped to [-127, 127] (-127 for an all-zero block),
 * stored as the byte X + 127; element codes = nearest E2M1 value of x / 2^X
 * (ties to the even code, saturating at +-6), two per byte, the even element
 * in the low nibble.
 *
 * mxfp4_quantize -- MXFP4 form of `rows` rows of d elements (d a multiple of
 *   32): x bf16 (x_is_f32 = 0) or f32, row stride ld_x elements; codes [rows]
 *   [d/2] bytes at row stride ld_codes (a multiple of 16), scales [rows][d/32]
 *   bytes at row stride ld_scales.  Bit-exact to the definition above.
 *
 * csa_indexer_topk_fp4 -- decode indexer + top-k (one query per request, as
 *   csa_indexer_topk in HCA_MODE_DECODE) with FP4 keys and queries and BF16
 *   scores: I(t,s) = bf16(sum_j w[t,j] ReLU(q4[t,j,:] . k4[s,:])), q4 and k4
 *   the MXFP4 values of q_I and K_I.  Takes the 64 x 128 indexer only.
 *   q_idx [B, 64, 128] bf16 (rounded to its MXFP4 values inside the call);
 *   w_idx [B, 64] f32; request r's keys: codes at k_codes + r*k_seq_stride*64
 *   ([N][64] bytes), scales at k_scales + r*k_seq_stride*4 ([N][4] bytes), both
 *   readable up to the next multiple of 4 keys; with B > 1, k_seq_stride >=
 *   that multiple of 4 and itself a multiple of 4.  topk_idx [B, topk] as in
 *   csa_indexer_topk.  ws: csa_indexer_topk_fp4_workspace(cfg, B, N) bytes.
 *   Device-side waits that give up are reported by hca_check_device.
 * ------------------------------------------------------------------------- */
int mxfp4_quantize(const void* x, int x_is_f32, long long ld_x, int rows, int d, uint8_t* codes,
                   long long ld_codes, uint8_t* scales, long long ld_scales, void* stream);
int csa_indexer_topk_fp4(const hca_bf16* q_idx, const float* w_idx, const uint8_t* k_codes,
                         const uint8_t* k_scales, long long k_seq_stride, int N, const int32_t* q_pos,
                         int B, const hca_layer_cfg* cfg, int32_t* topk_idx, void* ws, size_t ws_bytes,
                         void* stream);
size_t csa_indexer_topk_fp4_workspace(const hca_layer_cfg* cfg, int B, int N);

/* ---------------------------------------------------------------------------
 * FP8 storage of the KV channels outside the rotary part ([Tricks] "Partial
 * RoPE 和 Attention Sink": the rotary channels of the KV cache stay BF16, the
 * other channels are stored in FP8).  Cache form of a row of c channels, with
 * n = c - cfg->rope_dims (a multiple of 64) and rope_dims a multiple of 8:
 *   codes  [n] E4M3 bytes (sign bit 7, exponent bits 3-6 with bias 7 and field 0
 *          subnormal, mantissa bits 0-2): the E4M3 value nearest to x / scale of
 *          the channel's group (ties to the even mantissa, saturating at +-448;
 *          a negative value that rounds to zero keeps its sign);
 *   scales [n / 64] f32: scale of a group of 64 channels = f32(max |x| / 448),
 *          1 for an all-zero group;
 *   rope   [rope_dims] bf16: the last rope_dims channels, rounded to bf16.
 * A row's value is code * scale on the first n channels, then the rope part.
 *
 * kv_fp8_quantize -- the cache form of `rows` rows x [c] (x bf16, or f32 with
 *   x_is_f32 = 1; row stride ld_x elements); codes row stride ld_codes bytes (a
 *   multiple of 16), scales ld_scales floats, rope ld_rope bf16 (a multiple of 8).
 *   Every code is decided on the f64 quotient of the f32 values x and scale.
 * ------------------------------------------------------------------------- */
typedef struct {
  uint8_t* codes;      /* [rows][ld_codes] */
  float* scales;       /* [rows][ld_scales] */
  hca_bf16* rope;      /* [rows][ld_rope] */
  long long ld_codes, ld_scales, ld_rope;
  long long seq_rows;  /* rows between requests (decode) */
} hca_kv_fp8;
int kv_fp8_quantize(const void* x, int x_is_f32, long long ld_x, long long rows, const hca_layer_cfg* cfg,
                    uint8_t* codes, long long ld_codes, float* scales, long long ld_scales, hca_bf16* rope,
                    long long ld_rope, void* stream);

/* ---------------------------------------------------------------------------
 * sparse_mqa_attend -- core shared-KV multi-query attention over compressed
 * entries plus the sliding window, one softmax ([QbitAI] CSA step three, the
 * KV-entry-as-key-and-value remark and the sliding-window paragraph;
 * [Tricks] HCA and Sliding Window sections).
 *   For query t and head h, over the row set U(t):
 *     o[t, h, :] = sum_{u in U(t)} softmax_u(scale * q[t, h, :] . row_u) row_u
 *   U(t) = { kv[s] : s in idx[t, :], s >= 0 }             (CSA, idx != NULL)
 *        | { kv[s] : (s+1)*rate - 1 <= q_pos[t], s < N }  (HCA, idx == NULL)
 *        + window rows of t.
 *   Window rows: HCA_MODE_PREFILL: win[r] for r in [max(0, t-n_win+1), t]
 *   (win = the sequence's raw per-token KV rows, row stride cfg->c);
 *   HCA_MODE_DECODE: the first min(n_win, t+1) rows of request i's block
 *   win + i*win_seq_stride ([n_win, c]; any order).  In HCA_MODE_PREFILL
 *   win_seq_stride instead gives the number of rows in win (T >= 1 + every
 *   q_pos), so that no window tile reads past the sequence.
 *   q [Tq, H, c] bf16; kv: request r's entries at kv + r*kv_seq_stride, [N, c];
 *   idx [Tq, n_idx] int32 (entries < N, visible to the query; -1 = empty slot);
 *   out [Tq, H, c] bf16.  Logits, softmax and sums in f32.
 *   sink: NULL, or [H] f32 (device) learnable sink logits, one per head, in the
 *   units of scale * q . row: they join the softmax denominator only,
 *     o[t, h, :] = sum_u e^{s_u} row_u / (e^{sink[h]} + sum_u e^{s_u})
 *   ([QbitAI] attention-sink paragraph; [Tricks] "Partial RoPE 和 Attention
 *   Sink"), once per query also when the rows are split over CTAs.
 *   rotate_out: nonzero -> the last cfg->rope_dims channels of every output
 *   head are turned back by -q_pos[t] (the partial-RoPE output rotation, see
 *   rms_norm_rope; with shared K = V it leaves only relative positions).
 *   ws: hca_workspace_size(HCA_OP_SPARSE_MQA, cfg, Tq, N, mode) (split-K partials).
 * ------------------------------------------------------------------------- */
int sparse_mqa_attend(const hca_bf16* q, const hca_bf16* kv, long long kv_seq_stride, int N,
                      const int32_t* idx, int n_idx, int rate, const hca_bf16* win,
                      long long win_seq_stride, const int32_t* q_pos, int Tq, int mode,
                      const hca_layer_cfg* cfg, const float* sink, int rotate_out, hca_bf16* out,
                      void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * hybrid_attn_decode -- one decode step of a CSA layer and/or an HCA layer for
 * B requests, one query each at q_pos[b] (device int32 [B]).  Runs, in order:
 * the HCA compression of the newest complete block (if hca_block_cand), the
 * indexer + top-k, the CSA sparse attention, the HCA dense attention; split-K
 * over the context with a combine step.  A layer whose q pointer is NULL is
 * skipped.  Caches hold entries of request b at base + b*stride.
 * `events` (optional, may be NULL) is an array of n_events cudaEvent_t handles
 * that are recorded on `stream` at kernel boundaries, for profiling.
 * Q/KV normalisation (csa_norm / hca_norm = [2, c] f32: query weights, then KV
 * weights; NULL = none): the layer's queries and window rows are normalised
 * and rotated (rms_norm_rope) before its attention, its output is rotated
 * back (rotate_out), and the HCA entry compressed here is normalised and
 * rotated at its position, (hca_N-1)*m' + m'-1, before it is stored.  The
 * caches (csa_kv, hca_kv rows < hca_N-1) already hold entries in that form;
 * window blocks hold raw rows, oldest first (row w = token
 * max(0, q_pos-n_win+1) + w).
 * ------------------------------------------------------------------------- */
typedef struct {
  int B;
  const int32_t* q_pos;
  /* CSA layer */
  const hca_bf16* csa_q;      /* [B, H, c] */
  const hca_bf16* csa_q_idx;  /* [B, H_I, d_I] */
  const float* csa_w_idx;     /* [B, H_I] */
  const hca_bf16* csa_kv;     /* [B][csa_N, c] at csa_kv_stride */
  const hca_bf16* csa_k_idx;  /* [B][csa_N, d_I] at csa_k_stride */
  int csa_N;
  long long csa_kv_stride, csa_k_stride;
  const hca_bf16* csa_win;    /* [B][n_win, c] at csa_win_stride */
  long long csa_win_stride;
  int32_t* csa_topk_idx;      /* [B, topk] out */
  hca_bf16* csa_out;          /* [B, H, c] out */
  /* HCA layer */
  const hca_bf16* hca_q;      /* [B, H, c] */
  hca_bf16* hca_kv;           /* [B][hca_N, c] at hca_kv_stride.  With hca_block_cand, hca_N must equal
                                 floor((q_pos[b]+1)/m') for every b and row hca_N-1 is written */
  int hca_N;
  long long hca_kv_stride;
  const hca_bf16* hca_block_cand;   /* [B][m', c] newest complete block, or NULL */
  const hca_bf16* hca_block_logits; /* [B][m', c] */
  long long hca_block_stride;
  const float* hca_pos_bias;        /* [m', c] */
  const hca_bf16* hca_win;    /* [B][n_win, c] at hca_win_stride */
  long long hca_win_stride;
  hca_bf16* hca_out;          /* [B, H, c] out */
  void* const* events;
  int n_events;
  const float* csa_sink;      /* [H] sink logits of the CSA layer, or NULL (see sparse_mqa_attend) */
  const float* hca_sink;      /* [H] sink logits of the HCA layer, or NULL */
  const float* csa_norm;      /* [2, c] Q/KV normalisation weights of the CSA layer, or NULL */
  const float* hca_norm;      /* [2, c] of the HCA layer, or NULL */
  /* FP4 indexer variant (see csa_indexer_topk_fp4), or NULL: the CSA layer's indexer
   * reads MXFP4 keys instead of csa_k_idx (which is then not read): request b's codes
   * at csa_k_codes + b*csa_k4_stride*64 ([csa_N][64] bytes) and scales at
   * csa_k_scales + b*csa_k4_stride*4 ([csa_N][4] bytes), both readable up to the
   * next multiple of 4 keys; csa_k4_stride in keys, a multiple of 4 (B > 1). 64 x 128
   * indexer only; the index scores are BF16. */
  const uint8_t* csa_k_codes;
  const uint8_t* csa_k_scales;
  long long csa_k4_stride;
  /* Paged caches ([Tricks] "Heterogeneous KV Cache Layout": the compressed
   * ("classical") cache is allocated in blocks that each cover L = lcm(m, m')
   * raw tokens, i.e. L/m CSA entries with their indexer keys and L/m' HCA
   * entries; [Jiedu] 核心创新一: the window sits in a separate state cache), or
   * NULL: flat caches as above.  With block_table, request b's logical block j
   * is physical block block_table[b*bt_stride + j] (int32, device) of every
   * pool: csa_kv is a pool [n_pool_blocks][L/m][c], csa_k_idx
   * [n_pool_blocks][L/m][d_I], hca_kv [n_pool_blocks][L/m'][c]; entry i of a
   * request is row i % (L/m) of its block i / (L/m) (likewise for HCA); the
   * request strides csa_kv_stride, csa_k_stride and hca_kv_stride are not read.
   * The newest HCA entry (hca_block_cand) is written to its pool row.  Each
   * window block [n_win, c] is a ring: token tau at row tau mod n_win (this
   * only matters with Q/KV normalisation; rows >= q_pos+1 are not read).
   * Needs c = 512, 64 heads, the 64 x 128 indexer with bf16 keys, L/m a
   * multiple of 8 dividing 128, and bt_stride >= the blocks each layer's
   * entries span. */
  const int32_t* block_table;
  long long bt_stride;
  int n_pool_blocks;
  /* FP8 caches (see kv_fp8_quantize; host pointers to descriptors), or NULL: the
   * layer's entries are read from their FP8 form (csa_kv / hca_kv are not read):
   * request b's entry i is row b*seq_rows + i.  The rows an attention reads are
   * first widened to bf16 (code * scale, rounded once) in the workspace: the CSA
   * layer's selected rows, the HCA layer's visible rows.  With hca_block_cand the
   * newest HCA entry is written in FP8 form to row hca_N-1.  Not with paged caches. */
  const hca_kv_fp8* csa_kv8;
  const hca_kv_fp8* hca_kv8;
} hca_decode_args;

int hybrid_attn_decode(const hca_layer_cfg* cfg, const hca_decode_args* args, void* ws,
                       size_t ws_bytes, void* stream);
size_t hybrid_attn_decode_workspace(const hca_layer_cfg* cfg, const hca_decode_args* args);

/* ---------------------------------------------------------------------------
 * hybrid_attn_prefill -- a CSA layer (and optionally an HCA layer) over one
 * sequence of T raw tokens, every token a query (q_pos = 0..T-1, device).
 * Runs: CSA compression of KV and indexer keys (indexer-key logits/bias are
 * the first d_idx channels of logits/bias_csa), indexer + top-k, sparse MQA
 * with the causal window; then, if hca_kv != NULL, HCA compression and dense
 * causal MQA with the window.
 * Q/KV normalisation (csa_norm / hca_norm, as in hybrid_attn_decode): the
 * compressed entries are normalised and rotated at their positions
 * ((i+1)*rate - 1) before they are stored in csa_kv / hca_kv (one bf16
 * rounding), the queries and the window rows (cand) before the attention,
 * and the output is rotated back.  Indexer keys are not normalised.
 * ------------------------------------------------------------------------- */
typedef struct {
  int T;
  const int32_t* q_pos;       /* [T] */
  const hca_bf16* cand;       /* [T, c] raw per-token KV candidates (also the window rows) */
  const hca_bf16* logits;     /* [T, c] compression weight logits */
  const hca_bf16* kidx_cand;  /* [T, d_I] per-token indexer-key candidates */
  const float* bias_csa;      /* [2m, c] */
  const hca_bf16* q_idx;      /* [T, H_I, d_I] */
  const float* w_idx;         /* [T, H_I] */
  const hca_bf16* q;          /* [T, H, c] */
  hca_bf16* csa_kv;           /* [T/m, c] out */
  hca_bf16* csa_k_idx;        /* [T/m, d_I] out */
  int32_t* topk_idx;          /* [T, topk] out */
  hca_bf16* csa_out;          /* [T, H, c] out */
  const float* bias_hca;      /* [m', c] */
  const hca_bf16* hca_q;      /* [T, H, c] */
  hca_bf16* hca_kv;           /* [T/m', c] out, or NULL: no HCA layer */
  hca_bf16* hca_out;          /* [T, H, c] out */
  void* const* events;
  int n_events;
  const float* csa_sink;      /* [H] sink logits of the CSA layer, or NULL (see sparse_mqa_attend) */
  const float* hca_sink;      /* [H] sink logits of the HCA layer, or NULL */
  const float* csa_norm;      /* [2, c] Q/KV normalisation weights of the CSA layer, or NULL */
  const float* hca_norm;      /* [2, c] of the HCA layer, or NULL */
} hca_prefill_args;

int hybrid_attn_prefill(const hca_layer_cfg* cfg, const hca_prefill_args* args, void* ws,
                        size_t ws_bytes, void* stream);
size_t hybrid_attn_prefill_workspace(const hca_layer_cfg* cfg, const hca_prefill_args* args);

/* Workspace bytes for one op at Tq queries and N entries per request (mode
 * as in the calls).  For HCA_OP_SPARSE_MQA the size covers both the sparse
 * (idx, n_idx = cfg->topk) and the dense (idx = NULL) form.  Returns 0 for
 * calls that need none, (size_t)-1 for an unsupported configuration. */
size_t hca_workspace_size(int op, const hca_layer_cfg* cfg, int Tq, int N, int mode);

/* Number of kernels the last successful layer call (hybrid_attn_decode /
 * hybrid_attn_prefill) on the calling thread launched. */
int hca_last_launch_count(void);

/* Synchronise the current device and report kernels that gave up a bounded
 * wait since the last check (HCA_ERR_DEVICE_CHECK; the record is cleared).
 * The only entry point that synchronises; meant for tests and diagnostics. */
int hca_check_device(void);

/* Message describing the last error on the calling thread ("" if none). */
const char* hca_last_error(void);

/* Library version string. */
const char* hca_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HCA_H_ */
