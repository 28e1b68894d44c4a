// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace hca {

// Kernels launched on this thread (incremented by every launch_* below).
extern thread_local int g_launch_counter;

// ---- compress.cu ----------------------------------------------------------
cudaError_t launch_compress(const bf16* cand, int ld_cand, const bf16* logits, int ld_logits,
                            const float* bias, int ld_bias, int B, long long seq_in, int T, int c,
                            int rate, bool overlap, bf16* out, int ld_out, long long seq_out,
                            cudaStream_t stream, float* out_f32 = nullptr);
// (out_f32 != nullptr: the entries are written there in f32, same strides, and out is unused)
// Row b of src [B][c] into a paged pool [blocks * rpb][c]: row bt[b*bt_stride + entry/rpb]*rpb + entry%rpb.
cudaError_t launch_scatter_rows(const bf16* src, int B, int c, const int32_t* bt, long long bt_stride, int entry,
                                int rpb, bf16* pool, cudaStream_t stream);

// ---- indexer_fp4.cu (FP4 indexer variant) ----------------------------------------
cudaError_t launch_mxfp4_quantize(const void* x, bool x_f32, long long ld_x, int rows, int d, uint8_t* codes,
                                  long long ld_codes, uint8_t* scales, long long ld_scales, cudaStream_t stream);
cudaError_t launch_mxfp4_roundtrip(const bf16* x, int rows, int d, bf16* y, cudaStream_t stream);
// Decode indexer over MXFP4 keys (codes [N][64 B], scales [ceil4(N)][4 B] per request, requests
// k_seq_stride keys apart) with a bf16 query already rounded to its MXFP4 values; BF16 scores.
cudaError_t launch_indexer_decode_fp4(const bf16* q4, const float* w_idx, const uint8_t* k_codes,
                                      const uint8_t* k_scales, long long k_seq_stride, int N, const int32_t* q_pos,
                                      int B, int rate, float* scores, long long ld_scores, int num_sms,
                                      cudaStream_t stream, int* hist);
unsigned int read_and_clear_indexer_fp4_error();

// ---- kv_fp8.cu (FP8 storage of the non-rotary KV channels) -------------------------
// Cache form of KV rows: codes [rows][ld_codes] E4M3 bytes (the first c - rope_dims
// channels), scales [rows][ld_scales] f32 (one per 64 channels), rope [rows][ld_rope]
// bf16 (the last rope_dims channels); sequences seq_rows rows apart.
struct KvFp8 {
  const uint8_t* codes;
  const float* scales;
  const bf16* rope;
  long long ld_codes, ld_scales, ld_rope, seq_rows;
};
cudaError_t launch_kv_fp8_quantize(const void* x, bool x_f32, long long ld_x, long long rows, int c, int rope_dims,
                                   uint8_t* codes, long long ld_codes, float* scales, long long ld_scales, bf16* rope,
                                   long long ld_rope, cudaStream_t stream);
// bf16 rows [B][n_out][c] from an FP8 cache: row j of sequence b <- source row idx[b][j]
// (or j without idx); invalid or negative -> zeros (and idx_out -1, else j).
cudaError_t launch_kv_fp8_gather(const KvFp8& kv, int c, int rope_dims, int B, int n_out, const int32_t* idx,
                                 int n_src, bf16* out, int32_t* idx_out, cudaStream_t stream);

// ---- norm_rope.cu -------------------------------------------------------------
// Q/KV RMSNorm + partial RoPE of rows (see rms_norm_rope in hca.h for the row
// addressing and positions).
struct NormRope {
  const void* x;
  bool x_f32;
  long long ld_x, seq_x;
  int n_seq, rows_per_seq;
  const int32_t* pos;
  int pos_add, pos_step;
  const float* gamma;
  int c, rope_dims;
  float eps, rope_base;
  bf16* y;
  long long ld_y, seq_y;
  // ring != 0: the rows of a sequence are a ring buffer of rows_per_seq tokens ending
  // at pos[s]: row r holds the one token of [pos[s] - rows_per_seq + 1, pos[s]] that is
  // congruent to r mod rows_per_seq (pos_add and pos_step are not read)
  int ring = 0;
};
cudaError_t launch_norm_rope(const NormRope& p, cudaStream_t stream);

// ---- topk.cu ----------------------------------------------------------------
// Largest candidate-count a single select row may have (smem-resident).
constexpr int kSelectMaxN = 24576;     // 64-bit composites staged in shared memory
constexpr int kSelectRowMaxN = 49152;  // 32-bit score keys staged in shared memory (one row per CTA)

// Row r of a score matrix: scores at scores + r*ld_scores (f32), its entry
// indices are idx_base(r) + position; n(r) elements are candidates.
// Two ways to describe rows:
//   by query: row = query q (r = q), n = min(n_visible(q_pos[q]), N) - chunk0
//   by chunk: row = (q, j), scores + q*ld + j*chunk, n = clamp(nvis - j*chunk, 0, chunk)
// Launch, optionally with programmatic stream serialisation: the kernel may then
// start while the previous kernel of the stream finishes; it must call
// griddep_wait() (tc.cuh) before touching anything an earlier kernel writes or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct SelectRows {
  int n_rows;       // number of rows
  int chunks;       // chunks per query (rows = Tq * chunks)
  int chunk;        // chunk length (elements)
  int rate;         // compression rate for visibility
  int N;            // entries per request
  const int32_t* q_pos;
  long long ld_scores;  // elements between queries
};
// Select the top-k of each row of f32 scores and write either final indices
// (out_idx [rows, k], -1 padded) or composite candidates (out_cand [rows, k]).
cudaError_t launch_select_from_scores(const float* scores, const SelectRows& rows, int k,
                                      int32_t* out_idx, uint64_t* out_cand, cudaStream_t stream);
// Rows of at most kSelectRowMaxN visible entries, one CTA each (rows.chunks == 1):
// final indices to out_idx [rows, k].
cudaError_t launch_select_rows(const float* scores, const SelectRows& rows, int k, int32_t* out_idx,
                               cudaStream_t stream);
// Merge: row q has n_cand composite candidates at cand + q*n_cand; write the
// top-k indices to out_idx [rows, k].
cudaError_t launch_select_merge(const uint64_t* cand, int n_rows, int n_cand, int k,
                                int32_t* out_idx, cudaStream_t stream);
// Decode top-k from a per-request histogram of score keys (bins: key >> 20),
// built by the indexer.  Workspace regions as laid out by plan_indexer.
constexpr int kHistBins = 4096;
constexpr int kHistMaxCtas = 128;
constexpr int kHistSlice = 16384;  // entries per select CTA
struct HistSelect {
  const float* scores;
  long long ld;          // elements between requests' score rows
  const int32_t* q_pos;
  int rate, N, k;
  int* hist;             // [2][B][kHistBins]: level 1 by the indexer, level 2 here (zeroed before the indexer)
  int* done;             // [B] arrival tickets (zeroed with hist)
  int B;
  int2* cnt;             // [B][C] per-CTA (above, bin-T) counts
  int32_t* above;        // [B][C][k]
  uint64_t* eq;          // [B][C][slice] composites
  int C, slice;
  int32_t* out;          // [B][k]
};
cudaError_t launch_select_hist(const HistSelect& a, int B, cudaStream_t stream);
unsigned int read_and_clear_select_error();

// ---- indexer.cu ---------------------------------------------------------------
// scores[q, s] = sum_j w[q,j] relu(q_idx[q,j,:] . K[s,:]) for visible s (others untouched).
cudaError_t launch_indexer_scores(const bf16* q_idx, const float* w_idx, const bf16* k_idx,
                                  long long k_seq_stride, int N, const int32_t* q_pos, int Tq,
                                  int mode, int rate, int H_I, int d_I, float* scores,
                                  long long ld_scores, cudaStream_t stream);

// ---- indexer_tc.cu (tcgen05) -------------------------------------------------------
bool indexer_tc_supported(int H_I, int d_I);
// Paged indexer keys: request r's logical block j (rpb keys) is physical block
// bt[r*bt_stride + j] of a pool of n_blocks blocks, [n_blocks * rpb, d_I] bf16.
struct PagedKeys {
  const int32_t* bt;
  long long bt_stride;
  int rpb;
  long long n_blocks;
};
// Decode: query r scores request r's keys (k_idx + r*k_seq_stride), scores[r*ld + s].
cudaError_t launch_indexer_decode_tc(const bf16* q_idx, const float* w_idx, const bf16* k_idx, long long k_seq_stride,
                                     int N, const int32_t* q_pos, int B, int rate, float* scores, long long ld_scores,
                                     int num_sms, cudaStream_t stream,
                                     int* hist = nullptr, bool stall = false, const PagedKeys* paged = nullptr);
// (stall: tests of the bounded waits only -- the key producer issues nothing and every
// wait gives up after a few thousand polls; the kernel records an error and returns)
// Prefill: queries of one sequence against its keys [N, d_I].  With topk_idx (k <= the
// fused limit, indexer_prefill_topk_fused) the top-k is taken on chip and written to
// topk_idx [Tq, k] in entry order (-1 padded), scores unused; without it, scores[q*ld + s]
// for visible s.
bool indexer_prefill_topk_fused(int k);
cudaError_t launch_indexer_prefill_tc(const bf16* q_idx, const float* w_idx, const bf16* k_idx, int N,
                                      const int32_t* q_pos, int Tq, int rate, float* scores, long long ld_scores,
                                      int num_sms, cudaStream_t stream, int k = 0, int32_t* topk_idx = nullptr);
unsigned int read_and_clear_indexer_tc_error();

// SM count of the current device (cached per device).
int device_sm_count();

// ---- mqa.cu -----------------------------------------------------------------------
struct MqaProblem {
  const bf16* q;            // [Tq, H, c]
  const bf16* kv;           // compressed entries (request r at kv + r*kv_seq_stride)
  long long kv_seq_stride;
  int N;                    // entries per request
  const int32_t* idx;       // [Tq, n_idx] or nullptr (dense over visible)
  int n_idx;
  int rate;
  const bf16* win;
  long long win_seq_stride;  // decode: elements between requests' window blocks
  long long win_rows;        // prefill: raw token rows in win (>= 1 + every q_pos)
  const int32_t* q_pos;
  int Tq;
  int mode;
  int H, c, n_win;
  float scale;
  bf16* out;                // [Tq, H, c]
  const float* sink;        // [H] sink logits (natural units, like scale * q . k) or nullptr
  int rope_dims;            // > 0: the output's last rope_dims channels turn back by -q_pos
  float rope_base;
  // paged entries (decode, tensor-core kernel only): request r's entry e is row
  // bt[r*bt_stride + e / rpb] * rpb + e % rpb of a pool of pool_rows rows at kv
  const int32_t* bt = nullptr;
  long long bt_stride = 0;
  int rpb = 0;
  long long pool_rows = 0;
  // opt-in index check: record selected entries outside [-1, N), entries that the
  // query cannot see yet (last token after q_pos) and block-table entries outside
  // the pool; results are computed as without the check
  int check = 0;
};
// Bits of the index-check record (hca_check_device reports them).
constexpr unsigned int kIdxRange = 1u, kIdxCausal = 2u, kIdxBlock = 4u;
// Kind of a selected entry e of a query at position t (0: acceptable).
__host__ __device__ __forceinline__ unsigned int entry_check(int e, int t, int rate, int N) {
  if (e < -1 || e >= N) return kIdxRange;
  if (e >= 0 && (long long)(e + 1) * rate - 1 > t) return kIdxCausal;
  return 0u;
}
// Rows of one split; the workspace layout is decided by plan_mqa().
struct MqaPlan {
  int splits;          // splits per query (1 = no combine)
  int rows_per_split;  // rows of the query's row list per split
  int max_rows;        // upper bound of the row-list length
  size_t ws_bytes;
};
// plan_mqa / launch_mqa pick the tensor-core kernel when it supports the problem.
// pdl: launch it (and its combine) as programmatic dependents of the previous
// kernel of the stream (the caller's top-k); off for work started from events.
MqaPlan plan_mqa(const MqaProblem& p);
MqaPlan plan_mqa_sms(const MqaProblem& p, int sms);  // one wave of at most `sms` CTAs
MqaPlan plan_mqa_cuda_cores(const MqaProblem& p);
size_t mqa_ws_upper_bound(const MqaProblem& p);  // any idx / stride / mode, rows up to max(N, n_idx)
cudaError_t launch_mqa(const MqaProblem& p, const MqaPlan& plan, void* ws, cudaStream_t stream, bool pdl = false);
cudaError_t launch_mqa_combine(const float* ws_o, const float2* ws_ml, int Tq, int splits, int H, int C, bf16* out, const float* sink,
                               const int32_t* q_pos, int rope_dims, float rope_base,
                               cudaStream_t stream,
                               bool pdl = false);

// ---- mqa_tc.cu (tcgen05) -------------------------------------------------------------
bool mqa_tc_supported(const MqaProblem& p);
MqaPlan plan_mqa_tc(const MqaProblem& p, int num_sms);
cudaError_t launch_mqa_decode_tc(const MqaProblem& p, const MqaPlan& pl, void* ws, cudaStream_t stream, bool pdl);
unsigned int read_and_clear_mqa_tc_error();     // bit 0: a wait gave up; entry_check bits << 1
unsigned int read_and_clear_mqa_index_error();  // entry_check bits of the CUDA-core attention

}  // namespace hca
