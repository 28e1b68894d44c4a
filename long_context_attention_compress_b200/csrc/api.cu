// C ABI of libhca.so: argument checking, workspace planning and launch order.
// The operations are documented in include/hca.h.

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace hca {
thread_local int g_launch_counter = 0;

int device_sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}
}

using namespace hca;

namespace {

thread_local std::string g_err;
thread_local int g_last_launches = 0;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return HCA_OK;
  return fail(HCA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool injected(const char* name) {
  const char* v = getenv("HCA_INJECT_FAULT");
  if (!v || !*v) return false;
  return strcmp(v, "all") == 0 || strcmp(v, name) == 0;
}

// Tests of the bounded device waits: HCA_TEST_STALL=indexer makes the decode
// indexer's key producer issue nothing, with a tiny poll budget, so that every
// consumer wait runs out; the kernel records the error and returns.
bool test_stall_indexer() {
  const char* v = getenv("HCA_TEST_STALL");
  return v && strcmp(v, "indexer") == 0;
}

// HCA_DEBUG=1: the attention kernels record selected entries that are out of
// range or not causally visible, and block-table entries outside the pool
// (reported by hca_check_device; the results are as without the check).
bool debug_checks() {
  const char* v = getenv("HCA_DEBUG");
  return v && strcmp(v, "1") == 0;
}

// One NVTX range per entry point call (named after it), for timeline tools.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define HCA_RANGE(name) NvtxRange nvtx_range_(name)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define CHECK_PTR(p, name)                                                          \
  do {                                                                              \
    if (!(p)) return fail(HCA_ERR_INVALID_ARG, "%s: null pointer", name);           \
    if (!aligned16(p)) return fail(HCA_ERR_INVALID_ARG, "%s: not 16-byte aligned", name); \
  } while (0)

#define CHECK(cond, code, ...) \
  do {                         \
    if (!(cond)) return fail(code, __VA_ARGS__); \
  } while (0)

#define CUDA_TRY(expr, where)                      \
  do {                                             \
    int _s = cuda_status((expr), where);           \
    if (_s != HCA_OK) return _s;                   \
  } while (0)

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int check_cfg(const hca_layer_cfg* cfg) {
  if (!cfg) return fail(HCA_ERR_INVALID_ARG, "cfg: null");
  CHECK(cfg->c > 0 && cfg->m > 0 && cfg->m_hca > 0 && cfg->topk > 0 && cfg->n_idx_heads > 0 &&
            cfg->d_idx > 0 && cfg->n_heads > 0 && cfg->n_win > 0,
        HCA_ERR_INVALID_ARG, "cfg: sizes must be positive");
  CHECK(cfg->scale > 0.f, HCA_ERR_INVALID_ARG, "cfg: scale must be positive");
  CHECK((cfg->c == 512 && cfg->n_heads == 64) || (cfg->c == 64 && cfg->n_heads == 4), HCA_ERR_UNSUPPORTED,
        "cfg: (c=%d, n_heads=%d) not specialised; supported (512, 64) and (64, 4)", cfg->c, cfg->n_heads);
  CHECK(cfg->d_idx == 128 || cfg->d_idx == 32, HCA_ERR_UNSUPPORTED, "cfg: d_idx=%d not in {32, 128}", cfg->d_idx);
  CHECK(cfg->n_idx_heads <= 64 && cfg->n_idx_heads % 4 == 0, HCA_ERR_UNSUPPORTED,
        "cfg: n_idx_heads=%d (need <= 64, multiple of 4)", cfg->n_idx_heads);
  CHECK(cfg->topk <= 2048, HCA_ERR_UNSUPPORTED, "cfg: topk=%d > 2048", cfg->topk);
  CHECK(cfg->n_win <= 256, HCA_ERR_UNSUPPORTED, "cfg: n_win=%d > 256", cfg->n_win);
  CHECK(cfg->m <= 16, HCA_ERR_UNSUPPORTED, "cfg: m=%d > 16", cfg->m);
  CHECK(cfg->m_hca <= 1024, HCA_ERR_UNSUPPORTED, "cfg: m_hca=%d > 1024", cfg->m_hca);
  CHECK(cfg->rope_dims >= 0 && cfg->rope_dims % 8 == 0 && cfg->rope_dims <= cfg->c && cfg->rope_dims <= 256,
        HCA_ERR_UNSUPPORTED, "cfg: rope_dims=%d (need a multiple of 8, <= min(c, 256))", cfg->rope_dims);
  CHECK(cfg->rope_dims == 0 || cfg->rope_base > 0.f, HCA_ERR_INVALID_ARG, "cfg: rope_base must be positive");
  CHECK(cfg->norm_eps >= 0.f, HCA_ERR_INVALID_ARG, "cfg: norm_eps must be >= 0");
  return HCA_OK;
}

// Q/KV normalisation of rows (see rms_norm_rope in hca.h).
NormRope norm_rows(const hca_layer_cfg* cfg, const void* x, bool x_f32, long long ld_x, long long seq_x, int n_seq,
                   int rows_per_seq, const int32_t* pos, int pos_add, int pos_step, const float* gamma, void* y,
                   long long ld_y, long long seq_y) {
  NormRope r;
  r.x = x;
  r.x_f32 = x_f32;
  r.ld_x = ld_x;
  r.seq_x = seq_x;
  r.n_seq = n_seq;
  r.rows_per_seq = rows_per_seq;
  r.pos = pos;
  r.pos_add = pos_add;
  r.pos_step = pos_step;
  r.gamma = gamma;
  r.c = cfg->c;
  r.rope_dims = cfg->rope_dims;
  r.eps = cfg->norm_eps;
  r.rope_base = cfg->rope_base;
  r.y = reinterpret_cast<bf16*>(y);
  r.ld_y = ld_y;
  r.seq_y = seq_y;
  return r;
}

// ---- indexer workspace: score matrix [Tq, ldN] f32 + chunk candidates -------
struct IndexerPlan {
  long long ld;   // score row stride
  int chunk, chunks;
  size_t cand_off;  // chunked select: [Tq][chunks][k] composites
  // decode select from the indexer's score histogram (N > kSelectRowMaxN):
  int hist_ctas;    // select CTAs per request (kHistSlice entries each)
  size_t hist_off, done_off, cnt_off, above_off, eq_off;
  size_t bytes;
};

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Prefill on the tensor cores takes its top-k on chip (no workspace at all).
bool fused_prefill(const hca_layer_cfg* cfg, int mode) {
  return mode == HCA_MODE_PREFILL && indexer_tc_supported(cfg->n_idx_heads, cfg->d_idx) &&
         indexer_prefill_topk_fused(cfg->topk);
}

// Workspace: the f32 score rows, then either select layout (they share the space;
// only one is used per call); nothing for the fused prefill.
IndexerPlan plan_indexer(const hca_layer_cfg* cfg, int Tq, int N, int mode) {
  const int k = cfg->topk;
  IndexerPlan p;
  p.ld = ((long long)N + 3) / 4 * 4;
  if (N <= kSelectRowMaxN) {
    p.chunk = N > 0 ? N : 1;
    p.chunks = 1;
  } else {
    p.chunk = 16384;
    p.chunks = (N + p.chunk - 1) / p.chunk;
  }
  const size_t score_bytes = (size_t)Tq * (size_t)p.ld * sizeof(float);
  p.cand_off = align256(score_bytes);
  const size_t cand_bytes = p.chunks > 1 ? (size_t)Tq * p.chunks * k * sizeof(uint64_t) : 0;
  size_t end = p.cand_off + cand_bytes;
  p.hist_ctas = N > kSelectRowMaxN ? (N + kHistSlice - 1) / kHistSlice : 0;
  p.hist_off = p.done_off = p.cnt_off = p.above_off = p.eq_off = 0;
  if (p.hist_ctas > 0) {
    const size_t C = (size_t)p.hist_ctas;
    p.hist_off = align256(score_bytes);
    p.done_off = p.hist_off + 2 * (size_t)Tq * kHistBins * sizeof(int);  // zeroed together with the histograms
    p.cnt_off = align256(p.done_off + (size_t)Tq * sizeof(int));
    p.above_off = align256(p.cnt_off + (size_t)Tq * C * sizeof(int2));
    p.eq_off = align256(p.above_off + (size_t)Tq * C * k * sizeof(int32_t));
    const size_t hist_end = p.eq_off + (size_t)Tq * C * kHistSlice * sizeof(uint64_t);
    end = end > hist_end ? end : hist_end;
  }
  p.bytes = fused_prefill(cfg, mode) ? 0 : end;
  return p;
}

int indexer_ok(const hca_layer_cfg* cfg, int N, int mode) {
  const int k = cfg->topk;
  const IndexerPlan p = plan_indexer(cfg, 1, N, mode);
  if (fused_prefill(cfg, mode)) return HCA_OK;  // any number of entries
  if (mode == HCA_MODE_DECODE) {
    CHECK(p.hist_ctas <= kHistMaxCtas, HCA_ERR_UNSUPPORTED, "indexer: N=%d exceeds %d entries per request", N,
          kHistMaxCtas * kHistSlice);
    return HCA_OK;
  }
  CHECK((long long)p.chunks * k <= kSelectMaxN, HCA_ERR_UNSUPPORTED,
        "indexer: N=%d with topk=%d needs %d chunks (max merge %d candidates)", N, k, p.chunks, kSelectMaxN);
  return HCA_OK;
}

// Keys of the FP4 indexer variant (decode only): MXFP4 codes [N][64 B] and scales
// [N][4 B] per request, `stride` keys apart; q4 = workspace for the queries'
// MXFP4 values in bf16 [Tq, 64, 128].
struct Fp4Keys {
  const uint8_t* codes;
  const uint8_t* scales;
  long long stride;
  bf16* q4;
};

int run_indexer_topk(const bf16* q_idx, const float* w_idx, const bf16* k_idx, long long k_seq_stride, int N,
                     const int32_t* q_pos, int Tq, int mode, const hca_layer_cfg* cfg, int32_t* topk_idx,
                     void* ws, cudaStream_t st, void* const* ev, int n_ev, int& ev_i, int grid_sms = 0,
                     const Fp4Keys* fp4 = nullptr, const PagedKeys* paged = nullptr) {
  const IndexerPlan p = plan_indexer(cfg, Tq, N, mode);
  float* scores = reinterpret_cast<float*>(ws);
  // decode with more entries than one select CTA holds: the indexer also builds
  // each request's score-key histogram, and one threshold select follows
  const bool hist = mode == HCA_MODE_DECODE && p.hist_ctas > 0 &&
                    (fp4 != nullptr || indexer_tc_supported(cfg->n_idx_heads, cfg->d_idx));
  char* wsb = reinterpret_cast<char*>(ws);
  if (fp4) {
    // the queries' MXFP4 values (bf16), then the scores over the FP4 keys
    CUDA_TRY(launch_mxfp4_roundtrip(q_idx, Tq * cfg->n_idx_heads, cfg->d_idx, fp4->q4, st), "fp4 query rounding");
  }
  if (hist)
    CUDA_TRY(cudaMemsetAsync(wsb + p.hist_off, 0, (size_t)Tq * (2 * kHistBins + 1) * sizeof(int), st),
             "histogram reset");
  if (fp4) {
    CUDA_TRY(launch_indexer_decode_fp4(fp4->q4, w_idx, fp4->codes, fp4->scales, fp4->stride, N, q_pos, Tq, cfg->m,
                                       scores, p.ld, grid_sms > 0 ? grid_sms : device_sm_count(), st,
                                       hist ? reinterpret_cast<int*>(wsb + p.hist_off) : nullptr),
             "indexer scores (fp4)");
  } else if (mode == HCA_MODE_DECODE && indexer_tc_supported(cfg->n_idx_heads, cfg->d_idx)) {
    CUDA_TRY(launch_indexer_decode_tc(q_idx, w_idx, k_idx, k_seq_stride, N, q_pos, Tq, cfg->m, scores, p.ld,
                                      grid_sms > 0 ? grid_sms : device_sm_count(), st,
                                      hist ? reinterpret_cast<int*>(wsb + p.hist_off) : nullptr,
                                      test_stall_indexer(), paged),
             "indexer scores (tcgen05)");
  } else if (fused_prefill(cfg, mode)) {
    // scores and top-k in one kernel: nothing goes through memory but the indices
    CUDA_TRY(launch_indexer_prefill_tc(q_idx, w_idx, k_idx, N, q_pos, Tq, cfg->m, nullptr, 0,
                                       grid_sms > 0 ? grid_sms : device_sm_count(), st, cfg->topk, topk_idx),
             "indexer + top-k (tcgen05, prefill)");
    if (ev && ev_i < n_ev) CUDA_TRY(cudaEventRecord((cudaEvent_t)ev[ev_i++], st), "event");
    if (ev && ev_i < n_ev) CUDA_TRY(cudaEventRecord((cudaEvent_t)ev[ev_i++], st), "event");
    return HCA_OK;
  } else if (mode == HCA_MODE_PREFILL && indexer_tc_supported(cfg->n_idx_heads, cfg->d_idx)) {
    CUDA_TRY(launch_indexer_prefill_tc(q_idx, w_idx, k_idx, N, q_pos, Tq, cfg->m, scores, p.ld,
                                       grid_sms > 0 ? grid_sms : device_sm_count(), st),
             "indexer scores (tcgen05, prefill)");
  } else {
    CUDA_TRY(launch_indexer_scores(q_idx, w_idx, k_idx, k_seq_stride, N, q_pos, Tq, mode, cfg->m,
                                   cfg->n_idx_heads, cfg->d_idx, scores, p.ld, st),
             "indexer scores");
  }
  if (ev && ev_i < n_ev) CUDA_TRY(cudaEventRecord((cudaEvent_t)ev[ev_i++], st), "event");
  if (hist) {
    HistSelect a;
    a.scores = scores;
    a.ld = p.ld;
    a.q_pos = q_pos;
    a.rate = cfg->m;
    a.N = N;
    a.k = cfg->topk;
    a.hist = reinterpret_cast<int*>(wsb + p.hist_off);
    a.B = Tq;
    a.done = reinterpret_cast<int*>(wsb + p.done_off);
    a.cnt = reinterpret_cast<int2*>(wsb + p.cnt_off);
    a.above = reinterpret_cast<int32_t*>(wsb + p.above_off);
    a.eq = reinterpret_cast<uint64_t*>(wsb + p.eq_off);
    a.C = p.hist_ctas;
    a.slice = kHistSlice;
    a.out = topk_idx;
    CUDA_TRY(launch_select_hist(a, Tq, st), "select (histogram threshold)");
    if (ev && ev_i < n_ev) CUDA_TRY(cudaEventRecord((cudaEvent_t)ev[ev_i++], st), "event");
    return HCA_OK;
  }
  SelectRows rows;
  rows.chunks = p.chunks;
  rows.chunk = p.chunk;
  rows.n_rows = Tq * p.chunks;
  rows.rate = cfg->m;
  rows.N = N;
  rows.q_pos = q_pos;
  rows.ld_scores = p.ld;
  if (p.chunks == 1) {
    CUDA_TRY(launch_select_rows(scores, rows, cfg->topk, topk_idx, st), "select");
  } else {
    uint64_t* cand = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(ws) + p.cand_off);
    CUDA_TRY(launch_select_from_scores(scores, rows, cfg->topk, nullptr, cand, st), "select chunks");
    CUDA_TRY(launch_select_merge(cand, Tq, p.chunks * cfg->topk, cfg->topk, topk_idx, st), "select merge");
  }
  if (ev && ev_i < n_ev) CUDA_TRY(cudaEventRecord((cudaEvent_t)ev[ev_i++], st), "event");
  return HCA_OK;
}

MqaProblem make_mqa(const hca_layer_cfg* cfg, const hca_bf16* q, const hca_bf16* kv, long long kv_seq_stride, int N,
                    const int32_t* idx, int n_idx, int rate, const hca_bf16* win, long long win_seq_stride,
                    const int32_t* q_pos, int Tq, int mode, hca_bf16* out, const float* sink) {
  MqaProblem p;
  p.q = reinterpret_cast<const bf16*>(q);
  p.kv = reinterpret_cast<const bf16*>(kv);
  p.kv_seq_stride = kv_seq_stride;
  p.N = N;
  p.idx = idx;
  p.n_idx = n_idx;
  p.rate = rate;
  p.win = reinterpret_cast<const bf16*>(win);
  // the same argument carries the window's row count in prefill mode
  p.win_seq_stride = mode == HCA_MODE_DECODE ? win_seq_stride : 0;
  p.win_rows = mode == HCA_MODE_PREFILL ? win_seq_stride : 0;
  p.q_pos = q_pos;
  p.Tq = Tq;
  p.mode = mode;
  p.H = cfg->n_heads;
  p.c = cfg->c;
  p.n_win = cfg->n_win;
  p.scale = cfg->scale;
  p.out = reinterpret_cast<bf16*>(out);
  p.sink = sink;
  p.rope_dims = 0;
  p.rope_base = cfg->rope_base;
  p.check = debug_checks() ? 1 : 0;
  return p;
}

// The attention of a normalised layer reads its normalised queries and window
// rows from the workspace and rotates its output back.
void use_normalised(MqaProblem& p, const hca_layer_cfg* cfg, const void* qn, const void* wn, bool decode) {
  p.q = reinterpret_cast<const bf16*>(qn);
  p.win = reinterpret_cast<const bf16*>(wn);
  if (decode) p.win_seq_stride = (long long)cfg->n_win * cfg->c;
  p.rope_dims = cfg->rope_dims;
}

size_t mqa_ws_bound(const hca_layer_cfg* cfg, int Tq, int N, int n_idx) {
  MqaProblem p = make_mqa(cfg, nullptr, nullptr, 0, N > n_idx ? N : n_idx, nullptr, 0, 1, nullptr, 0, nullptr, Tq,
                          HCA_MODE_DECODE, nullptr, nullptr);
  return mqa_ws_upper_bound(p);
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" {

const char* hca_last_error(void) { return g_err.c_str(); }

int hca_last_launch_count(void) { return g_last_launches; }

const char* hca_version(void) { return "hca-b200 0.1 (sm_100a)"; }

int hca_check_device(void) {
  g_err.clear();
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e, "hca_check_device");
  const unsigned int w1 = read_and_clear_indexer_tc_error();
  const unsigned int w2 = read_and_clear_mqa_tc_error();
  const unsigned int w3 = read_and_clear_select_error();
  const unsigned int w4 = read_and_clear_indexer_fp4_error();
  if (w1 == 0xffffffffu || w2 == 0xffffffffu || w3 == 0xffffffffu || w4 == 0xffffffffu)
    return fail(HCA_ERR_CUDA, "hca_check_device: cannot read the device error word");
  const unsigned int w5 = read_and_clear_mqa_index_error();
  if (w5 == 0xffffffffu) return fail(HCA_ERR_CUDA, "hca_check_device: cannot read the device error word");
  const unsigned int w = w1 | ((w2 & 1u) << 1) | (w4 << 2);
  const unsigned int idx_bad = (w2 >> 1) | w5;
  if (w) return fail(HCA_ERR_DEVICE_CHECK, "hca_check_device: a kernel gave up waiting (error word 0x%x)", w);
  if (w3) return fail(HCA_ERR_DEVICE_CHECK, "hca_check_device: a top-k histogram disagreed with its scores");
  if (idx_bad)
    return fail(HCA_ERR_DEVICE_CHECK, "hca_check_device: the attention was given %s%s%s",
                (idx_bad & kIdxRange) ? "entries out of range; " : "",
                (idx_bad & kIdxCausal) ? "entries not yet visible to their query; " : "",
                (idx_bad & kIdxBlock) ? "block-table entries outside the pool; " : "");
  return HCA_OK;
}

int csa_compress(const hca_bf16* cand, int ld_cand, const hca_bf16* logits, int ld_logits, const float* pos_bias,
                 int ld_bias, int T, int c, int m, hca_bf16* out, int ld_out, void* stream) {
  HCA_RANGE("csa_compress");
  g_err.clear();
  CHECK(T >= 0 && c > 0 && m >= 1 && m <= 16, HCA_ERR_INVALID_ARG, "csa_compress: T=%d c=%d m=%d", T, c, m);
  CHECK(c % 8 == 0, HCA_ERR_UNSUPPORTED, "csa_compress: c=%d not a multiple of 8", c);
  CHECK(ld_cand >= c && ld_logits >= c && ld_bias >= c && ld_out >= c && ld_cand % 8 == 0 && ld_logits % 8 == 0 &&
            ld_out % 8 == 0 && ld_bias % 4 == 0,
        HCA_ERR_INVALID_ARG, "csa_compress: bad row strides");
  if (T / m == 0) return injected("csa_compress") ? fail(HCA_ERR_INJECTED, "csa_compress: injected") : HCA_OK;
  CHECK_PTR(cand, "csa_compress: cand");
  CHECK_PTR(logits, "csa_compress: logits");
  CHECK_PTR(pos_bias, "csa_compress: pos_bias");
  CHECK_PTR(out, "csa_compress: out");
  if (injected("csa_compress")) return fail(HCA_ERR_INJECTED, "csa_compress: injected");
  CUDA_TRY(launch_compress(reinterpret_cast<const bf16*>(cand), ld_cand, reinterpret_cast<const bf16*>(logits),
                           ld_logits, pos_bias, ld_bias, 1, 0, T, c, m, true, reinterpret_cast<bf16*>(out), ld_out, 0,
                           as_stream(stream)),
           "csa_compress");
  return HCA_OK;
}

int hca_compress(const hca_bf16* cand, int ld_cand, const hca_bf16* logits, int ld_logits, const float* pos_bias,
                 int ld_bias, int B, long long seq_stride_in, int T, int c, int m_hca, hca_bf16* out, int ld_out,
                 long long seq_stride_out, void* stream) {
  HCA_RANGE("hca_compress");
  g_err.clear();
  CHECK(B >= 0 && B <= 65535 && T >= 0 && c > 0 && m_hca >= 1 && m_hca <= 1024, HCA_ERR_INVALID_ARG,
        "hca_compress: B=%d T=%d c=%d m'=%d", B, T, c, m_hca);
  CHECK(c % 8 == 0, HCA_ERR_UNSUPPORTED, "hca_compress: c=%d not a multiple of 8", c);
  CHECK(ld_cand >= c && ld_logits >= c && ld_bias >= c && ld_out >= c && ld_cand % 8 == 0 && ld_logits % 8 == 0 &&
            ld_out % 8 == 0 && ld_bias % 4 == 0 && seq_stride_in % 8 == 0 && seq_stride_out % 8 == 0,
        HCA_ERR_INVALID_ARG, "hca_compress: bad strides");
  if (T / m_hca == 0 || B == 0) return injected("hca_compress") ? fail(HCA_ERR_INJECTED, "hca_compress: injected") : HCA_OK;
  CHECK_PTR(cand, "hca_compress: cand");
  CHECK_PTR(logits, "hca_compress: logits");
  CHECK_PTR(pos_bias, "hca_compress: pos_bias");
  CHECK_PTR(out, "hca_compress: out");
  if (injected("hca_compress")) return fail(HCA_ERR_INJECTED, "hca_compress: injected");
  CUDA_TRY(launch_compress(reinterpret_cast<const bf16*>(cand), ld_cand, reinterpret_cast<const bf16*>(logits),
                           ld_logits, pos_bias, ld_bias, B, seq_stride_in, T, c, m_hca, false,
                           reinterpret_cast<bf16*>(out), ld_out, seq_stride_out, as_stream(stream)),
           "hca_compress");
  return HCA_OK;
}

size_t hca_workspace_size(int op, const hca_layer_cfg* cfg, int Tq, int N, int mode) {
  if (check_cfg(cfg) != HCA_OK || Tq < 0 || N < 0) return (size_t)-1;
  switch (op) {
    case HCA_OP_INDEXER_TOPK:
      if (indexer_ok(cfg, N, mode) != HCA_OK) return (size_t)-1;
      return plan_indexer(cfg, Tq, N, mode).bytes;
    case HCA_OP_SPARSE_MQA:
      return mqa_ws_bound(cfg, Tq, N, cfg->topk);
    default:
      return (size_t)-1;
  }
}

int csa_indexer_topk(const hca_bf16* q_idx, const float* w_idx, const hca_bf16* k_idx, long long k_seq_stride, int N,
                     const int32_t* q_pos, int Tq, int mode, const hca_layer_cfg* cfg, int32_t* topk_idx, void* ws,
                     size_t ws_bytes, void* stream) {
  HCA_RANGE("csa_indexer_topk");
  g_err.clear();
  int s = check_cfg(cfg);
  if (s != HCA_OK) return s;
  CHECK(Tq >= 0 && N >= 0, HCA_ERR_INVALID_ARG, "csa_indexer_topk: Tq=%d N=%d", Tq, N);
  CHECK(mode == HCA_MODE_PREFILL || mode == HCA_MODE_DECODE, HCA_ERR_INVALID_ARG, "csa_indexer_topk: mode=%d", mode);
  CHECK(mode == HCA_MODE_PREFILL || k_seq_stride % 8 == 0, HCA_ERR_INVALID_ARG, "csa_indexer_topk: k_seq_stride");
  s = indexer_ok(cfg, N, mode);
  if (s != HCA_OK) return s;
  if (Tq == 0) return injected("csa_indexer_topk") ? fail(HCA_ERR_INJECTED, "injected") : HCA_OK;
  CHECK_PTR(q_idx, "csa_indexer_topk: q_idx");
  CHECK_PTR(w_idx, "csa_indexer_topk: w_idx");
  CHECK_PTR(q_pos, "csa_indexer_topk: q_pos");
  CHECK_PTR(topk_idx, "csa_indexer_topk: topk_idx");
  if (N > 0) CHECK_PTR(k_idx, "csa_indexer_topk: k_idx");
  const size_t need = plan_indexer(cfg, Tq, N, mode).bytes;
  CHECK(ws_bytes >= need, HCA_ERR_WORKSPACE, "csa_indexer_topk: workspace %zu < %zu", ws_bytes, need);
  if (need) CHECK(ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0, HCA_ERR_INVALID_ARG,
                  "csa_indexer_topk: ws null or not 256-byte aligned");
  if (injected("csa_indexer_topk")) return fail(HCA_ERR_INJECTED, "csa_indexer_topk: injected");
  int ev_i = 0;
  return run_indexer_topk(reinterpret_cast<const bf16*>(q_idx), w_idx, reinterpret_cast<const bf16*>(k_idx),
                          k_seq_stride, N, q_pos, Tq, mode, cfg, topk_idx, ws, as_stream(stream), nullptr, 0, ev_i);
}

// ---- csa_indexer_topk_noalloc ------------------------------------------------
// Scratch for callers that cannot allocate device memory: one file-scope
// device array, present on every GPU that loads this module until the
// process exits.  Host code only ever sees a stand-in symbol for it; the
// real device address comes from cudaGetSymbolAddress, taken once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HCA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

int noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "csa_indexer_topk_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return fail(HCA_ERR_UNSUPPORTED, "csa_indexer_topk_noalloc: device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e, "csa_indexer_topk_noalloc: cudaGetSymbolAddress");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return HCA_OK;
}
}  // namespace

int csa_indexer_topk_noalloc(const hca_bf16* q_idx, const float* w_idx, const hca_bf16* k_idx,
                             long long k_seq_stride, int N, const int32_t* q_pos, int Tq, int mode,
                             const hca_layer_cfg* cfg, int32_t* topk_idx, void* stream) {
  HCA_RANGE("csa_indexer_topk_noalloc");
  g_err.clear();
  int s = check_cfg(cfg);
  if (s != HCA_OK) return s;
  CHECK(Tq >= 0 && N >= 0, HCA_ERR_INVALID_ARG, "csa_indexer_topk_noalloc: Tq=%d N=%d", Tq, N);
  CHECK(mode == HCA_MODE_PREFILL || mode == HCA_MODE_DECODE, HCA_ERR_INVALID_ARG,
        "csa_indexer_topk_noalloc: mode=%d", mode);
  CHECK(mode == HCA_MODE_PREFILL || k_seq_stride % 8 == 0, HCA_ERR_INVALID_ARG,
        "csa_indexer_topk_noalloc: k_seq_stride");
  s = indexer_ok(cfg, N, mode);
  if (s != HCA_OK) return s;
  const size_t need = plan_indexer(cfg, Tq, N, mode).bytes;
  CHECK(need <= (size_t)HCA_NOALLOC_SCRATCH_BYTES, HCA_ERR_WORKSPACE,
        "csa_indexer_topk_noalloc: Tq=%d x N=%d needs %zu bytes of scratch, more than the built-in %zu; "
        "use csa_indexer_topk with a workspace",
        Tq, N, need, (size_t)HCA_NOALLOC_SCRATCH_BYTES);
  if (Tq == 0) return HCA_OK;
  CHECK_PTR(q_idx, "csa_indexer_topk_noalloc: q_idx");
  CHECK_PTR(w_idx, "csa_indexer_topk_noalloc: w_idx");
  CHECK_PTR(q_pos, "csa_indexer_topk_noalloc: q_pos");
  CHECK_PTR(topk_idx, "csa_indexer_topk_noalloc: topk_idx");
  if (N > 0) CHECK_PTR(k_idx, "csa_indexer_topk_noalloc: k_idx");
  if (injected("csa_indexer_topk_noalloc")) return fail(HCA_ERR_INJECTED, "csa_indexer_topk_noalloc: injected");
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != HCA_OK) return s;
  // Nothing in the scratch needs to start at zero: every score the select
  // reads and every chunk candidate the merge reads is written earlier in the
  // same call, so the previous call's contents are never observed.
  int ev_i = 0;
  return run_indexer_topk(reinterpret_cast<const bf16*>(q_idx), w_idx, reinterpret_cast<const bf16*>(k_idx),
                          k_seq_stride, N, q_pos, Tq, mode, cfg, topk_idx, scratch, as_stream(stream), nullptr, 0,
                          ev_i);
}

int rms_norm_rope(const void* x, int x_is_f32, long long ld_x, long long seq_stride_x, int n_seq, int rows_per_seq,
                  const int32_t* pos, int pos_add, int pos_step, const float* gamma, const hca_layer_cfg* cfg,
                  hca_bf16* y, long long ld_y, long long seq_stride_y, void* stream) {
  HCA_RANGE("rms_norm_rope");
  g_err.clear();
  int s = check_cfg(cfg);
  if (s != HCA_OK) return s;
  CHECK(n_seq >= 0 && rows_per_seq >= 0, HCA_ERR_INVALID_ARG, "rms_norm_rope: n_seq=%d rows_per_seq=%d", n_seq,
        rows_per_seq);
  const long long al = x_is_f32 ? 4 : 8;
  CHECK(ld_x >= cfg->c && ld_x % al == 0 && seq_stride_x >= 0 && seq_stride_x % al == 0, HCA_ERR_INVALID_ARG,
        "rms_norm_rope: x strides (%lld, %lld)", ld_x, seq_stride_x);
  CHECK(ld_y >= cfg->c && ld_y % 8 == 0 && seq_stride_y >= 0 && seq_stride_y % 8 == 0, HCA_ERR_INVALID_ARG,
        "rms_norm_rope: y strides (%lld, %lld)", ld_y, seq_stride_y);
  CHECK(!(x_is_f32 && (const void*)x == (const void*)y), HCA_ERR_INVALID_ARG,
        "rms_norm_rope: in place needs bf16 rows");
  if (n_seq == 0 || rows_per_seq == 0) return HCA_OK;
  CHECK_PTR(x, "rms_norm_rope: x");
  CHECK_PTR(gamma, "rms_norm_rope: gamma");
  CHECK_PTR(y, "rms_norm_rope: y");
  if (injected("rms_norm_rope")) return fail(HCA_ERR_INJECTED, "rms_norm_rope: injected");
  CUDA_TRY(launch_norm_rope(norm_rows(cfg, x, x_is_f32 != 0, ld_x, seq_stride_x, n_seq, rows_per_seq, pos, pos_add,
                                      pos_step, gamma, y, ld_y, seq_stride_y),
                            as_stream(stream)),
           "rms_norm_rope");
  return HCA_OK;
}

static int check_mqa(const hca_layer_cfg* cfg, const hca_bf16* q, const hca_bf16* kv, long long kv_seq_stride, int N,
                     const int32_t* idx, int n_idx, int rate, const hca_bf16* win, long long win_seq_stride,
                     const int32_t* q_pos, int Tq, int mode, hca_bf16* out, const char* who) {
  CHECK(Tq >= 0 && N >= 0 && rate >= 1, HCA_ERR_INVALID_ARG, "%s: Tq=%d N=%d rate=%d", who, Tq, N, rate);
  CHECK(mode == HCA_MODE_PREFILL || mode == HCA_MODE_DECODE, HCA_ERR_INVALID_ARG, "%s: mode=%d", who, mode);
  CHECK(!idx || (n_idx > 0 && n_idx <= 4096), HCA_ERR_INVALID_ARG, "%s: n_idx=%d", who, n_idx);
  CHECK(kv_seq_stride % 8 == 0 && (mode == HCA_MODE_PREFILL || win_seq_stride % 8 == 0), HCA_ERR_INVALID_ARG,
        "%s: strides", who);
  // prefill: the same argument is the window's row count (at least one row per query position)
  CHECK(mode == HCA_MODE_DECODE || win_seq_stride >= 1, HCA_ERR_INVALID_ARG, "%s: window row count %lld", who,
        win_seq_stride);
  if (Tq == 0) return HCA_OK;
  CHECK_PTR(q, who);
  CHECK_PTR(win, who);
  CHECK_PTR(q_pos, who);
  CHECK_PTR(out, who);
  if (N > 0) CHECK_PTR(kv, who);
  if (idx) CHECK_PTR(idx, who);
  return HCA_OK;
}

int sparse_mqa_attend(const hca_bf16* q, const hca_bf16* kv, long long kv_seq_stride, int N, const int32_t* idx,
                      int n_idx, int rate, const hca_bf16* win, long long win_seq_stride, const int32_t* q_pos, int Tq,
                      int mode, const hca_layer_cfg* cfg, const float* sink, int rotate_out, hca_bf16* out,
                      void* ws, size_t ws_bytes, void* stream) {
  HCA_RANGE("sparse_mqa_attend");
  g_err.clear();
  int s = check_cfg(cfg);
  if (s != HCA_OK) return s;
  s = check_mqa(cfg, q, kv, kv_seq_stride, N, idx, n_idx, rate, win, win_seq_stride, q_pos, Tq, mode, out,
                "sparse_mqa_attend");
  if (s != HCA_OK) return s;
  MqaProblem p = make_mqa(cfg, q, kv, kv_seq_stride, N, idx, n_idx, rate, win, win_seq_stride, q_pos, Tq, mode, out,
                          sink);
  if (rotate_out) p.rope_dims = cfg->rope_dims;
  const MqaPlan pl = plan_mqa(p);
  CHECK(ws_bytes >= pl.ws_bytes, HCA_ERR_WORKSPACE, "sparse_mqa_attend: workspace %zu < %zu", ws_bytes, pl.ws_bytes);
  if (pl.ws_bytes) CHECK(ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0, HCA_ERR_INVALID_ARG,
                         "sparse_mqa_attend: ws null or not 256-byte aligned");
  if (injected("sparse_mqa_attend")) return fail(HCA_ERR_INJECTED, "sparse_mqa_attend: injected");
  if (Tq == 0) return HCA_OK;
  CUDA_TRY(launch_mqa(p, pl, ws, as_stream(stream)), "sparse_mqa_attend");
  return HCA_OK;
}

// ---- FP8 storage of the non-rotary KV channels ----------------------------------
static int check_fp8_layout(const hca_layer_cfg* cfg, long long ld_codes, long long ld_scales, long long ld_rope,
                            const char* who) {
  const int n = cfg->c - cfg->rope_dims;
  CHECK(n > 0 && n % 64 == 0 && cfg->rope_dims % 8 == 0, HCA_ERR_UNSUPPORTED,
        "%s: c - rope_dims = %d must be a positive multiple of 64 (rope_dims a multiple of 8)", who, n);
  CHECK(ld_codes >= n && ld_codes % 16 == 0 && ld_scales >= n / 64 && ld_rope >= cfg->rope_dims && ld_rope % 8 == 0,
        HCA_ERR_INVALID_ARG, "%s: row strides (codes %lld, scales %lld, rope %lld)", who, ld_codes, ld_scales, ld_rope);
  return HCA_OK;
}

static KvFp8 kv_fp8_of(const hca_kv_fp8* d) {
  KvFp8 k;
  k.codes = d->codes;
  k.scales = d->scales;
  k.rope = reinterpret_cast<const bf16*>(d->rope);
  k.ld_codes = d->ld_codes;
  k.ld_scales = d->ld_scales;
  k.ld_rope = d->ld_rope;
  k.seq_rows = d->seq_rows;
  return k;
}

extern "C" int kv_fp8_quantize(const void* x, int x_is_f32, long long ld_x, long long rows, const hca_layer_cfg* cfg,
                               uint8_t* codes, long long ld_codes, float* scales, long long ld_scales, hca_bf16* rope,
                               long long ld_rope, void* stream) {
  HCA_RANGE("kv_fp8_quantize");
  g_err.clear();
  int s = check_cfg(cfg);
  if (s != HCA_OK) return s;
  CHECK(rows >= 0, HCA_ERR_INVALID_ARG, "kv_fp8_quantize: rows=%lld", rows);
  if ((s = check_fp8_layout(cfg, ld_codes, ld_scales, ld_rope, "kv_fp8_quantize")) != HCA_OK) return s;
  CHECK(ld_x >= cfg->c && ld_x % (x_is_f32 ? 4 : 8) == 0, HCA_ERR_INVALID_ARG, "kv_fp8_quantize: ld_x %lld", ld_x);
  if (rows == 0) return HCA_OK;
  CHECK_PTR(x, "kv_fp8_quantize: x");
  CHECK_PTR(codes, "kv_fp8_quantize: codes");
  CHECK(scales != nullptr && (reinterpret_cast<uintptr_t>(scales) & 3u) == 0, HCA_ERR_INVALID_ARG,
        "kv_fp8_quantize: scales null or misaligned");
  if (cfg->rope_dims) CHECK_PTR(rope, "kv_fp8_quantize: rope");
  if (injected("kv_fp8_quantize")) return fail(HCA_ERR_INJECTED, "kv_fp8_quantize: injected");
  CUDA_TRY(launch_kv_fp8_quantize(x, x_is_f32 != 0, ld_x, rows, cfg->c, cfg->rope_dims, codes, ld_codes, scales,
                                  ld_scales, reinterpret_cast<bf16*>(rope), ld_rope, as_stream(stream)),
           "kv_fp8_quantize");
  return HCA_OK;
}

static int check_kv8(const hca_layer_cfg* cfg, const hca_kv_fp8* d, const char* who) {
  int s = check_fp8_layout(cfg, d->ld_codes, d->ld_scales, d->ld_rope, who);
  if (s != HCA_OK) return s;
  CHECK_PTR(d->codes, who);
  CHECK(d->scales != nullptr && (reinterpret_cast<uintptr_t>(d->scales) & 3u) == 0, HCA_ERR_INVALID_ARG,
        "%s: scales null or misaligned", who);
  if (cfg->rope_dims) CHECK_PTR(d->rope, who);
  CHECK(d->seq_rows >= 0, HCA_ERR_INVALID_ARG, "%s: seq_rows", who);
  return HCA_OK;
}

// ---- decode ------------------------------------------------------------------
// When both layers are present, the HCA layer (its block compression and dense
// attention) runs on a side stream, concurrently with the CSA indexer, on a
// share of the SMs proportional to its bytes; the indexer's persistent grid
// leaves those SMs free.  The two then join before the call returns.  The HCA
// attention partials get their own workspace region.
struct DecodeSched {
  bool overlap = false;
  int sms = 0, r_hca = 0;
  MqaPlan csa_pl{}, hca_pl{};
  size_t main_bytes = 0, hca_off = 0, total = 0;
  // Q/KV normalisation: normalised queries [B, H, c] and window blocks [B, n_win, c]
  // (bf16) of each normalised layer, and the HCA entries in f32 [B, c] before theirs
  size_t csa_qn = 0, csa_wn = 0, hca_qn = 0, hca_wn = 0, hca_ef = 0;
  // FP4 indexer: the queries' MXFP4 values in bf16 [B, H_I, d_I]
  size_t q4 = 0;
  // paged caches: the newest HCA entries [B, c] bf16 before they go to their pool rows
  size_t hca_new = 0;
  // FP8 caches: the CSA layer's selected rows widened to bf16 [B, k, c] and their
  // slot indices [B, k]; the HCA layer's visible rows [B, hca_N, c]; the newest HCA
  // entries [B, c] (f32, or bf16 after normalisation) before their FP8 form
  size_t csa8_rows = 0, csa8_idx = 0, hca8_rows = 0, hca8_new = 0;
};

// Geometry of the paged (classical) cache: blocks of lcm(m, m') raw tokens.
struct PagedGeom {
  int rpb_csa = 0, rpb_hca = 0;
};
static PagedGeom paged_geom(const hca_layer_cfg* cfg) {
  int a = cfg->m, b = cfg->m_hca;
  while (b) { const int t = a % b; a = b; b = t; }
  const long long L = (long long)cfg->m / a * cfg->m_hca;
  PagedGeom g;
  g.rpb_csa = (int)(L / cfg->m);
  g.rpb_hca = (int)(L / cfg->m_hca);
  return g;
}
static void make_paged(MqaProblem& p, const hca_decode_args* a, int rpb) {
  p.bt = a->block_table;
  p.bt_stride = a->bt_stride;
  p.rpb = rpb;
  p.pool_rows = (long long)a->n_pool_blocks * rpb;
  p.kv_seq_stride = 0;
}

static MqaProblem decode_csa_problem(const hca_layer_cfg* cfg, const hca_decode_args* a) {
  MqaProblem p = make_mqa(cfg, a->csa_q, a->csa_kv, a->csa_kv_stride, a->csa_N,
                          a->csa_topk_idx ? a->csa_topk_idx : reinterpret_cast<const int32_t*>(1), cfg->topk, cfg->m,
                          a->csa_win, a->csa_win_stride, a->q_pos, a->B, HCA_MODE_DECODE, a->csa_out, a->csa_sink);
  if (a->block_table) make_paged(p, a, paged_geom(cfg).rpb_csa);
  return p;
}
static MqaProblem decode_hca_problem(const hca_layer_cfg* cfg, const hca_decode_args* a) {
  MqaProblem p = make_mqa(cfg, a->hca_q, a->hca_kv, a->hca_kv_stride, a->hca_N, nullptr, 0, cfg->m_hca, a->hca_win,
                          a->hca_win_stride, a->q_pos, a->B, HCA_MODE_DECODE, a->hca_out, a->hca_sink);
  if (a->block_table) make_paged(p, a, paged_geom(cfg).rpb_hca);
  return p;
}

static DecodeSched decode_schedule(const hca_layer_cfg* cfg, const hca_decode_args* a) {
  DecodeSched d;
  d.sms = device_sm_count();
  const bool csa = a->csa_q != nullptr, hcl = a->hca_q != nullptr;
  MqaProblem pc, ph;
  if (csa) pc = decode_csa_problem(cfg, a);
  if (hcl) ph = decode_hca_problem(cfg, a);
  d.overlap = csa && hcl && indexer_tc_supported(cfg->n_idx_heads, cfg->d_idx) && mqa_tc_supported(ph) && d.sms >= 16;
  if (d.overlap) {
    // Balance the two sides' SM-time: the attention costs about kAttnTileUs per
    // 64 rows on one SM, the indexer streams about kIdxBytesPerSmUs bytes per
    // microsecond per SM (calibrated on B200 by sweeping the HCA share of the
    // 8-request 1M-context step: 16 of 148 SMs is best there, 0.178 against
    // 0.188 ms with 24).  The HCA share is a whole number of splits per request
    // so that it runs as a single wave.
    constexpr double kAttnTileUs = 2.0, kIdxBytesPerSmUs = 35e3;
    const double hca_tiles = (double)a->B * std::ceil(((double)a->hca_N + cfg->n_win) / 64.0);
    const double hca_us = hca_tiles * kAttnTileUs;
    const double idx_us = (double)a->B * a->csa_N * cfg->d_idx * 2.0 / kIdxBytesPerSmUs;
    int r = (int)(d.sms * hca_us / (hca_us + idx_us) + 0.5);
    r = std::min(r, d.sms / 2);
    r = std::max(1, r / a->B) * a->B;
    if (r > d.sms / 2) {
      d.overlap = false;  // too many requests to share the machine this way
    } else {
      d.r_hca = r;
      d.hca_pl = plan_mqa_sms(ph, r);
    }
  }
  if (!d.overlap && hcl) {
    d.hca_pl = plan_mqa(ph);
  }
  if (csa) {
    d.csa_pl = plan_mqa(pc);
    d.main_bytes = std::max(plan_indexer(cfg, a->B, a->csa_N, HCA_MODE_DECODE).bytes, d.csa_pl.ws_bytes);
  }
  if (d.overlap) {
    d.hca_off = round256(d.main_bytes);
    d.total = round256(d.hca_off + d.hca_pl.ws_bytes);
  } else {
    d.hca_off = 0;
    d.total = round256(std::max(d.main_bytes, hcl ? d.hca_pl.ws_bytes : (size_t)0));
  }
  const size_t qbytes = round256((size_t)a->B * cfg->n_heads * cfg->c * 2);
  const size_t wbytes = round256((size_t)a->B * cfg->n_win * cfg->c * 2);
  if (csa && a->csa_norm) {
    d.csa_qn = d.total;
    d.csa_wn = d.csa_qn + qbytes;
    d.total = d.csa_wn + wbytes;
  }
  if (hcl && a->hca_norm) {
    d.hca_qn = d.total;
    d.hca_wn = d.hca_qn + qbytes;
    d.hca_ef = d.hca_wn + wbytes;
    d.total = d.hca_ef + round256((size_t)a->B * cfg->c * 4);
  }
  if (csa && a->csa_k_codes) {
    d.q4 = d.total;
    d.total = d.q4 + round256((size_t)a->B * cfg->n_idx_heads * cfg->d_idx * 2);
  }
  if (hcl && a->block_table && a->hca_block_cand) {
    d.hca_new = d.total;
    d.total = d.hca_new + round256((size_t)a->B * cfg->c * 2);
  }
  if (csa && a->csa_kv8) {
    d.csa8_rows = d.total;
    d.csa8_idx = d.csa8_rows + round256((size_t)a->B * cfg->topk * cfg->c * 2);
    d.total = d.csa8_idx + round256((size_t)a->B * cfg->topk * 4);
  }
  if (hcl && a->hca_kv8) {
    d.hca8_rows = d.total;
    d.hca8_new = d.hca8_rows + round256((size_t)a->B * a->hca_N * cfg->c * 2);
    d.total = d.hca8_new + round256((size_t)a->B * cfg->c * 4);
  }
  return d;
}

static size_t decode_ws(const hca_layer_cfg* cfg, const hca_decode_args* a) { return decode_schedule(cfg, a).total; }

// Side stream and fork/join events of the calling host thread on the current
// device (created on first use, kept for the thread's lifetime).
struct SideStream {
  int dev = -1;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
static int side_stream(SideStream** out) {
  static thread_local SideStream cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "side stream: cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(HCA_ERR_UNSUPPORTED, "side stream: device %d", dev);
  SideStream& ss = cache[dev];
  if (!ss.s) {
    if ((e = cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_status(e, "side stream: create");
    if ((e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_status(e, "side stream: event");
    if ((e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_status(e, "side stream: event");
    ss.dev = dev;
  }
  *out = &ss;
  return HCA_OK;
}

size_t hybrid_attn_decode_workspace(const hca_layer_cfg* cfg, const hca_decode_args* a) {
  if (check_cfg(cfg) != HCA_OK || !a || a->B < 0) return (size_t)-1;
  if (a->csa_q && indexer_ok(cfg, a->csa_N, HCA_MODE_DECODE) != HCA_OK) return (size_t)-1;
  return decode_ws(cfg, a);
}

int hybrid_attn_decode(const hca_layer_cfg* cfg, const hca_decode_args* a, void* ws, size_t ws_bytes, void* stream) {
  HCA_RANGE("hybrid_attn_decode");
  g_err.clear();
  int s = check_cfg(cfg);
  if (s != HCA_OK) return s;
  CHECK(a != nullptr, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: args null");
  CHECK(a->B >= 0 && a->B <= 65535, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: B=%d", a->B);
  CHECK(a->csa_q || a->hca_q, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: neither layer given");
  CHECK(a->n_events >= 0, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: n_events");
  if (a->B == 0) return HCA_OK;
  CHECK_PTR(a->q_pos, "hybrid_attn_decode: q_pos");
  const PagedGeom pg = paged_geom(cfg);
  if (a->block_table) {
    CHECK_PTR(a->block_table, "hybrid_attn_decode: block_table");
    CHECK(cfg->c == 512 && cfg->n_heads == 64, HCA_ERR_UNSUPPORTED,
          "hybrid_attn_decode: paged caches need c = 512 and 64 heads");
    CHECK(a->n_pool_blocks > 0, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: n_pool_blocks=%d", a->n_pool_blocks);
    if (a->csa_q) {
      CHECK(indexer_tc_supported(cfg->n_idx_heads, cfg->d_idx) && !a->csa_k_codes, HCA_ERR_UNSUPPORTED,
            "hybrid_attn_decode: paged caches need the 64 x 128 indexer with bf16 keys");
      CHECK(pg.rpb_csa % 8 == 0 && 128 % pg.rpb_csa == 0, HCA_ERR_UNSUPPORTED,
            "hybrid_attn_decode: paged CSA blocks of %d entries (need a multiple of 8 dividing 128)", pg.rpb_csa);
      CHECK(a->bt_stride >= ((long long)a->csa_N + pg.rpb_csa - 1) / pg.rpb_csa, HCA_ERR_INVALID_ARG,
            "hybrid_attn_decode: bt_stride %lld < the %d CSA blocks", a->bt_stride,
            (a->csa_N + pg.rpb_csa - 1) / pg.rpb_csa);
    }
    if (a->hca_q)
      CHECK(a->bt_stride >= ((long long)a->hca_N + pg.rpb_hca - 1) / pg.rpb_hca, HCA_ERR_INVALID_ARG,
            "hybrid_attn_decode: bt_stride %lld < the %d HCA blocks", a->bt_stride,
            (a->hca_N + pg.rpb_hca - 1) / pg.rpb_hca);
  }
  if (a->csa_kv8 || a->hca_kv8)
    CHECK(!a->block_table, HCA_ERR_UNSUPPORTED, "hybrid_attn_decode: FP8 caches are not paged");
  if (a->csa_q && a->csa_kv8 && (s = check_kv8(cfg, a->csa_kv8, "hybrid_attn_decode: csa_kv8")) != HCA_OK) return s;
  if (a->hca_q && a->hca_kv8 && (s = check_kv8(cfg, a->hca_kv8, "hybrid_attn_decode: hca_kv8")) != HCA_OK) return s;
  if (a->csa_q) {
    s = indexer_ok(cfg, a->csa_N, HCA_MODE_DECODE);
    if (s != HCA_OK) return s;
    CHECK(a->csa_N > 0, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: csa_N=%d", a->csa_N);
    CHECK_PTR(a->csa_q_idx, "hybrid_attn_decode: csa_q_idx");
    CHECK_PTR(a->csa_w_idx, "hybrid_attn_decode: csa_w_idx");
    if (a->csa_k_codes) {
      CHECK(indexer_tc_supported(cfg->n_idx_heads, cfg->d_idx), HCA_ERR_UNSUPPORTED,
            "hybrid_attn_decode: the FP4 indexer takes 64 heads x 128 (got %d x %d)", cfg->n_idx_heads, cfg->d_idx);
      CHECK_PTR(a->csa_k_codes, "hybrid_attn_decode: csa_k_codes");
      CHECK_PTR(a->csa_k_scales, "hybrid_attn_decode: csa_k_scales");
      const long long n4 = ((long long)a->csa_N + 3) / 4 * 4;
      CHECK(a->B <= 1 || (a->csa_k4_stride >= n4 && a->csa_k4_stride % 4 == 0), HCA_ERR_INVALID_ARG,
            "hybrid_attn_decode: csa_k4_stride %lld (need >= %lld keys, a multiple of 4)", a->csa_k4_stride, n4);
    } else {
      CHECK_PTR(a->csa_k_idx, "hybrid_attn_decode: csa_k_idx");
      CHECK(a->csa_k_stride % 8 == 0, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: csa_k_stride");
    }
    CHECK_PTR(a->csa_topk_idx, "hybrid_attn_decode: csa_topk_idx");
    s = check_mqa(cfg, a->csa_q, a->csa_kv, a->csa_kv_stride, a->csa_kv8 ? 0 : a->csa_N, a->csa_topk_idx, cfg->topk,
                  cfg->m,
                  a->csa_win, a->csa_win_stride, a->q_pos, a->B, HCA_MODE_DECODE, a->csa_out, "hybrid_attn_decode: csa");
    if (s != HCA_OK) return s;
    if (a->csa_norm) CHECK_PTR(a->csa_norm, "hybrid_attn_decode: csa_norm");
  }
  if (a->hca_q) {
    CHECK(a->hca_N > 0, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: hca_N=%d", a->hca_N);
    s = check_mqa(cfg, a->hca_q, a->hca_kv, a->hca_kv_stride, a->hca_kv8 ? 0 : a->hca_N, nullptr, 0, cfg->m_hca,
                  a->hca_win,
                  a->hca_win_stride, a->q_pos, a->B, HCA_MODE_DECODE, a->hca_out, "hybrid_attn_decode: hca");
    if (s != HCA_OK) return s;
    if (a->hca_norm) CHECK_PTR(a->hca_norm, "hybrid_attn_decode: hca_norm");
    if (a->hca_block_cand) {
      CHECK_PTR(a->hca_block_logits, "hybrid_attn_decode: hca_block_logits");
      CHECK_PTR(a->hca_pos_bias, "hybrid_attn_decode: hca_pos_bias");
      CHECK(a->hca_block_stride % 8 == 0, HCA_ERR_INVALID_ARG, "hybrid_attn_decode: hca_block_stride");
    }
  }
  const size_t need = decode_ws(cfg, a);
  CHECK(ws_bytes >= need, HCA_ERR_WORKSPACE, "hybrid_attn_decode: workspace %zu < %zu", ws_bytes, need);
  if (need) CHECK(ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0, HCA_ERR_INVALID_ARG,
                  "hybrid_attn_decode: ws null or not 256-byte aligned");
  if (injected("hybrid_attn_decode")) return fail(HCA_ERR_INJECTED, "hybrid_attn_decode: injected");

  cudaStream_t st = as_stream(stream);
  g_launch_counter = 0;
  g_last_launches = 0;
  int ev_i = 0;
  void* const* ev = a->events;
  const int n_ev = ev ? a->n_events : 0;
  auto mark = [&]() -> int {
    if (ev && ev_i < n_ev) return cuda_status(cudaEventRecord((cudaEvent_t)ev[ev_i++], st), "event");
    return HCA_OK;
  };
  const DecodeSched sched = decode_schedule(cfg, a);
  SideStream* side = nullptr;
  if (sched.overlap) {
    if ((s = side_stream(&side)) != HCA_OK) return s;
  }
  cudaStream_t hst = sched.overlap ? side->s : st;  // stream of the HCA layer
  void* hws = reinterpret_cast<char*>(ws) + sched.hca_off;
  if ((s = mark()) != HCA_OK) return s;
  if (sched.overlap) {
    CUDA_TRY(cudaEventRecord(side->fork, st), "decode: fork");
    CUDA_TRY(cudaStreamWaitEvent(side->s, side->fork, 0), "decode: fork wait");
  }
  // newest complete HCA block of every request -> its cache row.  All requests
  // share one position here (q_pos is on the device), so the row is hca_N - 1:
  // the caller passes caches sized to the complete blocks.
  char* wsb = reinterpret_cast<char*>(ws);
  const int c = cfg->c, H = cfg->n_heads, nw = cfg->n_win;
  auto run_hca_compress = [&]() -> int {
    if (a->hca_kv8) {
      // FP8 cache: the f32 entries (normalised to bf16 when asked), then their FP8 form in
      // row hca_N-1 of every request
      const hca_kv_fp8* d = a->hca_kv8;
      float* ef = reinterpret_cast<float*>(wsb + (a->hca_norm ? sched.hca_ef : sched.hca8_new));
      CUDA_TRY(launch_compress(reinterpret_cast<const bf16*>(a->hca_block_cand), c,
                               reinterpret_cast<const bf16*>(a->hca_block_logits), c, a->hca_pos_bias, c, a->B,
                               a->hca_block_stride, cfg->m_hca, c, cfg->m_hca, false, nullptr, c, c, hst, ef),
               "decode: hca compress");
      const void* src = ef;
      if (a->hca_norm) {
        CUDA_TRY(launch_norm_rope(norm_rows(cfg, ef, true, c, c, a->B, 1, nullptr, a->hca_N * cfg->m_hca - 1, 0,
                                            a->hca_norm + c, wsb + sched.hca8_new, c, c),
                                  hst),
                 "decode: hca entry normalisation");
        src = wsb + sched.hca8_new;
      }
      const long long r0 = a->hca_N - 1;
      CUDA_TRY(launch_kv_fp8_quantize(src, a->hca_norm == nullptr, c, a->B, c, cfg->rope_dims,
                                      d->codes + r0 * d->ld_codes, d->seq_rows * d->ld_codes,
                                      d->scales + r0 * d->ld_scales, d->seq_rows * d->ld_scales,
                                      reinterpret_cast<bf16*>(d->rope) + r0 * d->ld_rope, d->seq_rows * d->ld_rope,
                                      hst),
               "decode: hca entry to its FP8 form");
      return HCA_OK;
    }
    // flat: straight into row hca_N-1 of every request's cache; paged: into [B, c] in the
    // workspace, then each row to its pool row
    const bool pgd = a->block_table != nullptr;
    bf16* row = pgd ? reinterpret_cast<bf16*>(wsb + sched.hca_new)
                    : reinterpret_cast<bf16*>(a->hca_kv) + (long long)(a->hca_N - 1) * c;
    const long long row_stride = pgd ? (long long)c : a->hca_kv_stride;
    if (!a->hca_norm) {
      CUDA_TRY(launch_compress(reinterpret_cast<const bf16*>(a->hca_block_cand), c,
                               reinterpret_cast<const bf16*>(a->hca_block_logits), c, a->hca_pos_bias, c, a->B,
                               a->hca_block_stride, cfg->m_hca, c, cfg->m_hca, false, row, c, row_stride, hst),
               "decode: hca compress");
    } else {
      // f32 entries, then normalised and rotated at the entry's position into the cache row
      float* ef = reinterpret_cast<float*>(wsb + sched.hca_ef);
      CUDA_TRY(launch_compress(reinterpret_cast<const bf16*>(a->hca_block_cand), c,
                               reinterpret_cast<const bf16*>(a->hca_block_logits), c, a->hca_pos_bias, c, a->B,
                               a->hca_block_stride, cfg->m_hca, c, cfg->m_hca, false, nullptr, c, c, hst, ef),
               "decode: hca compress");
      CUDA_TRY(launch_norm_rope(norm_rows(cfg, ef, true, c, c, a->B, 1, nullptr, a->hca_N * cfg->m_hca - 1, 0,
                                          a->hca_norm + c, row, c, row_stride),
                                hst),
               "decode: hca entry normalisation");
    }
    if (pgd)
      CUDA_TRY(launch_scatter_rows(row, a->B, c, a->block_table, a->bt_stride, a->hca_N - 1, pg.rpb_hca,
                                   reinterpret_cast<bf16*>(a->hca_kv), hst),
               "decode: hca entry to its pool row");
    return HCA_OK;
  };
  // normalised queries and window blocks of a layer (window row w = token max(0, t-n_win+1) + w)
  auto normalise_layer = [&](const hca_bf16* q, const hca_bf16* win, long long win_stride, const float* norm,
                             size_t qn, size_t wn, cudaStream_t sm) -> int {
    CUDA_TRY(launch_norm_rope(norm_rows(cfg, q, false, c, (long long)H * c, a->B, H, a->q_pos, 0, 0, norm, wsb + qn,
                                        c, (long long)H * c),
                              sm),
             "decode: query normalisation");
    NormRope wr = norm_rows(cfg, win, false, c, win_stride, a->B, nw, a->q_pos, -(nw - 1), 1, norm + c, wsb + wn, c,
                            (long long)nw * c);
    wr.ring = a->block_table ? 1 : 0;  // paged: the window block is a ring of the last n_win tokens
    CUDA_TRY(launch_norm_rope(wr, sm), "decode: window normalisation");
    return HCA_OK;
  };
  auto run_hca_attention = [&]() -> int {
    MqaProblem p = decode_hca_problem(cfg, a);
    if (a->hca_kv8) {
      // the visible rows widened to bf16, read by the attention as its cache
      bf16* rows = reinterpret_cast<bf16*>(wsb + sched.hca8_rows);
      CUDA_TRY(launch_kv_fp8_gather(kv_fp8_of(a->hca_kv8), c, cfg->rope_dims, a->B, a->hca_N, nullptr, a->hca_N, rows,
                                    nullptr, hst),
               "decode: hca FP8 rows");
      p.kv = rows;
      p.kv_seq_stride = (long long)a->hca_N * c;
    }
    if (a->hca_norm) {
      int r = normalise_layer(a->hca_q, a->hca_win, a->hca_win_stride, a->hca_norm, sched.hca_qn, sched.hca_wn, hst);
      if (r != HCA_OK) return r;
      use_normalised(p, cfg, wsb + sched.hca_qn, wsb + sched.hca_wn, true);
    }
    CUDA_TRY(launch_mqa(p, sched.hca_pl, hws, hst), "decode: hca attention");
    return HCA_OK;
  };
  // Phase marks, in order: [hca compress] [indexer, top-k, csa attention] [hca attention].
  if (a->hca_q && sched.overlap) {
    // launched first so that its CTAs take their SMs before the indexer's persistent grid
    if (a->hca_block_cand && (s = run_hca_compress()) != HCA_OK) return s;
    if ((s = run_hca_attention()) != HCA_OK) return s;
    CUDA_TRY(cudaEventRecord(side->join, side->s), "decode: join");
    if (a->hca_block_cand && (s = mark()) != HCA_OK) return s;  // (the compression overlaps the rest)
  } else if (a->hca_q && a->hca_block_cand) {
    if ((s = run_hca_compress()) != HCA_OK) return s;
    if ((s = mark()) != HCA_OK) return s;
  }
  if (a->csa_q) {
    // (the normalisation runs before the indexer, outside the programmatic-launch chain
    // top-k -> attention, whose attention reads its queries before it waits)
    if (a->csa_norm) {
      s = normalise_layer(a->csa_q, a->csa_win, a->csa_win_stride, a->csa_norm, sched.csa_qn, sched.csa_wn, st);
      if (s != HCA_OK) return s;
    }
    Fp4Keys k4{a->csa_k_codes, a->csa_k_scales,
               a->B > 1 ? a->csa_k4_stride : ((long long)a->csa_N + 3) / 4 * 4,
               reinterpret_cast<bf16*>(wsb + sched.q4)};
    const PagedKeys pk{a->block_table, a->bt_stride, pg.rpb_csa, (long long)a->n_pool_blocks};
    s = run_indexer_topk(reinterpret_cast<const bf16*>(a->csa_q_idx), a->csa_w_idx,
                         reinterpret_cast<const bf16*>(a->csa_k_idx), a->csa_k_stride, a->csa_N, a->q_pos, a->B,
                         HCA_MODE_DECODE, cfg, a->csa_topk_idx, ws, st, ev, n_ev, ev_i,
                         sched.overlap ? sched.sms - sched.r_hca : 0, a->csa_k_codes ? &k4 : nullptr,
                         a->block_table ? &pk : nullptr);
    if (s != HCA_OK) return s;
    MqaProblem p = decode_csa_problem(cfg, a);
    if (a->csa_norm) use_normalised(p, cfg, wsb + sched.csa_qn, wsb + sched.csa_wn, true);
    if (a->csa_kv8) {
      // the selected rows widened to bf16 in slot order; the attention reads them as a
      // cache of k rows through the slot indices (empty slots stay -1)
      bf16* rows = reinterpret_cast<bf16*>(wsb + sched.csa8_rows);
      int32_t* slots = reinterpret_cast<int32_t*>(wsb + sched.csa8_idx);
      CUDA_TRY(launch_kv_fp8_gather(kv_fp8_of(a->csa_kv8), c, cfg->rope_dims, a->B, cfg->topk, a->csa_topk_idx,
                                    a->csa_N, rows, slots, st),
               "decode: csa FP8 rows");
      p.kv = rows;
      p.kv_seq_stride = (long long)cfg->topk * c;
      p.N = cfg->topk;
      p.idx = slots;
    }
    CUDA_TRY(launch_mqa(p, sched.csa_pl, ws, st, true), "decode: csa attention");
    if ((s = mark()) != HCA_OK) return s;
  }
  if (a->hca_q) {
    if (sched.overlap) {
      CUDA_TRY(cudaStreamWaitEvent(st, side->join, 0), "decode: join wait");
    } else if ((s = run_hca_attention()) != HCA_OK) {
      return s;
    }
    if ((s = mark()) != HCA_OK) return s;
  }
  g_last_launches = g_launch_counter;
  return HCA_OK;
}

// ---- prefill -----------------------------------------------------------------
// Workspace: indexer / attention scratch, then (with Q/KV normalisation) the
// normalised queries [T, H, c] and window rows [T, c] (bf16) and the f32
// entries [N, c] before theirs; the two layers reuse these in turn.
struct PrefillWs {
  size_t qn = 0, wn = 0, ef = 0, total = 0;
};
static PrefillWs prefill_ws_layout(const hca_layer_cfg* cfg, const hca_prefill_args* a) {
  const int T = a->T;
  const int Nc = T / cfg->m;
  size_t need = plan_indexer(cfg, T, Nc, HCA_MODE_PREFILL).bytes;
  MqaProblem p = make_mqa(cfg, nullptr, nullptr, 0, Nc, reinterpret_cast<const int32_t*>(1), cfg->topk, cfg->m,
                          nullptr, T, nullptr, T, HCA_MODE_PREFILL, nullptr, nullptr);
  need = std::max(need, plan_mqa(p).ws_bytes);
  if (a->hca_kv) {
    MqaProblem ph = make_mqa(cfg, nullptr, nullptr, 0, T / cfg->m_hca, nullptr, 0, cfg->m_hca, nullptr, T, nullptr, T,
                             HCA_MODE_PREFILL, nullptr, nullptr);
    need = std::max(need, plan_mqa(ph).ws_bytes);
  }
  PrefillWs w;
  w.total = round256(need);
  if (a->csa_norm || (a->hca_kv && a->hca_norm)) {
    w.qn = w.total;
    w.wn = w.qn + round256((size_t)T * cfg->n_heads * cfg->c * 2);
    w.ef = w.wn + round256((size_t)T * cfg->c * 2);
    const int Nh = a->hca_kv ? T / cfg->m_hca : 0;
    w.total = w.ef + round256((size_t)std::max(std::max(Nc, Nh), 1) * cfg->c * 4);
  }
  return w;
}
static size_t prefill_ws(const hca_layer_cfg* cfg, const hca_prefill_args* a) {
  return prefill_ws_layout(cfg, a).total;
}

size_t hybrid_attn_prefill_workspace(const hca_layer_cfg* cfg, const hca_prefill_args* a) {
  if (check_cfg(cfg) != HCA_OK || !a || a->T < 0) return (size_t)-1;
  if (indexer_ok(cfg, a->T / cfg->m, HCA_MODE_PREFILL) != HCA_OK) return (size_t)-1;
  return prefill_ws(cfg, a);
}

int hybrid_attn_prefill(const hca_layer_cfg* cfg, const hca_prefill_args* a, void* ws, size_t ws_bytes, void* stream) {
  HCA_RANGE("hybrid_attn_prefill");
  g_err.clear();
  int s = check_cfg(cfg);
  if (s != HCA_OK) return s;
  CHECK(a != nullptr, HCA_ERR_INVALID_ARG, "hybrid_attn_prefill: args null");
  CHECK(a->T >= 0, HCA_ERR_INVALID_ARG, "hybrid_attn_prefill: T=%d", a->T);
  CHECK(a->n_events >= 0, HCA_ERR_INVALID_ARG, "hybrid_attn_prefill: n_events");
  const int T = a->T;
  if (T == 0) return HCA_OK;
  const int Nc = T / cfg->m;
  s = indexer_ok(cfg, Nc, HCA_MODE_PREFILL);
  if (s != HCA_OK) return s;
  CHECK_PTR(a->q_pos, "hybrid_attn_prefill: q_pos");
  CHECK_PTR(a->cand, "hybrid_attn_prefill: cand");
  CHECK_PTR(a->logits, "hybrid_attn_prefill: logits");
  CHECK_PTR(a->kidx_cand, "hybrid_attn_prefill: kidx_cand");
  CHECK_PTR(a->bias_csa, "hybrid_attn_prefill: bias_csa");
  CHECK_PTR(a->q_idx, "hybrid_attn_prefill: q_idx");
  CHECK_PTR(a->w_idx, "hybrid_attn_prefill: w_idx");
  CHECK_PTR(a->q, "hybrid_attn_prefill: q");
  CHECK_PTR(a->topk_idx, "hybrid_attn_prefill: topk_idx");
  CHECK_PTR(a->csa_out, "hybrid_attn_prefill: csa_out");
  if (Nc > 0) {
    CHECK_PTR(a->csa_kv, "hybrid_attn_prefill: csa_kv");
    CHECK_PTR(a->csa_k_idx, "hybrid_attn_prefill: csa_k_idx");
  }
  if (a->hca_kv) {
    CHECK_PTR(a->bias_hca, "hybrid_attn_prefill: bias_hca");
    CHECK_PTR(a->hca_q, "hybrid_attn_prefill: hca_q");
    CHECK_PTR(a->hca_out, "hybrid_attn_prefill: hca_out");
    if (a->hca_norm) CHECK_PTR(a->hca_norm, "hybrid_attn_prefill: hca_norm");
  }
  if (a->csa_norm) CHECK_PTR(a->csa_norm, "hybrid_attn_prefill: csa_norm");
  const size_t need = prefill_ws(cfg, a);
  CHECK(ws_bytes >= need, HCA_ERR_WORKSPACE, "hybrid_attn_prefill: workspace %zu < %zu", ws_bytes, need);
  if (need) CHECK(ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0, HCA_ERR_INVALID_ARG,
                  "hybrid_attn_prefill: ws null or not 256-byte aligned");
  if (injected("hybrid_attn_prefill")) return fail(HCA_ERR_INJECTED, "hybrid_attn_prefill: injected");

  cudaStream_t st = as_stream(stream);
  g_launch_counter = 0;
  g_last_launches = 0;
  int ev_i = 0;
  void* const* ev = a->events;
  const int n_ev = ev ? a->n_events : 0;
  auto mark = [&]() -> int {
    if (ev && ev_i < n_ev) return cuda_status(cudaEventRecord((cudaEvent_t)ev[ev_i++], st), "event");
    return HCA_OK;
  };
  const int c = cfg->c, dI = cfg->d_idx, H = cfg->n_heads;
  const PrefillWs wl = prefill_ws_layout(cfg, a);
  char* wsb = reinterpret_cast<char*>(ws);
  float* ef = reinterpret_cast<float*>(wsb + wl.ef);
  // entries of one layer: f32 from the compressor, normalised and rotated at
  // (i+1)*rate - 1 into the cache (with normalisation), else bf16 directly
  auto compress_entries = [&](const float* bias, int rate, bool overlap, hca_bf16* kv, const float* norm,
                              const char* what) -> int {
    if (!norm) {
      CUDA_TRY(launch_compress(reinterpret_cast<const bf16*>(a->cand), c, reinterpret_cast<const bf16*>(a->logits), c,
                               bias, c, 1, 0, T, c, rate, overlap, reinterpret_cast<bf16*>(kv), c, 0, st),
               what);
      return HCA_OK;
    }
    CUDA_TRY(launch_compress(reinterpret_cast<const bf16*>(a->cand), c, reinterpret_cast<const bf16*>(a->logits), c,
                             bias, c, 1, 0, T, c, rate, overlap, nullptr, c, 0, st, ef),
             what);
    CUDA_TRY(launch_norm_rope(norm_rows(cfg, ef, true, c, 0, 1, T / rate, nullptr, rate - 1, rate, norm + c, kv, c, 0),
                              st),
             "prefill: entry normalisation");
    return HCA_OK;
  };
  // normalised queries [T, H, c] and window rows [T, c] (row r = token r) of a layer
  auto normalise_layer = [&](const hca_bf16* q, const float* norm) -> int {
    CUDA_TRY(launch_norm_rope(norm_rows(cfg, q, false, c, (long long)H * c, T, H, a->q_pos, 0, 0, norm, wsb + wl.qn, c,
                                        (long long)H * c),
                              st),
             "prefill: query normalisation");
    CUDA_TRY(launch_norm_rope(norm_rows(cfg, a->cand, false, c, 0, 1, T, nullptr, 0, 1, norm + c, wsb + wl.wn, c, 0),
                              st),
             "prefill: window normalisation");
    return HCA_OK;
  };
  if ((s = mark()) != HCA_OK) return s;
  // CSA compression of KV entries and of indexer keys (logits/bias: first d_I channels)
  if ((s = compress_entries(a->bias_csa, cfg->m, true, a->csa_kv, a->csa_norm, "prefill: csa compress")) != HCA_OK)
    return s;
  CUDA_TRY(launch_compress(reinterpret_cast<const bf16*>(a->kidx_cand), dI, reinterpret_cast<const bf16*>(a->logits),
                           c, a->bias_csa, c, 1, 0, T, dI, cfg->m, true, reinterpret_cast<bf16*>(a->csa_k_idx), dI, 0,
                           st),
           "prefill: indexer-key compress");
  // (before the indexer: outside the programmatic-launch chain top-k -> attention)
  if (a->csa_norm && (s = normalise_layer(a->q, a->csa_norm)) != HCA_OK) return s;
  if ((s = mark()) != HCA_OK) return s;
  s = run_indexer_topk(reinterpret_cast<const bf16*>(a->q_idx), a->w_idx, reinterpret_cast<const bf16*>(a->csa_k_idx),
                       0, Nc, a->q_pos, T, HCA_MODE_PREFILL, cfg, a->topk_idx, ws, st, ev, n_ev, ev_i);
  if (s != HCA_OK) return s;
  {
    MqaProblem p = make_mqa(cfg, a->q, a->csa_kv, 0, Nc, a->topk_idx, cfg->topk, cfg->m, a->cand, T, a->q_pos, T,
                            HCA_MODE_PREFILL, a->csa_out, a->csa_sink);
    if (a->csa_norm) use_normalised(p, cfg, wsb + wl.qn, wsb + wl.wn, false);
    CUDA_TRY(launch_mqa(p, plan_mqa(p), ws, st, true), "prefill: csa attention");
    if ((s = mark()) != HCA_OK) return s;
  }
  if (a->hca_kv) {
    const int Nh = T / cfg->m_hca;
    if ((s = compress_entries(a->bias_hca, cfg->m_hca, false, a->hca_kv, a->hca_norm, "prefill: hca compress")) !=
        HCA_OK)
      return s;
    MqaProblem p = make_mqa(cfg, a->hca_q, a->hca_kv, 0, Nh, nullptr, 0, cfg->m_hca, a->cand, T, a->q_pos, T,
                            HCA_MODE_PREFILL, a->hca_out, a->hca_sink);
    if (a->hca_norm) {
      // (the CSA layer's normalised rows are consumed: this stream ran its attention)
      if ((s = normalise_layer(a->hca_q, a->hca_norm)) != HCA_OK) return s;
      use_normalised(p, cfg, wsb + wl.qn, wsb + wl.wn, false);
    }
    CUDA_TRY(launch_mqa(p, plan_mqa(p), ws, st), "prefill: hca attention");
    if ((s = mark()) != HCA_OK) return s;
  }
  g_last_launches = g_launch_counter;
  return HCA_OK;
}

// ---- FP4 indexer variant -----------------------------------------------------------
int mxfp4_quantize(const void* x, int x_is_f32, long long ld_x, int rows, int d, uint8_t* codes, long long ld_codes,
                   uint8_t* scales, long long ld_scales, void* stream) {
  HCA_RANGE("mxfp4_quantize");
  g_err.clear();
  CHECK(rows >= 0 && d > 0 && d % 32 == 0, HCA_ERR_INVALID_ARG, "mxfp4_quantize: rows=%d d=%d (d a multiple of 32)",
        rows, d);
  CHECK(ld_x >= d && ld_codes >= d / 2 && ld_scales >= d / 32, HCA_ERR_INVALID_ARG, "mxfp4_quantize: row strides");
  CHECK(ld_codes % 16 == 0, HCA_ERR_INVALID_ARG, "mxfp4_quantize: ld_codes %lld not a multiple of 16", ld_codes);
  if (rows == 0) return HCA_OK;
  CHECK(x != nullptr && codes != nullptr && scales != nullptr, HCA_ERR_INVALID_ARG, "mxfp4_quantize: null pointer");
  CHECK(aligned16(codes), HCA_ERR_INVALID_ARG, "mxfp4_quantize: codes not 16-byte aligned");
  CHECK(((reinterpret_cast<uintptr_t>(x)) & (x_is_f32 ? 3u : 1u)) == 0, HCA_ERR_INVALID_ARG,
        "mxfp4_quantize: x misaligned");
  if (injected("mxfp4_quantize")) return fail(HCA_ERR_INJECTED, "mxfp4_quantize: injected");
  CUDA_TRY(launch_mxfp4_quantize(x, x_is_f32 != 0, ld_x, rows, d, codes, ld_codes, scales, ld_scales,
                                 as_stream(stream)),
           "mxfp4_quantize");
  return HCA_OK;
}

static size_t fp4_indexer_ws(const hca_layer_cfg* cfg, int B, int N) {
  const IndexerPlan p = plan_indexer(cfg, B, N, HCA_MODE_DECODE);
  return round256(p.bytes) + round256((size_t)B * cfg->n_idx_heads * cfg->d_idx * 2);
}

size_t csa_indexer_topk_fp4_workspace(const hca_layer_cfg* cfg, int B, int N) {
  if (check_cfg(cfg) != HCA_OK || B < 0 || N < 0) return (size_t)-1;
  if (indexer_ok(cfg, N, HCA_MODE_DECODE) != HCA_OK) return (size_t)-1;
  return fp4_indexer_ws(cfg, B, N);
}

int csa_indexer_topk_fp4(const hca_bf16* q_idx, const float* w_idx, const uint8_t* k_codes, const uint8_t* k_scales,
                         long long k_seq_stride, int N, const int32_t* q_pos, int B, const hca_layer_cfg* cfg,
                         int32_t* topk_idx, void* ws, size_t ws_bytes, void* stream) {
  HCA_RANGE("csa_indexer_topk_fp4");
  g_err.clear();
  int s = check_cfg(cfg);
  if (s != HCA_OK) return s;
  CHECK(indexer_tc_supported(cfg->n_idx_heads, cfg->d_idx), HCA_ERR_UNSUPPORTED,
        "csa_indexer_topk_fp4: the FP4 indexer takes 64 heads x 128 (got %d x %d)", cfg->n_idx_heads, cfg->d_idx);
  CHECK(B >= 0 && B <= 65535 && N > 0, HCA_ERR_INVALID_ARG, "csa_indexer_topk_fp4: B=%d N=%d", B, N);
  s = indexer_ok(cfg, N, HCA_MODE_DECODE);
  if (s != HCA_OK) return s;
  const long long n4 = ((long long)N + 3) / 4 * 4;
  CHECK(B <= 1 || (k_seq_stride >= n4 && k_seq_stride % 4 == 0), HCA_ERR_INVALID_ARG,
        "csa_indexer_topk_fp4: k_seq_stride %lld (need >= %lld keys, a multiple of 4)", k_seq_stride, n4);
  const size_t need = fp4_indexer_ws(cfg, B, N);
  CHECK(ws_bytes >= need, HCA_ERR_WORKSPACE, "csa_indexer_topk_fp4: workspace %zu < %zu", ws_bytes, need);
  if (B == 0) return HCA_OK;
  CHECK_PTR(q_idx, "csa_indexer_topk_fp4: q_idx");
  CHECK_PTR(w_idx, "csa_indexer_topk_fp4: w_idx");
  CHECK_PTR(k_codes, "csa_indexer_topk_fp4: k_codes");
  CHECK_PTR(k_scales, "csa_indexer_topk_fp4: k_scales");
  CHECK_PTR(topk_idx, "csa_indexer_topk_fp4: topk_idx");
  CHECK(q_pos != nullptr, HCA_ERR_INVALID_ARG, "csa_indexer_topk_fp4: q_pos null");
  CHECK(ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0, HCA_ERR_INVALID_ARG,
        "csa_indexer_topk_fp4: ws null or not 256-byte aligned");
  if (injected("csa_indexer_topk_fp4")) return fail(HCA_ERR_INJECTED, "csa_indexer_topk_fp4: injected");

  const IndexerPlan p = plan_indexer(cfg, B, N, HCA_MODE_DECODE);
  Fp4Keys k4{k_codes, k_scales, B > 1 ? k_seq_stride : (long long)(N + 3) / 4 * 4,
             reinterpret_cast<bf16*>(reinterpret_cast<char*>(ws) + round256(p.bytes))};
  int ev_i = 0;
  return run_indexer_topk(reinterpret_cast<const bf16*>(q_idx), w_idx, nullptr, 0, N, q_pos, B, HCA_MODE_DECODE,
                          cfg, topk_idx, ws, as_stream(stream), nullptr, 0, ev_i, 0, &k4);
}

}  // extern "C"
