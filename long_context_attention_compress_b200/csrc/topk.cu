// Exact per-row top-k selection by MSB-first radix select (sm_100a).
//
// Selection rule (the lightning-indexer top-k of the QbitAI write-up, CSA
// step two, and "DeepSeek V4 Architecture Tricks", CSA section): the k
// entries with the largest scores, ties broken towards the lower entry
// index; all candidates when there are at most k.  Each candidate is a
// 64-bit composite (order-preserving score key, bit-inverted index), so the
// k largest composites are exactly that set and the k-th largest is unique.
//
// One CTA per row.  The row's candidates (<= kSelectMaxN) are staged in
// shared memory once; eight 8-bit histogram passes (with early exit as soon
// as the threshold bucket holds exactly the remaining count) find the
// threshold; a block-wide scan writes the selected set in candidate order,
// so the output is deterministic.

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hca {

constexpr int kSelThreads = 1024;
__device__ unsigned int g_select_error = 0;

// Block-wide exclusive scan of two counters (NT threads, NT % 32 == 0).
template <int NT>
__device__ __forceinline__ void block_scan2(int a, int b, int& ea, int& eb, int& ta, int& tb, int2* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int va = __shfl_up_sync(0xffffffffu, ia, off);
    int vb = __shfl_up_sync(0xffffffffu, ib, off);
    if (lane >= off) { ia += va; ib += vb; }
  }
  if (lane == 31) s_warp[warp] = make_int2(ia, ib);
  __syncthreads();
  if (warp == 0) {
    int2 v = lane < NT / 32 ? s_warp[lane] : make_int2(0, 0);
    int xa = v.x, xb = v.y;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int va = __shfl_up_sync(0xffffffffu, xa, off);
      int vb = __shfl_up_sync(0xffffffffu, xb, off);
      if (lane >= off) { xa += va; xb += vb; }
    }
    if (lane < NT / 32) s_warp[lane] = make_int2(xa - v.x, xb - v.y);  // exclusive warp offsets
    if (lane == NT / 32 - 1) s_warp[NT / 32] = make_int2(xa, xb);        // totals
  }
  __syncthreads();
  ea = s_warp[warp].x + ia - a;
  eb = s_warp[warp].y + ib - b;
  ta = s_warp[NT / 32].x;
  tb = s_warp[NT / 32].y;
  __syncthreads();
}

// Core: select the top-k of s_c[0..n) (shared memory) and write them.
//
// MSB-first radix select over the 64-bit composites with 8-bit digits,
// starting at the highest bit where the candidates differ (bits above it are
// common to all and need no pass), so the first digit already spreads
// concentrated score distributions over many bins; the threshold bucket is
// found with a warp-shuffle suffix scan.
template <int NT>
__device__ void select_core(const uint64_t* s_c, int n, int k, int32_t* out_idx, uint64_t* out_cand) {
  __shared__ int s_hist[256];
  __shared__ int s_wsum[8];
  __shared__ int s_bucket, s_greater;
  __shared__ unsigned long long s_min, s_max;
  __shared__ int2 s_warp[NT / 32 + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (n <= k) {
    for (int e = tid; e < k; e += NT) {
      uint64_t c = e < n ? s_c[e] : 0ull;
      if (out_idx) out_idx[e] = e < n ? cand_index(c) : -1;
      else out_cand[e] = c;
    }
    return;
  }

  // range of the composites -> highest differing bit
  unsigned long long mn = ~0ull, mx = 0ull;
  for (int e = tid; e < n; e += NT) {
    const unsigned long long c = s_c[e];
    mn = c < mn ? c : mn;
    mx = c > mx ? c : mx;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, mn, o);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, mx, o);
    mn = a < mn ? a : mn;
    mx = b > mx ? b : mx;
  }
  if (tid == 0) { s_min = ~0ull; s_max = 0ull; }
  __syncthreads();
  if (lane == 0) { atomicMin(&s_min, mn); atomicMax(&s_max, mx); }
  __syncthreads();
  const unsigned long long cmin = s_min, cmax = s_max;
  // n > k >= 1 distinct composites except for empty slots: cmin < cmax unless
  // all are empty (then every slot is equal and any k of them will do)
  int hi = cmin == cmax ? -1 : 63 - __clzll((long long)(cmin ^ cmax));
  uint64_t prefix = hi >= 63 ? 0ull : (cmin >> (hi + 1)) << (hi + 1);
  int lo = hi + 1;  // lowest bit decided so far
  int remaining = k;
  while (hi >= 0) {
    lo = hi >= 7 ? hi - 7 : 0;
    const int width = hi - lo + 1;
    const uint32_t dmask = (1u << width) - 1u;
    for (int b = tid; b < 256; b += NT) s_hist[b] = 0;
    __syncthreads();
    for (int e = tid; e < n; e += NT) {
      const uint64_t c = s_c[e];
      if (hi >= 63 || (c >> (hi + 1)) == (prefix >> (hi + 1))) atomicAdd(&s_hist[(int)((c >> lo) & dmask)], 1);
    }
    __syncthreads();
    // suffix sums over the 256 bins: warps 0..7 hold 32 bins each
    if (tid < 256) {
      const int v = s_hist[tid];
      int suf = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
      }
      if (lane == 0) s_wsum[warp] = suf;
      // publish after every warp wrote its total
      asm volatile("bar.sync 3, 256;" ::: "memory");
      int above = 0;
      for (int w = warp + 1; w < 8; ++w) above += s_wsum[w];
      suf += above;
      const int nxt = suf - v;  // suffix of bin tid + 1
      if (suf >= remaining && nxt < remaining) { s_bucket = tid; s_greater = nxt; }
    }
    __syncthreads();
    const int b = s_bucket;
    remaining -= s_greater;
    prefix |= (uint64_t)b << lo;
    const int cnt = s_hist[b];
    __syncthreads();
    hi = lo - 1;
    if (cnt == remaining) break;
  }
  const int shift = lo;

  // Output in candidate order: all above the threshold prefix, then the first
  // `remaining` equal to it (only duplicates -- empty slots -- can tie here).
  // Warp w owns the contiguous range [w*seg, (w+1)*seg); lanes read it 32
  // consecutive candidates at a time (no bank conflicts), ranks come from
  // ballots, warp offsets from a scan of the 32 warp totals.
  const uint64_t P = prefix >> shift;
  constexpr int NW = NT / 32;
  const int seg = ((n + NW - 1) / NW + 31) / 32 * 32;
  const int w0 = warp * seg, w1 = min(n, w0 + seg);
  const unsigned lt = (1u << lane) - 1u;
  int ng = 0, ne = 0;
  for (int e = w0 + lane; e - lane < w1; e += 32) {
    const uint64_t v = e < w1 ? (s_c[e] >> shift) : 0ull;
    ng += __popc(__ballot_sync(0xffffffffu, e < w1 && v > P));
    ne += __popc(__ballot_sync(0xffffffffu, e < w1 && v == P));
  }
  int og, oe, tg, te;
  // one thread per warp carries the warp's totals into the block scan
  block_scan2<NT>(lane == 0 ? ng : 0, lane == 0 ? ne : 0, og, oe, tg, te, s_warp);
  og = __shfl_sync(0xffffffffu, og, 0);
  oe = __shfl_sync(0xffffffffu, oe, 0);
  for (int e = w0 + lane; e - lane < w1; e += 32) {
    const bool in = e < w1;
    const uint64_t c = in ? s_c[e] : 0ull;
    const uint64_t v = c >> shift;
    const bool g = in && v > P, q = in && v == P;
    const unsigned bg = __ballot_sync(0xffffffffu, g), bq = __ballot_sync(0xffffffffu, q);
    int slot = -1;
    if (g) slot = og + __popc(bg & lt);
    if (q) {
      const int r = oe + __popc(bq & lt);
      if (r < remaining) slot = tg + r;
    }
    if (slot >= 0) {
      if (out_idx) out_idx[slot] = cand_index(c);
      else out_cand[slot] = c;
    }
    og += __popc(bg);
    oe += __popc(bq);
  }
}

// The same selection over 32-bit score keys staged in index order (the index is
// the position): half the shared memory and at most four 8-bit passes.  Equal
// keys keep index order, so ties still go to the lower index.
template <int NT>
__device__ void select_core32(const uint32_t* s_c, int n, int k, int idx_base, int32_t* out_idx) {
  __shared__ int s_hist[256];
  __shared__ int s_wsum[8];
  __shared__ int s_bucket, s_greater;
  __shared__ unsigned int s_min, s_max;
  __shared__ int2 s_warp[NT / 32 + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (n <= k) {
    for (int e = tid; e < k; e += NT) out_idx[e] = e < n ? idx_base + e : -1;
    return;
  }

  // range of the composites -> highest differing bit
  unsigned int mn = ~0u, mx = 0u;
  for (int e = tid; e < n; e += NT) {
    const unsigned int c = s_c[e];
    mn = c < mn ? c : mn;
    mx = c > mx ? c : mx;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned int a = __shfl_xor_sync(0xffffffffu, mn, o);
    const unsigned int b = __shfl_xor_sync(0xffffffffu, mx, o);
    mn = a < mn ? a : mn;
    mx = b > mx ? b : mx;
  }
  if (tid == 0) { s_min = ~0u; s_max = 0u; }
  __syncthreads();
  if (lane == 0) { atomicMin(&s_min, mn); atomicMax(&s_max, mx); }
  __syncthreads();
  const unsigned int cmin = s_min, cmax = s_max;
  // n > k >= 1 distinct composites except for empty slots: cmin < cmax unless
  // all are empty (then every slot is equal and any k of them will do)
  int hi = cmin == cmax ? -1 : 31 - __clz((int)(cmin ^ cmax));
  uint32_t prefix = hi >= 31 ? 0u : (cmin >> (hi + 1)) << (hi + 1);
  int lo = hi + 1;  // lowest bit decided so far
  int remaining = k;
  while (hi >= 0) {
    lo = hi >= 7 ? hi - 7 : 0;
    const int width = hi - lo + 1;
    const uint32_t dmask = (1u << width) - 1u;
    for (int b = tid; b < 256; b += NT) s_hist[b] = 0;
    __syncthreads();
    for (int e = tid; e < n; e += NT) {
      const uint32_t c = s_c[e];
      if (hi >= 31 || (c >> (hi + 1)) == (prefix >> (hi + 1))) atomicAdd(&s_hist[(int)((c >> lo) & dmask)], 1);
    }
    __syncthreads();
    // suffix sums over the 256 bins: warps 0..7 hold 32 bins each
    if (tid < 256) {
      const int v = s_hist[tid];
      int suf = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
      }
      if (lane == 0) s_wsum[warp] = suf;
      // publish after every warp wrote its total
      asm volatile("bar.sync 3, 256;" ::: "memory");
      int above = 0;
      for (int w = warp + 1; w < 8; ++w) above += s_wsum[w];
      suf += above;
      const int nxt = suf - v;  // suffix of bin tid + 1
      if (suf >= remaining && nxt < remaining) { s_bucket = tid; s_greater = nxt; }
    }
    __syncthreads();
    const int b = s_bucket;
    remaining -= s_greater;
    prefix |= (uint32_t)b << lo;
    const int cnt = s_hist[b];
    __syncthreads();
    hi = lo - 1;
    if (cnt == remaining) break;
  }
  const int shift = lo;

  // Output in candidate order: all above the threshold prefix, then the first
  // `remaining` equal to it (only duplicates -- empty slots -- can tie here).
  // Warp w owns the contiguous range [w*seg, (w+1)*seg); lanes read it 32
  // consecutive candidates at a time (no bank conflicts), ranks come from
  // ballots, warp offsets from a scan of the 32 warp totals.
  const uint32_t P = prefix >> shift;
  constexpr int NW = NT / 32;
  const int seg = ((n + NW - 1) / NW + 31) / 32 * 32;
  const int w0 = warp * seg, w1 = min(n, w0 + seg);
  const unsigned lt = (1u << lane) - 1u;
  int ng = 0, ne = 0;
  for (int e = w0 + lane; e - lane < w1; e += 32) {
    const uint32_t v = e < w1 ? (s_c[e] >> shift) : 0u;
    ng += __popc(__ballot_sync(0xffffffffu, e < w1 && v > P));
    ne += __popc(__ballot_sync(0xffffffffu, e < w1 && v == P));
  }
  int og, oe, tg, te;
  // one thread per warp carries the warp's totals into the block scan
  block_scan2<NT>(lane == 0 ? ng : 0, lane == 0 ? ne : 0, og, oe, tg, te, s_warp);
  og = __shfl_sync(0xffffffffu, og, 0);
  oe = __shfl_sync(0xffffffffu, oe, 0);
  for (int e = w0 + lane; e - lane < w1; e += 32) {
    const bool in = e < w1;
    const uint32_t v = in ? (s_c[e] >> shift) : 0u;
    const bool g = in && v > P, q = in && v == P;
    const unsigned bg = __ballot_sync(0xffffffffu, g), bq = __ballot_sync(0xffffffffu, q);
    int slot = -1;
    if (g) slot = og + __popc(bg & lt);
    if (q) {
      const int r = oe + __popc(bq & lt);
      if (r < remaining) slot = tg + r;
    }
    if (slot >= 0) out_idx[slot] = idx_base + e;
    og += __popc(bg);
    oe += __popc(bq);
  }
}

__global__ void __launch_bounds__(kSelThreads) select_scores_kernel(const float* __restrict__ scores,
                                                                    SelectRows rows, int k,
                                                                    int32_t* out_idx, uint64_t* out_cand) {
  extern __shared__ uint64_t s_c[];
  tc::griddep_launch_dependents();
  tc::griddep_wait();  // the scores come from the previous kernel
  const int r = blockIdx.x;
  const int q = r / rows.chunks;
  const int j = r % rows.chunks;
  const int nvis = n_visible(rows.q_pos[q], rows.rate, rows.N);
  const int start = j * rows.chunk;
  int n = nvis - start;
  n = n < 0 ? 0 : (n > rows.chunk ? rows.chunk : n);
  const float* sp = scores + (long long)q * rows.ld_scores + start;
  // 8 independent loads in flight per thread before the shared-memory stores
  for (int b0 = 0; b0 < n; b0 += 8 * kSelThreads) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = b0 + u * kSelThreads + (int)threadIdx.x;
      v[u] = e < n ? sp[e] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = b0 + u * kSelThreads + (int)threadIdx.x;
      if (e < n) s_c[e] = make_cand(v[u], start + e);
    }
  }
  __syncthreads();
  select_core<kSelThreads>(s_c, n, k, out_idx ? out_idx + (long long)r * k : nullptr,
                           out_cand ? out_cand + (long long)r * k : nullptr);
}

// One row per CTA with at most kSelectRowMaxN visible entries: stage the score
// keys, select, write the final indices.
__global__ void __launch_bounds__(kSelThreads) select_row_kernel(const float* __restrict__ scores, SelectRows rows,
                                                                 int k, int32_t* out_idx) {
  extern __shared__ uint32_t s_k[];
  tc::griddep_launch_dependents();
  tc::griddep_wait();  // the scores come from the previous kernel
  const int q = blockIdx.x;
  const int n = n_visible(rows.q_pos[q], rows.rate, rows.N);
  const float* sp = scores + (long long)q * rows.ld_scores;
  // 8 independent loads in flight per thread before the shared-memory stores
  for (int b0 = 0; b0 < n; b0 += 8 * kSelThreads) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = b0 + u * kSelThreads + (int)threadIdx.x;
      v[u] = e < n ? sp[e] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = b0 + u * kSelThreads + (int)threadIdx.x;
      if (e < n) s_k[e] = float_key(v[u]);
    }
  }
  __syncthreads();
  select_core32<kSelThreads>(s_k, n, k, 0, out_idx + (long long)q * k);
}

__global__ void __launch_bounds__(kSelThreads) select_merge_kernel(const uint64_t* __restrict__ cand, int n_cand,
                                                                   int k, int32_t* out_idx) {
  extern __shared__ uint64_t s_c[];
  tc::griddep_launch_dependents();
  tc::griddep_wait();  // the candidates come from the previous kernel
  const int r = blockIdx.x;
  const uint64_t* cp = cand + (long long)r * n_cand;
  for (int b0 = 0; b0 < n_cand; b0 += 8 * kSelThreads) {
    uint64_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = b0 + u * kSelThreads + (int)threadIdx.x;
      v[u] = e < n_cand ? cp[e] : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = b0 + u * kSelThreads + (int)threadIdx.x;
      if (e < n_cand) s_c[e] = v[u];
    }
  }
  __syncthreads();
  const int n = n_cand;  // empty slots are zero composites and lose to any real candidate
  select_core<kSelThreads>(s_c, n, k, out_idx + (long long)r * k, nullptr);
}

// ---- decode: threshold select from a per-request score histogram ------------------
// The indexer counts each request's visible scores into 4096 bins of the top 12
// bits of their order-preserving key.  Bin T holding the k-th largest score splits
// every entry into three classes: above T (always selected), in T (candidates for
// the remaining k - above places) and below (never).  C CTAs per request scan
// slices of the scores and compact both classes in entry order; the last CTA to
// finish concatenates the "above" lists in slice order and runs the exact radix
// select over the bin-T candidates only.  The output is deterministic: the
// entries above T in index order, then the chosen bin-T entries in index order.
// Threshold over a 4096-bin histogram read from global memory: the bin holding the
// `k`-th largest entry, and the number of entries in higher bins.  All NT threads.
// The thread's four bins, as hist_threshold_from takes them.
template <int NT>
__device__ __forceinline__ int4 hist_bins(const int* h) {
  static_assert(NT * 4 == kHistBins, "four bins per thread");
  return __ldcg(reinterpret_cast<const int4*>(h + kHistBins - 4 * (threadIdx.x + 1)));
}
// (h4: this thread's bins, loaded by hist_bins)
template <int NT>
__device__ void hist_threshold_from(int4 h4, int k, int* s_bin, int* s_higher, int2* s_warp) {
  static_assert(NT * 4 == kHistBins, "four bins per thread");
  const int tid = threadIdx.x;
  if (tid == 0) { *s_bin = -1; *s_higher = 0; }
  const int hv[4] = {h4.w, h4.z, h4.y, h4.x};  // bins 4095 - 4t, 4094 - 4t, ...
  int ex, dummy, tot, tdummy;
  block_scan2<NT>(hv[0] + hv[1] + hv[2] + hv[3], 0, ex, dummy, tot, tdummy, s_warp);
  int run = ex;  // entries in higher bins
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    if (run < k && run + hv[u] >= k) { *s_bin = kHistBins - 1 - (4 * tid + u); *s_higher = run; }
    run += hv[u];
  }
  __syncthreads();
}
template <int NT>
__device__ void hist_threshold(const int* h, int k, int* s_bin, int* s_higher, int2* s_warp) {
  hist_threshold_from<NT>(hist_bins<NT>(h), k, s_bin, s_higher, s_warp);
}

// Largest j in [0, n) with off[j] <= i, for off[0] <= i < off[n] (a prefix sum:
// the list of a concatenation that holds element i, skipping empty lists).
__device__ __forceinline__ int list_of(const int* off, int stride, int n, int i) {
  int lo = 0, hi = n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid * stride] <= i) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kSelThreads) select_hist_kernel(HistSelect a) {
  extern __shared__ uint64_t s_c[];
  __shared__ int2 s_warp[kSelThreads / 32 + 1];
  __shared__ int s_T, s_above, s_T2, s_above2, s_last;
  __shared__ int2 s_cnt[kHistMaxCtas];
  __shared__ int2 s_off[kHistMaxCtas + 1];
  __shared__ uint64_t s_tie[32];
  tc::griddep_launch_dependents();
  tc::griddep_wait();  // scores and histograms come from the indexer
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = blockIdx.x / a.C, c = blockIdx.x % a.C;
  const int k = a.k;
  const int nvis = n_visible(a.q_pos[r], a.rate, a.N);
  int32_t* out = a.out + (long long)r * k;
  if (nvis <= k) {  // every visible entry (no histogram needed)
    if (c == 0)
      for (int e = tid; e < k; e += kSelThreads) out[e] = e < nvis ? e : -1;
    return;
  }
  // this CTA's slice, thread t owning 16 consecutive entries: loads issued first,
  // so their latency overlaps the threshold search
  const int e0 = c * a.slice + 16 * tid;
  const float* sp = a.scores + (long long)r * a.ld;
  float v[16];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int e = e0 + 4 * u;
    const float4 f = (e + 3 < nvis) ? __ldcg(reinterpret_cast<const float4*>(sp + e))
                                    : make_float4(e < nvis ? sp[e] : 0.f, e + 1 < nvis ? sp[e + 1] : 0.f,
                                                  e + 2 < nvis ? sp[e + 2] : 0.f, 0.f);
    v[4 * u] = f.x; v[4 * u + 1] = f.y; v[4 * u + 2] = f.z; v[4 * u + 3] = f.w;
  }
  // level 1: bin of the top 12 key bits holding the k-th largest score
  hist_threshold<kSelThreads>(a.hist + (long long)r * kHistBins, k, &s_T, &s_above, s_warp);
  if (s_T < 0) {  // fewer counted entries than visible ones: the histogram is not this call's
    if (tid == 0) atomicOr(&g_select_error, 1u);
    return;
  }
  const uint32_t T = (uint32_t)s_T;
  const int above_total = s_above;
  int* hist2 = a.hist + (long long)(a.B + r) * kHistBins;  // level-2 histograms follow the B level-1 ones
  int na = 0, ne = 0;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    if (e0 + u < nvis) {
      const uint32_t key = float_key(v[u]);
      na += (key >> 20) > T;
      if ((key >> 20) == T) {
        ++ne;
        atomicAdd(hist2 + ((key >> 8) & (kHistBins - 1)), 1);  // level 2: the next 12 key bits
      }
    }
  }
  int oa, oe, ta, te;
  block_scan2<kSelThreads>(na, ne, oa, oe, ta, te, s_warp);
  int32_t* above = a.above + ((long long)r * a.C + c) * k;
  uint64_t* eq = a.eq + ((long long)r * a.C + c) * a.slice;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int e = e0 + u;
    if (e < nvis) {
      const uint32_t b = float_key(v[u]) >> 20;
      // (a CTA never holds more than k - 1 entries above T; the bound only guards the
      // region if the histogram were not this call's -- the merge then reports it)
      if (b > T) { if (oa < k) above[oa] = e; ++oa; }
      else if (b == T) eq[oe++] = make_cand(v[u], e);
    }
  }
  // the last CTA of the request to finish merges
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    a.cnt[(long long)r * a.C + c] = make_int2(ta, te);
    __threadfence();
    s_last = atomicAdd(a.done + r, 1) == a.C - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // every CTA's counts (written by other CTAs: read from L2), exclusive offsets by warp 0;
  // the level-2 histogram is complete too: its bins load alongside
  if (tid < a.C) s_cnt[tid] = __ldcg(a.cnt + (long long)r * a.C + tid);
  const int4 h2 = hist_bins<kSelThreads>(hist2);
  __syncthreads();
  if (warp == 0) {
    int ca = 0, ce = 0;
    for (int j0 = 0; j0 < a.C; j0 += 32) {
      const int j = j0 + lane;
      const int2 n2 = j < a.C ? s_cnt[j] : make_int2(0, 0);
      int xa = n2.x, xe = n2.y;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, xa, o), ye = __shfl_up_sync(0xffffffffu, xe, o);
        if (lane >= o) { xa += ya; xe += ye; }
      }
      if (j < a.C) s_off[j] = make_int2(ca + xa - n2.x, ce + xe - n2.y);
      ca += __shfl_sync(0xffffffffu, xa, 31);
      ce += __shfl_sync(0xffffffffu, xe, 31);
    }
    if (lane == 0) s_off[a.C] = make_int2(ca, ce);
  }
  __syncthreads();
  const int n_above = s_off[a.C].x, n_eq = s_off[a.C].y;
  if (n_above != above_total || n_above >= k || n_eq < k - n_above) {
    // the histogram disagrees with the scores: report instead of selecting wrongly
    if (tid == 0) atomicOr(&g_select_error, 1u);
    return;
  }
  const int need = k - n_above;
  const bool staged = n_eq <= kSelectMaxN;
  // The "above" entries go straight to the output and, when they fit, the bin-T
  // candidates to shared memory, both in entry order: element i of the lists'
  // concatenation (above lists, then bin-T lists) is found in its list by a search
  // over the offsets, with all of a thread's loads in flight before its stores.
  {
    const int n_cp = n_above + (staged ? n_eq : 0);
    const int* off_a = &s_off[0].x;
    const int* off_e = &s_off[0].y;
    for (int i0 = 0; i0 < n_cp; i0 += 4 * kSelThreads) {
      uint64_t val[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kSelThreads + tid;
        val[u] = 0ull;
        if (i < n_above) {
          const int j = list_of(off_a, 2, a.C, i);
          val[u] = (uint32_t)__ldcg(a.above + ((long long)r * a.C + j) * k + (i - off_a[2 * j]));
        } else if (i < n_cp) {
          const int ie = i - n_above;
          const int j = list_of(off_e, 2, a.C, ie);
          val[u] = __ldcg(a.eq + ((long long)r * a.C + j) * a.slice + (ie - off_e[2 * j]));
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kSelThreads + tid;
        if (i < n_above) out[i] = (int32_t)(uint32_t)val[u];
        else if (i < n_cp) s_c[i - n_above] = val[u];
      }
    }
  }
  if (staged) {
    // level 2 threshold among the staged candidates (the histogram's total is n_eq;
    // its barriers also publish the staged candidates)
    hist_threshold_from<kSelThreads>(h2, need, &s_T2, &s_above2, s_warp);
    const int T2 = s_T2, above2 = s_above2;
    if (T2 < 0) {
      if (tid == 0) atomicOr(&g_select_error, 1u);
      return;
    }
    // one pass in entry order: level-2 bins above T2 are selected, bin T2 ties collected
    const int per = (n_eq + kSelThreads - 1) / kSelThreads;
    const int t0 = tid * per, t1 = min(n_eq, t0 + per);
    int ng = 0, nq = 0;
    for (int t = t0; t < t1; ++t) {
      const int b2 = (int)((s_c[t] >> 40) & (kHistBins - 1));
      ng += b2 > T2;
      nq += b2 == T2;
    }
    int og, oq, tg, tq;
    block_scan2<kSelThreads>(ng, nq, og, oq, tg, tq, s_warp);
    if (tg != above2) {
      if (tid == 0) atomicOr(&g_select_error, 1u);
      return;
    }
    const int need2 = need - above2;
    if (tq < need2) {
      if (tid == 0) atomicOr(&g_select_error, 1u);
      return;
    }
    // The level-2 ties go to a shared array when there are few (the usual case),
    // else to this request's candidate region in global memory, free now that its
    // lists are staged in shared memory.
    const bool few = tq <= 32;
    uint64_t* gties = a.eq + (long long)r * a.C * a.slice;
    for (int t = t0; t < t1; ++t) {
      const uint64_t cnd = s_c[t];
      const int b2 = (int)((cnd >> 40) & (kHistBins - 1));
      if (b2 > T2) {
        out[n_above + og++] = cand_index(cnd);
      } else if (b2 == T2) {
        if (few) s_tie[oq] = cnd;
        else gties[oq] = cnd;
        ++oq;
      }
    }
    __threadfence_block();
    __syncthreads();
    if (few) {
      // rank the ties within one warp (composites are distinct)
      if (warp == 0) {
        const uint64_t mine = lane < tq ? s_tie[lane] : 0ull;
        int rank = 0;
        for (int j = 0; j < tq; ++j) rank += s_tie[j] > mine;
        if (lane < tq && rank < need2) out[n_above + above2 + rank] = cand_index(mine);
      }
    } else {
      select_core<kSelThreads>(gties, tq, need2, out + n_above + above2, nullptr);
    }
  } else {
    // Many ties around the threshold: gather the candidates to the front of this
    // request's region (a left shift, chunk by chunk) and select from global memory.
    uint64_t* gdst = a.eq + (long long)r * a.C * a.slice;
    for (int j = 0; j < a.C; ++j) {
      const uint64_t* src = a.eq + ((long long)r * a.C + j) * a.slice;
      for (int t0 = 0; t0 < s_cnt[j].y; t0 += kSelThreads) {
        const int t = t0 + tid;
        const uint64_t x = t < s_cnt[j].y ? __ldcg(src + t) : 0ull;
        __syncthreads();
        if (t < s_cnt[j].y) gdst[s_off[j].y + t] = x;
        __syncthreads();
      }
    }
    __threadfence_block();
    __syncthreads();
    select_core<kSelThreads>(gdst, n_eq, need, out + n_above, nullptr);
  }
}

static cudaError_t set_smem(const void* fn, size_t bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_select_from_scores(const float* scores, const SelectRows& rows, int k,
                                      int32_t* out_idx, uint64_t* out_cand, cudaStream_t stream) {
  if (rows.n_rows == 0) return cudaSuccess;
  const size_t smem = (size_t)rows.chunk * sizeof(uint64_t);
  cudaError_t e = set_smem((const void*)select_scores_kernel, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(true, select_scores_kernel, dim3(rows.n_rows), dim3(kSelThreads), smem, stream, scores, rows, k,
                 out_idx, out_cand);
  if (e != cudaSuccess) return e;
  ++g_launch_counter;
  return cudaGetLastError();
}

cudaError_t launch_select_rows(const float* scores, const SelectRows& rows, int k, int32_t* out_idx,
                               cudaStream_t stream) {
  if (rows.n_rows == 0) return cudaSuccess;
  const size_t smem = (size_t)(rows.N < kSelectRowMaxN ? rows.N : kSelectRowMaxN) * sizeof(uint32_t) + 16;
  cudaError_t e = set_smem((const void*)select_row_kernel, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(true, select_row_kernel, dim3(rows.n_rows), dim3(kSelThreads), smem, stream, scores, rows, k,
                 out_idx);
  if (e != cudaSuccess) return e;
  ++g_launch_counter;
  return cudaGetLastError();
}

cudaError_t launch_select_merge(const uint64_t* cand, int n_rows, int n_cand, int k, int32_t* out_idx,
                                cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const size_t smem = (size_t)n_cand * sizeof(uint64_t);
  cudaError_t e = set_smem((const void*)select_merge_kernel, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(true, select_merge_kernel, dim3(n_rows), dim3(kSelThreads), smem, stream, cand, n_cand, k, out_idx);
  if (e != cudaSuccess) return e;
  ++g_launch_counter;
  return cudaGetLastError();
}

cudaError_t launch_select_hist(const HistSelect& a, int B, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  if (a.C > kHistMaxCtas || a.slice != 16 * kSelThreads) return cudaErrorInvalidValue;
  const size_t smem = (size_t)kSelectMaxN * sizeof(uint64_t);
  cudaError_t e = set_smem((const void*)select_hist_kernel, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(true, select_hist_kernel, dim3(B * a.C), dim3(kSelThreads), smem, stream, a);
  if (e != cudaSuccess) return e;
  ++g_launch_counter;
  return cudaGetLastError();
}

unsigned int read_and_clear_select_error() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_select_error, sizeof(v)) != cudaSuccess) return 0xffffffffu;
  if (v) cudaMemcpyToSymbol(g_select_error, &zero, sizeof(zero));
  return v;
}

}  // namespace hca
