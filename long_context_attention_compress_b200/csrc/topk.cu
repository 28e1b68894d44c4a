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

namespace hca {

constexpr int kSelThreads = 1024;

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

__global__ void __launch_bounds__(kSelThreads) select_scores_kernel(const float* __restrict__ scores,
                                                                    SelectRows rows, int k,
                                                                    int32_t* out_idx, uint64_t* out_cand) {
  extern __shared__ uint64_t s_c[];
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

__global__ void __launch_bounds__(kSelThreads) select_merge_kernel(const uint64_t* __restrict__ cand, int n_cand,
                                                                   int k, int32_t* out_idx) {
  extern __shared__ uint64_t s_c[];
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

static cudaError_t set_smem(const void* fn, size_t bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_select_from_scores(const float* scores, const SelectRows& rows, int k,
                                      int32_t* out_idx, uint64_t* out_cand, cudaStream_t stream) {
  if (rows.n_rows == 0) return cudaSuccess;
  const size_t smem = (size_t)rows.chunk * sizeof(uint64_t);
  cudaError_t e = set_smem((const void*)select_scores_kernel, smem);
  if (e != cudaSuccess) return e;
  select_scores_kernel<<<rows.n_rows, kSelThreads, smem, stream>>>(scores, rows, k, out_idx, out_cand);
  ++g_launch_counter;
  return cudaGetLastError();
}

cudaError_t launch_select_merge(const uint64_t* cand, int n_rows, int n_cand, int k, int32_t* out_idx,
                                cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const size_t smem = (size_t)n_cand * sizeof(uint64_t);
  cudaError_t e = set_smem((const void*)select_merge_kernel, smem);
  if (e != cudaSuccess) return e;
  select_merge_kernel<<<n_rows, kSelThreads, smem, stream>>>(cand, n_cand, k, out_idx);
  ++g_launch_counter;
  return cudaGetLastError();
}

}  // namespace hca
