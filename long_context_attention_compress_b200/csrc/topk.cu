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
template <int NT>
__device__ void select_core(const uint64_t* s_c, int n, int k, int32_t* out_idx, uint64_t* out_cand) {
  __shared__ int s_hist[256];
  __shared__ int s_suf[256];
  __shared__ int s_bucket, s_greater;
  __shared__ int2 s_warp[NT / 32 + 1];
  const int tid = threadIdx.x;

  if (n <= k) {
    for (int e = tid; e < k; e += NT) {
      uint64_t c = e < n ? s_c[e] : 0ull;
      if (out_idx) out_idx[e] = e < n ? cand_index(c) : -1;
      else out_cand[e] = c;
    }
    return;
  }

  uint64_t prefix = 0;
  int shift = 64;
  int remaining = k;
  for (int pass = 0; pass < 8; ++pass) {
    shift -= 8;
    for (int b = tid; b < 256; b += NT) s_hist[b] = 0;
    __syncthreads();
    const int hs = shift + 8;  // bits above this pass's digit
    for (int e = tid; e < n; e += NT) {
      const uint64_t c = s_c[e];
      if (pass == 0 || (c >> hs) == (prefix >> hs)) atomicAdd(&s_hist[(int)((c >> shift) & 255u)], 1);
    }
    __syncthreads();
    // suffix sums: s_suf[b] = sum_{d >= b} hist[d]
    if (tid < 256) s_suf[tid] = s_hist[tid];
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
      int v = 0;
      if (tid < 256 && tid + off < 256) v = s_suf[tid + off];
      __syncthreads();
      if (tid < 256) s_suf[tid] += v;
      __syncthreads();
    }
    if (tid < 256) {
      const int sb = s_suf[tid];
      const int sb1 = tid < 255 ? s_suf[tid + 1] : 0;
      if (sb >= remaining && sb1 < remaining) { s_bucket = tid; s_greater = sb1; }
    }
    __syncthreads();
    const int b = s_bucket;
    remaining -= s_greater;
    prefix |= (uint64_t)b << shift;
    const int cnt = s_hist[b];
    __syncthreads();
    if (cnt == remaining) break;
  }

  // Output in candidate order: all above the threshold prefix, then the first
  // `remaining` equal to it (only duplicates -- empty slots -- can tie here).
  const uint64_t P = prefix >> shift;
  const int per = (n + NT - 1) / NT;
  const int e0 = tid * per;
  const int e1 = min(n, e0 + per);
  int ng = 0, ne = 0;
  for (int e = e0; e < e1; ++e) {
    const uint64_t v = s_c[e] >> shift;
    ng += v > P;
    ne += v == P;
  }
  int og, oe, tg, te;
  block_scan2<NT>(ng, ne, og, oe, tg, te, s_warp);
  for (int e = e0; e < e1; ++e) {
    const uint64_t c = s_c[e];
    const uint64_t v = c >> shift;
    int slot = -1;
    if (v > P) slot = og++;
    else if (v == P) { if (oe < remaining) slot = tg + oe; ++oe; }
    if (slot >= 0) {
      if (out_idx) out_idx[slot] = cand_index(c);
      else out_cand[slot] = c;
    }
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
  for (int e = threadIdx.x; e < n; e += kSelThreads) s_c[e] = make_cand(sp[e], start + e);
  __syncthreads();
  select_core<kSelThreads>(s_c, n, k, out_idx ? out_idx + (long long)r * k : nullptr,
                           out_cand ? out_cand + (long long)r * k : nullptr);
}

__global__ void __launch_bounds__(kSelThreads) select_merge_kernel(const uint64_t* __restrict__ cand, int n_cand,
                                                                   int k, int32_t* out_idx) {
  extern __shared__ uint64_t s_c[];
  const int r = blockIdx.x;
  const uint64_t* cp = cand + (long long)r * n_cand;
  int n = 0;
  // compact the non-empty candidates (empty slots are zero) keeping order
  for (int e = threadIdx.x; e < n_cand; e += kSelThreads) s_c[e] = cp[e];
  __syncthreads();
  n = n_cand;
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
