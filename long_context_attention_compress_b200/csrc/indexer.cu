// Lightning-indexer scores (sm_100a), CUDA-core version.
//
//   I(t, s) = sum_j w[t, j] * ReLU(q_I[t, j, :] . K_I[s, :])
// over the causally complete entries s of the query's request (QbitAI
// write-up, "混合注意力機制", CSA step two: the lightweight indexer inherited
// from DeepSeek-V3.2; "DeepSeek V4 Architecture Tricks", CSA section:
// 64 indexer heads of dim 128).
//
// One CTA per (query, tile of 128 entries) -- grid.x queries, grid.y tiles, one thread per entry: the query's
// heads and weights sit in shared memory as f32 and are read as broadcasts;
// the thread's key row stays in registers.  Scores are written to a score
// matrix in the workspace for the radix select.

#include "common.cuh"
#include "internal.h"

namespace hca {

template <int D>
__global__ void __launch_bounds__(128) indexer_scores_kernel(
    const bf16* __restrict__ q_idx, const float* __restrict__ w_idx, const bf16* __restrict__ k_idx,
    long long k_seq_stride, int N, const int32_t* __restrict__ q_pos, int mode, int rate, int H_I,
    float* __restrict__ scores, long long ld_scores) {
  extern __shared__ float s_q[];  // [H_I][D] then w[H_I]
  float* s_w = s_q + H_I * D;
  const int q = blockIdx.x;
  const int t = q_pos[q];
  const int nvis = n_visible(t, rate, N);
  const int s0 = blockIdx.y * 128;
  if (s0 >= nvis) return;
  const bf16* qp = q_idx + (long long)q * H_I * D;
  for (int e = threadIdx.x * 8; e < H_I * D; e += 128 * 8) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(qp + e), f);
#pragma unroll
    for (int k = 0; k < 8; ++k) s_q[e + k] = f[k];
  }
  for (int j = threadIdx.x; j < H_I; j += 128) s_w[j] = w_idx[(long long)q * H_I + j];
  __syncthreads();
  const int s = s0 + threadIdx.x;
  if (s >= nvis) return;
  const bf16* kp = k_idx + (mode == HCA_MODE_DECODE ? (long long)q * k_seq_stride : 0ll) + (long long)s * D;
  float kf[D];
#pragma unroll
  for (int d = 0; d < D; d += 8) unpack8(*reinterpret_cast<const uint4*>(kp + d), kf + d);
  float score = 0.f;
  for (int j = 0; j < H_I; ++j) {
    const float* qj = s_q + j * D;
    float dot = 0.f;
#pragma unroll
    for (int d = 0; d < D; d += 4) {
      const float4 qv = *reinterpret_cast<const float4*>(qj + d);
      dot = fmaf(qv.x, kf[d], dot);
      dot = fmaf(qv.y, kf[d + 1], dot);
      dot = fmaf(qv.z, kf[d + 2], dot);
      dot = fmaf(qv.w, kf[d + 3], dot);
    }
    score = fmaf(s_w[j], fmaxf(dot, 0.f), score);
  }
  scores[(long long)q * ld_scores + s] = score;
}

cudaError_t launch_indexer_scores(const bf16* q_idx, const float* w_idx, const bf16* k_idx,
                                  long long k_seq_stride, int N, const int32_t* q_pos, int Tq,
                                  int mode, int rate, int H_I, int d_I, float* scores,
                                  long long ld_scores, cudaStream_t stream) {
  if (Tq == 0 || N == 0) return cudaSuccess;
  dim3 grid(Tq, (N + 127) / 128);
  const size_t smem = (size_t)(H_I * d_I + H_I) * sizeof(float);
  cudaError_t e;
  if (d_I == 128) {
    e = cudaFuncSetAttribute((const void*)indexer_scores_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    indexer_scores_kernel<128><<<grid, 128, smem, stream>>>(q_idx, w_idx, k_idx, k_seq_stride, N, q_pos,
                                                            mode, rate, H_I, scores, ld_scores);
  } else {
    indexer_scores_kernel<32><<<grid, 128, smem, stream>>>(q_idx, w_idx, k_idx, k_seq_stride, N, q_pos,
                                                           mode, rate, H_I, scores, ld_scores);
  }
  ++g_launch_counter;
  return cudaGetLastError();
}

}  // namespace hca
