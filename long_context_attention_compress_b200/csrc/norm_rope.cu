// Q/KV RMSNorm + partial RoPE of rows, sm_100a.
//
// What it computes (QbitAI write-up, "混合注意力機制": queries and KV entries
// are RMS-normalised before core attention and only their last 64 channels
// carry a rotary position; "DeepSeek V4 Architecture Tricks", "Partial RoPE 和
// Attention Sink"): y = x / sqrt(mean(x^2) + eps) * gamma, then pair j of the
// last rope_dims channels, (2j, 2j+1), turns by pos * base^(-2j/rope_dims).
//
// Design: HBM-bound (one read and one bf16 write per element).  One warp owns a
// row at a time: lane l holds the 8-channel chunks l and l+32 (16-byte bf16 or
// 32-byte f32 loads), the sum of squares is a warp all-reduce, and the rotated
// pairs sit inside a lane's chunk.  A warp walks a contiguous run of rows, so
// the query heads of one position (which share it) reuse the lane's cosines
// and sines; they are recomputed only when the position changes.
// Arithmetic is f64 (inputs are exact in it) up to one rounding to bf16 (via
// f32): the bf16 value is a quantisation of the normalised row, and taking it
// from an f32 normalisation would pick the other neighbour wherever the f32
// error crosses a rounding midpoint.  At the HBM rate this needs about a
// quarter of the f64 pipe.

#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {

constexpr int kNrThreads = 256;
constexpr int kNrMaxChunksPerLane = 2;  // c <= 512
constexpr int kNrMaxPairs = 128;        // rope_dims <= 256

template <bool F32>
__device__ __forceinline__ void load_chunk(const void* base, long long off, float* v) {
  if constexpr (F32) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    unpack8(*reinterpret_cast<const uint4*>(reinterpret_cast<const bf16*>(base) + off), v);
  }
}

template <bool F32>
__global__ void __launch_bounds__(kNrThreads) norm_rope_kernel(NormRope p, long long rows, long long rows_per_warp) {
  // per warp: (cos, sin) of every rotary pair at the warp's current position
  __shared__ double2 s_cs[kNrThreads / 32][kNrMaxPairs];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const long long warp = ((long long)blockIdx.x * kNrThreads + threadIdx.x) >> 5;
  const long long r0 = warp * rows_per_warp;
  const long long r1 = min(rows, r0 + rows_per_warp);
  if (r0 >= r1) return;
  const int nch = p.c >> 3;
  const int rope0 = p.c - p.rope_dims;
  const int n_pairs = p.rope_dims >> 1;
  long long last_pos = -1;
  for (long long R = r0; R < r1; ++R) {
    const long long sq = R / p.rows_per_seq, rr = R % p.rows_per_seq;
    const long long pos = (long long)max((p.pos ? p.pos[sq] : 0) + p.pos_add, 0) + rr * p.pos_step;
    if (pos != last_pos && n_pairs > 0) {  // warp-uniform
      last_pos = pos;
      __syncwarp();
      for (int j = lane; j < n_pairs; j += 32) {
        double cs, sn;
        rope_cos_sin_f64(pos, j, p.rope_dims, p.rope_base, cs, sn);
        s_cs[wib][j] = make_double2(cs, sn);
      }
      __syncwarp();
    }
    float v[kNrMaxChunksPerLane][8];
    double ss = 0.0;
    const long long xo = sq * p.seq_x + rr * p.ld_x;
#pragma unroll
    for (int k = 0; k < kNrMaxChunksPerLane; ++k) {
      const int ch = lane + 32 * k;
      if (ch < nch) {
        load_chunk<F32>(p.x, xo + 8 * ch, v[k]);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fma((double)v[k][e], (double)v[k][e], ss);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const double inv = 1.0 / sqrt(ss / p.c + (double)p.eps);
    const long long yo = sq * p.seq_y + rr * p.ld_y;
#pragma unroll
    for (int k = 0; k < kNrMaxChunksPerLane; ++k) {
      const int ch = lane + 32 * k;
      if (ch < nch) {
        float g[8];
        load_chunk<true>(p.gamma, 8 * ch, g);  // (L1-resident after the first row)
        float w[8];
        if (8 * ch >= rope0) {
          const int j0 = (8 * ch - rope0) >> 1;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const double2 r = s_cs[wib][j0 + i];
            const double a = (double)v[k][2 * i] * inv * (double)g[2 * i];
            const double b = (double)v[k][2 * i + 1] * inv * (double)g[2 * i + 1];
            w[2 * i] = (float)(a * r.x - b * r.y);
            w[2 * i + 1] = (float)(a * r.y + b * r.x);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = (float)((double)v[k][e] * inv * (double)g[e]);
        }
        uint4 o;
        o.x = pack_bf16x2(w[0], w[1]);
        o.y = pack_bf16x2(w[2], w[3]);
        o.z = pack_bf16x2(w[4], w[5]);
        o.w = pack_bf16x2(w[6], w[7]);
        *reinterpret_cast<uint4*>(p.y + yo + 8 * ch) = o;
      }
    }
  }
}

}  // namespace

cudaError_t launch_norm_rope(const NormRope& p, cudaStream_t stream) {
  const long long rows = (long long)p.n_seq * p.rows_per_seq;
  if (rows <= 0) return cudaSuccess;
  // up to 64 warps per SM (several waves when fewer fit), each over a contiguous run of rows
  const long long max_warps = (long long)device_sm_count() * 64;
  const long long warps = rows < max_warps ? rows : max_warps;
  const long long per = (rows + warps - 1) / warps;
  const long long used = (rows + per - 1) / per;
  const unsigned grid = (unsigned)((used * 32 + kNrThreads - 1) / kNrThreads);
  if (p.x_f32)
    norm_rope_kernel<true><<<grid, kNrThreads, 0, stream>>>(p, rows, per);
  else
    norm_rope_kernel<false><<<grid, kNrThreads, 0, stream>>>(p, rows, per);
  ++g_launch_counter;
  return cudaGetLastError();
}

}  // namespace hca
