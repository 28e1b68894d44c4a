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
// The bf16 value is a quantisation of the normalised row, taken as from the
// f64 value (rounded via f32): an f32 normalisation would pick the other
// neighbour wherever its error crosses a rounding midpoint.  The sum of squares
// and the scale are f64.  Unrotated channels are formed in f32 (within 3 f32
// ulps of the f64 value) and redone in f64 only when that lands within 16 f32
// ulps of a bf16 rounding midpoint, where the two could round apart; the
// rotated channels (whose f32 form can cancel) are always f64.

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

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

// Rows reach shared memory through a per-warp ring of kStages row buffers
// (cp.async, 16 bytes per copy): a warp keeps kStages - 1 rows in flight while
// it works on one.  Each lane copies, and later reads, only its own chunks, so
// the ring needs no synchronisation beyond the lane's own copy groups.
template <bool F32>
struct NrCfg {
  static constexpr int kEB = F32 ? 4 : 2;       // input bytes per element
  static constexpr int kStages = F32 ? 2 : 4;   // 32 KiB of rows per CTA at c = 512
};

template <bool F32>
size_t norm_rope_smem(int c) {
  return (size_t)(kNrThreads / 32) * NrCfg<F32>::kStages * c * NrCfg<F32>::kEB;
}

template <bool F32>
__global__ void __launch_bounds__(kNrThreads) norm_rope_kernel(NormRope p, long long rows, long long rows_per_warp) {
  using C = NrCfg<F32>;
  // per warp: (cos, sin) of every rotary pair at the warp's current position
  __shared__ double2 s_cs[kNrThreads / 32][kNrMaxPairs];
  extern __shared__ __align__(16) unsigned char s_rows[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const long long warp = ((long long)blockIdx.x * kNrThreads + threadIdx.x) >> 5;
  const long long r0 = warp * rows_per_warp;
  const long long r1 = min(rows, r0 + rows_per_warp);
  if (r0 >= r1) return;
  const int nch = p.c >> 3;
  const int rope0 = p.c - p.rope_dims;
  const int n_pairs = p.rope_dims >> 1;
  const int row_bytes = p.c * C::kEB;
  unsigned char* ring = s_rows + (size_t)wib * C::kStages * row_bytes;
  // (sequence, row) of the next row to copy (isq, irr) and of the row being worked on
  // (sq, rr), advanced one row at a time (no 64-bit divisions per row)
  long long isq = r0 / p.rows_per_seq, irr = r0 % p.rows_per_seq;
  long long sq = isq, rr = irr;
  // copy this lane's chunks of row R into ring slot `slot` (one commit group per call, empty
  // past r1); calls come with consecutive R, which (isq, irr) follows
  auto issue = [&](long long R, int slot) {
    if (R < r1) {
      const unsigned char* src =
          reinterpret_cast<const unsigned char*>(p.x) + (isq * p.seq_x + irr * p.ld_x) * C::kEB;
      const uint32_t dst = tc::smem_u32(ring + slot * row_bytes);
#pragma unroll
      for (int k = 0; k < kNrMaxChunksPerLane; ++k) {
        const int ch = lane + 32 * k;
        if (ch < nch) {
#pragma unroll
          for (int b = 0; b < 8 * C::kEB; b += 16) tc::cp_async16(dst + ch * 8 * C::kEB + b, src + ch * 8 * C::kEB + b, 16);
        }
      }
      if (++irr == p.rows_per_seq) { irr = 0; ++isq; }
    }
    tc::cp_async_commit();
  };
#pragma unroll
  for (int st = 0; st < C::kStages - 1; ++st) issue(r0 + st, st);
  long long last_pos = -1;
  int slot = 0;
  for (long long R = r0; R < r1; ++R) {
    issue(R + C::kStages - 1, slot == 0 ? C::kStages - 1 : slot - 1);
    long long pos;
    if (p.ring) {
      // ring block of rows_per_seq rows ending at t: row rr holds the token in
      // [t - rows_per_seq + 1, t] that is congruent to rr
      const long long t = p.pos ? p.pos[sq] : 0;
      const long long n = p.rows_per_seq;
      pos = t - (((t - rr) % n) + n) % n;
    } else {
      pos = (long long)max((p.pos ? p.pos[sq] : 0) + p.pos_add, 0) + rr * p.pos_step;
    }
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
    tc::cp_async_wait<C::kStages - 1>();  // this lane's copies of row R have landed
    const unsigned char* row = ring + slot * row_bytes;
    float v[kNrMaxChunksPerLane][8];
    double ss = 0.0;
#pragma unroll
    for (int k = 0; k < kNrMaxChunksPerLane; ++k) {
      const int ch = lane + 32 * k;
      if (ch < nch) {
        load_chunk<F32>(row, (long long)ch * 8, v[k]);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fma((double)v[k][e], (double)v[k][e], ss);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const double inv = rsqrt(ss / p.c + (double)p.eps);
    const float inv32 = (float)inv;
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
          for (int e = 0; e < 8; ++e) {
            float y = v[k][e] * inv32 * g[e];
            // low 16 bits = what bf16 rounding drops; 0x8000 is the midpoint
            const int low = (int)(__float_as_uint(y) & 0xffffu) - 0x8000;
            if (low > -16 && low < 16) y = (float)((double)v[k][e] * inv * (double)g[e]);
            w[e] = y;
          }
        }
        uint4 o;
        o.x = pack_bf16x2(w[0], w[1]);
        o.y = pack_bf16x2(w[2], w[3]);
        o.z = pack_bf16x2(w[4], w[5]);
        o.w = pack_bf16x2(w[6], w[7]);
        *reinterpret_cast<uint4*>(p.y + yo + 8 * ch) = o;
      }
    }
    slot = slot + 1 == C::kStages ? 0 : slot + 1;
    if (++rr == p.rows_per_seq) { rr = 0; ++sq; }
  }
  tc::cp_async_wait<0>();  // (nothing is left in flight at exit)
}

}  // namespace

template <bool F32>
static cudaError_t launch_norm_rope_t(const NormRope& p, long long rows, cudaStream_t stream) {
  const size_t smem = norm_rope_smem<F32>(p.c);
  cudaError_t e = cudaFuncSetAttribute((const void*)norm_rope_kernel<F32>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // up to 64 warps per SM (several waves when fewer fit), each over a contiguous run of rows
  const long long max_warps = (long long)device_sm_count() * 64;
  const long long warps = rows < max_warps ? rows : max_warps;
  const long long per = (rows + warps - 1) / warps;
  const long long used = (rows + per - 1) / per;
  const unsigned grid = (unsigned)((used * 32 + kNrThreads - 1) / kNrThreads);
  norm_rope_kernel<F32><<<grid, kNrThreads, smem, stream>>>(p, rows, per);
  return cudaGetLastError();
}

cudaError_t launch_norm_rope(const NormRope& p, cudaStream_t stream) {
  const long long rows = (long long)p.n_seq * p.rows_per_seq;
  if (rows <= 0) return cudaSuccess;
  const cudaError_t e = p.x_f32 ? launch_norm_rope_t<true>(p, rows, stream) : launch_norm_rope_t<false>(p, rows, stream);
  if (e == cudaSuccess) ++g_launch_counter;
  return e;
}

}  // namespace hca
