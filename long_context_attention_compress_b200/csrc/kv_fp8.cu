// FP8 (E4M3) storage of the KV channels outside the rotary part, sm_100a.
//
// What it stores ("DeepSeek V4 Architecture Tricks", "Partial RoPE 和 Attention
// Sink": the rotary channels of the KV cache stay BF16, the other channels are
// kept in FP8): the first n = c - rope_dims channels of a row as E4M3 codes
// with one f32 scale per 64 channels, scale = f32(group amax / 448) (1 for an
// all-zero group), code = the E4M3 value nearest to x / scale (ties to the
// even mantissa, saturating at +-448, the sign kept on values that round to
// zero); the last rope_dims channels as BF16.
//
// Exactness.  x / scale is formed as an f64 quotient of the two f32 values
// (correctly rounded, as any IEEE f64 division of them) and rounded to E4M3
// with exact f64 arithmetic (power-of-two steps), so every code is decided on
// the same number a float64 reference forms.
//
// Consumption.  The attention kernel's shared memory holds the query heads
// (64 KiB), one 128-row bf16 KV tile (128 KiB) and P (32 KiB); an FP8 staging
// area for widening in place does not fit beside them.  So the rows an
// attention call reads are widened first: kv_fp8_gather_kernel writes them as
// bf16 (the value code x scale, rounded once) into a workspace block that the
// attention then reads as an ordinary cache -- for the CSA layer the selected
// rows only (the top-k indices are rewritten to their slots), for the HCA
// layer every visible row.

#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {
constexpr int kFp8Group = 64;
constexpr double kE4m3Max = 448.0;

// E4M3 byte of q (f64), ties to even, saturating; sign bit 7, exponent bits 3-6
// (bias 7, field 0 = subnormal with spacing 2^-9), mantissa bits 0-2.
__device__ __forceinline__ uint32_t e4m3_encode(double q) {
  const uint32_t sign = q < 0.0 ? 0x80u : 0u;
  const double a = fabs(q);
  if (a >= kE4m3Max) return sign | 0x7Eu;  // 1.75 * 2^8 = 448
  int e = -6;
  if (a > 0.0) {
    int ex;
    frexp(a, &ex);  // a = f * 2^ex, f in [0.5, 1): floor(log2 a) = ex - 1
    e = ex - 1 < -6 ? -6 : ex - 1;
  }
  const double qq = ldexp(a, 3 - e);  // a / 2^(e-3), exact
  double fl = floor(qq);
  const double frac = qq - fl;
  if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) == 1.0)) fl += 1.0;
  int m = (int)fl;  // value = m * 2^(e-3), m in [0, 16]
  if (m >= 16) {    // rounded up into the next binade
    m = 8;
    ++e;
  }
  if (m < 8) return sign | (uint32_t)m;  // subnormal (e = -6): exponent field 0
  return sign | ((uint32_t)(e + 7) << 3) | (uint32_t)(m - 8);
}

__device__ __forceinline__ float e4m3_decode(uint32_t b) {
  const uint32_t ex = (b >> 3) & 15u, m = b & 7u;
  const float mag = ex ? __uint_as_float(((ex + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;  // m * 2^-9
  return (b & 0x80u) ? -mag : mag;
}

template <bool F32>
__device__ __forceinline__ float load_x(const void* x, long long i) {
  if constexpr (F32) return reinterpret_cast<const float*>(x)[i];
  return __bfloat162float(reinterpret_cast<const bf16*>(x)[i]);
}

// One thread per 64-channel group of the FP8 part, or per 8 rotary channels.
template <bool F32>
__global__ void __launch_bounds__(256) kv_fp8_quantize_kernel(const void* __restrict__ x, long long ld_x, long long rows,
                                                              int n_groups, int rope_dims, uint8_t* __restrict__ codes,
                                                              long long ld_codes, float* __restrict__ scales,
                                                              long long ld_scales, bf16* __restrict__ rope,
                                                              long long ld_rope) {
  const int per_row = n_groups + rope_dims / 8;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= rows * per_row) return;
  const long long r = gid / per_row;
  const int u = (int)(gid % per_row);
  const long long xr = r * ld_x;
  if (u >= n_groups) {  // rotary channels: bf16
    const int j0 = n_groups * kFp8Group + (u - n_groups) * 8;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = pack_bf16x2(load_x<F32>(x, xr + j0 + 2 * k), load_x<F32>(x, xr + j0 + 2 * k + 1));
    *reinterpret_cast<uint4*>(rope + r * ld_rope + (j0 - n_groups * kFp8Group)) = make_uint4(w[0], w[1], w[2], w[3]);
    return;
  }
  const int j0 = u * kFp8Group;
  float amax = 0.f;
  for (int j = 0; j < kFp8Group; ++j) amax = fmaxf(amax, fabsf(load_x<F32>(x, xr + j0 + j)));
  const float sc = amax > 0.f ? __double2float_rn((double)amax / kE4m3Max) : 1.f;
  const double sd = (double)sc;
  uint8_t* cp = codes + r * ld_codes + j0;
  for (int j = 0; j < kFp8Group; j += 16) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) word |= e4m3_encode((double)load_x<F32>(x, xr + j0 + j + 4 * k + b) / sd) << (8 * b);
      w[k] = word;
    }
    *reinterpret_cast<uint4*>(cp + j) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  scales[r * ld_scales + u] = sc;
}

// Widen rows of an FP8 cache to bf16: output row j of sequence b is source row
// e = idx ? idx[b*n_out + j] : j of sequence b (rows seq_rows apart); e < 0 or
// e >= n_src gives a zero row.  idx_out (optional) receives j for a copied
// selected row, -1 otherwise.  One thread per 8 channels.
__global__ void __launch_bounds__(256) kv_fp8_gather_kernel(KvFp8 kv, int c, int rope_dims, int B, int n_out,
                                                            const int32_t* __restrict__ idx, int n_src,
                                                            bf16* __restrict__ out, int32_t* __restrict__ idx_out) {
  const int per_row = c / 8;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)B * n_out * per_row) return;
  const long long orow = gid / per_row;
  const int u = (int)(gid % per_row);
  const int b = (int)(orow / n_out), j = (int)(orow % n_out);
  const int e = idx ? idx[orow] : j;
  const bool ok = e >= 0 && e < n_src;
  if (idx_out && u == 0) idx_out[orow] = ok ? j : -1;
  uint4 w = make_uint4(0u, 0u, 0u, 0u);
  if (ok) {
    const long long sr = (long long)b * kv.seq_rows + e;
    const int n = c - rope_dims;
    const int j0 = u * 8;
    if (j0 < n) {
      const uint2 cb = *reinterpret_cast<const uint2*>(kv.codes + sr * kv.ld_codes + j0);
      const float sc = kv.scales[sr * kv.ld_scales + j0 / kFp8Group];
      const uint32_t lo = cb.x, hi = cb.y;
      w.x = pack_bf16x2(e4m3_decode(lo & 255u) * sc, e4m3_decode((lo >> 8) & 255u) * sc);
      w.y = pack_bf16x2(e4m3_decode((lo >> 16) & 255u) * sc, e4m3_decode(lo >> 24) * sc);
      w.z = pack_bf16x2(e4m3_decode(hi & 255u) * sc, e4m3_decode((hi >> 8) & 255u) * sc);
      w.w = pack_bf16x2(e4m3_decode((hi >> 16) & 255u) * sc, e4m3_decode(hi >> 24) * sc);
    } else {
      w = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(kv.rope) + sr * kv.ld_rope + (j0 - n));
    }
  }
  *reinterpret_cast<uint4*>(out + orow * c + u * 8) = w;
}
}  // namespace

cudaError_t launch_kv_fp8_quantize(const void* x, bool x_f32, long long ld_x, long long rows, int c, int rope_dims,
                                   uint8_t* codes, long long ld_codes, float* scales, long long ld_scales, bf16* rope,
                                   long long ld_rope, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int n_groups = (c - rope_dims) / kFp8Group;
  const long long n = rows * (n_groups + rope_dims / 8);
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (x_f32)
    kv_fp8_quantize_kernel<true><<<grid, 256, 0, stream>>>(x, ld_x, rows, n_groups, rope_dims, codes, ld_codes, scales,
                                                           ld_scales, rope, ld_rope);
  else
    kv_fp8_quantize_kernel<false><<<grid, 256, 0, stream>>>(x, ld_x, rows, n_groups, rope_dims, codes, ld_codes,
                                                            scales, ld_scales, rope, ld_rope);
  ++g_launch_counter;
  return cudaGetLastError();
}

cudaError_t launch_kv_fp8_gather(const KvFp8& kv, int c, int rope_dims, int B, int n_out, const int32_t* idx,
                                 int n_src, bf16* out, int32_t* idx_out, cudaStream_t stream) {
  const long long n = (long long)B * n_out * (c / 8);
  if (n == 0) return cudaSuccess;
  kv_fp8_gather_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(kv, c, rope_dims, B, n_out, idx, n_src, out,
                                                                        idx_out);
  ++g_launch_counter;
  return cudaGetLastError();
}

}  // namespace hca
