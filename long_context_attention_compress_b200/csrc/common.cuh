// Shared device helpers for the hybrid CSA/HCA attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hca.h"

namespace hca {

typedef __nv_bfloat16 bf16;

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// 2^x with the hardware approximate exp2 (flush-to-zero); x = -inf gives 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16 <-> f32 on raw 16-bit patterns.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}
// Round-to-nearest-even f32 -> bf16 pair packed into one 32-bit word (lo = a).
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Order-preserving map of an f32 to u32: larger float -> larger key (NaN-free input).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}
// Top-k candidate: 64-bit composite, larger = preferred. High word: score key;
// low word: bit-inverted entry index, so equal scores prefer the lower index.
// The all-zero composite is an empty slot and decodes to index -1.
__device__ __forceinline__ uint64_t make_cand(float score, int idx) {
  return ((uint64_t)float_key(score) << 32) | (uint32_t)(~(uint32_t)idx);
}
__device__ __forceinline__ int cand_index(uint64_t c) { return (int)(~(uint32_t)(c & 0xffffffffu)); }

// Entries visible to a query at position t: s < floor((t+1)/rate), capped at N.
__device__ __forceinline__ int n_visible(int t, int rate, int N) {
  int v = (t + 1) / rate;
  return v < N ? v : N;
}

// Rotary angle of pair j (of d rotated channels) at position pos is
// pos * base^(-2j/d).  Positions reach 10^6, so the angle is formed and its
// cosine and sine taken in f64 (an f32 frequency alone would be off by
// ~0.06 rad there).
__device__ __forceinline__ void rope_cos_sin_f64(long long pos, int j, int d, float base, double& cs, double& sn) {
  const double theta = pow((double)base, -2.0 * j / d);
  sincos((double)pos * theta, &sn, &cs);
}
__device__ __forceinline__ void rope_cos_sin(long long pos, int j, int d, float base, float& cs, float& sn) {
  double cd, sd;
  rope_cos_sin_f64(pos, j, d, base, cd, sd);
  cs = (float)cd;
  sn = (float)sd;
}

}  // namespace hca
