// FP4 variant of the decode lightning indexer (sm_100a): MXFP4 keys and
// queries, BF16 index scores.
//
// What it computes ("DeepSeek V4 Architecture Tricks", "FP4 / FP8
// Quantization-Aware Training": the indexer's QK path is cached, loaded and
// multiplied in FP4 and the index scores are kept in BF16; FP4 values
// dequantise losslessly because the wider format's exponent absorbs the
// fine-grained scale):
//   I(t, s) = bf16( sum_j w[t, j] * ReLU(q4[t, j, :] . k4[s, :]) )
// with q4, k4 the MXFP4 values of q_I and K_I: E2M1 elements, one
// power-of-two scale 2^X per 32 consecutive elements along d_I,
// X = floor(log2 amax) - 2, nearest-even rounding saturating at +-6; codes
// two per byte, the even element in the low nibble; scales as E8M0 bytes X+127.
//
// Design.  A key costs 64 B of codes + 4 B of scales (bf16: 256 B), so the
// stream the decode step is bound by shrinks 3.8x.  E2M1 x 2^X has at most two
// significant bits, so it widens exactly to bf16, and the tile then runs
// through the same M = 128 entries x N = 64 heads x K = 16 bf16 tcgen05.mma and
// TMEM epilogue as the bf16 indexer.  Per CTA (persistent grid):
//   warp 0      TMA producer: a tile's codes [128 keys x 64 B] and scales
//               [128 keys x 4 B] into a 6-deep staging ring; the request's
//               (FP4-rounded, bf16) query on request change
//   warp 1      MMA issuer
//   warps 2..5  epilogue: ReLU, head weights, BF16 rounding, score-key histogram
//   warps 6..13 converters: half a key row per thread, codes x scale -> bf16 (byte
//               permutes and one bf16x2 multiply per pair) into the 128B-swizzled
//               K-major tile ring (3 deep) the MMA reads
// Every wait is bounded; a CTA that gives up records an error, lets its own
// copies and MMAs drain, frees its TMEM and returns.
//
// The quantiser (mxfp4_quantize_kernel) writes the cache form; the query
// round trip (mxfp4_roundtrip_kernel) writes the bf16 values of a row's MXFP4
// form.  Both decide every code with exact comparisons against the E2M1
// midpoints (x * 2^-X is exact), so the codes match the definition bit for bit.

#include <cudaTypedefs.h>

#include <cstddef>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hca {

namespace {
constexpr int kFStages = 6;   // staging ring (codes + scales)
constexpr int kFBuf = 3;      // bf16 tile ring
constexpr int kFTile = 128;   // entries per tile (MMA M)
constexpr int kFHeads = 64;   // indexer heads (MMA N)
constexpr int kFDim = 128;    // key dim (MMA K)
constexpr int kFAcc = 4;      // TMEM accumulators
constexpr int kFTmemCols = kFAcc * kFHeads;                // 256
constexpr uint32_t kFCodeBytes = kFTile * kFDim / 2;       // 8 KiB
constexpr uint32_t kFScaleBytes = kFTile * kFDim / 32;     // 512 B
constexpr uint32_t kFStageStride = 9216;                   // 1024-aligned slot of codes + scales
constexpr uint32_t kFTileBytes = kFTile * kFDim * 2;       // 32 KiB
constexpr uint32_t kFChunkBytes = kFTile * 128;            // 16 KiB (64 dims)
constexpr uint32_t kFQBytes = kFHeads * kFDim * 2;         // 16 KiB
constexpr uint32_t kFQChunkBytes = kFHeads * 128;          // 8 KiB
constexpr int kFConvWarps = 8;                             // converter warps (two per scheduler)
constexpr int kFThreads = 192 + 32 * kFConvWarps;          // producer, MMA, 4 epilogue warps, converters
constexpr int kFConv0 = 192;                               // first converter thread

struct __align__(8) FBars {
  uint64_t sfull[kFStages], sempty[kFStages];
  uint64_t cfull[kFBuf], bempty[kFBuf];
  uint64_t tfull[kFAcc], tempty[kFAcc];
  uint64_t qfull[2], qempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kFSmemBytes = 1024 /*align slack*/ + kFBuf * kFTileBytes + 2 * kFQBytes +
                               kFStages * kFStageStride + sizeof(FBars) + kHistBins * sizeof(int);
static_assert(kFSmemBytes <= 227 * 1024, "shared memory");

// E2M1 value of a 4-bit code (bit 3 sign, bits 1-2 exponent e with bias 1, bit 0
// mantissa m): e = 0 gives 0 or 0.5, else (1 + m/2) 2^(e-1); built as f32 bits.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const uint32_t mag = e ? (((126u + e) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
  return __uint_as_float(mag | ((c & 8u) << 28));
}

// Eight E2M1 codes (word nibbles 0..7, element order) times 2^X -> eight bf16, packed in
// pairs (o[k] = element 2k | element 2k+1 << 16).  The magnitudes come from byte
// tables by byte permutes (bf16 bits of 0, 0.5, 1, 1.5, 2, 3, 4, 6: high bytes
// 00 3F 3F 3F 40 40 40 40, low bytes 00 00 80 C0 00 40 80 C0; __byte_perm reads only
// bits 0-2 of each of the four low selector nibbles, so the codes serve as selectors
// as they are, sign bit included).  The signs (bit 3 of each nibble) join the high
// bytes before the pairs are formed: byte k of (codes << 4) holds element 2k's sign in
// its bit 7 and byte k of the codes element 2k+1's, so one permute per four elements
// and a mask line them up with the high bytes of those elements.  2^X is applied by one
// bf16x2 multiply, exact while every nonzero product stays a normal bf16
// (|X| <= 125: 0.5 * 2^X .. 6 * 2^X); beyond that the values are formed in f32 (as
// exact) and rounded once.
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t w, int X, uint32_t* o) {
  constexpr uint32_t kHiLo = 0x3F3F3F00u, kHiHi = 0x40404040u, kLoLo = 0xC0800000u, kLoHi = 0xC0804000u;
  if (X >= -125 && X <= 125) {
    const uint32_t w4 = w << 4, wh = w >> 16;
    // high bytes of elements 0-3 and 4-7, signs included; low bytes likewise
    const uint32_t h0 = __byte_perm(kHiLo, kHiHi, w) | (__byte_perm(w4, w, 0x5140u) & 0x80808080u);
    const uint32_t h1 = __byte_perm(kHiLo, kHiHi, wh) | (__byte_perm(w4, w, 0x7362u) & 0x80808080u);
    const uint32_t l0 = __byte_perm(kLoLo, kLoHi, w), l1 = __byte_perm(kLoLo, kLoHi, wh);
    uint32_t p[4];
    p[0] = __byte_perm(l0, h0, 0x5140u);
    p[1] = __byte_perm(l0, h0, 0x7362u);
    p[2] = __byte_perm(l1, h1, 0x5140u);
    p[3] = __byte_perm(l1, h1, 0x7362u);
    const uint32_t sb = (uint32_t)(127 + X) << 7;  // bf16 bits of 2^X
    const uint32_t sbits = sb | (sb << 16);
    __nv_bfloat162 sc;
    memcpy(&sc, &sbits, 4);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 v;
      memcpy(&v, &p[k], 4);
      v = __hmul2(v, sc);
      memcpy(&o[k], &v, 4);
    }
    return;
  }
  const float scf = ldexpf(1.f, X);
#pragma unroll
  for (int j = 0; j < 8; j += 2)
    o[j >> 1] = pack_bf16x2(e2m1_value((w >> (4 * j)) & 15u) * scf, e2m1_value((w >> (4 * j + 4)) & 15u) * scf);
}

// Nearest E2M1 code of a (already scaled) value, ties to the even code, saturating.
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  const float a = fabsf(y);
  const uint32_t m = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
                   : a <= 2.5f ? 4u : a < 3.5f ? 5u : a <= 5.0f ? 6u : 7u;
  return (y < 0.f && m != 0u) ? (m | 8u) : m;
}

// Shared exponent of a block: floor(log2 amax) - 2 in [-127, 127]; -127 for an all-zero block.
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  const int X = ilogbf(amax) - 2;
  return X < -127 ? -127 : (X > 127 ? 127 : X);
}

template <bool F32>
__device__ __forceinline__ float load_elem(const void* x, long long i) {
  if constexpr (F32) return reinterpret_cast<const float*>(x)[i];
  return __bfloat162float(reinterpret_cast<const bf16*>(x)[i]);
}

// One thread per 32-element block: codes (16 bytes) and the block's scale byte.
template <bool F32>
__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(const void* __restrict__ x, long long ld_x, int rows,
                                                             int d, uint8_t* __restrict__ codes, long long ld_codes,
                                                             uint8_t* __restrict__ scales, long long ld_scales) {
  const int bpr = d / 32;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)rows * bpr) return;
  const long long r = gid / bpr;
  const int blk = (int)(gid % bpr);
  const long long x0 = r * ld_x + blk * 32;
  float v[32];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = load_elem<F32>(x, x0 + i);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  const int X = mx_exponent(amax);
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) word |= e2m1_code(ldexpf(v[8 * q + j], -X)) << (4 * j);
    w[q] = word;
  }
  *reinterpret_cast<uint4*>(codes + r * ld_codes + blk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  scales[r * ld_scales + blk] = (uint8_t)(X + 127);
}

// One thread per 32-element block: the bf16 values of the block's MXFP4 form.
__global__ void __launch_bounds__(256) mxfp4_roundtrip_kernel(const bf16* __restrict__ x, int rows, int d,
                                                              bf16* __restrict__ y) {
  const int bpr = d / 32;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)rows * bpr) return;
  const long long o = (gid / bpr) * d + (gid % bpr) * 32;
  float v[32];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = __bfloat162float(x[o + i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  const int X = mx_exponent(amax);
  const float scf = ldexpf(1.f, X);  // 2^X, exact (subnormal at X = -127)
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const uint32_t c0 = e2m1_code(ldexpf(v[i], -X)), c1 = e2m1_code(ldexpf(v[i + 1], -X));
    *reinterpret_cast<uint32_t*>(y + o + i) = pack_bf16x2(e2m1_value(c0) * scf, e2m1_value(c1) * scf);
  }
}
}  // namespace

__device__ unsigned int g_indexer_fp4_error = 0;

namespace {
// This CTA's (request r, tile t) items in order, from flat index g0 on: one division at
// the start, then a carry into the next request; a request's visible entry count is
// read once per request (every role of the kernel walks the same items).
struct TileWalk {
  int r, t, nvis;
  __device__ __forceinline__ TileWalk(long long g0, int tiles, const int32_t* q_pos, int B, int rate, int N)
      : r((int)(g0 / tiles)), t((int)(g0 % tiles)), nvis(0) {
    if (r < B) nvis = n_visible(q_pos[r], rate, N);
  }
  __device__ __forceinline__ void next(int tiles, const int32_t* q_pos, int B, int rate, int N) {
    if (++t == tiles) {
      t = 0;
      if (++r < B) nvis = n_visible(q_pos[r], rate, N);
    }
  }
};
}  // namespace

__global__ void __launch_bounds__(kFThreads, 1) indexer_decode_fp4_kernel(
    const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales,
    const __grid_constant__ CUtensorMap tm_q, const float* __restrict__ w_idx, const int32_t* __restrict__ q_pos,
    int B, int N, int rate, int tiles_per_req, float* __restrict__ scores, long long ld_scores,
    int* __restrict__ hist_g) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = tc::smem_align1024(smem_raw);
  unsigned char* k_smem = base;                                   // [kFBuf][2][128][128 B] bf16, swizzled
  unsigned char* q_smem = k_smem + kFBuf * kFTileBytes;           // [2][2][64][128 B]
  unsigned char* st_smem = q_smem + 2 * kFQBytes;                 // [kFStages][codes 8 KiB | scales 512 B]
  FBars* bars = reinterpret_cast<FBars*>(st_smem + kFStages * kFStageStride);
  int* s_hist = reinterpret_cast<int*>(bars + 1);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long total = (long long)B * tiles_per_req;
  const long long g0 = total * blockIdx.x / gridDim.x;
  const long long g1 = total * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages; ++s) {
      tc::mbar_init(&bars->sfull[s], 1);
      tc::mbar_init(&bars->sempty[s], kFConvWarps);
    }
    for (int b = 0; b < kFBuf; ++b) {
      tc::mbar_init(&bars->cfull[b], kFConvWarps);
      tc::mbar_init(&bars->bempty[b], 1);
    }
    for (int a = 0; a < kFAcc; ++a) { tc::mbar_init(&bars->tfull[a], 1); tc::mbar_init(&bars->tempty[a], 4); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&bars->qfull[b], 1); tc::mbar_init(&bars->qempty[b], 1); }
    tc::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (hist_g)
    for (int i = threadIdx.x; i < kHistBins; i += kFThreads) s_hist[i] = 0;
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kFTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_codes);
      tc::tma_prefetch_desc(&tm_scales);
      tc::tma_prefetch_desc(&tm_q);
      int it = 0, rq = 0, cur_r = -1;
      TileWalk tw(g0, tiles_per_req, q_pos, B, rate, N);
      for (long long g = g0; g < g1; ++g, tw.next(tiles_per_req, q_pos, B, rate, N)) {
        const int r = tw.r;
        const int row0 = tw.t * kFTile;
        if (row0 >= tw.nvis) continue;
        if (r != cur_r) {
          const int qb = rq & 1;
          if (!tc::mbar_wait(&bars->qempty[qb], ((rq >> 1) & 1) ^ 1, abort)) break;
          tc::mbar_arrive_expect_tx(&bars->qfull[qb], kFQBytes);
          tc::tma_load_2d(q_smem + qb * kFQBytes, &tm_q, &bars->qfull[qb], 0, r * kFHeads);
          tc::tma_load_2d(q_smem + qb * kFQBytes + kFQChunkBytes, &tm_q, &bars->qfull[qb], 64, r * kFHeads);
          cur_r = r;
          ++rq;
        }
        const int s = it % kFStages;
        if (!tc::mbar_wait(&bars->sempty[s], ((it / kFStages) & 1) ^ 1, abort)) break;
        tc::mbar_arrive_expect_tx(&bars->sfull[s], kFCodeBytes + kFScaleBytes);
        unsigned char* slot = st_smem + s * kFStageStride;
        tc::tma_load_3d(slot, &tm_codes, &bars->sfull[s], 0, row0 / 2, r);              // [64][128 B]
        tc::tma_load_3d(slot + kFCodeBytes, &tm_scales, &bars->sfull[s], 0, row0 / 4, r);  // [32][16 B]
        ++it;
      }
      // make sure no copy of ours is still landing in shared memory
      for (int j = (it > kFStages ? it - kFStages : 0); j < it; ++j) {
        for (uint32_t i = 0; i < tc::kSpinLimit && !tc::mbar_try_wait(&bars->sfull[j % kFStages], (j / kFStages) & 1);
             ++i)
          __nanosleep(64);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kFTile, kFHeads, false, false);
      const uint32_t k_base = tc::smem_u32(k_smem), q_base = tc::smem_u32(q_smem);
      int it = 0, rq = 0, cur_r = -1, qb = 0;
      TileWalk tw(g0, tiles_per_req, q_pos, B, rate, N);
      for (long long g = g0; g < g1; ++g, tw.next(tiles_per_req, q_pos, B, rate, N)) {
        const int r = tw.r;
        const int row0 = tw.t * kFTile;
        if (row0 >= tw.nvis) continue;
        if (r != cur_r) {
          if (cur_r >= 0) tc::mma_commit(&bars->qempty[qb]);
          qb = rq & 1;
          if (!tc::mbar_wait(&bars->qfull[qb], (rq >> 1) & 1, abort)) break;
          tc::fence_after_sync();
          cur_r = r;
          ++rq;
        }
        const int b = it % kFBuf;
        const int a = it % kFAcc;
        if (!tc::mbar_wait(&bars->cfull[b], (it / kFBuf) & 1, abort)) break;
        if (!tc::mbar_wait(&bars->tempty[a], ((it / kFAcc) & 1) ^ 1, abort)) break;
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < kFDim / 16; ++k) {
          const uint32_t koff = (k >> 2) * kFChunkBytes + (k & 3) * 32;
          const uint32_t qoff = (k >> 2) * kFQChunkBytes + (k & 3) * 32;
          const uint64_t ad = tc::sdesc_sw128(k_base + b * kFTileBytes + koff, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(q_base + qb * kFQBytes + qoff, 16, 1024);
          tc::mma_bf16(tmem + a * kFHeads, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars->bempty[b]);
        tc::mma_commit(&bars->tfull[a]);
        ++it;
      }
      tc::mma_commit(&bars->drain);
      for (uint32_t i = 0; i < tc::kSpinLimit && !tc::mbar_try_wait(&bars->drain, 0); ++i) __nanosleep(64);
    }
  } else if (warp < 6) {
    // ------------------------------ epilogue ------------------------------
    const int lq = warp & 3;
    const int row_in_tile = lq * 32 + lane;
    const int et = (warp - 2) * 32 + lane;
    float w[kFHeads];
    int it = 0, cur_r = -1;
    bool failed = false;
    auto flush = [&](int r) {
      if (tc::named_bar_or(1, 128, failed || *abort)) { failed = true; return; }
#pragma unroll 4
      for (int b = et * (kHistBins / 128); b < (et + 1) * (kHistBins / 128); ++b) {
        const int c = s_hist[b];
        if (c) {
          atomicAdd(hist_g + (long long)r * kHistBins + b, c);
          s_hist[b] = 0;
        }
      }
      tc::named_bar(1, 128);
    };
    TileWalk tw(g0, tiles_per_req, q_pos, B, rate, N);
    for (long long g = g0; g < g1; ++g, tw.next(tiles_per_req, q_pos, B, rate, N)) {
      const int r = tw.r;
      const int row0 = tw.t * kFTile;
      const int nvis = tw.nvis;
      if (row0 >= nvis) continue;
      if (r != cur_r) {
        if (hist_g && cur_r >= 0) flush(cur_r);
#pragma unroll
        for (int j = 0; j < kFHeads; ++j) w[j] = w_idx[(long long)r * kFHeads + j];
        cur_r = r;
      }
      const int a = it % kFAcc;
      ++it;
      if (!failed) failed = !tc::warp_wait(&bars->tfull[a], ((it - 1) / kFAcc) & 1, abort);
      if (failed) continue;
      tc::fence_after_sync();
      uint32_t v[kFHeads];
      const uint32_t taddr = tmem + ((uint32_t)(lq * 32) << 16) + a * kFHeads;
      tc::tmem_ld32(taddr, v);
      tc::tmem_ld32(taddr + 32, v + 32);
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->tempty[a]);
      float sc0 = 0.f, sc1 = 0.f;
#pragma unroll
      for (int j = 0; j < kFHeads; j += 2) {
        sc0 = fmaf(w[j], fmaxf(__uint_as_float(v[j]), 0.f), sc0);
        sc1 = fmaf(w[j + 1], fmaxf(__uint_as_float(v[j + 1]), 0.f), sc1);
      }
      const int e = row0 + row_in_tile;
      const float sc = __bfloat162float(__float2bfloat16_rn(sc0 + sc1));  // BF16 index scores
      if (e < nvis) scores[(long long)r * ld_scores + e] = sc;
      if (hist_g) {
        const uint32_t bin = e < nvis ? float_key(sc) >> 20 : 0xffffffffu;
        const unsigned same = __match_any_sync(0xffffffffu, bin);
        if (e < nvis && (int)(__ffs(same) - 1) == lane) atomicAdd(s_hist + bin, __popc(same));
      }
    }
    if (hist_g && cur_r >= 0) flush(cur_r);
  } else {
    // ------------------------------ converters ------------------------------
    // thread ci widens half a key row of each tile: row ci % 128, 64-dim chunk ci / 128
    // (its 32 code bytes and 2 block scales) -> bf16, written in the K-major
    // 128B-swizzled layout (16-byte unit u of the chunk at row * 128 + ((u ^ (row & 7)) * 16)).
    const int ci = threadIdx.x - kFConv0;
    const int crw = ci & (kFTile - 1), chh = ci >> 7;
    int it = 0;
    TileWalk tw(g0, tiles_per_req, q_pos, B, rate, N);
    for (long long g = g0; g < g1; ++g, tw.next(tiles_per_req, q_pos, B, rate, N)) {
      if (tw.t * kFTile >= tw.nvis) continue;
      const int s = it % kFStages, b = it % kFBuf;
      if (!tc::warp_wait(&bars->sfull[s], (it / kFStages) & 1, abort)) break;
      if (!tc::warp_wait(&bars->bempty[b], ((it / kFBuf) & 1) ^ 1, abort)) break;
      const unsigned char* slot = st_smem + s * kFStageStride;
      const uint4* crow = reinterpret_cast<const uint4*>(slot + crw * 64 + chh * 32);
      const uint32_t sc2 = *reinterpret_cast<const uint32_t*>(slot + kFCodeBytes + crw * 4) >> (16 * chh);
      unsigned char* trow = k_smem + b * kFTileBytes + chh * kFChunkBytes + crw * 128;
#pragma unroll
      for (int q = 0; q < 2; ++q) {  // 32-dim block q of the chunk: codes crow[q], scale byte q
        const uint4 cw = crow[q];
        const int X = (int)((sc2 >> (8 * q)) & 0xffu) - 127;
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // 8 dims: unit 4q + h of the chunk
          uint32_t o[4];
          e2m1x8_to_bf16(words[h], X, o);
          const int uu = 4 * q + h;
          *reinterpret_cast<uint4*>(trow + ((uu ^ (crw & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      tc::fence_proxy_async_smem();  // the tensor cores read the tile through the async proxy
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&bars->cfull[b]);
        tc::mbar_arrive(&bars->sempty[s]);
      }
      ++it;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && bars->abort) atomicOr(&g_indexer_fp4_error, 1u);
  if (warp == 1) tc::tmem_dealloc(tmem, kFTmemCols);
}

namespace {
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn_fp4() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// byte tensor map, no swizzle, rank 3, box = {box_x bytes, box_rows, 1}
cudaError_t make_tmap_u8(CUtensorMap* m, const void* ptr, const uint64_t* dims, const uint64_t* strides_bytes,
                         uint32_t box_x, uint32_t box_rows) {
  auto fn = encode_fn_fp4();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t gdim[3] = {dims[0], dims[1], dims[2]}, gstride[2] = {strides_bytes[0], strides_bytes[1]};
  cuuint32_t box[3] = {box_x, box_rows, 1}, estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), gdim, gstride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

extern cudaError_t make_tmap_bf16(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                                  const uint64_t* strides_bytes, uint32_t box_rows);

cudaError_t launch_mxfp4_quantize(const void* x, bool x_f32, long long ld_x, int rows, int d, uint8_t* codes,
                                  long long ld_codes, uint8_t* scales, long long ld_scales, cudaStream_t stream) {
  const long long n = (long long)rows * (d / 32);
  if (n <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (x_f32)
    mxfp4_quantize_kernel<true><<<grid, 256, 0, stream>>>(x, ld_x, rows, d, codes, ld_codes, scales, ld_scales);
  else
    mxfp4_quantize_kernel<false><<<grid, 256, 0, stream>>>(x, ld_x, rows, d, codes, ld_codes, scales, ld_scales);
  ++g_launch_counter;
  return cudaGetLastError();
}

cudaError_t launch_mxfp4_roundtrip(const bf16* x, int rows, int d, bf16* y, cudaStream_t stream) {
  const long long n = (long long)rows * (d / 32);
  if (n <= 0) return cudaSuccess;
  mxfp4_roundtrip_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(x, rows, d, y);
  ++g_launch_counter;
  return cudaGetLastError();
}

cudaError_t launch_indexer_decode_fp4(const bf16* q4, const float* w_idx, const uint8_t* k_codes,
                                      const uint8_t* k_scales, long long k_seq_stride, int N, const int32_t* q_pos,
                                      int B, int rate, float* scores, long long ld_scores, int num_sms,
                                      cudaStream_t stream, int* hist) {
  if (B == 0 || N == 0) return cudaSuccess;
  CUtensorMap tm_codes, tm_scales, tm_q;
  const long long per_req = B > 1 ? k_seq_stride : (long long)(N + 3) / 4 * 4;  // keys between requests
  // codes as 128-byte rows of two keys (contiguous, so the staged bytes are the same as
  // key rows of 64 B): half the row requests of 64-byte rows
  const uint64_t cd[3] = {128, (uint64_t)(N + 3) / 4 * 2, (uint64_t)B};
  const uint64_t cs[2] = {128, (uint64_t)per_req * 64};
  cudaError_t e = make_tmap_u8(&tm_codes, k_codes, cd, cs, 128, kFTile / 2);
  if (e != cudaSuccess) return e;
  const uint64_t sd[3] = {16, (uint64_t)(N + 3) / 4, (uint64_t)B};
  const uint64_t ss[2] = {16, (uint64_t)per_req * 4};
  e = make_tmap_u8(&tm_scales, k_scales, sd, ss, 16, kFTile / 4);
  if (e != cudaSuccess) return e;
  const uint64_t qd[2] = {(uint64_t)kFDim, (uint64_t)B * kFHeads};
  const uint64_t qs[1] = {(uint64_t)kFDim * 2};
  e = make_tmap_bf16(&tm_q, q4, 2, qd, qs, kFHeads);
  if (e != cudaSuccess) return e;
  const int tiles_per_req = (N + kFTile - 1) / kFTile;
  const long long total = (long long)B * tiles_per_req;
  const int grid = (int)(total < num_sms ? total : num_sms);
  e = cudaFuncSetAttribute((const void*)indexer_decode_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kFSmemBytes);
  if (e != cudaSuccess) return e;
  indexer_decode_fp4_kernel<<<grid, kFThreads, kFSmemBytes, stream>>>(tm_codes, tm_scales, tm_q, w_idx, q_pos, B, N,
                                                                      rate, tiles_per_req, scores, ld_scores, hist);
  ++g_launch_counter;
  return cudaGetLastError();
}

unsigned int read_and_clear_indexer_fp4_error() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_indexer_fp4_error, sizeof(v)) != cudaSuccess) return 0xffffffffu;
  if (v) cudaMemcpyToSymbol(g_indexer_fp4_error, &zero, sizeof(zero));
  return v;
}

}  // namespace hca
