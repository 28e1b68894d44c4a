// Shared-KV multi-query attention on the 5th-generation tensor cores (sm_100a),
// decode shape: one query (64 heads x 512) per request, split over CTAs along
// its row list, partial softmax states merged by the combine kernel.
//
// What it computes (QbitAI write-up, "混合注意力機制": CSA step three, KV
// entries act as both key and value, sliding-window branch; "DeepSeek V4
// Architecture Tricks", HCA section):
//   o[h, :] = sum_u softmax_u(scale * q[h, :] . row_u) row_u
// over U = selected CSA entries (idx) or all visible HCA entries, then the
// window rows.
//
// Design.  Rows are the MMA's M dimension and heads its N dimension, so one
// 64-row KV tile staged in shared memory (128B-swizzled, eight 64-dim
// chunks) serves as the K-major A operand of S^T = R . Q^T and, read
// MN-major, as the A operand of O^T += V^T . P^T.  Shared memory holds Q
// (64 KiB) and two 64-row stages interleaved per chunk (128 KiB); the
// QK^T MMA runs with M = 128 and reads the other stage's rows as its upper
// 64 rows, whose results are ignored (decode is bandwidth-bound; the MMA
// has time to spare).  Dense rows arrive as TMA tiles, selected rows as
// tile::gather4 loads of four 1 KiB rows per 64-dim chunk.
//   warp 0     producer (all lanes issue loads)
//   warp 1     MMA issuer; QK^T of tile i+1 overlaps the softmax of tile i
//   warps 4,5  softmax of the 64 rows (TMEM lanes 0..63): per-head tile
//              maximum by a warp reduce-scatter, P = 2^(s - m) written to
//              shared memory as two bf16 terms P_hi + P_lo (MN-major B
//              operands of PV; two MMAs give P ~16 significant bits)
//   warps 2..5 lazy rescale of the TMEM accumulators (only when a head's
//              maximum grows by more than 2^8) and the final epilogue
// Row sums l_h come from a small MMA of a ones matrix with P^T, so they use
// exactly the bf16 P that the PV product uses.
// TMEM: S^T 2 x 64 columns, O^T 4 blocks x 64, l 64.

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hca {

namespace {
constexpr int kThreads = 192;
constexpr int kRows = 64;
constexpr int kC = 512;
constexpr int kH = 64;
constexpr int kChunks = kC / 64;
constexpr uint32_t kQBytes = kH * kC * 2;            // 64 KiB
constexpr uint32_t kQChunk = kH * 128;               // 8 KiB
constexpr uint32_t kStageOff = kRows * 128;          // 8 KiB (stage within a chunk)
constexpr uint32_t kKvChunk = 2 * kStageOff;         // 16 KiB (both stages of a chunk)
constexpr uint32_t kKvBytes = kChunks * kKvChunk;    // 128 KiB
constexpr uint32_t kTileBytes = kRows * kC * 2;      // 64 KiB per stage
constexpr uint32_t kPBytes = kRows * kH * 2;         // 8 KiB
constexpr uint32_t kOnesBytes = 128 * 16 * 2;        // 4 KiB
constexpr uint32_t kOffQ = 0, kOffKv = kQBytes, kOffP = kOffKv + kKvBytes, kOffOnes = kOffP + 2 * kPBytes,
                   kOffBars = kOffOnes + kOnesBytes;
constexpr uint32_t kColS = 0, kColO = 128, kColL = 384, kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;

struct __align__(8) Bars {
  uint64_t qfull, kvfull[2], kvempty[2], sfull[2], sempty[2], pfull[2], odone, drain;
  uint32_t tmem_base;
  int abort;
  int rescale;
  float red[2][kH];
  float mref[kH];
  float alpha[kH];
};
constexpr size_t kSmemBytes = 1024 + kOffBars + sizeof(Bars);

struct Tile {
  int seg;    // 0: entries, 1: window
  int row0;   // first row within the segment
  int nrows;  // valid rows
};

// Tiles of one split: the split's range of the row list cut at the
// entries/window boundary, 64 rows per tile.
struct SplitTiles {
  int a0, a1, b0, b1, na, nb;
  __device__ __forceinline__ SplitTiles(int n_first, int n_win, int ub, int ue) {
    a0 = ub;
    a1 = min(ue, n_first);
    if (a1 < a0) a1 = a0;
    b0 = max(ub, n_first) - n_first;
    b1 = ue - n_first;
    if (b1 < b0) b1 = b0;
    if (b1 > n_win) b1 = n_win;
    if (b0 > b1) b0 = b1;
    na = (a1 - a0 + kRows - 1) / kRows;
    nb = (b1 - b0 + kRows - 1) / kRows;
  }
  __device__ __forceinline__ int count() const { return na + nb; }
  __device__ __forceinline__ Tile get(int i) const {
    Tile t;
    if (i < na) {
      t.seg = 0;
      t.row0 = a0 + i * kRows;
      t.nrows = min(kRows, a1 - t.row0);
    } else {
      t.seg = 1;
      t.row0 = b0 + (i - na) * kRows;
      t.nrows = min(kRows, b1 - t.row0);
    }
    return t;
  }
};

// One reduce-scatter step over lane bit O: of the n values held, keep the
// half selected by the bit and fold in the partner's copy of that half.
template <int O, int NV>
__device__ __forceinline__ void rs_max_step(float (&a)[kH], int lane) {
  const bool hi = (lane & O) != 0;
#pragma unroll
  for (int j = 0; j < NV / 2; ++j) {
    const float send = hi ? a[j] : a[j + NV / 2];
    const float keep = hi ? a[j + NV / 2] : a[j];
    a[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, O));
  }
}
// Afterwards lane l holds the warp-wide maxima of heads 2l and 2l+1 (62 shuffles).
__device__ __forceinline__ void warp_max2(float (&a)[kH], int lane, float (&out)[2]) {
  rs_max_step<16, 64>(a, lane);
  rs_max_step<8, 32>(a, lane);
  rs_max_step<4, 16>(a, lane);
  rs_max_step<2, 8>(a, lane);
  rs_max_step<1, 4>(a, lane);
  out[0] = a[0];
  out[1] = a[1];
}
}  // namespace

__device__ unsigned int g_mqa_tc_error = 0;

struct MqaTcParams {
  const int32_t* idx;      // [Tq, n_idx] or nullptr
  int n_idx;
  const int32_t* q_pos;
  int rate, N, n_win;
  int prefill;                // one sequence (window = raw token rows) rather than per-request blocks
  long long kv_rows_stride;   // rows between requests in the kv map
  long long win_rows_stride;  // rows between requests in the window map
  float scale_log2;
  int splits, rows_per_split;
  bf16* out;
  float* ws_o;
  float2* ws_ml;
};

__global__ void __launch_bounds__(kThreads, 1) mqa_decode_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
    const __grid_constant__ CUtensorMap tm_kvg, const __grid_constant__ CUtensorMap tm_win, MqaTcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(base + kOffBars);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = blockIdx.x / p.splits;
  const int sp = blockIdx.x % p.splits;

  // this query's row list
  const int t_pos = p.q_pos[q];
  const int n_first = p.idx ? p.n_idx : n_visible(t_pos, p.rate, p.N);
  const int n_win = min(p.n_win, t_pos + 1);
  const int ub = sp * p.rows_per_split;
  const int ue = min(n_first + n_win, ub + p.rows_per_split);
  const SplitTiles tiles(n_first, n_win, ub, max(ub, ue));
  const int nt = tiles.count();
  const int32_t* idx_q = p.idx ? p.idx + (long long)q * p.n_idx : nullptr;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->qfull, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->kvfull[s], 1);
      tc::mbar_init(&bars->kvempty[s], 1);
      tc::mbar_init(&bars->sfull[s], 1);
      tc::mbar_init(&bars->sempty[s], 2);
      tc::mbar_init(&bars->pfull[s], 2);
    }
    tc::mbar_init(&bars->odone, 1);
    tc::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    bars->rescale = 0;
    tc::fence_mbar_init();
  }
  // ones matrix for the row-sum MMA (4 KiB of bf16 1.0)
  for (int i = threadIdx.x; i < (int)(kOnesBytes / 16); i += kThreads)
    reinterpret_cast<uint4*>(base + kOffOnes)[i] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  for (int h = threadIdx.x; h < kH; h += kThreads) { bars->mref[h] = neg_inf(); bars->alpha[h] = 1.f; }
  tc::fence_proxy_async_smem();
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_kv);
      tc::mbar_arrive_expect_tx(&bars->qfull, kQBytes);
      for (int c = 0; c < kChunks; ++c) tc::tma_load_2d(base + kOffQ + c * kQChunk, &tm_q, &bars->qfull, c * 64, q * kH);
    }
    // decode: request q's cache and window block; prefill: one sequence whose
    // window is the raw token rows [max(0, t - n_win + 1), t]
    const long long kv_row_base = p.prefill ? 0ll : (long long)q * p.kv_rows_stride;
    const long long win_row_base = p.prefill ? (long long)max(0, t_pos - p.n_win + 1)
                                             : (long long)q * p.win_rows_stride;
    int i = 0;
    for (; i < nt; ++i) {
      const Tile t = tiles.get(i);
      const int s = i & 1;
      bool ok = true;
      if (lane == 0) {
        ok = tc::mbar_wait(&bars->kvempty[s], ((i >> 1) & 1) ^ 1, abort);
        if (ok) tc::mbar_arrive_expect_tx(&bars->kvfull[s], kTileBytes);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      unsigned char* st = base + kOffKv + s * kStageOff;
      if (t.seg == 0 && idx_q != nullptr) {
        // gathered rows: lane g < 16 loads rows 4g..4g+3 (invalid slots read row 0, masked later)
        if (lane < 16) {
          int y[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = 4 * lane + j;
            int e = r < t.nrows ? idx_q[t.row0 + r] : 0;
            if (e < 0 || e >= p.N) e = 0;
            y[j] = (int)(kv_row_base + e);
          }
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
            tc::tma_gather4(st + c * kKvChunk + lane * 512, &tm_kvg, &bars->kvfull[s], c * 64, y[0], y[1], y[2], y[3]);
        }
      } else if (lane < kChunks) {
        const int c = lane;
        if (t.seg == 0)
          tc::tma_load_2d(st + c * kKvChunk, &tm_kv, &bars->kvfull[s], c * 64, (int)(kv_row_base + t.row0));
        else
          tc::tma_load_2d(st + c * kKvChunk, &tm_win, &bars->kvfull[s], c * 64, (int)(win_row_base + t.row0));
      }
      __syncwarp();
    }
    // drain: every stage we filled has landed before the CTA may exit
    if (lane == 0) {
      for (int j = (i > 2 ? i - 2 : 0); j < i; ++j)
        for (uint32_t k = 0; k < tc::kSpinLimit && !tc::mbar_try_wait(&bars->kvfull[j & 1], (j >> 1) & 1); ++k)
          __nanosleep(64);
      for (uint32_t k = 0; k < tc::kSpinLimit && !tc::mbar_try_wait(&bars->qfull, 0); ++k) __nanosleep(64);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t id_qk = tc::idesc_bf16_f32(128, kH, false, false);
      constexpr uint32_t id_pv = tc::idesc_bf16_f32(128, kH, true, true);
      constexpr uint32_t id_l = tc::idesc_bf16_f32(128, kH, false, true);
      const uint32_t q_base = tc::smem_u32(base + kOffQ), kv_base = tc::smem_u32(base + kOffKv),
                     p_base = tc::smem_u32(base + kOffP), ones = tc::smem_u32(base + kOffOnes);
      const uint64_t q_desc0 = tc::sdesc_sw128(q_base, 16, 1024);
      const uint64_t p_hi_desc0 = tc::sdesc_sw128(p_base, kPBytes, 1024);
      const uint64_t p_lo_desc0 = tc::sdesc_sw128(p_base + kPBytes, kPBytes, 1024);
      const uint64_t ones_desc = tc::sdesc_noswz(ones, 128, 256);
      bool ok = tc::mbar_wait(&bars->qfull, 0, abort);
      auto issue_qk = [&](int j) -> bool {
        const int s = j & 1;
        if (!tc::mbar_wait(&bars->kvfull[s], (j >> 1) & 1, abort)) return false;
        if (!tc::mbar_wait(&bars->sempty[s], ((j >> 1) & 1) ^ 1, abort)) return false;
        tc::fence_after_sync();
        // Descriptors are built once; each K-step only adds a compile-time
        // offset (>> 4) to the start-address field, which keeps the single
        // issuing thread from becoming the bottleneck.
        const uint64_t a0 = tc::sdesc_sw128(kv_base + s * kStageOff, 16, 1024);
        const uint32_t d_s = tmem + kColS + s * kH;
#pragma unroll
        for (int k = 0; k < kC / 16; ++k) {
          const uint32_t aoff = ((k >> 2) * kKvChunk + (k & 3) * 32) >> 4;
          const uint32_t boff = ((k >> 2) * kQChunk + (k & 3) * 32) >> 4;
          tc::mma_bf16(d_s, a0 + aoff, q_desc0 + boff, id_qk, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars->sfull[s]);
        return true;
      };
      if (ok && nt > 0) ok = issue_qk(0);
      // Issue whichever is ready first: QK^T of the next tile (its rows have
      // landed and its S buffer is free) or PV of the oldest tile whose P is
      // published.  QK(j) runs at most one tile ahead of PV, so every barrier
      // is waited on at most one phase ahead.
      int next_qk = 1;
      for (int i = 0; ok && i < nt; ++i) {
        const int s = i & 1;
        uint32_t spins = 0;
        for (;;) {
          if (next_qk < nt && next_qk <= i + 1 && tc::mbar_try_wait(&bars->kvfull[next_qk & 1], (next_qk >> 1) & 1) &&
              tc::mbar_try_wait(&bars->sempty[next_qk & 1], ((next_qk >> 1) & 1) ^ 1)) {
            ok = issue_qk(next_qk);  // both waits inside succeed at once
            ++next_qk;
            if (!ok) break;
            continue;
          }
          if (tc::mbar_try_wait(&bars->pfull[0], i & 1)) break;  // P(i) ready
          if (++spins > tc::kSpinLimit || *abort) { *abort = 1; ok = false; break; }
          if ((spins & 255u) == 0) __nanosleep(64);
        }
        if (!ok) break;
        tc::fence_after_sync();
        const uint64_t va0 = tc::sdesc_sw128(kv_base + s * kStageOff, kKvChunk, 1024);
        const uint32_t acc0 = i > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {
          const uint64_t bhi = p_hi_desc0 + ((kk * 2048) >> 4);
          const uint64_t blo = p_lo_desc0 + ((kk * 2048) >> 4);
          const uint32_t first = kk > 0 ? 1u : acc0;
#pragma unroll
          for (int mb = 0; mb < 4; ++mb) {
            const uint64_t ad = va0 + (((2 * mb) * kKvChunk + kk * 2048) >> 4);
            tc::mma_bf16(tmem + kColO + mb * kH, ad, bhi, id_pv, first);
            tc::mma_bf16(tmem + kColO + mb * kH, ad, blo, id_pv, 1u);
          }
          tc::mma_bf16(tmem + kColL, ones_desc, bhi, id_l, first);
          tc::mma_bf16(tmem + kColL, ones_desc, blo, id_l, 1u);
        }
        tc::mma_commit(&bars->kvempty[s]);
        tc::mma_commit(&bars->odone);
      }
      tc::mma_commit(&bars->drain);
      for (uint32_t k = 0; k < tc::kSpinLimit && !tc::mbar_try_wait(&bars->drain, 0); ++k) __nanosleep(64);
    }
  } else {
    // ------------------------------ softmax / correction / epilogue ------------------------------
    const int quarter = warp & 3;                  // TMEM lane quarter
    const bool smx = quarter < 2;                  // warps 4, 5: rows 0..63
    const int row = quarter * 32 + lane;           // S^T lane (softmax) / O^T lane
    const int st = (warp - 2) * 32 + lane;         // 0..127 within the compute group
    const int sm_t = row;                          // 0..63 for the softmax threads
    // Every named barrier below is reached by all of its participants on every
    // iteration; failures are agreed through bar.red.or before anyone leaves.
    bool failed = false;
    for (int i = 0; i < nt; ++i) {
      const Tile t = tiles.get(i);
      const int s = i & 1;
      float sv[kH];
      if (smx) {
        if (!failed) failed = !tc::warp_wait(&bars->sfull[s], (i >> 1) & 1, abort);
        if (!failed) {
          tc::fence_after_sync();
          uint32_t v[kH];
          const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + kColS + s * kH;
          tc::tmem_ld32(ta, v);
          tc::tmem_ld32(ta + 32, v + 32);
          tc::tmem_ld_wait();
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bars->sempty[s]);
          bool valid = row < t.nrows;
          if (valid && t.seg == 0 && idx_q != nullptr) {
            const int e = idx_q[t.row0 + row];
            valid = e >= 0 && e < p.N;
          }
#pragma unroll
          for (int h = 0; h < kH; ++h) sv[h] = valid ? __uint_as_float(v[h]) * p.scale_log2 : neg_inf();
          float tmp[kH];
#pragma unroll
          for (int h = 0; h < kH; ++h) tmp[h] = sv[h];
          float m2[2];
          warp_max2(tmp, lane, m2);
          bars->red[quarter][2 * lane] = m2[0];
          bars->red[quarter][2 * lane + 1] = m2[1];
        }
        tc::named_bar(1, 64);
        if (!failed) {
          const int h = sm_t;
          const float mt = fmaxf(bars->red[0][h], bars->red[1][h]);
          const float mo = bars->mref[h];
          if (mt > mo + kRescaleLog2 || (mo == neg_inf() && mt != neg_inf())) {
            bars->alpha[h] = (mo == neg_inf()) ? 0.f : fast_exp2(mo - mt);
            bars->mref[h] = mt;
            bars->rescale = 1;
          } else {
            bars->alpha[h] = 1.f;
          }
        }
      }
      if (tc::named_bar_or(2, 128, failed || *abort)) { failed = true; break; }
      if (i > 0) {
        // Wait for PV(i-1) on every tile, in order: the odone barrier completes once per
        // tile, and a parity wait is only unambiguous while the waiter is at most one
        // phase behind (PV(i) cannot complete before this group publishes P(i)).
        if (!tc::warp_wait(&bars->odone, (i - 1) & 1, abort)) failed = true;
      }
      if (bars->rescale && i > 0) {
        // O^T and l hold the sums up to tile i-1: scale column h by alpha[h]
        if (!failed) {
          tc::fence_after_sync();
          const uint32_t lanebase = (uint32_t)(quarter * 32) << 16;
#pragma unroll 1
          for (int blk = 0; blk < 5; ++blk) {
            const uint32_t ta = tmem + lanebase + (blk < 4 ? kColO + blk * kH : kColL);
            uint32_t v[kH];
            tc::tmem_ld32(ta, v);
            tc::tmem_ld32(ta + 32, v + 32);
            tc::tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < kH; ++h) v[h] = __float_as_uint(__uint_as_float(v[h]) * bars->alpha[h]);
            tc::tmem_st32(ta, v);
            tc::tmem_st32(ta + 32, v + 32);
          }
          tc::tmem_st_wait();
          tc::fence_before_sync();
        }
      }
      if (tc::named_bar_or(2, 128, failed || *abort)) { failed = true; break; }
      if (smx) {
        if (sm_t == 0) bars->rescale = 0;
        // PV(i-1), the last reader of the P buffer, has completed (waited above).
        // P = P_hi + P_lo, both bf16: the PV and row-sum MMAs run on both halves,
        // so the probabilities carry ~16 significant bits instead of 8.
        unsigned char* phi = base + kOffP + row * 128;
        unsigned char* plo = phi + kPBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t wh[4], wl[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int h = c * 8 + 2 * j;
            const float m0 = bars->mref[h], m1 = bars->mref[h + 1];
            const float p0 = (m0 == neg_inf()) ? 0.f : fast_exp2(sv[h] - m0);
            const float p1 = (m1 == neg_inf()) ? 0.f : fast_exp2(sv[h + 1] - m1);
            wh[j] = pack_bf16x2(p0, p1);
            wl[j] = pack_bf16x2(p0 - bf16_lo(wh[j]), p1 - bf16_hi(wh[j]));
          }
          const uint32_t sw = (uint32_t)((c ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(phi + sw) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          *reinterpret_cast<uint4*>(plo + sw) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->pfull[0]);
      }
    }
    // ---- epilogue: O^T (dims x heads) and l ----
    bool ok = !failed;
    if (ok && nt > 0) ok = tc::warp_wait(&bars->odone, (nt - 1) & 1, abort);
    if (ok) {
      tc::fence_after_sync();
      const uint32_t lanebase = (uint32_t)(quarter * 32) << 16;
      uint32_t lv[kH];
      if (nt > 0) {
        tc::tmem_ld32(tmem + lanebase + kColL, lv);
        tc::tmem_ld32(tmem + lanebase + kColL + 32, lv + 32);
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int h = 0; h < kH; ++h) lv[h] = 0u;
      }
      const int dim_lane = quarter * 32 + lane;
      if (p.splits == 1) {
        bf16* op = p.out + (long long)q * kH * kC;
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
          uint32_t v[kH];
          if (nt > 0) {
            tc::tmem_ld32(tmem + lanebase + kColO + mb * kH, v);
            tc::tmem_ld32(tmem + lanebase + kColO + mb * kH + 32, v + 32);
            tc::tmem_ld_wait();
          }
          const int d = mb * 128 + dim_lane;
#pragma unroll
          for (int h = 0; h < kH; ++h) {
            const float l = __uint_as_float(lv[h]);
            const float o = (nt > 0 && l > 0.f) ? __uint_as_float(v[h]) / l : 0.f;
            op[h * kC + d] = __float2bfloat16_rn(o);
          }
        }
      } else {
        float* wo = p.ws_o + ((long long)q * p.splits + sp) * kH * kC;
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
          uint32_t v[kH];
          if (nt > 0) {
            tc::tmem_ld32(tmem + lanebase + kColO + mb * kH, v);
            tc::tmem_ld32(tmem + lanebase + kColO + mb * kH + 32, v + 32);
            tc::tmem_ld_wait();
          }
          const int d = mb * 128 + dim_lane;
#pragma unroll
          for (int h = 0; h < kH; ++h) wo[h * kC + d] = nt > 0 ? __uint_as_float(v[h]) : 0.f;
        }
        if (st < kH) {
          float l = 0.f;  // lv[st] without a dynamically indexed register array
#pragma unroll
          for (int h = 0; h < kH; ++h) l = (h == st && nt > 0) ? __uint_as_float(lv[h]) : l;
          p.ws_ml[((long long)q * p.splits + sp) * kH + st] = make_float2(l > 0.f ? bars->mref[st] : neg_inf(), l);
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && bars->abort) atomicOr(&g_mqa_tc_error, 1u);
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- host side ------------------------------------------------------------------
bool mqa_tc_supported(const MqaProblem& p) {
  if (p.H != kH || p.c != kC || p.n_win > 256) return false;
  if (p.mode == HCA_MODE_PREFILL) return p.win_rows > 0;
  return p.mode == HCA_MODE_DECODE && p.kv_seq_stride % kC == 0 && p.win_seq_stride % kC == 0;
}

// Splits per query: one wave of at most num_sms CTAs, fewest tiles per CTA.
MqaPlan plan_mqa_tc(const MqaProblem& p, int num_sms) {
  MqaPlan pl;
  const int first = p.idx ? p.n_idx : p.N;
  pl.max_rows = first + p.n_win;
  const int tiles = (first + kRows - 1) / kRows + (p.n_win + kRows - 1) / kRows;
  int best_s = 1;
  long long best_cost = -1;
  const int smax = p.Tq > 0 ? min(1024, max(1, (2 * num_sms) / p.Tq)) : 1;  // combine handles <= 1024
  for (int s = 1; s <= smax && s <= tiles; ++s) {
    const int tpc = (tiles + s - 1) / s;
    const int s_eff = (tiles + tpc - 1) / tpc;
    const long long ctas = (long long)p.Tq * s_eff;
    const long long waves = (ctas + num_sms - 1) / num_sms;
    const long long cost = waves * tpc * 4 + (s_eff > 1 ? 1 : 0);  // tiles on the critical path, + combine
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best_s = s_eff; }
  }
  const int tpc = (tiles + best_s - 1) / best_s;
  pl.splits = best_s;
  pl.rows_per_split = tpc * kRows;
  // A split boundary must not cut a tile of the window segment out of step with
  // the entries segment: rows_per_split is a multiple of 64 and the first
  // segment is tiled from its own start, so splits only ever start on a tile.
  pl.ws_bytes = best_s > 1 ? (size_t)p.Tq * best_s * kH * ((size_t)kC * sizeof(float) + sizeof(float2)) : 0;
  return pl;
}

extern cudaError_t make_tmap_bf16(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                                  const uint64_t* strides_bytes, uint32_t box_rows);

cudaError_t launch_mqa_decode_tc(const MqaProblem& p, const MqaPlan& pl, void* ws, cudaStream_t stream) {
  if (p.Tq == 0) return cudaSuccess;
  CUtensorMap tm_q, tm_kv, tm_kvg, tm_win;
  const uint64_t rstride[1] = {(uint64_t)kC * 2};
  const uint64_t qd[2] = {(uint64_t)kC, (uint64_t)p.Tq * kH};
  cudaError_t e = make_tmap_bf16(&tm_q, p.q, 2, qd, rstride, 64);
  if (e != cudaSuccess) return e;
  const long long kv_rs = p.mode == HCA_MODE_PREFILL ? 0 : p.kv_seq_stride / kC;
  const uint64_t kvd[2] = {(uint64_t)kC, (uint64_t)((long long)(p.Tq - 1) * kv_rs + (p.N > 0 ? p.N : 1))};
  e = make_tmap_bf16(&tm_kv, p.kv, 2, kvd, rstride, 64);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tm_kvg, p.kv, 2, kvd, rstride, 1);
  if (e != cudaSuccess) return e;
  const bool prefill = p.mode == HCA_MODE_PREFILL;
  const long long win_rs = prefill ? 0 : p.win_seq_stride / kC;
  const uint64_t wd[2] = {(uint64_t)kC,
                          prefill ? (uint64_t)p.win_rows : (uint64_t)((long long)(p.Tq - 1) * win_rs + p.n_win)};
  e = make_tmap_bf16(&tm_win, p.win, 2, wd, rstride, 64);
  if (e != cudaSuccess) return e;
  MqaTcParams a;
  a.idx = p.idx;
  a.n_idx = p.n_idx;
  a.q_pos = p.q_pos;
  a.rate = p.rate;
  a.N = p.N;
  a.n_win = p.n_win;
  a.kv_rows_stride = prefill ? 0 : kv_rs;
  a.prefill = prefill ? 1 : 0;
  a.win_rows_stride = win_rs;
  a.scale_log2 = p.scale * kLog2e;
  a.splits = pl.splits;
  a.rows_per_split = pl.rows_per_split;
  a.out = p.out;
  a.ws_o = pl.splits > 1 ? reinterpret_cast<float*>(ws) : nullptr;
  a.ws_ml = pl.splits > 1 ? reinterpret_cast<float2*>(reinterpret_cast<float*>(ws) + (size_t)p.Tq * pl.splits * kH * kC)
                          : nullptr;
  e = cudaFuncSetAttribute((const void*)mqa_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  mqa_decode_tc_kernel<<<p.Tq * pl.splits, kThreads, kSmemBytes, stream>>>(tm_q, tm_kv, tm_kvg, tm_win, a);
  ++g_launch_counter;
  e = cudaGetLastError();
  if (e != cudaSuccess || pl.splits == 1) return e;
  return launch_mqa_combine(a.ws_o, a.ws_ml, p.Tq, pl.splits, kH, kC, p.out, stream);
}

unsigned int read_and_clear_mqa_tc_error() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_mqa_tc_error, sizeof(v)) != cudaSuccess) return 0xffffffffu;
  if (v) cudaMemcpyToSymbol(g_mqa_tc_error, &zero, sizeof(zero));
  return v;
}

}  // namespace hca
