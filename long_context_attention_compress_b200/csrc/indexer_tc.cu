// Lightning-indexer scores on the 5th-generation tensor cores (sm_100a).
//
//   I(t, s) = sum_j w[t, j] * ReLU(q_I[t, j, :] . K_I[s, :])
// (QbitAI write-up, "混合注意力機制", CSA step two; "DeepSeek V4 Architecture
// Tricks", CSA section: 64 indexer heads of dim 128.)
//
// Decode shape: one query per request, the request's whole key cache
// streamed once.  The (request, 128-entry tile) space is split evenly over a
// persistent grid (one CTA per SM).  Per CTA:
//   warp 0      TMA producer: key tiles [128 entries x 128 dims] bf16 (two
//               64-dim 128B-swizzled boxes, 32 KiB, L2 evict-first) into a
//               ring of stages;
//               the request's q_I [64 heads x 128] when the request changes.
//   warp 1      MMA issuer (one thread): S^T[128 entries, 64 heads] =
//               K_tile . q_I^T with eight M=128 N=64 K=16 tcgen05.mma into one
//               of four TMEM accumulators (64 f32 columns each).
//   warps 2..5  epilogue: each thread owns one TMEM lane = one entry, loads
//               its 64 head dot products, applies ReLU and the head weights
//               and writes the entry's score (4 bytes per 256-byte key row).
// The entry is the MMA's M dimension, so the head sum needs no shuffles.
// Every wait is bounded; a CTA that runs out of budget records an error,
// lets its own copies and MMAs drain, frees its TMEM and returns.

#include <cudaTypedefs.h>

#include <cstddef>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hca {

namespace {
constexpr int kStages = 5;
constexpr int kTile = 128;   // entries per tile (MMA M)
constexpr int kHeads = 64;   // indexer heads (MMA N)
constexpr int kDim = 128;    // key dim (MMA K)
constexpr int kAcc = 4;      // TMEM accumulators
constexpr int kTmemCols = kAcc * kHeads;  // 256
constexpr uint32_t kTileBytes = kTile * kDim * 2;   // 32 KiB
constexpr uint32_t kChunkBytes = kTile * 128;       // 16 KiB (64 dims)
constexpr uint32_t kQBytes = kHeads * kDim * 2;     // 16 KiB
constexpr uint32_t kQChunkBytes = kHeads * 128;     // 8 KiB
constexpr int kThreads = 192;

struct __align__(8) Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t tfull[kAcc], tempty[kAcc];
  uint64_t qfull[2], qempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes =
    1024 /*align slack*/ + kStages * kTileBytes + 2 * kQBytes + sizeof(Bars) + kHistBins * sizeof(int);
}  // namespace

__device__ unsigned int g_indexer_tc_error = 0;

__global__ void __launch_bounds__(kThreads, 1) indexer_decode_tc_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
    const float* __restrict__ w_idx, const int32_t* __restrict__ q_pos, int B, int N, int rate,
    int tiles_per_req, float* __restrict__ scores, long long ld_scores, int* __restrict__ hist_g,
    uint32_t spin, int stall, const int32_t* __restrict__ bt, long long bt_stride, int rpb) {
  // bt != nullptr: paged keys -- request r's logical block j (rpb keys) is physical block
  // bt[r*bt_stride + j] of a pool that tm_k maps as [blocks * rpb rows, 128 dims].
  // spin: poll budget of every wait (tc::kSpinLimit in normal use).  stall != 0 (tests of
  // the bounded waits only): the producer issues nothing, so every consumer wait runs out.
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = tc::smem_align1024(smem_raw);
  unsigned char* k_smem = base;                              // [stages][2][128][128 B]
  unsigned char* q_smem = base + kStages * kTileBytes;        // [2][2][64][128 B]
  Bars* bars = reinterpret_cast<Bars*>(q_smem + 2 * kQBytes);
  int* s_hist = reinterpret_cast<int*>(bars + 1);             // [kHistBins] score-key histogram
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long total = (long long)B * tiles_per_req;
  const long long g0 = total * blockIdx.x / gridDim.x;
  const long long g1 = total * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { tc::mbar_init(&bars->full[s], 1); tc::mbar_init(&bars->empty[s], 1); }
    for (int a = 0; a < kAcc; ++a) { tc::mbar_init(&bars->tfull[a], 1); tc::mbar_init(&bars->tempty[a], 4); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&bars->qfull[b], 1); tc::mbar_init(&bars->qempty[b], 1); }
    tc::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (hist_g)
    for (int i = threadIdx.x; i < kHistBins; i += kThreads) s_hist[i] = 0;
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_k);
      tc::tma_prefetch_desc(&tm_q);
      // the keys are read once per step: their lines go first, so that the scores and
      // histograms stay in L2 for the select that reads them next
      const uint64_t stream_pol = tc::l2_evict_first_policy();
      int it = 0, rq = 0, cur_r = -1;
      for (long long g = stall ? g1 : g0; g < g1; ++g) {
        const int r = (int)(g / tiles_per_req);
        const int row0 = (int)(g % tiles_per_req) * kTile;
        if (row0 >= n_visible(q_pos[r], rate, N)) continue;
        if (r != cur_r) {
          const int qb = rq & 1;
          if (!tc::mbar_wait(&bars->qempty[qb], ((rq >> 1) & 1) ^ 1, abort, spin)) break;
          tc::mbar_arrive_expect_tx(&bars->qfull[qb], kQBytes);
          tc::tma_load_2d(q_smem + qb * kQBytes, &tm_q, &bars->qfull[qb], 0, r * kHeads);
          tc::tma_load_2d(q_smem + qb * kQBytes + kQChunkBytes, &tm_q, &bars->qfull[qb], 64, r * kHeads);
          cur_r = r;
          ++rq;
        }
        const int s = it % kStages;
        // paged: the tile's blocks that hold visible keys (their ids are loaded before the
        // wait for a free stage, so the loads' latency hides behind it)
        int pb[kTile / 8];
        int nb = 0;
        if (bt) {
          const int nvis = n_visible(q_pos[r], rate, N);
          nb = min(kTile / rpb, (nvis - row0 + rpb - 1) / rpb);
          const int32_t* btr = bt + (long long)r * bt_stride + row0 / rpb;
#pragma unroll
          for (int i = 0; i < kTile / 8; ++i) pb[i] = i < nb ? __ldg(btr + i) : 0;
        }
        if (!tc::mbar_wait(&bars->empty[s], ((it / kStages) & 1) ^ 1, abort, spin)) break;
        if (bt) {
          // one box of rpb rows per block and 64-dim chunk (rows past the visible blocks
          // keep stale data: their scores are never used)
          tc::mbar_arrive_expect_tx(&bars->full[s], (uint32_t)(nb * rpb * kDim * 2));
#pragma unroll
          for (int i = 0; i < kTile / 8; ++i) {
            if (i < nb) {
              const int prow = pb[i] * rpb;
              tc::tma_load_2d_hint(k_smem + s * kTileBytes + i * rpb * 128, &tm_k, &bars->full[s], 0, prow, stream_pol);
              tc::tma_load_2d_hint(k_smem + s * kTileBytes + kChunkBytes + i * rpb * 128, &tm_k, &bars->full[s], 64,
                                   prow, stream_pol);
            }
          }
        } else {
          tc::mbar_arrive_expect_tx(&bars->full[s], kTileBytes);
          tc::tma_load_3d_hint(k_smem + s * kTileBytes, &tm_k, &bars->full[s], 0, row0, r, stream_pol);
          tc::tma_load_3d_hint(k_smem + s * kTileBytes + kChunkBytes, &tm_k, &bars->full[s], 64, row0, r, stream_pol);
        }
        ++it;
      }
      // make sure no copy of ours is still landing in shared memory
      for (int j = (it > kStages ? it - kStages : 0); j < it; ++j) {
        for (uint32_t i = 0; i < tc::kSpinLimit && !tc::mbar_try_wait(&bars->full[j % kStages], (j / kStages) & 1); ++i)
          __nanosleep(64);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kTile, kHeads, false, false);
      const uint32_t k_base = tc::smem_u32(k_smem), q_base = tc::smem_u32(q_smem);
      int it = 0, rq = 0, cur_r = -1, qb = 0;
      for (long long g = g0; g < g1; ++g) {
        const int r = (int)(g / tiles_per_req);
        const int row0 = (int)(g % tiles_per_req) * kTile;
        if (row0 >= n_visible(q_pos[r], rate, N)) continue;
        if (r != cur_r) {
          if (cur_r >= 0) tc::mma_commit(&bars->qempty[qb]);  // previous q buffer free once its MMAs finish
          qb = rq & 1;
          if (!tc::mbar_wait(&bars->qfull[qb], (rq >> 1) & 1, abort, spin)) break;
          tc::fence_after_sync();
          cur_r = r;
          ++rq;
        }
        const int s = it % kStages;
        const int a = it % kAcc;
        if (!tc::mbar_wait(&bars->full[s], (it / kStages) & 1, abort, spin)) break;
        if (!tc::mbar_wait(&bars->tempty[a], ((it / kAcc) & 1) ^ 1, abort, spin)) break;
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < kDim / 16; ++k) {
          const uint32_t koff = (k >> 2) * kChunkBytes + (k & 3) * 32;
          const uint32_t qoff = (k >> 2) * kQChunkBytes + (k & 3) * 32;
          const uint64_t ad = tc::sdesc_sw128(k_base + s * kTileBytes + koff, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(q_base + qb * kQBytes + qoff, 16, 1024);
          tc::mma_bf16(tmem + a * kHeads, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars->empty[s]);
        tc::mma_commit(&bars->tfull[a]);
        ++it;
      }
      // wait for every MMA of ours before the TMEM is freed
      tc::mma_commit(&bars->drain);
      for (uint32_t i = 0; i < tc::kSpinLimit && !tc::mbar_try_wait(&bars->drain, 0); ++i) __nanosleep(64);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int lq = warp & 3;  // TMEM lane quarter this warp may access
    const int row_in_tile = lq * 32 + lane;
    const int et = (warp - 2) * 32 + lane;  // 0..127 within the epilogue warps
    float w[kHeads];
    int it = 0, cur_r = -1;
    // A failed wait does not leave the loop: every epilogue thread still reaches
    // the histogram flushes, whose barriers agree on the failure first.
    bool failed = false;
    // Add this CTA's counts for request r to the request's global histogram.
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
    for (long long g = g0; g < g1; ++g) {
      const int r = (int)(g / tiles_per_req);
      const int row0 = (int)(g % tiles_per_req) * kTile;
      const int nvis = n_visible(q_pos[r], rate, N);
      if (row0 >= nvis) continue;
      if (r != cur_r) {
        if (hist_g && cur_r >= 0) flush(cur_r);
#pragma unroll
        for (int j = 0; j < kHeads; ++j) w[j] = w_idx[(long long)r * kHeads + j];
        cur_r = r;
      }
      const int a = it % kAcc;
      ++it;
      if (!failed) failed = !tc::warp_wait(&bars->tfull[a], ((it - 1) / kAcc) & 1, abort, spin);
      if (failed) continue;
      tc::fence_after_sync();
      uint32_t v[kHeads];
      const uint32_t taddr = tmem + ((uint32_t)(lq * 32) << 16) + a * kHeads;
      tc::tmem_ld32(taddr, v);
      tc::tmem_ld32(taddr + 32, v + 32);
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->tempty[a]);
      float sc0 = 0.f, sc1 = 0.f;
#pragma unroll
      for (int j = 0; j < kHeads; j += 2) {
        sc0 = fmaf(w[j], fmaxf(__uint_as_float(v[j]), 0.f), sc0);
        sc1 = fmaf(w[j + 1], fmaxf(__uint_as_float(v[j + 1]), 0.f), sc1);
      }
      const int e = row0 + row_in_tile;
      const float sc = sc0 + sc1;
      if (e < nvis) scores[(long long)r * ld_scores + e] = sc;
      if (hist_g) {
        // neighbouring entries share few bins: one shared-memory atomic per distinct bin of the warp
        const uint32_t bin = e < nvis ? float_key(sc) >> 20 : 0xffffffffu;
        const unsigned same = __match_any_sync(0xffffffffu, bin);
        if (e < nvis && (int)(__ffs(same) - 1) == lane) atomicAdd(s_hist + bin, __popc(same));
      }
    }
    if (hist_g && cur_r >= 0) flush(cur_r);
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && bars->abort) atomicOr(&g_indexer_tc_error, 1u);
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- prefill: groups of 4 queries (N = 4 x 64 heads = 256), top-k on chip -----------
// One sequence: query t sees entries s < n_visible(q_pos[t]).  A CTA owns
// groups of four consecutive queries (their q_I rows form the 256-row B
// operand, 64 KiB) and streams the key tiles visible to the group's queries
// through a 3-stage ring; two 256-column TMEM accumulators let the epilogue of
// one tile overlap the MMAs of the next.  Groups are dealt to the persistent
// grid largest first, interleaved, which balances the causal triangle.
// Epilogue: per query, ReLU of 64 head dot products weighted by the f32 head
// weights (staged in shared memory per group).
//
// Top-k fused into the epilogue (the per-query selection of the QbitAI
// write-up, CSA step two; "DeepSeek V4 Architecture Tricks", CSA section,
// top-k 1024): the scores never leave the SM.  Each query of the group keeps,
// in shared memory, a list of candidates -- 64-bit composites (order-
// preserving score key, inverted entry index; distinct, and larger = preferred,
// so ties go to the lower index) in entry order -- and a threshold, the
// smallest composite of its last cut.  Per tile, the two warps of each TMEM
// lane quarter append the entries that beat the threshold, at offsets agreed
// per lane quarter so that the list stays in entry order.  When the next tile
// could overflow the list, an exact MSB-first radix select cuts it back to its
// k largest, in order, and raises the threshold to the smallest one kept (no
// later entry below it can be among the k largest).  After the group's last
// tile a final cut leaves exactly the k largest, written out in entry order.
// A query that sees at most k entries takes all of them without scoring.
// Without the fused top-k (k above kPCand - kTile) the epilogue writes the f32
// scores instead, for a separate select.
namespace {
constexpr int kPStages = 3;
constexpr int kPQ = 4;                       // queries per group
constexpr int kPN = kPQ * kHeads;            // 256 = MMA N
constexpr uint32_t kPQBytes = kPN * kDim * 2;        // 64 KiB
constexpr uint32_t kPQChunkBytes = kPN * 128;        // 32 KiB
constexpr int kPAcc = 2;
constexpr int kPEpi = 16;       // epilogue warps (four per TMEM lane quarter)
constexpr int kPQT = kPQ * 4 / kPEpi;  // queries per epilogue thread (1)
constexpr int kPParts = kPQ / kPQT;    // 128-thread parts of the epilogue, one per query
constexpr int kPThreads = 64 + 32 * kPEpi;  // producer, MMA, epilogue
constexpr int kPCand = 1792;    // candidate slots per query
constexpr int kPPer = kPCand / 128;  // candidates per thread of a half in a cut

// Scratch of one part of the epilogue (the 128 threads serving kPQT queries).
struct __align__(16) PHalf {
  unsigned long long wmin[4], wmax[4];
  int hist[256];
  int wsum[4];
  int wcnt[2][4][kPQT];  // [tile parity][TMEM lane quarter][query of the part]: appends per warp
  int bucket, greater;
};
struct __align__(16) PBars {
  float w[kPN];  // first: read with 16-byte vector loads
  int nvis[kPQ];
  uint64_t full[kPStages], empty[kPStages];
  uint64_t tfull[kPAcc], tempty[kPAcc];
  uint64_t qfull, qempty, drain;
  uint32_t tmem_base;
  int abort;
  PHalf half[kPParts];
};
static_assert(offsetof(PBars, w) % 16 == 0 && offsetof(PBars, full) % 8 == 0, "PBars alignment");
static_assert((kPStages * kTileBytes + kPQBytes) % 1024 == 0, "candidate lists start 1024-byte aligned");
constexpr size_t kPCandBytes = (size_t)kPQ * kPCand * sizeof(uint64_t);  // 48 KiB
constexpr size_t kPSmemBytes = 1024 + kPStages * kTileBytes + kPQBytes + kPCandBytes + sizeof(PBars);
static_assert(kPSmemBytes <= 232448, "shared memory budget");

// Exclusive prefix of v over the 128 threads of a half (hl = 0..127, in order);
// *total receives the sum.  Every thread of the half calls it.
__device__ __forceinline__ int half_scan(int v, int hl, PHalf* hs, uint32_t bar, int* total) {
  const int lane = hl & 31, w = hl >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) hs->wsum[w] = x;
  tc::named_bar(bar, 128);
  int before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int s = hs->wsum[i];
    before += i < w ? s : 0;
    tot += s;
  }
  tc::named_bar(bar, 128);  // wsum is free again
  *total = tot;
  return before + x - v;
}

// Cut the candidate list buf[0..n) (distinct composites, k < n <= kPCand) to its k
// largest, keeping their order; returns the smallest composite kept.  All 128
// threads of the half call it with the same n and k.  Thread hl holds the
// contiguous run [hl*per, hl*per + per) in registers, so the ordered rewrite is
// a scan of the per-thread counts; every write stays inside [0, n).
__device__ __forceinline__ uint64_t cut_to_topk(uint64_t* buf, int n, int k, PHalf* hs, uint32_t bar, int hl) {
  const int lane = hl & 31, w = hl >> 5;
  tc::named_bar(bar, 128);  // every warp's appends are in place
  const int per = (n + 127) / 128;
  const int i0 = hl * per;
  uint64_t v[kPPer];
  unsigned long long mn = ~0ull, mx = 0ull;
#pragma unroll
  for (int u = 0; u < kPPer; ++u) {
    const int i = i0 + u;
    const bool ok = u < per && i < n;
    v[u] = ok ? buf[i] : 0ull;
    if (ok) {
      mn = v[u] < mn ? v[u] : mn;
      mx = v[u] > mx ? v[u] : mx;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, mn, o);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, mx, o);
    mn = a < mn ? a : mn;
    mx = b > mx ? b : mx;
  }
  if (lane == 0) {
    hs->wmin[w] = mn;
    hs->wmax[w] = mx;
  }
  tc::named_bar(bar, 128);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mn = hs->wmin[i] < mn ? hs->wmin[i] : mn;
    mx = hs->wmax[i] > mx ? hs->wmax[i] : mx;
  }
  // MSB-first radix select of the k-th largest, 8-bit digits, from the highest bit
  // where the candidates differ (distinct and n > k >= 1, so mn < mx)
  int hi = mn == mx ? -1 : 63 - __clzll((long long)(mn ^ mx));
  uint64_t prefix = hi >= 63 ? 0ull : (mn >> (hi + 1)) << (hi + 1);
  int lo = hi + 1;
  int remaining = k;
  while (hi >= 0) {
    lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dmask = (1u << (hi - lo + 1)) - 1u;
    hs->hist[hl] = 0;
    hs->hist[hl + 128] = 0;
    tc::named_bar(bar, 128);
#pragma unroll
    for (int u = 0; u < kPPer; ++u) {
      const int i = i0 + u;
      if (u < per && i < n && (hi >= 63 || (v[u] >> (hi + 1)) == (prefix >> (hi + 1))))
        atomicAdd(&hs->hist[(int)((v[u] >> lo) & dmask)], 1);
    }
    tc::named_bar(bar, 128);
    // thread hl owns bins 255 - 2hl and 254 - 2hl: a prefix over the threads is a
    // suffix over the bins
    const int b0 = 255 - 2 * hl, b1 = b0 - 1;
    const int h0 = hs->hist[b0], h1 = hs->hist[b1];
    int tot;
    const int ex = half_scan(h0 + h1, hl, hs, bar, &tot);  // candidates in bins above b0
    if (ex < remaining && ex + h0 >= remaining) {
      hs->bucket = b0;
      hs->greater = ex;
    } else if (ex + h0 < remaining && ex + h0 + h1 >= remaining) {
      hs->bucket = b1;
      hs->greater = ex + h0;
    }
    tc::named_bar(bar, 128);
    const int b = hs->bucket;
    remaining -= hs->greater;
    prefix |= (uint64_t)b << lo;
    const int cnt = hs->hist[b];
    tc::named_bar(bar, 128);  // bucket and histogram read by all before they are rewritten
    hi = lo - 1;
    if (cnt == remaining) break;
  }
  // kept: the composites whose decided bits are at least the prefix's (exactly k of them)
  const int shift = lo;
  const uint64_t P = prefix >> shift;
  int nk = 0;
  unsigned long long kmin = ~0ull;
#pragma unroll
  for (int u = 0; u < kPPer; ++u) {
    const int i = i0 + u;
    if (u < per && i < n && (v[u] >> shift) >= P) {
      ++nk;
      kmin = v[u] < kmin ? v[u] : kmin;
    }
  }
  int tot;
  int off = half_scan(nk, hl, hs, bar, &tot);
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o);
    kmin = a < kmin ? a : kmin;
  }
  if (lane == 0) hs->wmin[w] = kmin;
#pragma unroll
  for (int u = 0; u < kPPer; ++u) {
    const int i = i0 + u;
    if (u < per && i < n && (v[u] >> shift) >= P) buf[off++] = v[u];
  }
  tc::named_bar(bar, 128);  // the cut list and the warp minima are in place
#pragma unroll
  for (int i = 0; i < 4; ++i) kmin = hs->wmin[i] < kmin ? hs->wmin[i] : kmin;
  return kmin;
}
// Cut the candidate list buf[0..n) (distinct composites, k < n <= kPCand) to the
// candidates at or above the bucket of its k-th largest, in one histogram pass over
// the 8 highest bits where the list differs; keeps their order and returns how many
// were kept (at least k) through *kept, and as the new threshold the largest
// composite below every kept one.  No later entry at or under it can be among the k
// largest: the kept ones are at least k and all larger.  Falls back to the exact cut
// when the bucket would leave less than two tiles of room.
__device__ __forceinline__ uint64_t cut_coarse(uint64_t* buf, int n, int k, PHalf* hs, uint32_t bar, int hl,
                                               int* kept) {
  const int lane = hl & 31, w = hl >> 5;
  tc::named_bar(bar, 128);  // every warp's appends are in place
  const int per = (n + 127) / 128;
  const int i0 = hl * per;
  uint64_t v[kPPer];
  unsigned long long mn = ~0ull, mx = 0ull;
#pragma unroll
  for (int u = 0; u < kPPer; ++u) {
    const int i = i0 + u;
    const bool ok = u < per && i < n;
    v[u] = ok ? buf[i] : 0ull;
    if (ok) {
      mn = v[u] < mn ? v[u] : mn;
      mx = v[u] > mx ? v[u] : mx;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, mn, o);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, mx, o);
    mn = a < mn ? a : mn;
    mx = b > mx ? b : mx;
  }
  if (lane == 0) {
    hs->wmin[w] = mn;
    hs->wmax[w] = mx;
  }
  tc::named_bar(bar, 128);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mn = hs->wmin[i] < mn ? hs->wmin[i] : mn;
    mx = hs->wmax[i] > mx ? hs->wmax[i] : mx;
  }
  const int hi = 63 - __clzll((long long)(mn ^ mx));  // mn < mx: distinct and n > k >= 1
  const int lo = hi >= 7 ? hi - 7 : 0;
  const uint32_t dmask = (1u << (hi - lo + 1)) - 1u;
  hs->hist[hl] = 0;
  hs->hist[hl + 128] = 0;
  tc::named_bar(bar, 128);
#pragma unroll
  for (int u = 0; u < kPPer; ++u) {
    const int i = i0 + u;
    if (u < per && i < n) atomicAdd(&hs->hist[(int)((v[u] >> lo) & dmask)], 1);
  }
  tc::named_bar(bar, 128);
  const int b0 = 255 - 2 * hl, b1 = b0 - 1;
  const int h0 = hs->hist[b0], h1 = hs->hist[b1];
  int tot;
  const int ex = half_scan(h0 + h1, hl, hs, bar, &tot);  // candidates in bins above b0
  if (ex < k && ex + h0 >= k) {
    hs->bucket = b0;
    hs->greater = ex + h0;  // kept: everything in bin b0 and above
  } else if (ex + h0 < k && ex + h0 + h1 >= k) {
    hs->bucket = b1;
    hs->greater = ex + h0 + h1;
  }
  tc::named_bar(bar, 128);
  const int nkeep = hs->greater;
  const uint64_t P = ((mn >> lo) & ~(uint64_t)dmask) | (uint64_t)hs->bucket;  // bucket's value of v >> lo
  tc::named_bar(bar, 128);  // bucket read by all before it is rewritten
  if (nkeep > kPCand - 2 * kTile) {  // a fat bucket: the exact cut
    // (buf is unchanged; cut_to_topk reloads it)
    *kept = k;
    return cut_to_topk(buf, n, k, hs, bar, hl);
  }
  int nk = 0;
#pragma unroll
  for (int u = 0; u < kPPer; ++u) {
    const int i = i0 + u;
    nk += (u < per && i < n && (v[u] >> lo) >= P) ? 1 : 0;
  }
  int off = half_scan(nk, hl, hs, bar, &tot);
#pragma unroll
  for (int u = 0; u < kPPer; ++u) {
    const int i = i0 + u;
    if (u < per && i < n && (v[u] >> lo) >= P) buf[off++] = v[u];
  }
  tc::named_bar(bar, 128);  // the cut list is in place
  *kept = tot;
  return (P << lo) - 1;  // every kept composite is >= P << lo > 0
}
}  // namespace

bool indexer_prefill_topk_fused(int k) { return k >= 1 && k <= kPCand - kTile; }

__global__ void __launch_bounds__(kPThreads, 1) indexer_prefill_tc_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
    const float* __restrict__ w_idx, const int32_t* __restrict__ q_pos, int Tq, int N, int rate,
    float* __restrict__ scores, long long ld_scores, int k, int32_t* __restrict__ topk_idx) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = tc::smem_align1024(smem_raw);
  unsigned char* k_smem = base;                           // [stages][2][128][128 B]
  unsigned char* q_smem = base + kPStages * kTileBytes;   // [2][256][128 B]
  uint64_t* cand_smem = reinterpret_cast<uint64_t*>(q_smem + kPQBytes);  // [4][kPCand]
  PBars* bars = reinterpret_cast<PBars*>(q_smem + kPQBytes + kPCandBytes);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_groups = (Tq + kPQ - 1) / kPQ;
  const bool fused = topk_idx != nullptr;
  // tiles of group g: entries visible to its queries (q_pos is non-decreasing within a group
  // in the layer call; the maximum over the group is used in general).  With the fused
  // top-k a group whose queries all see at most k entries needs no scores at all.
  auto group_tiles = [&](int g) -> int {
    int nv = 0;
    for (int j = 0; j < kPQ; ++j) {
      const int q = g * kPQ + j;
      if (q < Tq) nv = max(nv, n_visible(q_pos[q], rate, N));
    }
    if (fused && nv <= k) return 0;
    return (nv + kTile - 1) / kTile;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) { tc::mbar_init(&bars->full[s], 1); tc::mbar_init(&bars->empty[s], 1); }
    for (int a = 0; a < kPAcc; ++a) { tc::mbar_init(&bars->tfull[a], 1); tc::mbar_init(&bars->tempty[a], kPEpi); }
    tc::mbar_init(&bars->qfull, 1);
    tc::mbar_init(&bars->qempty, 1);
    tc::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kPAcc * kPN);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_k);
      tc::tma_prefetch_desc(&tm_q);
      int it = 0, gi = 0;  // gi counts the groups actually processed (one q-buffer phase each)
      bool ok = true;
      for (int g = n_groups - 1 - (int)blockIdx.x; ok && g >= 0; g -= (int)gridDim.x) {
        const int nt = group_tiles(g);
        if (nt == 0) continue;
        if (!tc::mbar_wait(&bars->qempty, (gi++ & 1) ^ 1, abort)) break;
        tc::mbar_arrive_expect_tx(&bars->qfull, kPQBytes);
        tc::tma_load_2d(q_smem, &tm_q, &bars->qfull, 0, g * kPN);
        tc::tma_load_2d(q_smem + kPQChunkBytes, &tm_q, &bars->qfull, 64, g * kPN);
        // the next group's queries into L2 while this group streams: its load above
        // then waits on L2, not on HBM (the q buffer holds one group)
        {
          int gn = g - (int)gridDim.x;
          while (gn >= 0 && group_tiles(gn) == 0) gn -= (int)gridDim.x;
          if (gn >= 0) tc::tma_prefetch_2d(&tm_q, 0, gn * kPN), tc::tma_prefetch_2d(&tm_q, 64, gn * kPN);
        }
        for (int t = 0; t < nt; ++t, ++it) {
          const int s = it % kPStages;
          if (!tc::mbar_wait(&bars->empty[s], ((it / kPStages) & 1) ^ 1, abort)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&bars->full[s], kTileBytes);
          tc::tma_load_3d(k_smem + s * kTileBytes, &tm_k, &bars->full[s], 0, t * kTile, 0);
          tc::tma_load_3d(k_smem + s * kTileBytes + kChunkBytes, &tm_k, &bars->full[s], 64, t * kTile, 0);
        }
      }
      for (int j = (it > kPStages ? it - kPStages : 0); j < it; ++j)
        for (uint32_t i = 0; i < tc::kSpinLimit && !tc::mbar_try_wait(&bars->full[j % kPStages], (j / kPStages) & 1); ++i)
          __nanosleep(64);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kTile, kPN, false, false);
      const uint64_t qd0 = tc::sdesc_sw128(tc::smem_u32(q_smem), 16, 1024);
      const uint32_t k_base = tc::smem_u32(k_smem);
      int it = 0, gi = 0;
      bool ok = true;
      for (int g = n_groups - 1 - (int)blockIdx.x; ok && g >= 0; g -= (int)gridDim.x) {
        const int nt = group_tiles(g);
        if (nt == 0) continue;
        if (!tc::mbar_wait(&bars->qfull, gi++ & 1, abort)) break;
        tc::fence_after_sync();
        for (int t = 0; t < nt; ++t, ++it) {
          const int s = it % kPStages, a = it % kPAcc;
          if (!tc::mbar_wait(&bars->full[s], (it / kPStages) & 1, abort)) { ok = false; break; }
          if (!tc::mbar_wait(&bars->tempty[a], ((it / kPAcc) & 1) ^ 1, abort)) { ok = false; break; }
          tc::fence_after_sync();
          const uint64_t ad0 = tc::sdesc_sw128(k_base + s * kTileBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kDim / 16; ++kk) {
            const uint32_t aoff = ((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4;
            const uint32_t boff = ((kk >> 2) * kPQChunkBytes + (kk & 3) * 32) >> 4;
            tc::mma_bf16(tmem + a * kPN, ad0 + aoff, qd0 + boff, idesc, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&bars->empty[s]);
          tc::mma_commit(&bars->tfull[a]);
        }
        tc::mma_commit(&bars->qempty);  // q buffer free once this group's MMAs finish
      }
      tc::mma_commit(&bars->drain);
      for (uint32_t i = 0; i < tc::kSpinLimit && !tc::mbar_try_wait(&bars->drain, 0); ++i) __nanosleep(64);
    }
    __syncwarp();
  } else {
    // epilogue: warps 2..17, one TMEM lane (= entry) per thread; the four warps of a
    // lane quarter score one of the group's four queries each.  Warps 2-5 (part 0)
    // serve query 0, warps 6-9 query 1, and so on.
    const int lq = warp & 3;
    const int row_in_tile = lq * 32 + lane;
    const int et = threadIdx.x - 64;  // 0..255
    const int half = (warp - 2) >> 2;  // the part: kPQT queries
    const int j0 = kPQT * half;
    const int hl = et - 128 * half;  // 0..127 within the part
    const uint32_t hbar = 2 + half;
    PHalf* hs = &bars->half[half];
    uint64_t* cbuf[kPQT];
#pragma unroll
    for (int jj = 0; jj < kPQT; ++jj) cbuf[jj] = cand_smem + (size_t)(j0 + jj) * kPCand;
    const unsigned lt = (1u << lane) - 1u;
    int it = 0, par = 0;
    bool failed = false;
    for (int g = n_groups - 1 - (int)blockIdx.x; g >= 0; g -= (int)gridDim.x) {
      const int nt = group_tiles(g);
      if (nt == 0 && !fused) continue;
      // stage this group's weights and visible counts (the previous group's readers are done)
      tc::named_bar(1, 32 * kPEpi);
      for (int e = et; e < kPN; e += 32 * kPEpi) {
        const int q = g * kPQ + e / kHeads;
        bars->w[e] = q < Tq ? w_idx[(long long)q * kHeads + (e % kHeads)] : 0.f;
      }
      if (et < kPQ) {
        const int q = g * kPQ + et;
        bars->nvis[et] = q < Tq ? n_visible(q_pos[q], rate, N) : 0;
      }
      tc::named_bar(1, 32 * kPEpi);
      // fused top-k state of this part's queries (uniform over the part)
      bool sel[kPQT];
      int cnt[kPQT];
      uint64_t thr[kPQT];  // every real composite is > 0
#pragma unroll
      for (int jj = 0; jj < kPQT; ++jj) { cnt[jj] = 0; thr[jj] = 0ull; }
#pragma unroll
      for (int jj = 0; jj < kPQT; ++jj) sel[jj] = fused && g * kPQ + j0 + jj < Tq && bars->nvis[j0 + jj] > k;
      for (int t = 0; t < nt; ++t, ++it) {
        const int a = it % kPAcc;
        if (!failed) failed = !tc::warp_wait(&bars->tfull[a], (it / kPAcc) & 1, abort);
        const int e = t * kTile + row_in_tile;
        float sc[kPQT];
#pragma unroll
        for (int jj = 0; jj < kPQT; ++jj) sc[jj] = 0.f;
        if (!failed) {
          tc::fence_after_sync();
          static_assert(kPQT == 1, "the accumulator is released right after its one read below");
#pragma unroll
          for (int jj = 0; jj < kPQT; ++jj) {
            const int j = j0 + jj;
            uint32_t v[kHeads];
            const uint32_t taddr = tmem + ((uint32_t)(lq * 32) << 16) + a * kPN + j * kHeads;
            tc::tmem_ld32(taddr, v);
            tc::tmem_ld32(taddr + 32, v + 32);
            tc::tmem_ld_wait();
            // the accumulator may take tile it + 2's MMAs while this warp sums
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->tempty[a]);
            const float* w = bars->w + j * kHeads;
            // eight independent chains (a fixed association, the same for every entry)
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int h = 0; h < kHeads; h += 8) {
              const float4 wa = *reinterpret_cast<const float4*>(w + h);
              const float4 wb = *reinterpret_cast<const float4*>(w + h + 4);
              acc[0] = fmaf(wa.x, fmaxf(__uint_as_float(v[h]), 0.f), acc[0]);
              acc[1] = fmaf(wa.y, fmaxf(__uint_as_float(v[h + 1]), 0.f), acc[1]);
              acc[2] = fmaf(wa.z, fmaxf(__uint_as_float(v[h + 2]), 0.f), acc[2]);
              acc[3] = fmaf(wa.w, fmaxf(__uint_as_float(v[h + 3]), 0.f), acc[3]);
              acc[4] = fmaf(wb.x, fmaxf(__uint_as_float(v[h + 4]), 0.f), acc[4]);
              acc[5] = fmaf(wb.y, fmaxf(__uint_as_float(v[h + 5]), 0.f), acc[5]);
              acc[6] = fmaf(wb.z, fmaxf(__uint_as_float(v[h + 6]), 0.f), acc[6]);
              acc[7] = fmaf(wb.w, fmaxf(__uint_as_float(v[h + 7]), 0.f), acc[7]);
            }
            sc[jj] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
          }
        }
        if (!fused) {
          if (failed) continue;
#pragma unroll
          for (int jj = 0; jj < kPQT; ++jj) {
            const int q = g * kPQ + j0 + jj;
            if (q < Tq && e < bars->nvis[j0 + jj]) scores[(long long)q * ld_scores + e] = sc[jj];
          }
          continue;
        }
        // fused: candidates that beat the threshold, appended in entry order
        uint64_t c[kPQT];
        unsigned bal[kPQT];
#pragma unroll
        for (int jj = 0; jj < kPQT; ++jj) {
          c[jj] = make_cand(sc[jj], e);
          const bool take = !failed && sel[jj] && e < bars->nvis[j0 + jj] && c[jj] > thr[jj];
          bal[jj] = __ballot_sync(0xffffffffu, take);
          if (lane == 0) hs->wcnt[par][lq][jj] = __popc(bal[jj]);
        }
        // one barrier per tile: the warps' counts are in, and every thread agrees on failure
        if (tc::named_bar_or(hbar, 128, failed || *abort)) { failed = true; break; }
#pragma unroll
        for (int jj = 0; jj < kPQT; ++jj) {
          int off = cnt[jj], tot = 0;
#pragma unroll
          for (int l = 0; l < 4; ++l) {
            const int n_l = hs->wcnt[par][l][jj];
            off += l < lq ? n_l : 0;
            tot += n_l;
          }
          if ((bal[jj] >> lane) & 1u) cbuf[jj][off + __popc(bal[jj] & lt)] = c[jj];
          cnt[jj] += tot;
        }
        par ^= 1;
        // room for one more tile of appends in each list, else cut it back (coarsely: the
        // exact k largest are taken once, after the group's last tile)
#pragma unroll
        for (int jj = 0; jj < kPQT; ++jj) {
          if (cnt[jj] > kPCand - kTile) {
            int kept;
            thr[jj] = cut_coarse(cbuf[jj], cnt[jj], k, hs, hbar, hl, &kept);
            cnt[jj] = kept;
          }
        }
      }
      if (!fused) continue;
      if (failed) continue;  // (uniform over the half: agreed at the per-tile barrier)
      tc::named_bar(hbar, 128);  // the last tile's appends are in place
#pragma unroll
      for (int jj = 0; jj < kPQT; ++jj) {
        const int q = g * kPQ + j0 + jj;
        if (q >= Tq) continue;
        int32_t* out = topk_idx + (long long)q * k;
        if (!sel[jj]) {
          // at most k visible entries: all of them, then empty slots
          const int nv = bars->nvis[j0 + jj];
          for (int i = hl; i < k; i += 128) out[i] = i < nv ? i : -1;
          continue;
        }
        if (cnt[jj] > k) {
          thr[jj] = cut_to_topk(cbuf[jj], cnt[jj], k, hs, hbar, hl);
          cnt[jj] = k;
        }
        for (int i = hl; i < k; i += 128) out[i] = cand_index(cbuf[jj][i]);
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && bars->abort) atomicOr(&g_indexer_tc_error, 2u);
  if (warp == 1) tc::tmem_dealloc(tmem, kPAcc * kPN);
}

// ---- host side ------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// bf16 tensor map, 128B swizzle, box = {64, box_rows, 1}; dims innermost first.
cudaError_t make_tmap_bf16(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t gdim[3], gstride[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) gdim[i] = dims[i];
  for (int i = 0; i < rank - 1; ++i) gstride[i] = strides_bytes[i];
  box[0] = 64;
  box[1] = box_rows;
  box[2] = 1;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), gdim, gstride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

bool indexer_tc_supported(int H_I, int d_I) { return H_I == kHeads && d_I == kDim; }

cudaError_t launch_indexer_decode_tc(const bf16* q_idx, const float* w_idx, const bf16* k_idx, long long k_seq_stride,
                                     int N, const int32_t* q_pos, int B, int rate, float* scores, long long ld_scores,
                                     int num_sms, cudaStream_t stream, int* hist, bool stall, const PagedKeys* paged) {
  constexpr uint32_t kStallSpin = 4096;  // a stalled test launch gives up after ~4k polls
  if (B == 0 || N == 0) return cudaSuccess;
  CUtensorMap tm_k, tm_q;
  cudaError_t e;
  if (paged) {
    if (paged->rpb < 8 || paged->rpb > kTile || kTile % paged->rpb != 0 || paged->rpb % 8 != 0)
      return cudaErrorInvalidValue;
    const uint64_t kd[2] = {(uint64_t)kDim, (uint64_t)paged->n_blocks * paged->rpb};
    const uint64_t ks[1] = {(uint64_t)kDim * 2};
    e = make_tmap_bf16(&tm_k, k_idx, 2, kd, ks, (uint32_t)paged->rpb);
  } else {
    const uint64_t kd[3] = {(uint64_t)kDim, (uint64_t)N, (uint64_t)B};
    const uint64_t ks[2] = {(uint64_t)kDim * 2, (uint64_t)(B > 1 ? k_seq_stride : (long long)N * kDim) * 2};
    e = make_tmap_bf16(&tm_k, k_idx, 3, kd, ks, kTile);
  }
  if (e != cudaSuccess) return e;
  const uint64_t qd[2] = {(uint64_t)kDim, (uint64_t)B * kHeads};
  const uint64_t qs[1] = {(uint64_t)kDim * 2};
  e = make_tmap_bf16(&tm_q, q_idx, 2, qd, qs, kHeads);
  if (e != cudaSuccess) return e;
  const int tiles_per_req = (N + kTile - 1) / kTile;
  const long long total = (long long)B * tiles_per_req;
  const int grid = (int)(total < num_sms ? total : num_sms);
  e = cudaFuncSetAttribute((const void*)indexer_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  indexer_decode_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm_k, tm_q, w_idx, q_pos, B, N, rate,
                                                                   tiles_per_req, scores, ld_scores, hist,
                                                                   stall ? kStallSpin : tc::kSpinLimit,
                                                                   stall ? 1 : 0, paged ? paged->bt : nullptr,
                                                                   paged ? paged->bt_stride : 0,
                                                                   paged ? paged->rpb : 0);
  ++g_launch_counter;
  return cudaGetLastError();
}

cudaError_t launch_indexer_prefill_tc(const bf16* q_idx, const float* w_idx, const bf16* k_idx, int N,
                                      const int32_t* q_pos, int Tq, int rate, float* scores, long long ld_scores,
                                      int num_sms, cudaStream_t stream, int k, int32_t* topk_idx) {
  if (Tq == 0) return cudaSuccess;
  if (N == 0) {
    // nothing is visible to any query: every slot of the fused top-k is empty (-1)
    if (!topk_idx) return cudaSuccess;
    ++g_launch_counter;
    return cudaMemsetAsync(topk_idx, 0xff, (size_t)Tq * k * sizeof(int32_t), stream);
  }
  if (topk_idx && !indexer_prefill_topk_fused(k)) return cudaErrorInvalidValue;
  CUtensorMap tm_k, tm_q;
  const uint64_t kd[3] = {(uint64_t)kDim, (uint64_t)N, 1};
  const uint64_t ks[2] = {(uint64_t)kDim * 2, (uint64_t)N * kDim * 2};
  cudaError_t e = make_tmap_bf16(&tm_k, k_idx, 3, kd, ks, kTile);
  if (e != cudaSuccess) return e;
  const uint64_t qd[2] = {(uint64_t)kDim, (uint64_t)Tq * kHeads};
  const uint64_t qs[1] = {(uint64_t)kDim * 2};
  e = make_tmap_bf16(&tm_q, q_idx, 2, qd, qs, kPN);
  if (e != cudaSuccess) return e;
  const int n_groups = (Tq + kPQ - 1) / kPQ;
  const int grid = n_groups < num_sms ? n_groups : num_sms;
  e = cudaFuncSetAttribute((const void*)indexer_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kPSmemBytes);
  if (e != cudaSuccess) return e;
  indexer_prefill_tc_kernel<<<grid, kPThreads, kPSmemBytes, stream>>>(tm_k, tm_q, w_idx, q_pos, Tq, N, rate, scores,
                                                                      ld_scores, k, topk_idx);
  ++g_launch_counter;
  return cudaGetLastError();
}

unsigned int read_and_clear_indexer_tc_error() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_indexer_tc_error, sizeof(v)) != cudaSuccess) return 0xffffffffu;
  if (v) cudaMemcpyToSymbol(g_indexer_tc_error, &zero, sizeof(zero));
  return v;
}

}  // namespace hca
