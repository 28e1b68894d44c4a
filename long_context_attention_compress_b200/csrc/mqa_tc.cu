// Shared-KV multi-query attention on the 5th-generation tensor cores (sm_100a),
// for decode (one query of 64 heads x 512 per request, split over CTAs along
// its row list, partial softmax states merged by the combine kernel) and for
// prefill (one CTA per query of one sequence).
//
// What it computes (QbitAI write-up, "混合注意力機制": CSA step three, KV
// entries act as both key and value, sliding-window branch; "DeepSeek V4
// Architecture Tricks", HCA section):
//   o[h, :] = sum_u softmax_u(scale * q[h, :] . row_u) row_u
// over U = selected CSA entries (idx) or all visible HCA entries, then the
// window rows.
//
// Design.  Rows are the MMA's M dimension and heads its N dimension, so one
// 128-row KV tile in shared memory (128B-swizzled, eight 64-dim chunks of
// [128 rows x 128 B]) is the K-major A operand of S^T = R . Q^T (M = 128) and,
// read MN-major, the A operand of O^T += V^T . P^T (M = 128 dims per block,
// K = rows).  The tile is tracked as four 128-dim column blocks (two chunks
// each) with their own full/empty barriers: PV runs block by block and
// releases each block as soon as its MMAs finish, so the next tile's loads of
// that block, and its QK^T over it, start while PV is still running.
// Dense rows arrive as 3-D TMA tiles.  Selected (gathered) rows are copied by
// the compute threads with 16-byte cp.async, the 128-byte swizzle applied by
// hand: the TMA unit gathers only about 36 bytes per clock (tile::gather4 of
// 128-byte row pieces), less than the tile rate PV sustains, while the
// threads' copies keep up; each column block is signalled as soon as its
// copies have landed.  The query's output leaves as one contiguous 64 KiB bulk
// copy staged in the free tile buffer.
//   warp 0     MMA issuer (and TMEM owner)
//   warps 1-8  two per TMEM lane quarter (32 rows of S^T), each owning 32 of
//              the 64 heads: per-head tile maxima by a warp reduce-scatter plus
//              a 4-way shared-memory step; P = 2^(s - m) written as two bf16
//              terms P_hi + P_lo, each truncated (MN-major B operands of PV; P
//              keeps ~15 significant bits); lazy rescale of the TMEM accumulators (only
//              when a head's maximum grows by more than 2^8); the loads of the
//              next tile; the final epilogue.
// Row sums l_h are warp reduce-scatter sums of exactly the bf16 P_hi + P_lo
// that PV multiplies (kept per warp across tiles, rescaled with O).
// TMEM: S^T 64 columns, O^T 3 blocks x 128 (P_hi and P_lo products apart) + 1 x 64.

#include <cudaTypedefs.h>

#include <cstddef>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hca {

namespace {
constexpr int kCompute = 16;                         // compute warps (four per TMEM lane quarter)
constexpr int kThreads = 32 * (1 + kCompute);
constexpr int kRows = 128;                           // rows per tile
constexpr int kC = 512;
constexpr int kH = 64;
constexpr int kChunks = kC / 64;
constexpr int kBlocks = 4;                           // 128-dim column blocks
// Gathered rows: warp w copies tile rows [8 w, 8 w + 8) of every column block,
// lane l the 16-byte unit l % 8 of rows 8 w + 4 k + l / 8 (k < 2), both chunks.
constexpr int kCopyRows = 2;
constexpr uint32_t kQBytes = kH * kC * 2;            // 64 KiB
constexpr uint32_t kQChunk = kH * 128;               // 8 KiB
constexpr uint32_t kKvChunk = kRows * 128;           // 16 KiB
constexpr uint32_t kKvBytes = kChunks * kKvChunk;    // 128 KiB
constexpr uint32_t kBlockBytes = 2 * kKvChunk;       // 32 KiB
constexpr uint32_t kPBytes = kRows * kH * 2;         // 16 KiB per P term
constexpr uint32_t kOffQ = 0, kOffKv = kQBytes, kOffP = kOffKv + kKvBytes, kOffBars = kOffP + 2 * kPBytes;
constexpr uint32_t kColS = 0, kColO = 64, kTmemCols = 512;
// O^T column blocks.  Blocks 0-2 keep the P_hi and P_lo products apart (128
// columns, hi then lo: one N = 128 MMA per K-step reads the V^T tile once for
// both terms); block 3 accumulates both terms in 64 columns (two N = 64 MMAs).
// TMEM: S^T 64 + 3 x 128 + 64 = 512 columns.
constexpr int kWideBlocks = 3;
__host__ __device__ constexpr bool wide_block(int b) { return b < kWideBlocks; }
__host__ __device__ constexpr uint32_t col_o(int b) {
  return kColO + (b < kWideBlocks ? b * 2 * kH : kWideBlocks * 2 * kH + (b - kWideBlocks) * kH);
}
static_assert(col_o(kBlocks - 1) + kH == kTmemCols, "TMEM columns");
constexpr float kRescaleLog2 = 8.f;
constexpr int kHpt = kH * 4 / kCompute;  // heads per compute thread (16)
static_assert(kCompute * 8 == kRows && kCopyRows * 4 == 8, "copies cover the tile");
static_assert(kHpt == 16, "the reductions below are written for 16 heads per thread");

struct __align__(16) Bars {
  // float arrays first: mref is read with 16-byte vector loads
  float red[4][kH];
  float mref[kH];
  float alpha[kH];
  uint64_t qfull, kvfull[kBlocks], kvempty[kBlocks], sfull, sempty, pfull, odone, drain;
  uint32_t tmem_base;
  int abort;
  int rescale;
  int need[3];  // per tile (mod 3): some score exceeds its head's running maximum by > 2^8
};
static_assert(offsetof(Bars, mref) % 16 == 0 && offsetof(Bars, red) % 16 == 0, "vector-loaded arrays");
static_assert(offsetof(Bars, qfull) % 8 == 0, "mbarriers are 8-byte aligned");
static_assert(kOffBars % 1024 == 0, "operand buffers keep 1024-byte alignment");
constexpr size_t kSmemBytes = 1024 + kOffBars + sizeof(Bars);
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Tile {
  int seg;    // 0: entries, 1: window
  int row0;   // first row within the segment
  int nrows;  // valid rows
};

// Tiles of one split: the split's range of the row list cut at the
// entries/window boundary, 128 rows per tile.
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

// One reduce-scatter step over lane bit O: of the NV values held, keep the
// half selected by the bit and fold in the partner's copy of that half.
template <int O, int NV, int SZ>
__device__ __forceinline__ void rs_max_step(float (&a)[SZ], int lane) {
  const bool hi = (lane & O) != 0;
#pragma unroll
  for (int j = 0; j < NV / 2; ++j) {
    const float send = hi ? a[j] : a[j + NV / 2];
    const float keep = hi ? a[j + NV / 2] : a[j];
    a[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, O));
  }
}
template <int O, int NV, int SZ>
__device__ __forceinline__ void rs_sum_step(float (&a)[SZ], int lane) {
  const bool hi = (lane & O) != 0;
#pragma unroll
  for (int j = 0; j < NV / 2; ++j) {
    const float send = hi ? a[j] : a[j + NV / 2];
    const float keep = hi ? a[j + NV / 2] : a[j];
    a[j] = keep + __shfl_xor_sync(0xffffffffu, send, O);
  }
}
// Afterwards lane l holds the warp-wide sum of value l % 16 (16 shuffles).
__device__ __forceinline__ float warp_sum16(float (&a)[16], int lane) {
  rs_sum_step<8, 16>(a, lane);
  rs_sum_step<4, 8>(a, lane);
  rs_sum_step<2, 4>(a, lane);
  rs_sum_step<1, 2>(a, lane);
  return a[0] + __shfl_xor_sync(0xffffffffu, a[0], 16);
}
// Afterwards lane l holds the warp-wide maximum of value l % 16 (16 shuffles).
__device__ __forceinline__ float warp_max16(float (&a)[16], int lane) {
  rs_max_step<8, 16>(a, lane);
  rs_max_step<4, 8>(a, lane);
  rs_max_step<2, 4>(a, lane);
  rs_max_step<1, 2>(a, lane);
  return fmaxf(a[0], __shfl_xor_sync(0xffffffffu, a[0], 16));
}
}  // namespace

__device__ unsigned int g_mqa_tc_error = 0;

struct MqaTcParams {
  const int32_t* idx;         // [Tq, n_idx] or nullptr
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
  const float* sink;          // [H] sink logits (natural units) or nullptr; unsplit queries add it here,
                              // split ones in the combine
  int rope_dims;              // > 0: unsplit queries turn their output's last rope_dims channels back by
  float rope_base;            // -t here, split ones in the combine
  const int32_t* bt;          // paged entries (see MqaProblem), or nullptr
  long long bt_stride;
  int rpb;
  long long pool_blocks;      // blocks of the pool the block table points into
  int check;                  // record entry_check failures (bits << 1 of the error word)
  const bf16* kvg;            // base of the gathered-row map (rows of kC elements)
  long long kvg_rows;         // its rows (a copy never reads outside them)
};

__global__ void __launch_bounds__(kThreads, 1) mqa_decode_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
    const __grid_constant__ CUtensorMap tm_win, const __grid_constant__ CUtensorMap tm_out, MqaTcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      tc::smem_align1024(smem_raw);
  Bars* bars = reinterpret_cast<Bars*>(base + kOffBars);
  volatile int* abort = &bars->abort;
  volatile int* need_flag = bars->need;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = blockIdx.x / p.splits;
  const int sp = blockIdx.x % p.splits;

  // this query's row list
  const int t_pos = p.q_pos[q];
  // (no entries at all, e.g. a sequence shorter than one block: only the window;
  // every selected slot is then empty and nothing may be read from the cache)
  const int n_first = p.N <= 0 ? 0 : (p.idx ? p.n_idx : n_visible(t_pos, p.rate, p.N));
  const int n_win = min(p.n_win, t_pos + 1);
  const int ub = sp * p.rows_per_split;
  const int ue = min(n_first + n_win, ub + p.rows_per_split);
  const SplitTiles tiles(n_first, n_win, ub, max(ub, ue));
  const int nt = tiles.count();
  const int32_t* idx_q = p.idx ? p.idx + (long long)q * p.n_idx : nullptr;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->qfull, 1);
    for (int b = 0; b < kBlocks; ++b) {
      tc::mbar_init(&bars->kvfull[b], kCompute);  // one arrival per compute warp
      tc::mbar_init(&bars->kvempty[b], 1);
    }
    tc::mbar_init(&bars->sfull, 1);
    tc::mbar_init(&bars->sempty, kCompute);
    tc::mbar_init(&bars->pfull, kCompute);
    tc::mbar_init(&bars->odone, 1);
    tc::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    bars->rescale = 0;
    for (int k = 0; k < 3; ++k) bars->need[k] = 0;
    tc::fence_mbar_init();
  }
  for (int h = threadIdx.x; h < kH; h += kThreads) { bars->mref[h] = neg_inf(); bars->alpha[h] = 1.f; }
  if (warp == 0) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  tc::griddep_launch_dependents();
  // The queries are a call input: their load may start before the previous kernel
  // (the top-k) has finished; everything else waits for it.
  if (warp == 0 && lane == 0) {
    tc::mbar_arrive_expect_tx(&bars->qfull, kQBytes);
    for (int c = 0; c < kChunks; ++c) tc::tma_load_2d(base + kOffQ + c * kQChunk, &tm_q, &bars->qfull, c * 64, q * kH);
  }
  tc::griddep_wait();

  if (warp == 0) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t id_qk = tc::idesc_bf16_f32(kRows, kH, false, false);
      constexpr uint32_t id_pv = tc::idesc_bf16_f32(128, kH, true, true);
      constexpr uint32_t id_pv2 = tc::idesc_bf16_f32(128, 2 * kH, true, true);  // B = [P_hi | P_lo]
      const uint32_t q_base = tc::smem_u32(base + kOffQ), kv_base = tc::smem_u32(base + kOffKv),
                     p_base = tc::smem_u32(base + kOffP);
      // Descriptors are built once; each K-step only adds a compile-time
      // offset (>> 4) to the start-address field.
      uint64_t q_desc0 = tc::sdesc_sw128(q_base, 16, 1024);
      uint64_t k_desc0 = tc::sdesc_sw128(kv_base, 16, 1024);
      uint64_t v_desc0 = tc::sdesc_sw128(kv_base, kKvChunk, 1024);
      uint64_t p_hi0 = tc::sdesc_sw128(p_base, kPBytes, 1024);
      uint64_t p_lo0 = tc::sdesc_sw128(p_base + kPBytes, kPBytes, 1024);
      bool ok = tc::mbar_wait(&bars->qfull, 0, abort);
      for (int i = 0; ok && i < nt; ++i) {
        const uint32_t ph = i & 1;
        // keep the per-step descriptors from being hoisted out of the loop (96 live 64-bit values)
        asm volatile("" : "+l"(q_desc0), "+l"(k_desc0), "+l"(v_desc0), "+l"(p_hi0), "+l"(p_lo0));
        if (!tc::mbar_wait(&bars->sempty, ph ^ 1, abort)) { ok = false; break; }
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {
          if (!tc::mbar_wait(&bars->kvfull[b], ph, abort)) { ok = false; break; }
          tc::fence_after_sync();
#pragma unroll
          for (int k = 8 * b; k < 8 * b + 8; ++k) {
            const uint32_t aoff = ((k >> 2) * kKvChunk + (k & 3) * 32) >> 4;
            const uint32_t boff = ((k >> 2) * kQChunk + (k & 3) * 32) >> 4;
            tc::mma_bf16(tmem + kColS, k_desc0 + aoff, q_desc0 + boff, id_qk, k > 0 ? 1u : 0u);
          }
        }
        if (!ok) break;
        tc::mma_commit(&bars->sfull);
        if (!tc::mbar_wait(&bars->pfull, ph, abort)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t acc0 = i > 0 ? 1u : 0u;
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk) {
            const uint32_t koff = (kk * 2048) >> 4;
            const uint32_t first = kk > 0 ? 1u : acc0;
            const uint64_t ad = v_desc0 + (((2 * b) * kKvChunk) >> 4) + koff;
            if (wide_block(b)) {
              // N = 128: the P_lo columns are the next 64-column block of the operand (LBO)
              tc::mma_bf16(tmem + col_o(b), ad, p_hi0 + koff, id_pv2, first);
            } else {
              tc::mma_bf16(tmem + col_o(b), ad, p_hi0 + koff, id_pv, first);
              tc::mma_bf16(tmem + col_o(b), ad, p_lo0 + koff, id_pv, 1u);
            }
          }
          tc::mma_commit(&bars->kvempty[b]);  // this block's columns of the tile may be reloaded
        }
        tc::mma_commit(&bars->odone);
      }
      tc::mma_commit(&bars->drain);
      for (uint32_t k = 0; k < tc::kSpinLimit && !tc::mbar_try_wait(&bars->drain, 0); ++k) __nanosleep(64);
      for (uint32_t k = 0; k < tc::kSpinLimit && !tc::mbar_try_wait(&bars->qfull, 0); ++k) __nanosleep(64);
    }
  } else {
    // --------------------- loads, softmax / correction / epilogue ---------------------
    const int cw = warp - 1;                       // compute warp 0..7
    const int quarter = warp & 3;                  // TMEM lane quarter
    const int hsel = cw >> 2;                      // heads [16 hsel, 16 hsel + 16)
    const int row = quarter * 32 + lane;           // S^T row (tile row) / O^T lane
    const int st = cw * 32 + lane;                 // 0..255 within the compute group
    const uint32_t lanebase = (uint32_t)(quarter * 32) << 16;
    // decode: request q's cache and window block; prefill: one sequence whose
    // window is the raw token rows [max(0, t - n_win + 1), t]
    const long long kv_row_base = p.prefill ? 0ll : (long long)q * p.kv_rows_stride;
    const int req = p.prefill ? 0 : q;
    const int win_row0 = p.prefill ? max(0, t_pos - p.n_win + 1) : 0;
    int loaded = 0;  // tiles whose loads were issued (thread st == 0 drains them)

    const int32_t* bt_q = p.bt ? p.bt + (long long)q * p.bt_stride : nullptr;
    // Map rows of entries (invalid slots read the request's row 0, masked by the
    // softmax).  With paged entries every entry row is gathered: selected rows
    // (idx) or the dense rows, translated through the request's block table.
    auto rows_of = [&](const auto& e, auto& y) {
#pragma unroll
      for (int k = 0; k < (int)(sizeof(e) / sizeof(e[0])); ++k) {
        int v = e[k];
        if (v < 0 || v >= p.N) v = 0;
        y[k] = bt_q ? bt_q[v / p.rpb] * p.rpb + v % p.rpb : (int)(kv_row_base + v);
      }
    };
    // Entries of the rows this lane copies in tile j (rows 8 cw + 4 k + lane / 8),
    // loaded one tile ahead of their use so that no global-load latency lies on
    // the path from one tile to the next.
    auto load_copy_entries = [&](int j, int (&e)[kCopyRows]) {
      const Tile t = tiles.get(j);
#pragma unroll
      for (int k = 0; k < kCopyRows; ++k) {
        const int r = 8 * cw + 4 * k + (lane >> 3);
        int v = 0;
        if (t.seg == 0 && r < t.nrows) v = idx_q != nullptr ? idx_q[t.row0 + r] : t.row0 + r;
        e[k] = v;
      }
    };
    // The entry of this thread's row of tile j (its validity), also loaded a tile ahead.
    auto row_entry = [&](int j) -> int {
      const Tile t = tiles.get(j);
      if (row >= t.nrows || t.seg != 0) return 0;
      return idx_q != nullptr ? idx_q[t.row0 + row] : t.row0 + row;
    };
    // Issue the loads of tile j, block by block, each once PV of the previous
    // tile has released it.  Returns false on a failed wait (warp-uniform).
    auto issue_tile = [&](int j, const int (&ly)[kCopyRows]) -> bool {
      const Tile t = tiles.get(j);
      const bool gathered = t.seg == 0 && (idx_q != nullptr || bt_q != nullptr);
      const int u = lane & 7;
      for (int b = 0; b < kBlocks; ++b) {
        if (!tc::warp_wait(&bars->kvempty[b], (j & 1) ^ 1, abort)) return false;
        unsigned char* dst = base + kOffKv + 2 * b * kKvChunk;
        if (gathered) {
          // four 16-byte copies per lane: (row group k, chunk c), swizzled as TMA would
#pragma unroll
          for (int k = 0; k < kCopyRows; ++k) {
            const int r = 8 * cw + 4 * k + (lane >> 3);
            const long long mr = (ly[k] >= 0 && ly[k] < p.kvg_rows) ? ly[k] : 0;
            const bf16* src = p.kvg + mr * kC + 2 * b * 64 + u * 8;
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tc::cp_async16(tc::smem_u32(dst + c * kKvChunk + r * 128 + ((u ^ (r & 7)) << 4)), src + c * 64, 16);
          }
          tc::cp_async_commit();
          if (b > 0) {
            // block b-1 has landed: visible to the tensor core (async proxy), one arrival per warp
            tc::cp_async_wait<1>();
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->kvfull[b - 1]);
          }
        } else {
          // 3-D maps (dims, rows, request): rows past the request's own extent read as zeros
          if (st == 0) {
            tc::mbar_arrive_expect_tx(&bars->kvfull[b], kBlockBytes);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (t.seg == 0)
                tc::tma_load_3d(dst + c * kKvChunk, &tm_kv, &bars->kvfull[b], (2 * b + c) * 64, t.row0, req);
              else
                tc::tma_load_3d(dst + c * kKvChunk, &tm_win, &bars->kvfull[b], (2 * b + c) * 64,
                                (int)(win_row0 + t.row0), req);
            }
          } else if (lane == 0) {
            tc::mbar_arrive(&bars->kvfull[b]);
          }
          __syncwarp();
        }
      }
      if (gathered) {
        tc::cp_async_wait<0>();
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->kvfull[kBlocks - 1]);
      }
      return true;
    };

    // Every named barrier below is reached by all compute threads on every
    // iteration; failures are agreed through bar.red.or before anyone leaves.
    bool failed = false;
    // Row sums: lane l of this warp carries the sum over its quarter's rows of
    // P[row, 16 hsel + l % 16] (exactly the bf16 P_hi + P_lo that PV multiplies), over
    // all tiles so far, relative to the running maxima.
    float lw = 0.f;
    int ly[kCopyRows];  // map rows this lane copies in the next tile to load
    int le[kCopyRows];  // entries of those rows in the tile after it (loads in flight)
    int ev = 0;         // entry of this thread's row in the current tile
    if (nt > 0) {
      load_copy_entries(0, le);
      ev = row_entry(0);
      rows_of(le, ly);
      failed = !issue_tile(0, ly);
      if (!failed) loaded = 1;
      if (nt > 1) load_copy_entries(1, le);
    }
    for (int i = 0; i < nt; ++i) {
      const Tile t = tiles.get(i);
      const uint32_t ph = i & 1;
      bool valid = row < t.nrows;
      const int e_row = ev;
      if (i + 1 < nt) {
        ev = row_entry(i + 1);
        rows_of(le, ly);  // entries loaded during the previous tile
        if (i + 2 < nt) load_copy_entries(i + 2, le);
      }
      if (valid && t.seg == 0) {
        const int e = e_row;
        if (idx_q != nullptr) valid = e >= 0 && e < p.N;
        if (p.check) {
          unsigned int k = idx_q != nullptr ? entry_check(e, t_pos, p.rate, p.N) : 0u;
          if (valid && p.bt) {
            const int blk = p.bt[(long long)q * p.bt_stride + e / p.rpb];
            if (blk < 0 || blk >= p.pool_blocks) k |= kIdxBlock;
          }
          if (k) atomicOr(&g_mqa_tc_error, k << 1);
        }
      }
      float sv[kHpt];
      bool need = false;  // a score above its head's running maximum + 2^8 (or the first valid one)
      if (!failed) failed = !tc::warp_wait(&bars->sfull, ph, abort);
      if (!failed) {
        tc::fence_after_sync();
        uint32_t v[kHpt];
        tc::tmem_ld16(tmem + lanebase + kColS + kHpt * hsel, v);
        tc::tmem_ld_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->sempty);
#pragma unroll
        for (int c = 0; c < kHpt / 4; ++c) {
          const float4 m4 = *reinterpret_cast<const float4*>(bars->mref + kHpt * hsel + 4 * c);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int h = 4 * c + j;
            sv[h] = valid ? __uint_as_float(v[h]) * p.scale_log2 : neg_inf();
            need |= sv[h] > mm[j] + kRescaleLog2;  // -inf + 2^8 = -inf: any valid score of an empty head
          }
        }
        if (need) need_flag[i % 3] = 1;
      }
      if (tc::named_bar_or(1, 32 * kCompute, failed || *abort)) { failed = true; break; }
      // The flag of tile i+2 is cleared here: its writers are past the next barrier,
      // which this thread reaches first, and its last readers (tile i-1) are past this one.
      if (st == 0) need_flag[(i + 2) % 3] = 0;
      // Full path, only when some head's maximum grew by more than 2^8: exact tile
      // maxima, new running maxima and the rescale of the accumulators.  Otherwise
      // every head keeps its running maximum, exactly as the full path would decide.
      const bool full = need_flag[i % 3] != 0;
      if (full) {
        float tmp[kHpt];
#pragma unroll
        for (int h = 0; h < kHpt; ++h) tmp[h] = sv[h];
        const float tmax = warp_max16(tmp, lane);
        if (lane < kHpt) bars->red[quarter][kHpt * hsel + lane] = tmax;
        if (tc::named_bar_or(1, 32 * kCompute, failed || *abort)) { failed = true; break; }
        if (st < kH) {
          const int h = st;
          const float mt = fmaxf(fmaxf(bars->red[0][h], bars->red[1][h]), fmaxf(bars->red[2][h], bars->red[3][h]));
          const float mo = bars->mref[h];
          if (mt > mo + kRescaleLog2 || (mo == neg_inf() && mt != neg_inf())) {
            bars->alpha[h] = (mo == neg_inf()) ? 0.f : fast_exp2(mo - mt);
            bars->mref[h] = mt;
            bars->rescale = 1;
          } else {
            bars->alpha[h] = 1.f;
          }
        }
        if (tc::named_bar_or(1, 32 * kCompute, failed || *abort)) { failed = true; break; }
      }
      // PV(i-1) has completed here: the MMA thread issued it before QK(i), and the
      // commit that signalled S(i) tracks every MMA issued before it.  So the O^T
      // accumulators may be rescaled and the P buffers rewritten without a wait.
      if (full) {
        lw *= bars->alpha[kHpt * hsel + (lane & (kHpt - 1))];
        if (!failed && bars->rescale && i > 0) {
          // O^T holds the sums up to tile i-1: scale column h by alpha[h]
          tc::fence_after_sync();
#pragma unroll 1
          for (int part = 0; part < kBlocks + kWideBlocks; ++part) {
            const int blk = part < kBlocks ? part : part - kBlocks;  // then the lo halves of the wide blocks
            const uint32_t ta = tmem + lanebase + col_o(blk) + (part < kBlocks ? 0u : (uint32_t)kH) + kHpt * hsel;
            uint32_t v[kHpt];
            tc::tmem_ld16(ta, v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < kHpt; ++h) v[h] = __float_as_uint(__uint_as_float(v[h]) * bars->alpha[kHpt * hsel + h]);
            tc::tmem_st16(ta, v);
          }
          tc::tmem_st_wait();
          tc::fence_before_sync();
        }
        if (tc::named_bar_or(1, 32 * kCompute, failed || *abort)) { failed = true; break; }
        if (st == 0) bars->rescale = 0;  // every reader has passed the barrier above
      }
      // P = P_hi + P_lo, both bf16 (PV(i-1), the last reader of the P buffers, has completed)
      unsigned char* phi = base + kOffP + row * 128;
      unsigned char* plo = phi + kPBytes;
#pragma unroll
      for (int cc = 0; cc < kHpt / 8; ++cc) {
        const int c = (kHpt / 8) * hsel + cc;  // 16-byte unit of the row: heads 8c .. 8c+7
        const float4 ma = *reinterpret_cast<const float4*>(bars->mref + c * 8);
        const float4 mb = *reinterpret_cast<const float4*>(bars->mref + c * 8 + 4);
        const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int h = cc * 8 + 2 * j;
          const float m0 = mm[2 * j], m1 = mm[2 * j + 1];
          const float p0 = (m0 == neg_inf()) ? 0.f : fast_exp2(sv[h] - m0);
          const float p1 = (m1 == neg_inf()) ? 0.f : fast_exp2(sv[h + 1] - m1);
          // P_hi = p truncated to bf16, P_lo = the (exact) remainder truncated to bf16:
          // relative error below 2^-14, by integer masks instead of conversions
          const uint32_t h0 = __float_as_uint(p0) & 0xffff0000u, h1 = __float_as_uint(p1) & 0xffff0000u;
          const uint32_t l0 = __float_as_uint(p0 - __uint_as_float(h0)) & 0xffff0000u;
          const uint32_t l1 = __float_as_uint(p1 - __uint_as_float(h1)) & 0xffff0000u;
          wh[j] = __byte_perm(h0, h1, 0x7632);
          wl[j] = __byte_perm(l0, l1, 0x7632);
          sv[h] = __uint_as_float(h0) + __uint_as_float(l0);  // the probability PV uses (exact in f32)
          sv[h + 1] = __uint_as_float(h1) + __uint_as_float(l1);
        }
        const uint32_t sw = (uint32_t)((c ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(phi + sw) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        *reinterpret_cast<uint4*>(plo + sw) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->pfull);
      lw += warp_sum16(sv, lane);
      // next tile's rows, block by block as PV(i) releases them
      if (!failed && i + 1 < nt) {
        if (issue_tile(i + 1, ly)) loaded = i + 2;
        else failed = true;
      }
    }
    // ---- epilogue: O^T (dims x heads) and l ----
    // The four quarters' row-sum partials meet in shared memory.  Every compute
    // thread reaches this barrier (the loop only ends together or normally) and
    // it also settles, for all of them, whether a wait failed on the last tile.
    if (lane < kHpt) bars->red[quarter][kHpt * hsel + lane] = lw;
    bool ok = !tc::named_bar_or(1, 32 * kCompute, failed || *abort);
    if (ok && nt > 0) ok = tc::warp_wait(&bars->odone, (nt - 1) & 1, abort);
    // every compute warp takes the same branch below (the unsplit path has a barrier)
    ok = !tc::named_bar_or(1, 32 * kCompute, !ok);
    if (ok) {
      tc::fence_after_sync();
      uint32_t lv[kHpt];
      // an unsplit query's sink logit joins its denominator here (base-2 scale, against the
      // head's running maximum); split queries leave it to the combine
      const bool sink_here = p.sink != nullptr && p.splits == 1;
#pragma unroll
      for (int h = 0; h < kHpt; ++h) {
        const int hh = kHpt * hsel + h;
        float l = (bars->red[0][hh] + bars->red[1][hh]) + (bars->red[2][hh] + bars->red[3][hh]);
        if (sink_here) l += fast_exp2(p.sink[hh] * kLog2e - bars->mref[hh]);
        lv[h] = __float_as_uint(l);
      }
      const int dim_lane = quarter * 32 + lane;
      if (p.splits == 1) {
        // The output leaves block by block as TMA tensor stores (a map of the same
        // shape as the queries'): each 128-dim block is staged as two 128B-swizzled
        // [64 heads x 64 dims] boxes in the tile buffer, which the last PV has
        // released and no load refills, and its store overlaps the next block's staging.
        const int rope0 = kC - p.rope_dims;
        float inv[kHpt];
#pragma unroll
        for (int h = 0; h < kHpt; ++h) {
          const float l = __uint_as_float(lv[h]);
          inv[h] = (nt > 0 && l > 0.f) ? __fdividef(1.f, l) : 0.f;
        }
        const int dl = dim_lane & 63;                    // dim within its 64-dim chunk
        const uint32_t ubyte = (uint32_t)(dl * 2);       // byte within the 128-byte row
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
          uint32_t v[kHpt];
          if (nt > 0) {
            tc::tmem_ld16(tmem + lanebase + col_o(mb) + kHpt * hsel, v);
            if (wide_block(mb)) {
              uint32_t w[kHpt];
              tc::tmem_ld16(tmem + lanebase + col_o(mb) + kH + kHpt * hsel, w);
              tc::tmem_ld_wait();
#pragma unroll
              for (int h = 0; h < kHpt; ++h) v[h] = __float_as_uint(__uint_as_float(v[h]) + __uint_as_float(w[h]));
            }
            tc::tmem_ld_wait();
          } else {
#pragma unroll
            for (int h = 0; h < kHpt; ++h) v[h] = 0u;
          }
          const int d = mb * 128 + dim_lane;
          // chunk 2 mb + dim_lane / 64 of the output, rows = heads
          unsigned char* box = base + kOffKv + (2 * mb + (dim_lane >> 6)) * kQChunk;
          // partial-RoPE output rotation by -t: channel d pairs with d ^ 1, the
          // neighbouring TMEM lane (lane ^ 1 of this warp); whole warps take the branch
          const bool rot = p.rope_dims > 0 && mb * 128 + quarter * 32 + 31 >= rope0;
          float rc = 1.f, rsx = 0.f;
          if (rot && d >= rope0) {
            float sn;
            rope_cos_sin(t_pos, (d - rope0) >> 1, p.rope_dims, p.rope_base, rc, sn);
            rsx = (d & 1) ? -sn : sn;
          }
#pragma unroll
          for (int h = 0; h < kHpt; ++h) {
            float o = inv[h] != 0.f ? __uint_as_float(v[h]) * inv[h] : 0.f;
            if (rot) o = fmaf(o, rc, __shfl_xor_sync(0xffffffffu, o, 1) * rsx);
            const int hh = kHpt * hsel + h;
            *reinterpret_cast<bf16*>(box + hh * 128 + ((((ubyte >> 4) ^ (hh & 7)) << 4) | (ubyte & 15))) =
                __float2bfloat16_rn(o);
          }
          tc::fence_proxy_async_smem();
          tc::named_bar(1, 32 * kCompute);
          if (st == 0) {
            for (int c = 0; c < 2; ++c)
              tc::tma_store_2d(&tm_out, (2 * mb + c) * 64, q * kH,
                               tc::smem_u32(base + kOffKv + (2 * mb + c) * kQChunk));
            tc::bulk_commit();
          }
        }
        if (st == 0) tc::bulk_wait_read_all();
      } else {
        float* wo = p.ws_o + ((long long)q * p.splits + sp) * kH * kC + (long long)(kHpt * hsel) * kC;
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
          uint32_t v[kHpt];
          if (nt > 0) {
            tc::tmem_ld16(tmem + lanebase + col_o(mb) + kHpt * hsel, v);
            if (wide_block(mb)) {
              uint32_t w[kHpt];
              tc::tmem_ld16(tmem + lanebase + col_o(mb) + kH + kHpt * hsel, w);
              tc::tmem_ld_wait();
#pragma unroll
              for (int h = 0; h < kHpt; ++h) v[h] = __float_as_uint(__uint_as_float(v[h]) + __uint_as_float(w[h]));
            }
            tc::tmem_ld_wait();
          }
          const int d = mb * 128 + dim_lane;
#pragma unroll
          for (int h = 0; h < kHpt; ++h) wo[h * kC + d] = nt > 0 ? __uint_as_float(v[h]) : 0.f;
        }
        if (quarter == 0) {
          // lane l < 16 of the quarter-0 warps: head 16 hsel + l (l is the same in every TMEM lane)
          float l = 0.f;  // lv[lane] without a dynamically indexed register array
#pragma unroll
          for (int h = 0; h < kHpt; ++h) l = (h == lane && nt > 0) ? __uint_as_float(lv[h]) : l;
          const int hh = kHpt * hsel + lane;
          if (lane < kHpt)
            p.ws_ml[((long long)q * p.splits + sp) * kH + hh] = make_float2(l > 0.f ? bars->mref[hh] : neg_inf(), l);
        }
      }
    }
    // drain: every block load issued has landed before the CTA may exit
    tc::cp_async_wait<0>();
    if (st == 0 && loaded > 0) {
      const int j = loaded - 1;
      for (int b = 0; b < kBlocks; ++b)
        for (uint32_t k = 0; k < tc::kSpinLimit && !tc::mbar_try_wait(&bars->kvfull[b], j & 1); ++k) __nanosleep(64);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && bars->abort) atomicOr(&g_mqa_tc_error, 1u);
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- host side ------------------------------------------------------------------
bool mqa_tc_supported(const MqaProblem& p) {
  if (p.H != kH || p.c != kC || p.n_win > 256) return false;
  if (p.mode == HCA_MODE_PREFILL) return p.win_rows > 0 && p.bt == nullptr;
  if (p.bt) return p.mode == HCA_MODE_DECODE && p.rpb >= 1 && p.pool_rows >= 1 && p.win_seq_stride % kC == 0;
  return p.mode == HCA_MODE_DECODE && p.kv_seq_stride % kC == 0 && p.win_seq_stride % kC == 0;
}

// Splits per query: at most num_sms CTAs per wave, fewest tiles on the critical path.
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
    const long long cost = waves * (tpc * 4 + 3) + (s_eff > 1 ? 2 : 0);  // tiles + per-CTA setup, + combine
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best_s = s_eff; }
  }
  const int tpc = (tiles + best_s - 1) / best_s;
  pl.splits = best_s;
  // Splits start on tile boundaries of the entries segment (rows_per_split is a
  // multiple of the tile height and each segment is tiled from its own start).
  pl.rows_per_split = tpc * kRows;
  pl.ws_bytes = best_s > 1 ? (size_t)p.Tq * best_s * kH * ((size_t)kC * sizeof(float) + sizeof(float2)) : 0;
  return pl;
}

extern cudaError_t make_tmap_bf16(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                                  const uint64_t* strides_bytes, uint32_t box_rows);

cudaError_t launch_mqa_decode_tc(const MqaProblem& p, const MqaPlan& pl, void* ws, cudaStream_t stream, bool pdl) {
  if (p.Tq == 0) return cudaSuccess;
  CUtensorMap tm_q, tm_kv, tm_win, tm_out;
  const uint64_t rstride[1] = {(uint64_t)kC * 2};
  const uint64_t qd[2] = {(uint64_t)kC, (uint64_t)p.Tq * kH};
  cudaError_t e = make_tmap_bf16(&tm_q, p.q, 2, qd, rstride, 64);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tm_out, p.out, 2, qd, rstride, 64);  // unsplit queries store through it
  if (e != cudaSuccess) return e;
  const bool prefill = p.mode == HCA_MODE_PREFILL;
  const long long kv_rs = (prefill || p.bt) ? 0 : p.kv_seq_stride / kC;
  // (paged: the maps cover the whole pool; only the gather map is used)
  const uint64_t n_kv = p.bt ? (uint64_t)p.pool_rows : (uint64_t)(p.N > 0 ? p.N : 1);
  // With no entries the entry maps are never used (no entry tiles): point them at
  // the window rows, which exist, instead of a cache that may have no rows.
  const void* kv_base = p.N > 0 ? (const void*)p.kv : (const void*)p.win;
  // dense tiles: (dims, rows of one request, request), so a tile never reads
  // another request's rows or the unused capacity behind a request's entries
  const uint64_t kvd3[3] = {(uint64_t)kC, n_kv, (prefill || p.bt) ? 1ull : (uint64_t)p.Tq};
  const long long kv_req_elems =
      (prefill || p.bt || p.Tq == 1 || p.N <= 0) ? (long long)n_kv * kC : p.kv_seq_stride;
  const uint64_t kvs3[2] = {(uint64_t)kC * 2, (uint64_t)kv_req_elems * 2};
  e = make_tmap_bf16(&tm_kv, kv_base, 3, kvd3, kvs3, kRows);
  if (e != cudaSuccess) return e;
  // gathered rows: copied by the threads from one range over every request's rows
  const long long kvg_rows = (long long)(p.Tq - 1) * kv_rs + (long long)n_kv;
  const long long win_rs = prefill ? 0 : p.win_seq_stride / kC;
  const uint64_t wd3[3] = {(uint64_t)kC, prefill ? (uint64_t)p.win_rows : (uint64_t)p.n_win,
                           prefill ? 1ull : (uint64_t)p.Tq};
  const long long win_req_elems = prefill ? p.win_rows * kC : (p.Tq == 1 ? (long long)p.n_win * kC : p.win_seq_stride);
  const uint64_t ws3[2] = {(uint64_t)kC * 2, (uint64_t)win_req_elems * 2};
  e = make_tmap_bf16(&tm_win, p.win, 3, wd3, ws3, kRows);
  if (e != cudaSuccess) return e;
  MqaTcParams a;
  a.idx = p.idx;
  a.n_idx = p.n_idx;
  a.q_pos = p.q_pos;
  a.rate = p.rate;
  a.N = p.N;
  a.n_win = p.n_win;
  a.prefill = prefill ? 1 : 0;
  a.kv_rows_stride = kv_rs;
  a.win_rows_stride = win_rs;
  a.scale_log2 = p.scale * kLog2e;
  a.splits = pl.splits;
  a.rows_per_split = pl.rows_per_split;
  a.out = p.out;
  a.sink = p.sink;
  a.rope_dims = p.rope_dims;
  a.rope_base = p.rope_base;
  a.bt = p.bt;
  a.bt_stride = p.bt_stride;
  a.rpb = p.rpb > 0 ? p.rpb : 1;
  a.pool_blocks = p.bt ? p.pool_rows / a.rpb : 0;
  a.check = p.check;
  a.kvg = reinterpret_cast<const bf16*>(kv_base);
  a.kvg_rows = kvg_rows;
  a.ws_o = pl.splits > 1 ? reinterpret_cast<float*>(ws) : nullptr;
  a.ws_ml = pl.splits > 1 ? reinterpret_cast<float2*>(reinterpret_cast<float*>(ws) + (size_t)p.Tq * pl.splits * kH * kC)
                          : nullptr;
  e = cudaFuncSetAttribute((const void*)mqa_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(pdl, mqa_decode_tc_kernel, dim3(p.Tq * pl.splits), dim3(kThreads), kSmemBytes, stream, tm_q, tm_kv,
                 tm_win, tm_out, a);
  ++g_launch_counter;
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || pl.splits == 1) return e;
  return launch_mqa_combine(a.ws_o, a.ws_ml, p.Tq, pl.splits, kH, kC, p.out, p.sink, p.q_pos, p.rope_dims,
                            p.rope_base, stream, pdl);
}

unsigned int read_and_clear_mqa_tc_error() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_mqa_tc_error, sizeof(v)) != cudaSuccess) return 0xffffffffu;
  if (v) cudaMemcpyToSymbol(g_mqa_tc_error, &zero, sizeof(zero));
  return v;
}

}  // namespace hca
