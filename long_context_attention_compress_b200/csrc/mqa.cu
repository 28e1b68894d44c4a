// Shared-KV multi-query attention over compressed entries + sliding window
// (sm_100a), CUDA-core version with split-K and a combine kernel.
//
// For query t and head h over the row set U(t) (QbitAI write-up,
// "混合注意力機制": CSA step three, KV entries serve as both key and value,
// and the sliding-window branch of the most recent 128 raw tokens;
// "DeepSeek V4 Architecture Tricks", HCA section: dense over all entries):
//   o[t,h,:] = sum_u softmax_u(scale * q[t,h,:] . row_u) row_u
// U(t) = selected CSA entries (idx) or all visible HCA entries, then the
// window rows.  Each query's row list is cut into `splits` contiguous ranges;
// one CTA runs an online softmax over its range in tiles of TR rows and
// writes either the normalised output (one split) or its softmax state
// (m, l, unnormalised o) for the combine kernel:
//   o = sum_i e^{m_i - M} o_i / sum_i e^{m_i - M} l_i.

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hca {

constexpr int kMqaThreads = 256;

// index-check record of this kernel (entry_check bits)
__device__ unsigned int g_mqa_index_error = 0;
constexpr int kTR = 16;  // rows per tile

struct RowList {
  const bf16* kv;       // this request's entries
  const int32_t* idx;   // this query's selected entries or nullptr
  int n_first;          // length of the entry part
  int N;                // entries of the request
  int t;                // the query's position
  const bf16* win;      // first window row
  int n_win;            // window rows
  int c;
  __device__ __forceinline__ int length() const { return n_first + n_win; }
  // pointer of list row u, or nullptr for an empty (or out-of-range) selected slot
  __device__ __forceinline__ const bf16* row(int u) const {
    if (u < n_first) {
      int s = idx ? idx[u] : u;
      return (s < 0 || s >= N) ? nullptr : kv + (long long)s * c;
    }
    return win + (long long)(u - n_first) * c;
  }
};

__device__ __forceinline__ RowList make_rows(const MqaProblem& p, int q) {
  RowList L;
  const int t = p.q_pos[q];
  const long long rs = p.mode == HCA_MODE_DECODE ? q : 0;
  L.kv = p.kv + rs * p.kv_seq_stride;
  L.c = p.c;
  L.N = p.N;
  L.t = t;
  if (p.idx) {
    L.idx = p.idx + (long long)q * p.n_idx;
    L.n_first = p.n_idx;
  } else {
    L.idx = nullptr;
    L.n_first = n_visible(t, p.rate, p.N);
  }
  if (p.mode == HCA_MODE_DECODE) {
    L.win = p.win + rs * p.win_seq_stride;
    L.n_win = min(p.n_win, t + 1);
  } else {
    const int w0 = max(0, t - p.n_win + 1);
    L.win = p.win + (long long)w0 * p.c;
    L.n_win = t - w0 + 1;
  }
  return L;
}

template <int H, int C>
__global__ void __launch_bounds__(kMqaThreads) mqa_split_kernel(MqaProblem p, int splits, int rows_per_split,
                                                                float* __restrict__ ws_o, float2* __restrict__ ws_ml) {
  constexpr int CP = C + 8;  // padded smem row stride (bf16 elements)
  constexpr int DPT = H * C / kMqaThreads;
  static_assert(H * C % kMqaThreads == 0, "outputs per thread");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  bf16* s_q = reinterpret_cast<bf16*>(smem_raw);                   // [H][CP]
  bf16* s_r = s_q + H * CP;                                         // [TR][CP]
  float* s_s = reinterpret_cast<float*>(s_r + kTR * CP);            // [H][TR] scores
  float* s_p = s_s + H * kTR;                                       // [TR][H] probabilities
  float* s_m = s_p + kTR * H;                                       // [H]
  float* s_l = s_m + H;                                             // [H]
  float* s_a = s_l + H;                                             // [H] rescale factor
  __shared__ int s_valid[kTR];

  const int tid = threadIdx.x;
  const int q = blockIdx.x / splits;
  const int sp = blockIdx.x % splits;
  const RowList L = make_rows(p, q);
  const int u_begin = sp * rows_per_split;
  const int u_end = min(L.length(), u_begin + rows_per_split);

  // stage q [H][C]
  const bf16* qp = p.q + (long long)q * H * C;
  for (int e = tid; e < H * C / 8; e += kMqaThreads) {
    const int h = e / (C / 8), d = (e % (C / 8)) * 8;
    *reinterpret_cast<uint4*>(s_q + h * CP + d) = *reinterpret_cast<const uint4*>(qp + h * C + d);
  }
  for (int h = tid; h < H; h += kMqaThreads) { s_m[h] = neg_inf(); s_l[h] = 0.f; }
  float o[DPT];
#pragma unroll
  for (int j = 0; j < DPT; ++j) o[j] = 0.f;
  const float sl2 = p.scale * kLog2e;

  for (int u0 = u_begin; u0 < u_end; u0 += kTR) {
    __syncthreads();  // previous tile fully consumed
    // load TR rows (zeros for missing rows)
    for (int e = tid; e < kTR * (C / 8); e += kMqaThreads) {
      const int r = e / (C / 8), d = (e % (C / 8)) * 8;
      const int u = u0 + r;
      const bf16* rp = u < u_end ? L.row(u) : nullptr;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (rp) v = *reinterpret_cast<const uint4*>(rp + d);
      *reinterpret_cast<uint4*>(s_r + r * CP + d) = v;
      if (d == 0) {
        s_valid[r] = rp != nullptr;
        if (p.check && L.idx && u < u_end && u < L.n_first) {
          const unsigned int k = entry_check(L.idx[u], L.t, p.rate, p.N);
          if (k) atomicOr(&g_mqa_index_error, k);
        }
      }
    }
    __syncthreads();
    // scores S[h][u] (base-2 scaled)
    for (int pr = tid; pr < H * kTR; pr += kMqaThreads) {
      const int h = pr / kTR, r = pr % kTR;
      const bf16* a = s_q + h * CP;
      const bf16* b = s_r + r * CP;
      float acc = 0.f;
#pragma unroll 4
      for (int d = 0; d < C; d += 8) {
        float fa[8], fb[8];
        unpack8(*reinterpret_cast<const uint4*>(a + d), fa);
        unpack8(*reinterpret_cast<const uint4*>(b + d), fb);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc = fmaf(fa[k], fb[k], acc);
      }
      s_s[h * kTR + r] = s_valid[r] ? acc * sl2 : neg_inf();
    }
    __syncthreads();
    // online softmax per head
    for (int h = tid; h < H; h += kMqaThreads) {
      float mx = s_m[h];
      float tm = neg_inf();
#pragma unroll
      for (int r = 0; r < kTR; ++r) tm = fmaxf(tm, s_s[h * kTR + r]);
      const float mn = fmaxf(mx, tm);
      float alpha = 1.f, lsum = 0.f;
      if (mn == neg_inf()) {
#pragma unroll
        for (int r = 0; r < kTR; ++r) s_p[r * H + h] = 0.f;
      } else {
        alpha = fast_exp2(mx - mn);
#pragma unroll
        for (int r = 0; r < kTR; ++r) {
          const float e = fast_exp2(s_s[h * kTR + r] - mn);
          s_p[r * H + h] = e;
          lsum += e;
        }
        s_m[h] = mn;
      }
      s_l[h] = s_l[h] * alpha + lsum;
      s_a[h] = alpha;
    }
    __syncthreads();
    // o = o * alpha + P V
#pragma unroll
    for (int j = 0; j < DPT; ++j) {
      const int oi = tid + kMqaThreads * j;
      o[j] *= s_a[oi / C];
    }
#pragma unroll 2
    for (int r = 0; r < kTR; ++r) {
      const bf16* rr = s_r + r * CP;
      const float* pr = s_p + r * H;
#pragma unroll
      for (int j = 0; j < DPT; ++j) {
        const int oi = tid + kMqaThreads * j;
        const int h = oi / C, d = oi % C;
        o[j] = fmaf(pr[h], __bfloat162float(rr[d]), o[j]);
      }
    }
  }
  __syncthreads();
  if (splits == 1) {
    if (p.sink) {
      // the sink joins the denominator (in the base-2 scale of the running maxima)
      for (int h = tid; h < H; h += kMqaThreads) s_l[h] += fast_exp2(p.sink[h] * kLog2e - s_m[h]);
      __syncthreads();
    }
    bf16* op = p.out + (long long)q * H * C;
    const int rope0 = C - p.rope_dims;
#pragma unroll
    for (int j = 0; j < DPT; ++j) {
      const int oi = tid + kMqaThreads * j;
      const float l = s_l[oi / C];
      float v = l > 0.f ? o[j] / l : 0.f;
      if (p.rope_dims > 0) {
        // partial-RoPE output rotation by -t: channel d pairs with d ^ 1, held by lane ^ 1
        const float pr = __shfl_xor_sync(0xffffffffu, v, 1);
        const int d = oi % C;
        if (d >= rope0) {
          float cs, sn;
          rope_cos_sin(p.q_pos[q], (d - rope0) >> 1, p.rope_dims, p.rope_base, cs, sn);
          v = fmaf(v, cs, pr * ((d & 1) ? -sn : sn));
        }
      }
      op[oi] = __float2bfloat16_rn(v);
    }
  } else {
    float* wo = ws_o + ((long long)q * splits + sp) * H * C;
#pragma unroll
    for (int j = 0; j < DPT; ++j) wo[tid + kMqaThreads * j] = o[j];
    for (int h = tid; h < H; h += kMqaThreads)
      ws_ml[((long long)q * splits + sp) * H + h] = make_float2(s_m[h], s_l[h]);
  }
}

// combine: o = sum_i e^{m_i - M} o_i / sum_i e^{m_i - M} l_i per (query, head).
// 256 threads per CTA, TPH per head (256 / TPH heads per CTA), each thread owning
// the float4s t, t + TPH, ... of its head's output (C <= 512).  The first BATCH
// splits' float4s are loaded before the weights are formed, so that their latency
// overlaps the reductions over the splits' (m, l); later batches follow one load
// round each.  The sum runs over the splits in order with the normalised weights
// w_i / den formed at use.  Few queries take TPH = 128 with 16 splits in flight
// (one wave at two CTAs per SM); many take TPH = 64 with 4, which needs fewer
// registers, so that more CTAs share an SM.
constexpr int kCombMaxSplits = 1024;  // planners never exceed this
template <int TPH, int BATCH>
__global__ void __launch_bounds__(256) mqa_combine_kernel(const float* __restrict__ ws_o,
                                                          const float2* __restrict__ ws_ml, int splits,
                                                          int H, int C, bf16* __restrict__ out,
                                                          const float* __restrict__ sink,
                                                          const int32_t* __restrict__ q_pos, int rope_dims,
                                                          float rope_base) {
  constexpr int kHeads = 256 / TPH, kWarps = TPH / 32, kF = 128 / TPH;
  __shared__ float s_w[kHeads][kCombMaxSplits];
  __shared__ float s_red[kHeads][2][kWarps];
  tc::griddep_wait();  // the partial states come from the attention kernel
  const int hh = threadIdx.x / TPH, t = threadIdx.x % TPH, lane = t & 31, wq = t >> 5;
  const int q = blockIdx.x, h = blockIdx.y * kHeads + hh;
  if (h >= H) return;  // the whole TPH-thread group: its named barrier counts no one else
  const int bar = 1 + hh;
  const int per_head = C >> 2;
  const long long sstride = (long long)H * C / 4;  // float4s between splits
  const float4* src = reinterpret_cast<const float4*>(ws_o + ((long long)q * splits * H + h) * C) + t;
  float4 v[BATCH][kF];
#pragma unroll
  for (int u = 0; u < BATCH; ++u)
#pragma unroll
    for (int f = 0; f < kF; ++f)
      v[u][f] = (t + f * TPH < per_head && u < splits) ? src[u * sstride + f * TPH] : make_float4(0.f, 0.f, 0.f, 0.f);
  // weights: the maximum over the splits (and the sink logit), then the denominator
  const float2* ml = ws_ml + (long long)q * splits * H + h;  // split s at ml[s * H]
  float M = neg_inf();
  for (int s = t; s < splits; s += TPH) M = fmaxf(M, ml[(long long)s * H].x);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) s_red[hh][0][wq] = M;
  asm volatile("bar.sync %0, %1;" ::"r"(bar), "n"(TPH) : "memory");
  M = s_red[hh][0][0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) M = fmaxf(M, s_red[hh][0][w]);
  // a sink logit (base-2 scale like the maxima) joins the denominator once per query
  const float z = sink ? sink[h] * kLog2e : neg_inf();
  M = fmaxf(M, z);
  float den = 0.f;
  for (int s = t; s < splits; s += TPH) {
    const float2 m_l = ml[(long long)s * H];
    const float w = m_l.y > 0.f ? fast_exp2(m_l.x - M) : 0.f;
    s_w[hh][s] = w;
    den += w * m_l.y;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane == 0) s_red[hh][1][wq] = den;
  asm volatile("bar.sync %0, %1;" ::"r"(bar), "n"(TPH) : "memory");
  den = s_red[hh][1][0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) den += s_red[hh][1][w];
  if (sink) den += fast_exp2(z - M);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float4 acc[kF];
#pragma unroll
  for (int f = 0; f < kF; ++f) acc[f] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < splits; s0 += BATCH) {
    if (s0 > 0) {
#pragma unroll
      for (int u = 0; u < BATCH; ++u)
#pragma unroll
        for (int f = 0; f < kF; ++f)
          if (t + f * TPH < per_head && s0 + u < splits) v[u][f] = src[(s0 + u) * sstride + f * TPH];
    }
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      if (s0 + u < splits) {
        const float w = s_w[hh][s0 + u] * inv;
#pragma unroll
        for (int f = 0; f < kF; ++f) {
          acc[f].x = fmaf(w, v[u][f].x, acc[f].x); acc[f].y = fmaf(w, v[u][f].y, acc[f].y);
          acc[f].z = fmaf(w, v[u][f].z, acc[f].z); acc[f].w = fmaf(w, v[u][f].w, acc[f].w);
        }
      }
    }
  }
#pragma unroll
  for (int f = 0; f < kF; ++f) {
    const int d4 = t + f * TPH;
    if (d4 >= per_head) break;
    float4 o = acc[f];
    if (rope_dims > 0 && d4 * 4 >= C - rope_dims) {
      // partial-RoPE output rotation by -t of the pairs (x, y) and (z, w):
      // a' = a cos + b sin, b' = b cos - a sin
      const int j = (d4 * 4 - (C - rope_dims)) >> 1;
      float c0, s0, c1, s1;
      rope_cos_sin(q_pos[q], j, rope_dims, rope_base, c0, s0);
      rope_cos_sin(q_pos[q], j + 1, rope_dims, rope_base, c1, s1);
      o = make_float4(fmaf(o.x, c0, o.y * s0), fmaf(o.y, c0, -o.x * s0), fmaf(o.z, c1, o.w * s1),
                      fmaf(o.w, c1, -o.z * s1));
    }
    uint2 pk;
    pk.x = pack_bf16x2(o.x, o.y);
    pk.y = pack_bf16x2(o.z, o.w);
    *reinterpret_cast<uint2*>(out + ((long long)q * H + h) * C + d4 * 4) = pk;
  }
}

template <int H, int C>
static size_t mqa_smem() {
  return (size_t)(H + kTR) * (C + 8) * sizeof(bf16) + (size_t)(2 * H * kTR + 3 * H) * sizeof(float);
}

cudaError_t launch_mqa_combine(const float* ws_o, const float2* ws_ml, int Tq, int splits, int H, int C, bf16* out,
                               const float* sink, const int32_t* q_pos, int rope_dims, float rope_base,
                               cudaStream_t stream, bool pdl) {
  if (C % 4 != 0 || C > 4 * 128 || splits < 1 || splits > kCombMaxSplits) return cudaErrorInvalidValue;
  cudaError_t e;
  if ((long long)Tq * ((H + 1) / 2) <= 2ll * device_sm_count())
    e = launch_pdl(pdl, mqa_combine_kernel<128, 16>, dim3(Tq, (H + 1) / 2), dim3(256), 0, stream, ws_o, ws_ml, splits,
                   H, C, out, sink, q_pos, rope_dims, rope_base);
  else
    e = launch_pdl(pdl, mqa_combine_kernel<64, 4>, dim3(Tq, (H + 3) / 4), dim3(256), 0, stream, ws_o, ws_ml, splits,
                   H, C, out, sink, q_pos, rope_dims, rope_base);
  if (e != cudaSuccess) return e;
  ++g_launch_counter;
  return cudaGetLastError();
}

size_t mqa_ws_upper_bound(const MqaProblem& p) {
  MqaProblem v0 = p;
  v0.mode = HCA_MODE_PREFILL;  // the CUDA-core plan, for any row count up to max(N, n_idx)
  size_t b = plan_mqa_cuda_cores(v0).ws_bytes;
  const int sms = device_sm_count();
  const long long smax = p.Tq > 0 ? std::max(1, (2 * sms) / p.Tq) : 1;
  const size_t tc_bound = (size_t)p.Tq * smax * p.H * ((size_t)p.c * sizeof(float) + sizeof(float2));
  MqaProblem d = p;
  d.mode = HCA_MODE_DECODE;
  const size_t v0d = plan_mqa_cuda_cores(d).ws_bytes;
  return std::max(b, std::max(tc_bound, v0d));
}

MqaPlan plan_mqa(const MqaProblem& p) { return plan_mqa_sms(p, device_sm_count()); }

MqaPlan plan_mqa_sms(const MqaProblem& p, int sms) {
  if (mqa_tc_supported(p)) return plan_mqa_tc(p, sms);
  return plan_mqa_cuda_cores(p);
}

MqaPlan plan_mqa_cuda_cores(const MqaProblem& p) {
  MqaPlan pl;
  const int first = p.idx ? p.n_idx : p.N;
  pl.max_rows = first + p.n_win;
  const int target_ctas = 148 * 4;
  int splits = 1;
  if (p.Tq < target_ctas) {
    splits = (target_ctas + p.Tq - 1) / p.Tq;
    const int max_splits = (pl.max_rows + kTR - 1) / kTR;
    if (splits > max_splits) splits = max_splits;
    if (splits > kCombMaxSplits) splits = kCombMaxSplits;
    if (splits < 1) splits = 1;
  }
  int rps = (pl.max_rows + splits - 1) / splits;
  rps = (rps + kTR - 1) / kTR * kTR;
  splits = (pl.max_rows + rps - 1) / rps;
  if (splits < 1) splits = 1;
  pl.splits = splits;
  pl.rows_per_split = rps;
  pl.ws_bytes = splits > 1 ? (size_t)p.Tq * splits * p.H * ((size_t)p.c * sizeof(float) + sizeof(float2)) : 0;
  return pl;
}

template <int H, int C>
static cudaError_t launch_mqa_t(const MqaProblem& p, const MqaPlan& pl, void* ws, cudaStream_t stream) {
  const size_t smem = mqa_smem<H, C>();
  cudaError_t e = cudaFuncSetAttribute((const void*)mqa_split_kernel<H, C>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  float* ws_o = nullptr;
  float2* ws_ml = nullptr;
  if (pl.splits > 1) {
    ws_o = reinterpret_cast<float*>(ws);
    ws_ml = reinterpret_cast<float2*>(ws_o + (size_t)p.Tq * pl.splits * H * C);
  }
  mqa_split_kernel<H, C><<<p.Tq * pl.splits, kMqaThreads, smem, stream>>>(p, pl.splits, pl.rows_per_split,
                                                                          ws_o, ws_ml);
  ++g_launch_counter;
  e = cudaGetLastError();
  if (e != cudaSuccess || pl.splits == 1) return e;
  return launch_mqa_combine(ws_o, ws_ml, p.Tq, pl.splits, H, C, p.out, p.sink, p.q_pos, p.rope_dims, p.rope_base,
                            stream, false);
}

unsigned int read_and_clear_mqa_index_error() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_mqa_index_error, sizeof(v)) != cudaSuccess) return 0xffffffffu;
  if (v) cudaMemcpyToSymbol(g_mqa_index_error, &zero, sizeof(zero));
  return v;
}

cudaError_t launch_mqa(const MqaProblem& p, const MqaPlan& pl, void* ws, cudaStream_t stream, bool pdl) {
  if (p.Tq == 0) return cudaSuccess;
  if (mqa_tc_supported(p)) return launch_mqa_decode_tc(p, pl, ws, stream, pdl);
  if (p.bt) return cudaErrorInvalidValue;  // paged entries: tensor-core kernel only
  if (p.H == 64 && p.c == 512) return launch_mqa_t<64, 512>(p, pl, ws, stream);
  if (p.H == 4 && p.c == 64) return launch_mqa_t<4, 64>(p, pl, ws, stream);
  return cudaErrorInvalidValue;
}

}  // namespace hca
