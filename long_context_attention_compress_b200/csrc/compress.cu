// Softmax-gated KV compression (CSA overlapped, HCA plain), sm_100a.
//
// What it computes ("DeepSeek V4 Architecture Tricks", section
// "压缩 KV 的具体 trick"; QbitAI write-up, "混合注意力機制", CSA step one and
// the HCA paragraph): each compressed entry is, per channel, a softmax over
// the entry's tokens of (weight logit + learnable positional bias), used to
// weight the tokens' KV candidates.  CSA entry i pools the previous and the
// current block of m tokens (bias rows 0..m-1 / m..2m-1); HCA entry i pools
// its own block of m' tokens.
//
// Design: HBM-bound (reads 2 bf16 per token and channel, writes 1 bf16 per
// entry and channel).  One thread owns 8 consecutive channels (16-byte
// vector loads of candidates and logits) of one entry and a group of G
// tokens; the TG = window/G threads of an entry sit in consecutive lanes of
// a warp and merge their partial softmax states with xor-shuffles.  Softmax
// runs online in f32 with exp2.

#include "common.cuh"
#include "internal.h"

namespace hca {

struct SoftState {
  float mx[8], l[8], acc[8];
};

__device__ __forceinline__ void merge_state(SoftState& a, const float* mx2, const float* l2, const float* acc2) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float mn = fmaxf(a.mx[k], mx2[k]);
    float s1 = (a.l[k] == 0.f) ? 0.f : fast_exp2(a.mx[k] - mn);
    float s2 = (l2[k] == 0.f) ? 0.f : fast_exp2(mx2[k] - mn);
    a.l[k] = a.l[k] * s1 + l2[k] * s2;
    a.acc[k] = a.acc[k] * s1 + acc2[k] * s2;
    a.mx[k] = (a.l[k] == 0.f) ? neg_inf() : mn;
  }
}

// grid: x over (entry, 8-channel vector, token group) units; y over sequences.
__global__ void __launch_bounds__(256) compress_kernel(
    const bf16* __restrict__ cand, int ld_cand, const bf16* __restrict__ logits, int ld_logits,
    const float* __restrict__ bias, int ld_bias, int T, int c, int rate, int overlap,
    int n_entries, long long seq_in, bf16* __restrict__ out, int ld_out, long long seq_out,
    int tg_log2, int toks_per_group, float* __restrict__ out_f32) {
  const int TG = 1 << tg_log2;
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int grp = (int)(gtid & (TG - 1));
  const long long unit = gtid >> tg_log2;
  const int vpr = c >> 3;
  const bool valid = unit < (long long)n_entries * vpr;
  const int i = valid ? (int)(unit / vpr) : 0;
  const int j0 = valid ? (int)(unit % vpr) * 8 : 0;
  const long long b = blockIdx.y;
  cand += b * seq_in;
  logits += b * seq_in;
  if (out_f32) out_f32 += b * seq_out;
  else out += b * seq_out;

  SoftState st;
#pragma unroll
  for (int k = 0; k < 8; ++k) { st.mx[k] = neg_inf(); st.l[k] = 0.f; st.acc[k] = 0.f; }

  if (valid) {
    // window [lo, hi) and the bias row of token lo
    int lo, hi, brow0;
    if (overlap) {
      lo = (i - 1) * rate; brow0 = 0;
      if (lo < 0) { lo = 0; brow0 = rate; }
      hi = (i + 1) * rate;
    } else {
      lo = i * rate; hi = lo + rate; brow0 = 0;
    }
    if (hi > T) hi = T;
    const int r0 = lo + grp * toks_per_group;
    int r1 = r0 + toks_per_group;
    if (r1 > hi) r1 = hi;
    for (int r = r0; r < r1; ++r) {
      const uint4 cv = *reinterpret_cast<const uint4*>(cand + (long long)r * ld_cand + j0);
      const uint4 zv = *reinterpret_cast<const uint4*>(logits + (long long)r * ld_logits + j0);
      const float* bp = bias + (long long)(brow0 + r - lo) * ld_bias + j0;
      const float4 b0 = *reinterpret_cast<const float4*>(bp);
      const float4 b1 = *reinterpret_cast<const float4*>(bp + 4);
      float cf[8], zf[8];
      unpack8(cv, cf);
      unpack8(zv, zf);
      const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float z = (zf[k] + bb[k]) * kLog2e;  // base-2 logits
        const float mn = fmaxf(st.mx[k], z);
        const float a = fast_exp2(st.mx[k] - mn);  // 0 when mx = -inf
        const float e = fast_exp2(z - mn);
        st.l[k] = st.l[k] * a + e;
        st.acc[k] = st.acc[k] * a + e * cf[k];
        st.mx[k] = mn;
      }
    }
  }
  // merge token groups (lanes grp ^ off belong to the same unit)
  for (int off = 1; off < TG; off <<= 1) {
    float mx2[8], l2[8], acc2[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      mx2[k] = __shfl_xor_sync(0xffffffffu, st.mx[k], off);
      l2[k] = __shfl_xor_sync(0xffffffffu, st.l[k], off);
      acc2[k] = __shfl_xor_sync(0xffffffffu, st.acc[k], off);
    }
    merge_state(st, mx2, l2, acc2);
  }
  if (valid && grp == 0) {
    float o[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = st.acc[k] / st.l[k];
    if (out_f32) {  // handed on, unrounded, to the Q/KV normalisation
      float4* d = reinterpret_cast<float4*>(out_f32 + (long long)i * ld_out + j0);
      d[0] = make_float4(o[0], o[1], o[2], o[3]);
      d[1] = make_float4(o[4], o[5], o[6], o[7]);
      return;
    }
    uint4 w;
    w.x = pack_bf16x2(o[0], o[1]);
    w.y = pack_bf16x2(o[2], o[3]);
    w.z = pack_bf16x2(o[4], o[5]);
    w.w = pack_bf16x2(o[6], o[7]);
    *reinterpret_cast<uint4*>(out + (long long)i * ld_out + j0) = w;
  }
}

cudaError_t launch_compress(const bf16* cand, int ld_cand, const bf16* logits, int ld_logits,
                            const float* bias, int ld_bias, int B, long long seq_in, int T, int c,
                            int rate, bool overlap, bf16* out, int ld_out, long long seq_out,
                            cudaStream_t stream, float* out_f32) {
  const int n_entries = T / rate;
  if (n_entries == 0 || B == 0) return cudaSuccess;
  const int window = overlap ? 2 * rate : rate;
  // Aim for <= 8 tokens per thread; TG a power of two <= 32.
  int tg_log2 = 0;
  while ((1 << tg_log2) < 32 && (window + (1 << tg_log2) - 1) / (1 << tg_log2) > 8) ++tg_log2;
  const int TG = 1 << tg_log2;
  const int per = (window + TG - 1) / TG;
  const long long threads = (long long)n_entries * (c / 8) * TG;
  const int block = 256;
  const long long grid = (threads + block - 1) / block;
  dim3 g((unsigned)grid, (unsigned)B);
  compress_kernel<<<g, block, 0, stream>>>(cand, ld_cand, logits, ld_logits, bias, ld_bias, T, c,
                                           rate, overlap ? 1 : 0, n_entries, seq_in, out, ld_out,
                                           seq_out, tg_log2, per, out_f32);
  ++g_launch_counter;
  return cudaGetLastError();
}

// Row b of src [B][c] (bf16) into its paged pool row:
// pool + (bt[b*bt_stride + entry / rpb] * rpb + entry % rpb) * c.
__global__ void __launch_bounds__(64) scatter_rows_kernel(const bf16* __restrict__ src, int c,
                                                          const int32_t* __restrict__ bt, long long bt_stride,
                                                          int entry, int rpb, bf16* __restrict__ pool) {
  const long long b = blockIdx.x;
  const long long row = (long long)bt[b * bt_stride + entry / rpb] * rpb + entry % rpb;
  for (int j = threadIdx.x * 8; j < c; j += blockDim.x * 8)
    *reinterpret_cast<uint4*>(pool + row * c + j) = *reinterpret_cast<const uint4*>(src + b * c + j);
}

cudaError_t launch_scatter_rows(const bf16* src, int B, int c, const int32_t* bt, long long bt_stride, int entry,
                                int rpb, bf16* pool, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  scatter_rows_kernel<<<B, 64, 0, stream>>>(src, c, bt, bt_stride, entry, rpb, pool);
  ++g_launch_counter;
  return cudaGetLastError();
}

}  // namespace hca
