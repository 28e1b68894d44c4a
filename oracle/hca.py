"""Oracle arithmetic for the hybrid CSA/HCA attention layer (float64 NumPy).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py`` for who may use it).

Everything here is the plain definition, computed one entry / one query at a
time, with no blocking, fusion or reordering beyond what the definition
states.  Sources, by page title and section:

  [Tricks]  "DeepSeek V4 Architecture Tricks" (pinktalk.online), sections
            "CSA: Compressed Sparse Attention", "HCA: Heavily Compressed
            Attention", "压缩 KV 的具体 trick", "Sliding Window Branch".
  [QbitAI]  QbitAI write-up of the V4 report (admirer.cn), section
            "混合注意力機制" (steps one to three of CSA, HCA, the sliding
            window branch and its strict-causality remark).
  [Report]  "[DeepSeek-5] DeepSeek-V4 Technical Report: Hybrid Attention and
            Post-Training for Million-Token Contexts" (xutianle.me),
            section 3 (CSA), section 4 (HCA), section 5 (heterogeneous cache).
  [Jiedu]   "DeepSeek-V4技术报告解读" (yetianai.com), section
            "核心创新一：混合注意力机制（CSA+HCA）".

Readings taken where the pages are silent (each is also listed in the design
notes):
  * Overlapped CSA compression: entry i pools the 2m tokens
    [(i-1)m, (i+1)m); positional-bias rows 0..m-1 go with the previous block,
    rows m..2m-1 with the current block; the same candidate and logit tensors
    serve both halves.  Entry 0 has no previous block: the missing slots are
    left out of the softmax (not zero-padded).
  * A trailing incomplete block produces no entry: N = floor(T / m).
  * Causality: a query at 0-based position t sees compressed entry s iff the
    last token of the entry's block, (s+1)*rate - 1, is <= t.
  * Sliding window: raw tokens [max(0, t-n_win+1), t] (t itself included),
    attended in the same softmax as the compressed entries, even where they
    cover the same tokens.
  * Lightning-indexer score: I(t,s) = sum_j w[t,j] * ReLU(q[t,j,:] . K[s,:]),
    no scale; the pages only say the indexer is the lightweight one inherited
    from DeepSeek-V3.2 ([QbitAI], CSA step two) with 64 heads of dim 128
    ([Tricks], CSA section).
  * Top-k order: score descending, ties by entry index ascending; all visible
    entries when fewer than k are visible.
  * Compressed entries are stored as bf16 (the cache format); the oracle
    rounds its float64 compressor output to bf16 (round-to-nearest-even, via
    float32) before it is attended or indexed.
  * Q/KV normalisation and partial RoPE (optional, ``norm=``): RMSNorm over
    the c channels of every query head and every KV row, with one learned
    weight vector for the queries and one for the KV rows of a layer, eps
    1e-6; RoPE then rotates the last rope_dims (64) channels in adjacent
    pairs (2j, 2j+1) by pos * base^(-2j/rope_dims), base 10000; the
    attention output is rotated back by -t.  A compressed entry sits at the
    position of the last token of its own block, (i+1)*rate - 1; a window row
    at its token's position.  Entries are cached after normalisation and
    rotation (one bf16 rounding); window rows are kept raw (they are the
    compressor's input too) and normalised when attended.  Normalised queries
    and window rows enter the attention as bf16 values, like the entries.
    The indexer is not core attention and is left as it is.
  * FP4 indexer variant: the FP4 format is MXFP4 (E2M1 elements, one
    power-of-two E8M0 scale per 32 consecutive elements along d_I, shared
    exponent floor(log2 amax) - 2, nearest-even rounding saturating at +-6):
    the pages give no format, but say FP4 values dequantise losslessly into
    FP8 because FP8's exponent absorbs the scale -- true for power-of-two
    scales.  Codes are packed two per byte, the even element in the low
    nibble.  Index scores are rounded to BF16.
  * FP8 KV channels: the channels outside the rotary part are stored as
    E4M3 (nearest even, saturating at +-448) with one f32 scale per 64
    channels of a row, scale = group amax / 448; the rotary channels stay
    BF16.  The pages name the split (FP8 / BF16) but no scale convention.
  * Paged cache: a classical block holds the entries of lcm(m, m') raw
    tokens -- lcm/m CSA entries (and their indexer keys) and lcm/m' HCA
    entries -- reached through a per-request block table (logical block j
    covers tokens [j L, (j+1) L)); entry i sits in logical block i // (L/rate),
    slot i % (L/rate).  The state cache keeps the window as a ring of n_win raw
    rows, token tau at slot tau % n_win.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "round_bf16", "softmax", "csa_compress", "hca_compress",
    "compress_weights_csa", "compress_weights_hca", "n_visible",
    "indexer_scores", "topk_select", "window_rows", "mqa_attend",
    "mqa_partial", "combine_partials", "csa_layer_prefill",
    "hca_layer_prefill", "csa_layer_decode", "hca_layer_decode",
    "rms_norm", "rope_theta", "rope", "entry_position", "QKNorm",
    "norm_rope_rows", "attend_norm_rope", "cache_entries",
    "E2M1_GRID", "MX_BLOCK", "e2m1_value", "mxfp4_quantize", "mxfp4_dequantize", "mxfp4_pack",
    "mxfp4_unpack", "indexer_scores_fp4", "topk_recall",
    "classical_block_tokens", "paged_rows", "ring_window", "csa_layer_decode_paged",
    "hca_attend_decode_paged", "round_e4m3", "fp8_kv_quantize", "fp8_kv_dequantize",
]


# ----------------------------------------------------------------------------
# storage format
# ----------------------------------------------------------------------------
def round_bf16(x) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as float64.

    bf16 keeps the top 16 bits of an IEEE float32.  The value is first
    rounded to float32 (NumPy's cast, nearest-even), then the low 16 bits
    are rounded away with ties to even.  Finite inputs only.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def softmax(z: np.ndarray, axis: int) -> np.ndarray:
    """Max-subtracted softmax in float64."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - np.max(z, axis=axis, keepdims=True))
    return e / np.sum(e, axis=axis, keepdims=True)


# ----------------------------------------------------------------------------
# (1) KV compressor  ([Tricks] "压缩 KV 的具体 trick"; [QbitAI] CSA step one,
#     HCA paragraph; [Report] sections 3 and 4)
# ----------------------------------------------------------------------------
def _csa_window(i: int, m: int, T: int):
    """Token range pooled by CSA entry i, and the bias row of its first token."""
    lo = max(0, (i - 1) * m)
    hi = min(T, (i + 1) * m)
    bias_row0 = lo - (i - 1) * m  # m for entry 0 (no previous block), else 0
    return lo, hi, bias_row0


def compress_weights_csa(logits: np.ndarray, pos_bias: np.ndarray, m: int, i: int) -> np.ndarray:
    """Softmax weights [tokens, channels] that CSA entry i puts on its tokens.

    Per channel j: softmax over the tokens r of the window of
    (logit Z[r, j] + positional bias B[r - (i-1)m, j]).
    """
    T = logits.shape[0]
    lo, hi, b0 = _csa_window(i, m, T)
    z = logits[lo:hi] + pos_bias[b0:b0 + (hi - lo)]
    return softmax(z, axis=0)


def csa_compress(cand: np.ndarray, logits: np.ndarray, pos_bias: np.ndarray, m: int) -> np.ndarray:
    """Overlapped CSA compression: [T, c] -> [floor(T/m), c] (float64, unrounded).

    E[i, j] = sum_{r in W(i)} softmax_r(Z[r, j] + B[r - (i-1)m, j]) * C[r, j],
    W(i) = [(i-1)m, (i+1)m) intersected with [0, T).  Each token therefore
    contributes to its own block's entry and to the next one (the overlap
    with the previous adjacent block that [Tricks] describes).
    """
    cand = np.asarray(cand, dtype=np.float64)
    logits = np.asarray(logits, dtype=np.float64)
    pos_bias = np.asarray(pos_bias, dtype=np.float64)
    T, c = cand.shape
    assert logits.shape == (T, c) and pos_bias.shape == (2 * m, c)
    n = T // m
    out = np.zeros((n, c), dtype=np.float64)
    for i in range(n):
        lo, hi, _ = _csa_window(i, m, T)
        w = compress_weights_csa(logits, pos_bias, m, i)
        out[i] = np.sum(w * cand[lo:hi], axis=0)
    return out


def compress_weights_hca(logits: np.ndarray, pos_bias: np.ndarray, m_hca: int, i: int) -> np.ndarray:
    """Softmax weights [m', channels] of HCA entry i (block [i m', (i+1) m'))."""
    lo = i * m_hca
    return softmax(logits[lo:lo + m_hca] + pos_bias, axis=0)


def hca_compress(cand: np.ndarray, logits: np.ndarray, pos_bias: np.ndarray, m_hca: int) -> np.ndarray:
    """HCA compression, no overlap: [T, c] -> [floor(T/m'), c] (float64, unrounded).

    E_h[i, j] = sum_{r in [i m', (i+1) m')} softmax_r(Z[r, j] + B[r - i m', j]) * C[r, j].
    """
    cand = np.asarray(cand, dtype=np.float64)
    logits = np.asarray(logits, dtype=np.float64)
    pos_bias = np.asarray(pos_bias, dtype=np.float64)
    T, c = cand.shape
    assert logits.shape == (T, c) and pos_bias.shape == (m_hca, c)
    n = T // m_hca
    out = np.zeros((n, c), dtype=np.float64)
    for i in range(n):
        w = compress_weights_hca(logits, pos_bias, m_hca, i)
        out[i] = np.sum(w * cand[i * m_hca:(i + 1) * m_hca], axis=0)
    return out


# ----------------------------------------------------------------------------
# (4) causal visibility  ([QbitAI] sliding-window paragraph: compressed
#     attention is strictly causal, a query cannot see its own incomplete block)
# ----------------------------------------------------------------------------
def n_visible(t: int, rate: int, n_entries: int) -> int:
    """Number of compressed entries visible to a query at position t.

    Entry s is visible iff (s+1)*rate - 1 <= t, i.e. s < floor((t+1)/rate);
    the entries visible are therefore always the prefix [0, n_visible).
    """
    return int(min(n_entries, (t + 1) // rate))


def window_rows(t: int, n_win: int) -> np.ndarray:
    """Raw-token positions of the sliding window of a query at t ([Tricks]
    "Sliding Window Branch": the most recent n_win = 128 uncompressed tokens)."""
    return np.arange(max(0, t - n_win + 1), t + 1)


# ----------------------------------------------------------------------------
# (2) lightning indexer and top-k  ([QbitAI] CSA step two; [Tricks] CSA section)
# ----------------------------------------------------------------------------
def indexer_scores(q_idx: np.ndarray, w_idx: np.ndarray, k_idx: np.ndarray) -> np.ndarray:
    """Scores of one query against entries: I(s) = sum_j w[j] * ReLU(q[j,:] . K[s,:]).

    q_idx [H_I, d_I], w_idx [H_I], k_idx [N, d_I] -> [N] float64.
    """
    q = np.asarray(q_idx, dtype=np.float64)
    w = np.asarray(w_idx, dtype=np.float64)
    k = np.asarray(k_idx, dtype=np.float64)
    dots = k @ q.T                      # [N, H_I]: q_j . K_s
    return np.maximum(dots, 0.0) @ w    # sum_j w_j ReLU(.)


def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the min(k, N) largest scores, ordered by (score desc, index asc)."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    order = np.lexsort((np.arange(n), -scores))
    return order[:min(k, n)].astype(np.int64)


# ----------------------------------------------------------------------------
# (3) core multi-query attention with shared K = V  ([QbitAI] CSA step three
#     and the remark that KV entries serve as both key and value; c = 512)
# ----------------------------------------------------------------------------
def mqa_partial(q: np.ndarray, rows: np.ndarray, scale: float):
    """Unnormalised softmax state of MQA over a row set.

    q [H, c], rows [U, c] (each row is key and value) ->
    (m [H], l [H], o [H, c]) with m_h = max_u s_hu, l_h = sum_u exp(s_hu - m_h),
    o_h = sum_u exp(s_hu - m_h) rows_u, s_hu = scale * q_h . rows_u.
    """
    q = np.asarray(q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    s = scale * (q @ rows.T)                       # [H, U]
    mx = np.max(s, axis=1)
    e = np.exp(s - mx[:, None])
    return mx, np.sum(e, axis=1), e @ rows


def mqa_attend(q: np.ndarray, rows: np.ndarray, scale: float, sink=None) -> np.ndarray:
    """o_h = sum_u softmax_u(scale * q_h . rows_u) rows_u; q [H, c], rows [U, c].

    sink [H] (optional): a learnable logit per head added to the softmax
    denominator only, so that the weights of the rows may sum to less than one
    ([QbitAI] "混合注意力機制", attention-sink paragraph; [Tricks] "Partial RoPE
    和 Attention Sink"):  o_h = sum_u e^{s_hu} rows_u / (e^{z_h} + sum_u e^{s_hu}).
    """
    mx, l, o = mqa_partial(q, rows, scale)
    if sink is not None:
        l = l + np.exp(np.asarray(sink, dtype=np.float64) - mx)
    return o / l[:, None]


def combine_partials(parts, sink=None) -> np.ndarray:
    """Merge softmax states of disjoint row subsets:
    o = sum_i e^{m_i - M} o_i / (sum_i e^{m_i - M} l_i [+ e^{z - M}]), M = max_i m_i
    (the sink logit z, if any, enters the denominator once, not per subset)."""
    ms = np.stack([p[0] for p in parts])          # [P, H]
    M = np.max(ms, axis=0)
    num = sum(np.exp(p[0] - M)[:, None] * p[2] for p in parts)
    den = sum(np.exp(p[0] - M) * p[1] for p in parts)
    if sink is not None:
        den = den + np.exp(np.asarray(sink, dtype=np.float64) - M)
    return num / den[:, None]


# ----------------------------------------------------------------------------
# (5) Q/KV RMSNorm, partial RoPE and the output's inverse rotation
#     ([QbitAI] "混合注意力機制": the Q/KV normalisation and partial-RoPE
#     tricks; [Tricks] "Partial RoPE 和 Attention Sink")
# ----------------------------------------------------------------------------
class QKNorm:
    """Parameters of the Q/KV normalisation of one layer: weight vectors
    q_gamma [c] and kv_gamma [c], eps, and the rotary part (the last
    rope_dims channels, frequency base `base`)."""

    def __init__(self, q_gamma, kv_gamma, eps=1e-6, rope_dims=64, base=10000.0):
        self.q_gamma = np.asarray(q_gamma, dtype=np.float64)
        self.kv_gamma = np.asarray(kv_gamma, dtype=np.float64)
        self.eps = float(eps)
        self.rope_dims = int(rope_dims)
        self.base = float(base)


def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def rope_theta(rope_dims: int, base: float) -> np.ndarray:
    """Frequencies of the rotary pairs: theta_j = base^(-2j / rope_dims)."""
    j = np.arange(rope_dims // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * j / rope_dims)


def rope(x: np.ndarray, pos, rope_dims: int, base: float) -> np.ndarray:
    """Rotate the last rope_dims channels of x [..., c] at position(s) pos.

    Pair j of the rotary part, channels (c - rope_dims + 2j, c - rope_dims + 2j + 1),
    turns by the angle pos * theta_j:  (a, b) -> (a cos - b sin, a sin + b cos).
    `pos` is a scalar or broadcasts against x's leading axes.  The other
    channels pass through unchanged."""
    x = np.array(x, dtype=np.float64, copy=True)
    if rope_dims == 0:
        return x
    c = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_theta(rope_dims, base)
    cs, sn = np.cos(ang), np.sin(ang)
    a = x[..., c - rope_dims::2].copy()
    b = x[..., c - rope_dims + 1::2].copy()
    x[..., c - rope_dims::2] = a * cs - b * sn
    x[..., c - rope_dims + 1::2] = a * sn + b * cs
    return x


def entry_position(i, rate: int):
    """Position of compressed entry i: the last token of its own block."""
    return (np.asarray(i) + 1) * rate - 1


def norm_rope_rows(rows: np.ndarray, pos, gamma: np.ndarray, nrm: "QKNorm") -> np.ndarray:
    """RMSNorm with `gamma`, then RoPE at `pos` ([U] or scalar), row by row."""
    return rope(rms_norm(rows, gamma, nrm.eps), pos, nrm.rope_dims, nrm.base)


def attend_norm_rope(q: np.ndarray, t: int, rows: np.ndarray, row_pos, scale: float, nrm: "QKNorm",
                     sink=None, rows_ready=None, bf16_operands: bool = True) -> np.ndarray:
    """Core attention of one query at position t with Q/KV normalisation.

    q [H, c] raw query heads; rows [U, c] raw KV rows at positions row_pos [U]
    (normalised and rotated here), or, for rows already in the cache's form,
    rows_ready [U', c] appended as they are.  The output is rotated back by -t,
    which leaves only relative positions in it (a KV row is both key and value,
    so its own rotation reaches the output).

    bf16_operands: the normalised, rotated queries and rows enter the attention
    as bf16 values, like the cached entries (the pages keep the rotated KV
    channels in BF16 in the cache; bf16 is the attention's operand type).
    False gives the unrounded definition."""
    qn = norm_rope_rows(q, t, nrm.q_gamma, nrm)
    kv = norm_rope_rows(rows, np.asarray(row_pos), nrm.kv_gamma, nrm) if len(rows) else np.zeros((0, q.shape[1]))
    if bf16_operands:
        qn, kv = round_bf16(qn), round_bf16(kv)
    if rows_ready is not None:
        kv = np.concatenate([np.asarray(rows_ready, dtype=np.float64), kv], axis=0)
    o = mqa_attend(qn, kv, scale, sink)
    return rope(o, -t, nrm.rope_dims, nrm.base)


def cache_entries(E_exact: np.ndarray, rate: int, nrm: "QKNorm" = None, first: int = 0) -> np.ndarray:
    """Compressed entries in the cache's form: bf16, after the KV normalisation
    and rotation at their own positions when `nrm` is given (entry indices
    start at `first`)."""
    if nrm is None:
        return round_bf16(E_exact)
    pos = entry_position(np.arange(first, first + E_exact.shape[0]), rate)
    return round_bf16(norm_rope_rows(E_exact, pos, nrm.kv_gamma, nrm))


# ----------------------------------------------------------------------------
# (6) FP4 indexer variant  ([Tricks] "FP4 / FP8 Quantization-Aware Training":
#     the indexer's QK activations are cached, loaded and multiplied in FP4,
#     the index scores are kept in BF16; FP4 values dequantise losslessly into
#     FP8 because FP8's wider exponent absorbs the fine-grained scale)
# ----------------------------------------------------------------------------
# E2M1 magnitudes by 3-bit code (sign in bit 3): 0, 0.5, 1, 1.5, 2, 3, 4, 6.
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MX_BLOCK = 32        # elements sharing one scale
E2M1_EMAX = 2        # exponent of E2M1's largest normal value (6 = 1.5 * 2^2)


def _e2m1_code(y: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code of each value (ties to the even code), saturating at +-6."""
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), 6.0)
    # candidates: the grid points below and above |y|
    hi = np.searchsorted(E2M1_GRID, a, side="left").clip(0, 7)
    lo = (hi - 1).clip(0, 7)
    d_lo = a - E2M1_GRID[lo]
    d_hi = E2M1_GRID[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo)
    neg = (y < 0) & (mag != 0)
    return (mag + 8 * neg).astype(np.uint8)


def e2m1_value(code) -> np.ndarray:
    """Value of E2M1 codes (bit 3 = sign, bits 0-2 index E2M1_GRID)."""
    code = np.asarray(code, dtype=np.int64)
    v = E2M1_GRID[code & 7]
    return np.where(code & 8, -v, v)


def mxfp4_quantize(x: np.ndarray):
    """MXFP4 quantisation along the last axis (length a multiple of 32).

    Each block of 32 elements gets one power-of-two scale 2^X with
    X = floor(log2(max |x|)) - 2, clamped to [-127, 127] (X = -127 for an
    all-zero block), stored as the E8M0 byte X + 127; each element becomes
    the E2M1 code nearest to x / 2^X (ties to even, saturating at +-6).
    Returns (codes uint8 [..., d], scales uint8 [..., d/32])."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    assert d % MX_BLOCK == 0
    xb = x.reshape(x.shape[:-1] + (d // MX_BLOCK, MX_BLOCK))
    amax = np.max(np.abs(xb), axis=-1)
    with np.errstate(divide="ignore"):
        X = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - E2M1_EMAX, -127.0)
    X = np.clip(X, -127, 127)
    codes = _e2m1_code(xb / np.exp2(X)[..., None])
    return codes.reshape(x.shape).astype(np.uint8), (X + 127).astype(np.uint8)


def mxfp4_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Values of MXFP4 data: e2m1_value(code) * 2^(scale - 127), block by block."""
    codes = np.asarray(codes)
    d = codes.shape[-1]
    v = e2m1_value(codes).reshape(codes.shape[:-1] + (d // MX_BLOCK, MX_BLOCK))
    return (v * np.exp2(np.asarray(scales, dtype=np.float64) - 127.0)[..., None]).reshape(codes.shape)


def mxfp4_pack(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte along the last axis: element 2i in the low nibble,
    element 2i+1 in the high nibble (the cache format)."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def mxfp4_unpack(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


def indexer_scores_fp4(q_idx: np.ndarray, w_idx: np.ndarray, k_idx: np.ndarray) -> np.ndarray:
    """Index scores of the FP4 variant: the queries and keys enter as their
    MXFP4 values (quantised along d_I), the score is formed as in
    indexer_scores and kept in BF16 (rounded to nearest even)."""
    qd = mxfp4_dequantize(*mxfp4_quantize(q_idx))
    kd = mxfp4_dequantize(*mxfp4_quantize(k_idx))
    return round_bf16(indexer_scores(qd, w_idx, kd))


def topk_recall(sel: np.ndarray, ref: np.ndarray) -> float:
    """Fraction of the reference selection that `sel` also selects."""
    ref = np.asarray(ref)
    if ref.size == 0:
        return 1.0
    return float(np.intersect1d(np.asarray(sel), ref).size) / float(ref.size)


# ----------------------------------------------------------------------------
# (6b) FP8 storage of the non-rotated KV channels  ([Tricks] "Partial RoPE 和
#      Attention Sink": the RoPE channels stay BF16 in the KV cache, the other
#      KV channels are stored in FP8)
# ----------------------------------------------------------------------------
E4M3_MAX = 448.0
FP8_GROUP = 64       # channels sharing one scale


def round_e4m3(y) -> np.ndarray:
    """Nearest FP8 E4M3 value (ties to even), saturating at +-448.  E4M3 keeps 3
    mantissa bits; normal exponents -6..8, subnormals in steps of 2^-9."""
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), E4M3_MAX)
    with np.errstate(divide="ignore"):
        e = np.where(a > 0, np.floor(np.log2(np.where(a > 0, a, 1.0))), -6.0)
    e = np.maximum(e, -6.0)                     # below 2^-6: the subnormal spacing 2^-9
    step = np.exp2(e - 3.0)
    q = a / step
    fl = np.floor(q)
    frac = q - fl
    up = (frac > 0.5) | ((frac == 0.5) & (fl % 2 == 1))
    r = (fl + up) * step
    return np.where(y < 0, -r, r)


def fp8_kv_quantize(rows: np.ndarray, rope_dims: int):
    """Cache form of KV rows [.., c]: the first c - rope_dims channels in E4M3
    with one f32 scale per FP8_GROUP channels (scale = group amax / 448, 1 for
    an all-zero group), the last rope_dims channels in BF16.
    Returns (fp8 values / scale [.., c-r], scales [.., (c-r)/64], rope part bf16 [.., r])."""
    rows = np.asarray(rows, dtype=np.float64)
    c = rows.shape[-1]
    n = c - rope_dims
    assert n % FP8_GROUP == 0
    body = rows[..., :n].reshape(rows.shape[:-1] + (n // FP8_GROUP, FP8_GROUP))
    amax = np.max(np.abs(body), axis=-1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0).astype(np.float32).astype(np.float64)
    codes = round_e4m3(body / scale[..., None])
    return codes.reshape(rows.shape[:-1] + (n,)), scale, round_bf16(rows[..., n:])


def fp8_kv_dequantize(codes: np.ndarray, scales: np.ndarray, rope_part: np.ndarray) -> np.ndarray:
    """Row values of the FP8 cache form: codes * scale per group, then the BF16 rope part."""
    codes = np.asarray(codes, dtype=np.float64)
    n = codes.shape[-1]
    body = codes.reshape(codes.shape[:-1] + (n // FP8_GROUP, FP8_GROUP)) * np.asarray(scales)[..., None]
    return np.concatenate([body.reshape(codes.shape), np.asarray(rope_part, dtype=np.float64)], axis=-1)


# ----------------------------------------------------------------------------
# (7) paged heterogeneous cache  ([Jiedu] cache layout: a fixed per-request
#     state cache for the sliding window and the uncompressed tail, and a
#     block-allocated classical cache for the compressed entries; [Tricks]
#     "Heterogeneous KV Cache Layout": each classical block covers lcm(m, m')
#     raw tokens)
# ----------------------------------------------------------------------------
def classical_block_tokens(m: int, m_hca: int) -> int:
    """Raw tokens a classical cache block covers: lcm(m, m')."""
    return int(np.lcm(m, m_hca))


def paged_rows(pool: np.ndarray, block_table, idx, rows_per_block: int) -> np.ndarray:
    """Rows of a paged cache: logical row i lives in physical block
    block_table[i // rows_per_block], slot i % rows_per_block.
    pool [P, rows_per_block, width]; idx: logical row indices."""
    idx = np.asarray(idx, dtype=np.int64)
    bt = np.asarray(block_table, dtype=np.int64)
    return np.asarray(pool, dtype=np.float64)[bt[idx // rows_per_block], idx % rows_per_block]


def ring_window(ring: np.ndarray, t: int, n_win: int) -> np.ndarray:
    """Window rows of a query at t from a ring buffer of n_win rows in which
    token tau sits at slot tau % n_win: tokens max(0, t-n_win+1) .. t, oldest first."""
    toks = window_rows(t, n_win)
    return np.asarray(ring, dtype=np.float64)[toks % n_win]


def csa_layer_decode_paged(kv_pool, k_pool, block_table, N, ring, q, q_idx, w_idx, t, *, m, m_hca, topk, n_win,
                           scale, sink=None, norm=None):
    """csa_layer_decode with the cache in its paged form: N entries reached
    through the request's block table (lcm(m, m')/m entry rows per block, the
    keys in a pool of the same blocks) and the window read from the request's
    ring buffer."""
    rpb = classical_block_tokens(m, m_hca) // m
    E = paged_rows(kv_pool, block_table, np.arange(N), rpb)
    K = paged_rows(k_pool, block_table, np.arange(N), rpb)
    return csa_layer_decode(E, K, ring_window(ring, t, n_win), q, q_idx, w_idx, t, m=m, topk=topk, n_win=n_win,
                            scale=scale, sink=sink, norm=norm)


def hca_attend_decode_paged(kv_pool, block_table, N, ring, q, t, *, m, m_hca, n_win, scale, sink=None, norm=None):
    """Dense HCA attention of one decode query with the entries reached through
    the block table (lcm(m, m')/m' rows per block) and the window from the ring."""
    rpb = classical_block_tokens(m, m_hca) // m_hca
    nv = n_visible(t, m_hca, N)
    E = paged_rows(kv_pool, block_table, np.arange(nv), rpb)
    win = ring_window(ring, t, n_win)
    if norm is None:
        return mqa_attend(q, np.concatenate([E, win], axis=0), scale, sink)
    return attend_norm_rope(q, t, win, window_rows(t, n_win), scale, norm, sink, rows_ready=E)


# ----------------------------------------------------------------------------
# whole layers
# ----------------------------------------------------------------------------
def csa_layer_prefill(cand, logits, kidx_cand, pos_bias, q_idx, w_idx, q, *,
                      m, topk, d_idx, n_win, scale, queries=None, sink=None, norm=None):
    """CSA layer over one sequence of T raw tokens, for the given query positions.

    cand/logits [T, c]; kidx_cand [T, d_I] (per-token indexer-key candidates,
    compressed with the same compressor using logits[:, :d_I] and
    pos_bias[:, :d_I]); q_idx [T, H_I, d_I]; w_idx [T, H_I]; q [T, H, c].
    Returns dict with E [N, c] and K_I [N, d_I] (bf16-valued float64), and per
    query: the selected indices (ordered), their scores, the visible count and
    the output o [H, c].  norm (a QKNorm, optional): Q/KV normalisation and
    partial RoPE; E is then the cache form (normalised and rotated).
    """
    T = cand.shape[0]
    E = cache_entries(csa_compress(cand, logits, pos_bias, m), m, norm)
    K_I = round_bf16(csa_compress(kidx_cand, np.asarray(logits)[:, :d_idx],
                                  np.asarray(pos_bias)[:, :d_idx], m))
    N = E.shape[0]
    qs = range(T) if queries is None else queries
    res = {"E": E, "K_I": K_I, "idx": {}, "scores": {}, "n_vis": {}, "O": {}}
    cand64 = np.asarray(cand, dtype=np.float64)
    for t in qs:
        nv = n_visible(t, m, N)
        sc = indexer_scores(q_idx[t], w_idx[t], K_I[:nv])
        sel = topk_select(sc, topk)
        wr = window_rows(t, n_win)
        res["idx"][t] = sel
        res["scores"][t] = sc
        res["n_vis"][t] = nv
        if norm is None:
            rows = np.concatenate([E[sel], cand64[wr]], axis=0)
            res["O"][t] = mqa_attend(q[t], rows, scale, sink)
        else:
            res["O"][t] = attend_norm_rope(q[t], t, cand64[wr], wr, scale, norm, sink, rows_ready=E[sel])
    return res


def hca_layer_prefill(cand, logits, pos_bias, q, *, m_hca, n_win, scale, queries=None, sink=None, norm=None):
    """HCA layer over one sequence: dense attention over every visible HCA
    entry plus the sliding window ([Tricks] HCA section: no top-k selector).
    norm: as in csa_layer_prefill."""
    T = cand.shape[0]
    E = cache_entries(hca_compress(cand, logits, pos_bias, m_hca), m_hca, norm)
    N = E.shape[0]
    qs = range(T) if queries is None else queries
    cand64 = np.asarray(cand, dtype=np.float64)
    res = {"E": E, "n_vis": {}, "O": {}}
    for t in qs:
        nv = n_visible(t, m_hca, N)
        wr = window_rows(t, n_win)
        res["n_vis"][t] = nv
        if norm is None:
            rows = np.concatenate([E[:nv], cand64[wr]], axis=0)
            res["O"][t] = mqa_attend(q[t], rows, scale, sink)
        else:
            res["O"][t] = attend_norm_rope(q[t], t, cand64[wr], wr, scale, norm, sink, rows_ready=E[:nv])
    return res


def csa_layer_decode(E, K_I, win, q, q_idx, w_idx, t, *, m, topk, n_win, scale, sink=None, norm=None):
    """One decode query of one request against its CSA cache.

    E [N, c] compressed entries (the cache's form), K_I [N, d_I] indexer keys,
    win [n_win, c] the raw rows of the last min(n_win, t+1) tokens (first rows
    valid; oldest first, which matters only with `norm`), q [H, c],
    q_idx [H_I, d_I], w_idx [H_I].
    """
    nv = n_visible(t, m, E.shape[0])
    sc = indexer_scores(q_idx, w_idx, K_I[:nv])
    sel = topk_select(sc, topk)
    nw = min(n_win, t + 1)
    E64, win64 = np.asarray(E, dtype=np.float64), np.asarray(win, dtype=np.float64)
    if norm is None:
        O = mqa_attend(q, np.concatenate([E64[sel], win64[:nw]], axis=0), scale, sink)
    else:
        O = attend_norm_rope(q, t, win64[:nw], window_rows(t, n_win), scale, norm, sink, rows_ready=E64[sel])
    return {"idx": sel, "scores": sc, "n_vis": nv, "O": O}


def hca_layer_decode(E_h, block_cand, block_logits, pos_bias, win, q, t, *, m_hca, n_win, scale, sink=None,
                     norm=None):
    """One decode query of one request against its HCA cache, including the
    compression of the newest complete block ([Report] section 5 and [Jiedu]
    cache layout: the tail block is kept raw until it completes).

    E_h [N_h, c] holds entries 0..n-2 where n = floor((t+1)/m') is the number
    of complete blocks; block_cand/block_logits [m', c] are the raw rows of the
    newest complete block (tokens [(n-1) m', n m')), whose entry n-1 is
    computed here.  Returns the new entry and o [H, c].
    """
    n = (t + 1) // m_hca
    assert (t + 1) % m_hca == 0, "the newest block completes at t"
    new = cache_entries(hca_compress(block_cand, block_logits, pos_bias, m_hca), m_hca, norm, first=n - 1)
    Eh = np.concatenate([np.asarray(E_h, dtype=np.float64)[:n - 1], new], axis=0)
    nw = min(n_win, t + 1)
    win64 = np.asarray(win, dtype=np.float64)
    if norm is None:
        O = mqa_attend(q, np.concatenate([Eh, win64[:nw]], axis=0), scale, sink)
    else:
        O = attend_norm_rope(q, t, win64[:nw], window_rows(t, n_win), scale, norm, sink, rows_ready=Eh)
    return {"new_entry": new[0], "O": O}
