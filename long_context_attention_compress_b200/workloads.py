"""Seeded synthetic inputs for the hybrid CSA/HCA attention layer.

This module only draws random tensors of the right shapes and distributions;
it holds none of the layer's arithmetic.  Both the CUDA path and the CPU
oracle are fed from here.

Shapes follow the DeepSeek-V4-Pro attention hyper-parameters the write-ups
give ("DeepSeek V4 Architecture Tricks", CSA / HCA / Sliding Window sections:
m = 4, m' = 128, top-k = 1024, 64 indexer heads of dim 128, n_win = 128; the
QbitAI write-up, CSA step four: head dim c = 512), plus a tiny shape for
checks that a CPU reference finishes in seconds.

Distributions (all bf16 unless noted; per-request seeds are ``seed + b``):
  * raw per-token KV candidates, weight logits, indexer-key candidates,
    queries and indexer queries: N(0, 1);
  * indexer head weights: U(0, 1), float32;
  * compressor positional bias: N(0, 0.1), float32;
  * decode caches: N(0, 1) scaled by ``cache_std`` (1/sqrt(512) for the CSA
    and HCA decode workloads, 1 for the hybrid 1M-context workload); window
    rows use the cache's distribution.
Tensors are generated on the CPU with ``torch.Generator`` by default; the
benchmark may pass ``device='cuda'`` to draw the same recipe with the CUDA
generator (different numbers, same distributions).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LayerShape:
    """Hyper-parameters of one attention layer (c: KV/head dim, m: CSA rate,
    m_hca: HCA rate, topk: CSA selection size, n_idx_heads x d_idx: indexer
    heads, n_heads: query heads sharing one KV, n_win: sliding window;
    rope_dims / rope_base / norm_eps: the rotary part, its frequency base and
    the RMSNorm epsilon of the optional Q/KV normalisation)."""
    c: int
    m: int
    m_hca: int
    topk: int
    n_idx_heads: int
    d_idx: int
    n_heads: int
    n_win: int
    rope_dims: int = 64
    rope_base: float = 10000.0
    norm_eps: float = 1e-6

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.c)


TINY = LayerShape(c=64, m=4, m_hca=32, topk=64, n_idx_heads=4, d_idx=32, n_heads=4, n_win=32, rope_dims=16)
PRO = LayerShape(c=512, m=4, m_hca=128, topk=1024, n_idx_heads=64, d_idx=128, n_heads=64, n_win=128)


def _gen(seed: int, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(g, shape, std=1.0, device="cpu", dtype=torch.bfloat16, chunk_rows=None):
    """N(0, std) drawn in float32 and cast; large tensors are drawn in row chunks."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=dtype, device=device)
    rows = shape[0]
    per_row = max(1, math.prod(shape[1:]))
    if chunk_rows is None:
        chunk_rows = max(1, (1 << 26) // per_row)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = torch.randn((r1 - r0,) + shape[1:], generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[r0:r1] = x.to(dtype)
    return out


def _uniform(g, shape, device="cpu"):
    return torch.rand(tuple(shape), generator=g, device=device, dtype=torch.float32)


def prefill_inputs(shape: LayerShape, T: int, seed: int = 0, device: str = "cpu", with_hca: bool = True):
    """Raw inputs of one sequence of T tokens for a CSA layer (and an HCA layer).

    Returns a dict: cand [T,c], logits [T,c], kidx_cand [T,d_I] (per-token
    indexer-key candidates), q_idx [T,H_I,d_I], w_idx [T,H_I] f32, q [T,H,c],
    bias_csa [2m,c] f32, bias_hca [m',c] f32 (if with_hca), q_pos [T] int32.
    """
    g = _gen(seed, device)
    d = {}
    d["cand"] = _normal(g, (T, shape.c), device=device)
    d["logits"] = _normal(g, (T, shape.c), device=device)
    d["kidx_cand"] = _normal(g, (T, shape.d_idx), device=device)
    d["q_idx"] = _normal(g, (T, shape.n_idx_heads, shape.d_idx), device=device)
    d["w_idx"] = _uniform(g, (T, shape.n_idx_heads), device=device)
    d["q"] = _normal(g, (T, shape.n_heads, shape.c), device=device)
    d["bias_csa"] = _normal(g, (2 * shape.m, shape.c), std=0.1, device=device, dtype=torch.float32)
    if with_hca:
        d["bias_hca"] = _normal(g, (shape.m_hca, shape.c), std=0.1, device=device, dtype=torch.float32)
    d["q_pos"] = torch.arange(T, dtype=torch.int32, device=device)
    return d


def norm_weights(shape: LayerShape, seed: int = 0, device: str = "cpu") -> torch.Tensor:
    """Synthetic Q/KV normalisation weights of one layer: [2, c] float32 (row 0
    for the queries, row 1 for the KV rows), U(0.5, 1.5)."""
    g = _gen(seed + 424_243, device)
    return 0.5 + _uniform(g, (2, shape.c), device=device)


def csa_decode_inputs(shape: LayerShape, B: int, ctx: int, seed: int = 0, cache_std: float = 1.0,
                      device: str = "cpu"):
    """B decode requests, one query each at position ctx-1, against a CSA cache
    of N = ctx // m compressed entries.

    Returns E [B,N,c], K_I [B,N,d_I], win [B,n_win,c], q [B,H,c],
    q_idx [B,H_I,d_I], w_idx [B,H_I] f32, q_pos [B] int32.
    """
    N = ctx // shape.m
    E = torch.empty((B, N, shape.c), dtype=torch.bfloat16, device=device)
    K = torch.empty((B, N, shape.d_idx), dtype=torch.bfloat16, device=device)
    win = torch.empty((B, shape.n_win, shape.c), dtype=torch.bfloat16, device=device)
    q = torch.empty((B, shape.n_heads, shape.c), dtype=torch.bfloat16, device=device)
    qi = torch.empty((B, shape.n_idx_heads, shape.d_idx), dtype=torch.bfloat16, device=device)
    wi = torch.empty((B, shape.n_idx_heads), dtype=torch.float32, device=device)
    for b in range(B):
        g = _gen(seed + b, device)
        E[b] = _normal(g, (N, shape.c), std=cache_std, device=device)
        K[b] = _normal(g, (N, shape.d_idx), device=device)
        win[b] = _normal(g, (shape.n_win, shape.c), std=cache_std, device=device)
        q[b] = _normal(g, (shape.n_heads, shape.c), device=device)
        qi[b] = _normal(g, (shape.n_idx_heads, shape.d_idx), device=device)
        wi[b] = _uniform(g, (shape.n_idx_heads,), device=device)
    q_pos = torch.full((B,), ctx - 1, dtype=torch.int32, device=device)
    return {"E": E, "K_I": K, "win": win, "q": q, "q_idx": qi, "w_idx": wi, "q_pos": q_pos}


def hca_decode_inputs(shape: LayerShape, B: int, ctx: int, seed: int = 0, cache_std: float = 1.0,
                      device: str = "cpu", with_block: bool = True):
    """B decode requests at position ctx-1 against an HCA cache of
    N_h = ctx // m' entries.

    With ``with_block`` the newest complete block is given raw
    (block_cand / block_logits [B,m',c], shared positional bias [m',c] f32)
    and row N_h-1 of E_h is left zero for the compressor to fill; otherwise
    every row of E_h is drawn.  Also win [B,n_win,c], q [B,H,c], q_pos [B].
    """
    Nh = ctx // shape.m_hca
    Eh = torch.zeros((B, Nh, shape.c), dtype=torch.bfloat16, device=device)
    win = torch.empty((B, shape.n_win, shape.c), dtype=torch.bfloat16, device=device)
    q = torch.empty((B, shape.n_heads, shape.c), dtype=torch.bfloat16, device=device)
    out = {}
    if with_block:
        bc = torch.empty((B, shape.m_hca, shape.c), dtype=torch.bfloat16, device=device)
        bl = torch.empty((B, shape.m_hca, shape.c), dtype=torch.bfloat16, device=device)
    for b in range(B):
        g = _gen(seed + b, device)
        n_drawn = Nh - 1 if with_block else Nh
        Eh[b, :n_drawn] = _normal(g, (n_drawn, shape.c), std=cache_std, device=device)
        win[b] = _normal(g, (shape.n_win, shape.c), std=cache_std, device=device)
        q[b] = _normal(g, (shape.n_heads, shape.c), device=device)
        if with_block:
            bc[b] = _normal(g, (shape.m_hca, shape.c), std=cache_std, device=device)
            bl[b] = _normal(g, (shape.m_hca, shape.c), device=device)
    if with_block:
        gb = _gen(seed + 1_000_003, device)
        out["bias_hca"] = _normal(gb, (shape.m_hca, shape.c), std=0.1, device=device, dtype=torch.float32)
        out["block_cand"] = bc
        out["block_logits"] = bl
    out.update({"E_h": Eh, "win": win, "q": q,
                "q_pos": torch.full((B,), ctx - 1, dtype=torch.int32, device=device)})
    return out


def hybrid_decode_inputs(shape: LayerShape, B: int, ctx: int, seed: int = 0, cache_std: float = 1.0,
                         device: str = "cpu"):
    """A CSA layer and an HCA layer decoded back to back for B requests at
    position ctx-1 (independently seeded queries, caches and windows)."""
    csa = csa_decode_inputs(shape, B, ctx, seed=seed, cache_std=cache_std, device=device)
    hca = hca_decode_inputs(shape, B, ctx, seed=seed + 7919, cache_std=cache_std, device=device,
                            with_block=False)
    return {"csa": csa, "hca": hca}


# The five workloads, by what they are.
WORKLOADS = {
    "tiny_prefill_1k": dict(shape=TINY, kind="prefill", T=1024, seed=0),
    "csa_decode_b32_128k": dict(shape=PRO, kind="csa_decode", B=32, ctx=131072, seed=0,
                                cache_std=1.0 / math.sqrt(512)),
    "hca_decode_b16_1m": dict(shape=PRO, kind="hca_decode", B=16, ctx=1048576, seed=0,
                              cache_std=1.0 / math.sqrt(512)),
    "csa_prefill_64k": dict(shape=PRO, kind="prefill", T=65536, seed=0),
    "hybrid_decode_b8_1m": dict(shape=PRO, kind="hybrid_decode", B=8, ctx=1048576, seed=0,
                                cache_std=1.0),
}
