"""Prefill of a CSA layer at the V4-Pro shape (c = 512, 64 heads, 64 x 128
indexer, top-1024, n_win = 128) through hybrid_attn_prefill, against the
oracle on sampled queries: a ragged 3001-token sequence and the full
65,536-token workload (queries at the edges of causality and of the window,
plus a seeded random sample)."""

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import assert_bf16_close, assert_norm_close, check_topk_row, to64, to_dev

pytestmark = pytest.mark.gpu


def _prefill(hca, s, d):
    g = to_dev(d)
    T = d["cand"].shape[0]
    Nc = T // s.m
    dev = "cuda"
    csa_kv = torch.empty((Nc, s.c), dtype=torch.bfloat16, device=dev)
    csa_k = torch.empty((Nc, s.d_idx), dtype=torch.bfloat16, device=dev)
    topk = torch.empty((T, s.topk), dtype=torch.int32, device=dev)
    out = torch.empty((T, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_prefill_args(g, csa_kv, csa_k, topk, out)
    hca.hybrid_attn_prefill(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    return csa_kv, csa_k, topk, out


class _Rows:
    """Float64 view of a bf16 tensor's rows, converted one row at a time."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, i):
        return self.t[i].float().numpy().astype(np.float64)


def _check(s, d, csa_kv, csa_k, topk, out, queries, check_all_entries):
    f = lambda x: x.float().numpy().astype(np.float64)  # noqa: E731
    C, Z, KC, Bc = f(d["cand"]), f(d["logits"]), f(d["kidx_cand"]), f(d["bias_csa"])
    E_ref = oracle.csa_compress(C, Z, Bc, s.m)
    K_ref = oracle.csa_compress(KC, Z[:, :s.d_idx], Bc[:, :s.d_idx], s.m)
    if check_all_entries:
        assert_bf16_close(to64(csa_kv), E_ref, "E")
        assert_bf16_close(to64(csa_k), K_ref, "K_I")
    res = oracle.csa_layer_prefill(C, Z, KC, Bc, _Rows(d["q_idx"]), d["w_idx"].double().numpy(), _Rows(d["q"]),
                                   m=s.m, topk=s.topk, d_idx=s.d_idx, n_win=s.n_win, scale=s.scale,
                                   queries=queries)
    ti = topk.cpu().numpy()
    o = out.cpu()
    for t in queries:
        check_topk_row(ti[t], res["idx"][t], res["scores"][t], s.topk, res["n_vis"][t])
        assert_norm_close(to64(o[t]), res["O"][t], what=f"prefill query {t}")


def test_prefill_pro_shape_ragged(hca=None):
    import long_context_attention_compress_b200 as hca
    s = wl.PRO
    T = 3001
    d = wl.prefill_inputs(s, T=T, seed=5, with_hca=False)
    csa_kv, csa_k, topk, out = _prefill(hca, s, d)
    qs = list(range(0, 8)) + [63, 64, 127, 128, 129, 511, 1000, 2047, 2999, 3000]
    _check(s, d, csa_kv, csa_k, topk, out, qs, check_all_entries=True)


def cfg4_subsample(T=65536):
    """The 1,024-query subsample of the 64K prefill: every 64th position, shifted by
    i mod 4 so that all four queries of a 4-query indexer group occur (t = 64 i + i mod 4),
    plus the edges of causality and of the window and the last query."""
    qs = [64 * i + (i % 4) for i in range(T // 64)]
    return sorted(set(qs + [0, 1, 2, 3, 4, 127, 128, 4095, 4096, 4097, T - 1]))


def test_prefill_64k_sampled():
    import long_context_attention_compress_b200 as hca
    s = wl.PRO
    T = 65536
    d = wl.prefill_inputs(s, T=T, seed=0, with_hca=False)
    csa_kv, csa_k, topk, out = _prefill(hca, s, d)
    rng = np.random.default_rng(0)
    qs = cfg4_subsample(T)
    assert len(qs) >= 1024 and {t % 4 for t in qs} == {0, 1, 2, 3}
    # entries compared on a sample (the float64 compressor over 16,384 entries is checked in full elsewhere)
    _check(s, d, csa_kv, csa_k, topk, out, qs, check_all_entries=False)
    f = lambda x: x.float().numpy().astype(np.float64)  # noqa: E731
    for i in [0, 1, 2, 1023, 1024, 16383] + rng.integers(0, T // s.m, 40).tolist():
        lo = max(0, (i - 1) * s.m)
        ref = oracle.csa_compress(f(d["cand"][lo:(i + 1) * s.m]), f(d["logits"][lo:(i + 1) * s.m]),
                                  f(d["bias_csa"]), s.m)[-1]
        assert_bf16_close(to64(csa_kv[i]), ref, f"entry {i}")


def test_prefill_indexer_long_rows():
    """Prefill-mode indexer + top-k on queries whose visible rows cross 49,152
    entries (the most one on-chip select pass of 32-bit keys holds), up to
    65,536 entries, plus short rows in the same call."""
    import long_context_attention_compress_b200 as hca
    s = wl.PRO
    N = 65536
    g = torch.Generator().manual_seed(77)
    K = torch.randn((N, s.d_idx), generator=g).bfloat16()
    pos = [0, 3, 4 * 1024 - 1, 4 * 1024, 4 * 49152 - 2, 4 * 49152 - 1, 4 * 49152 + 3, 4 * 50000 + 1,
           4 * 60000 + 2, 4 * 65535, 4 * 65536 - 2, 4 * 65536 - 1]
    Tq = len(pos)
    q_idx = torch.randn((Tq, s.n_idx_heads, s.d_idx), generator=g).bfloat16()
    w_idx = torch.rand((Tq, s.n_idx_heads), generator=g)
    q_pos = torch.tensor(pos, dtype=torch.int32)
    cfg = hca.make_cfg(s)
    ti = hca.csa_indexer_topk(q_idx.cuda(), w_idx.cuda(), K.cuda(), q_pos.cuda(), cfg, mode=hca.HCA_MODE_PREFILL)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    ti = ti.cpu().numpy()
    K64 = to64(K)
    for i, t in enumerate(pos):
        nv = oracle.n_visible(t, s.m, N)
        sc = oracle.indexer_scores(to64(q_idx[i]), w_idx[i].double().numpy(), K64[:nv])
        check_topk_row(ti[i], oracle.topk_select(sc, s.topk), sc, s.topk, nv)
