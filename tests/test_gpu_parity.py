"""CUDA path (through the C ABI) against the CPU oracle, on the same seeded inputs.

Sizes: the tiny shape (c=64, 4 heads) over several tiles with ragged tails,
and the full-size decode workloads with the oracle run per request.  The
64K-token prefill is covered in test_gpu_prefill.py on sampled queries.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import (assert_bf16_close, assert_bf16_ulps, assert_norm_close, check_topk_row, to64,
                         to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hca():
    import long_context_attention_compress_b200 as h
    return h


# ----------------------------------------------------------------------------
# compressor
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("T", [0, 3, 4, 37, 1024, 1001])
def test_csa_compress_tiny(hca, T):
    s = wl.TINY
    d = wl.prefill_inputs(s, T=max(T, 1), seed=11)
    d = {k: v[:T] if k in ("cand", "logits", "kidx_cand") else v for k, v in d.items()}
    g = to_dev(d)
    E = hca.csa_compress(g["cand"], g["logits"], g["bias_csa"], s.m)
    torch.cuda.synchronize()
    assert E.shape == (T // s.m, s.c)
    if T // s.m:
        ref = oracle.csa_compress(to64(d["cand"]), to64(d["logits"]), to64(d["bias_csa"]), s.m)
        assert_bf16_close(to64(E), ref, "csa_compress")
        # indexer keys: first d_I channels of logits / bias
        K = hca.csa_compress(g["kidx_cand"], g["logits"], g["bias_csa"], s.m)
        refk = oracle.csa_compress(to64(d["kidx_cand"]), to64(d["logits"])[:, :s.d_idx],
                                   to64(d["bias_csa"])[:, :s.d_idx], s.m)
        assert_bf16_close(to64(K), refk, "indexer-key compress")


@pytest.mark.parametrize("T,m_hca", [(1024, 32), (1001, 32), (31, 32), (384, 128), (100, 1)])
def test_hca_compress_tiny(hca, T, m_hca):
    s = wl.TINY
    d = wl.prefill_inputs(s, T=T, seed=12)
    bias = torch.randn((m_hca, s.c), generator=torch.Generator().manual_seed(5)) * 0.1
    g = to_dev(d)
    E = hca.hca_compress(g["cand"], g["logits"], bias.cuda(), m_hca)
    torch.cuda.synchronize()
    assert E.shape == (T // m_hca, s.c)
    if T // m_hca:
        ref = oracle.hca_compress(to64(d["cand"]), to64(d["logits"]), bias.double().numpy(), m_hca)
        assert_bf16_close(to64(E), ref, "hca_compress")


def test_csa_compress_full_64k_sampled(hca):
    s = wl.PRO
    T = 65536
    g = torch.Generator().manual_seed(0)
    C = torch.randn((T, s.c), generator=g).bfloat16()
    Z = torch.randn((T, s.c), generator=g).bfloat16()
    B = (torch.randn((2 * s.m, s.c), generator=g) * 0.1).float()
    E = hca.csa_compress(C.cuda(), Z.cuda(), B.cuda(), s.m)
    torch.cuda.synchronize()
    E = to64(E)
    rng = np.random.default_rng(0)
    sample = sorted(set([0, 1, 2, T // s.m - 1] + rng.integers(0, T // s.m, 200).tolist()))
    C64, Z64, B64 = to64(C), to64(Z), to64(B)
    for i in sample:
        lo = max(0, (i - 1) * s.m)
        ref = oracle.csa_compress(C64[lo:(i + 1) * s.m], Z64[lo:(i + 1) * s.m], B64, s.m)[-1]
        assert_bf16_close(E[i], ref, f"entry {i}")


# ----------------------------------------------------------------------------
# indexer + top-k
# ----------------------------------------------------------------------------
def _rand_keys(N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((N, d), generator=g).bfloat16()


@pytest.mark.parametrize("T", [1024, 777])
def test_indexer_topk_tiny_prefill(hca, T):
    s = wl.TINY
    d = wl.prefill_inputs(s, T=T, seed=13)
    K = _rand_keys(T // s.m, s.d_idx, 14)
    cfg = hca.make_cfg(s)
    idx = hca.csa_indexer_topk(d["q_idx"].cuda(), d["w_idx"].cuda(), K.cuda(), d["q_pos"].cuda(), cfg)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    K64, q64, w64 = to64(K), to64(d["q_idx"]), d["w_idx"].double().numpy()
    swaps = 0
    for t in range(T):
        nv = oracle.n_visible(t, s.m, K.shape[0])
        sc = oracle.indexer_scores(q64[t], w64[t], K64[:nv])
        sel = oracle.topk_select(sc, s.topk)
        swaps += check_topk_row(idx[t], sel, sc, s.topk, nv)
    assert swaps <= T // 50


def test_indexer_topk_ties_take_lowest_index(hca):
    # all weights zero: every score is 0, the top-k is the k lowest visible indices
    s = wl.TINY
    T = 600
    d = wl.prefill_inputs(s, T=T, seed=15)
    K = _rand_keys(T // s.m, s.d_idx, 16)
    cfg = hca.make_cfg(s)
    idx = hca.csa_indexer_topk(d["q_idx"].cuda(), torch.zeros_like(d["w_idx"]).cuda(), K.cuda(),
                               d["q_pos"].cuda(), cfg).cpu().numpy()
    for t in range(T):
        nv = oracle.n_visible(t, s.m, K.shape[0])
        row = idx[t]
        assert sorted(row[row >= 0].tolist()) == list(range(min(nv, s.topk)))


def test_indexer_topk_decode_csa_128k(hca):
    """Full-size CSA decode indexer: 32 requests x 32768 entries, top-1024."""
    s = wl.PRO
    d = wl.csa_decode_inputs(s, B=32, ctx=131072, seed=0, cache_std=1 / np.sqrt(512))
    g = to_dev(d)
    cfg = hca.make_cfg(s)
    idx = hca.csa_indexer_topk(g["q_idx"], g["w_idx"], g["K_I"], g["q_pos"], cfg, mode=hca.HCA_MODE_DECODE)
    idx = idx.cpu().numpy()
    swaps = 0
    for b in range(32):
        sc = oracle.indexer_scores(to64(d["q_idx"][b]), d["w_idx"][b].double().numpy(), to64(d["K_I"][b]))
        sel = oracle.topk_select(sc, s.topk)
        swaps += check_topk_row(idx[b], sel, sc, s.topk, sc.shape[0])
    assert swaps <= 32 * 8


@pytest.mark.parametrize("N", [40000, 60000])
def test_indexer_topk_decode_threshold_ties(hca, N):
    """Decode top-k when thousands of scores tie at the threshold, for a row that one
    CTA selects from shared memory (40,000 entries) and for the histogram path
    (60,000).  Request 0: every third key is the same vector and the rest are zero,
    so N/3 equal scores compete for the 1024 places (ties go to the lower index).
    Request 1: all keys zero, so all N scores are equal (on the histogram path, more
    threshold candidates than one CTA stages in shared memory).  Request 2: ordinary
    random keys."""
    s = wl.PRO
    d = wl.csa_decode_inputs(s, B=3, ctx=4 * N, seed=11)
    K = d["K_I"].clone()
    assert K.shape[1] == N
    K[0] = 0
    K[0, ::3] = d["K_I"][0, 7]
    K[1] = 0
    d["K_I"] = K
    g = to_dev(d)
    cfg = hca.make_cfg(s)
    idx = hca.csa_indexer_topk(g["q_idx"], g["w_idx"], g["K_I"], g["q_pos"], cfg, mode=hca.HCA_MODE_DECODE)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    idx = idx.cpu().numpy()
    for b in range(3):
        sc = oracle.indexer_scores(to64(d["q_idx"][b]), d["w_idx"][b].double().numpy(), to64(d["K_I"][b]))
        sel = oracle.topk_select(sc, s.topk)
        if b < 2:
            # exactly tied scores: the lower indices win, on both sides
            assert sorted(idx[b].tolist()) == sorted(sel.tolist())
        else:
            check_topk_row(idx[b], sel, sc, s.topk, N)
    assert sorted(idx[0].tolist()) == list(range(0, 3 * s.topk, 3))
    assert sorted(idx[1].tolist()) == list(range(s.topk))


@pytest.mark.parametrize("B,ctx", [(300, 4 * 2048), (5, 4 * 1000 + 3), (7, 4 * 128 * 3 - 1)])
def test_indexer_topk_decode_many_requests_ragged(hca, B, ctx):
    """Many short requests per CTA (the q_I buffer switches mid-range), ragged last tiles,
    and a position whose newest block is still incomplete."""
    s = wl.PRO
    d = wl.csa_decode_inputs(s, B=B, ctx=ctx, seed=B)
    g = to_dev(d)
    cfg = hca.make_cfg(s)
    idx = hca.csa_indexer_topk(g["q_idx"], g["w_idx"], g["K_I"], g["q_pos"], cfg, mode=hca.HCA_MODE_DECODE)
    idx = idx.cpu().numpy()
    N = d["K_I"].shape[1]
    for b in range(B):
        nv = oracle.n_visible(ctx - 1, s.m, N)
        sc = oracle.indexer_scores(to64(d["q_idx"][b]), d["w_idx"][b].double().numpy(), to64(d["K_I"][b])[:nv])
        check_topk_row(idx[b], oracle.topk_select(sc, s.topk), sc, s.topk, nv)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def test_sparse_mqa_tiny_prefill_with_oracle_indices(hca):
    s = wl.TINY
    T = 1024
    d = wl.prefill_inputs(s, T=T, seed=17)
    E = torch.randn((T // s.m, s.c), generator=torch.Generator().manual_seed(18)).bfloat16()
    K = _rand_keys(T // s.m, s.d_idx, 19)
    E64, K64, cand64 = to64(E), to64(K), to64(d["cand"])
    q64, qi64, w64 = to64(d["q"]), to64(d["q_idx"]), d["w_idx"].double().numpy()
    idx = np.full((T, s.topk), -1, dtype=np.int32)
    refs = np.zeros((T, s.n_heads, s.c))
    for t in range(T):
        nv = oracle.n_visible(t, s.m, E.shape[0])
        sel = oracle.topk_select(oracle.indexer_scores(qi64[t], w64[t], K64[:nv]), s.topk)
        idx[t, :len(sel)] = sel[::-1]  # any order
        rows = np.concatenate([E64[sel], cand64[oracle.window_rows(t, s.n_win)]])
        refs[t] = oracle.mqa_attend(q64[t], rows, s.scale)
    cfg = hca.make_cfg(s)
    out = hca.sparse_mqa_attend(d["q"].cuda(), E.cuda(), d["cand"].cuda(), d["q_pos"].cuda(), cfg,
                                idx=torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    assert_norm_close(to64(out), refs, what="sparse MQA tiny")


def test_dense_mqa_tiny_prefill(hca):
    s = wl.TINY
    T = 1001
    d = wl.prefill_inputs(s, T=T, seed=20)
    Nh = T // s.m_hca
    E = torch.randn((Nh, s.c), generator=torch.Generator().manual_seed(21)).bfloat16()
    cfg = hca.make_cfg(s)
    out = hca.sparse_mqa_attend(d["q"].cuda(), E.cuda(), d["cand"].cuda(), d["q_pos"].cuda(), cfg, idx=None)
    torch.cuda.synchronize()
    E64, cand64, q64 = to64(E), to64(d["cand"]), to64(d["q"])
    refs = np.zeros((T, s.n_heads, s.c))
    for t in range(T):
        nv = oracle.n_visible(t, s.m_hca, Nh)
        rows = np.concatenate([E64[:nv], cand64[oracle.window_rows(t, s.n_win)]])
        refs[t] = oracle.mqa_attend(q64[t], rows, s.scale)
    assert_norm_close(to64(out), refs, what="dense MQA tiny")


def test_sparse_mqa_permutation_invariant(hca):
    """Shuffling a query's selected indices leaves the output unchanged (up to f32 order)."""
    s = wl.PRO
    d = wl.csa_decode_inputs(s, B=4, ctx=16384, seed=3)
    g = to_dev(d)
    cfg = hca.make_cfg(s)
    N = d["E"].shape[1]
    rng = np.random.default_rng(0)
    idx = np.stack([rng.choice(N, s.topk, replace=False) for _ in range(4)]).astype(np.int32)
    o1 = hca.sparse_mqa_attend(g["q"], g["E"], g["win"], g["q_pos"], cfg, idx=torch.from_numpy(idx).cuda(),
                               mode=hca.HCA_MODE_DECODE)
    idx2 = np.stack([rng.permutation(r) for r in idx]).astype(np.int32)
    o2 = hca.sparse_mqa_attend(g["q"], g["E"], g["win"], g["q_pos"], cfg, idx=torch.from_numpy(idx2).cuda(),
                               mode=hca.HCA_MODE_DECODE)
    torch.cuda.synchronize()
    # A permutation moves rows between tiles and splits, which changes the f32
    # summation order and which running maximum each probability is rounded
    # against; both orders must meet the parity bar, and agree with each other
    # to one bf16 rounding of the output (a flat softmax over ~1,150 rows moves
    # the output by ~3% of its RMS for a dropped or doubled row, far above the
    # 2^-10 RMS slack for cancelling elements).
    ref = np.stack([oracle.mqa_attend(to64(d["q"][b]),
                                      np.concatenate([to64(d["E"][b])[idx[b]], to64(d["win"][b])]), s.scale)
                    for b in range(4)])
    assert_norm_close(to64(o1), ref, what="sparse MQA decode")
    assert_norm_close(to64(o2), ref, what="sparse MQA decode, permuted")
    assert_bf16_ulps(to64(o1), to64(o2), ulps=1, rms_slack=2.0 ** -10, what="permutation")


def test_mqa_decode_rescale_path(hca):
    """Scores that grow along the row list force the running maximum up by more
    than 2^8 several times inside one split (the lazy rescale of the TMEM
    accumulators), for dense and gathered rows."""
    s = wl.PRO
    B = 3
    d = wl.hca_decode_inputs(s, B=B, ctx=128 * 1024, seed=9, cache_std=1.0, with_block=False)
    ramp = torch.linspace(0.2, 12.0, d["E_h"].shape[1]).reshape(1, -1, 1)
    d["E_h"] = (d["E_h"].float() * ramp).bfloat16()
    idx = hca_idx = None
    g = to_dev(d)
    cfg = hca.make_cfg(s)
    out = hca.sparse_mqa_attend(g["q"], g["E_h"], g["win"], g["q_pos"], cfg, idx=None, rate=s.m_hca,
                                mode=hca.HCA_MODE_DECODE)
    N = d["E_h"].shape[1]
    rng = np.random.default_rng(1)
    idx = np.sort(np.stack([rng.choice(N, 512, replace=False) for _ in range(B)]), axis=1).astype(np.int32)
    out2 = hca.sparse_mqa_attend(g["q"], g["E_h"], g["win"], g["q_pos"], cfg, idx=torch.from_numpy(idx).cuda(),
                                 mode=hca.HCA_MODE_DECODE)
    torch.cuda.synchronize()
    for b in range(B):
        E = to64(d["E_h"][b])
        ref = oracle.mqa_attend(to64(d["q"][b]), np.concatenate([E, to64(d["win"][b])]), s.scale)
        assert_norm_close(to64(out[b]), ref, what=f"dense rescale request {b}")
        ref2 = oracle.mqa_attend(to64(d["q"][b]), np.concatenate([E[idx[b]], to64(d["win"][b])]), s.scale)
        assert_norm_close(to64(out2[b]), ref2, what=f"gathered rescale request {b}")


# ----------------------------------------------------------------------------
# whole layers
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("T", [1024, 1001, 3])
def test_hybrid_prefill_tiny(hca, T):
    s = wl.TINY
    d = wl.prefill_inputs(s, T=T, seed=0)
    g = to_dev(d)
    Nc, Nh = T // s.m, T // s.m_hca
    dev = "cuda"
    csa_kv = torch.empty((Nc, s.c), dtype=torch.bfloat16, device=dev)
    csa_k = torch.empty((Nc, s.d_idx), dtype=torch.bfloat16, device=dev)
    topk = torch.empty((T, s.topk), dtype=torch.int32, device=dev)
    csa_out = torch.empty((T, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    hca_kv = torch.empty((max(Nh, 1), s.c), dtype=torch.bfloat16, device=dev)
    hca_out = torch.empty_like(csa_out)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_prefill_args(g, csa_kv, csa_k, topk, csa_out, hca_kv=hca_kv, hca_q=g["q"],
                                       hca_out=hca_out)
    hca.hybrid_attn_prefill(cfg, args)
    torch.cuda.synchronize()
    n = {k: (to64(v) if v.is_floating_point() else v.numpy()) for k, v in d.items()}
    res = oracle.csa_layer_prefill(n["cand"], n["logits"], n["kidx_cand"], n["bias_csa"], n["q_idx"], n["w_idx"],
                                   n["q"], m=s.m, topk=s.topk, d_idx=s.d_idx, n_win=s.n_win, scale=s.scale)
    if Nc:
        # against the unrounded float64 compressor (res holds the bf16-rounded cache)
        assert_bf16_close(to64(csa_kv), oracle.csa_compress(n["cand"], n["logits"], n["bias_csa"], s.m), "E")
        assert_bf16_close(to64(csa_k), oracle.csa_compress(n["kidx_cand"], n["logits"][:, :s.d_idx],
                                                           n["bias_csa"][:, :s.d_idx], s.m), "K_I")
    ti = topk.cpu().numpy()
    for t in range(T):
        check_topk_row(ti[t], res["idx"][t], res["scores"][t], s.topk, res["n_vis"][t])
    assert_norm_close(to64(csa_out), np.stack([res["O"][t] for t in range(T)]), what="CSA layer output")
    hres = oracle.hca_layer_prefill(n["cand"], n["logits"], n["bias_hca"], n["q"], m_hca=s.m_hca, n_win=s.n_win,
                                    scale=s.scale)
    if Nh:
        assert_bf16_close(to64(hca_kv[:Nh]), oracle.hca_compress(n["cand"], n["logits"], n["bias_hca"], s.m_hca),
                          "E_h")
    assert_norm_close(to64(hca_out), np.stack([hres["O"][t] for t in range(T)]), what="HCA layer output")


def _decode_check(hca, s, csa, hcad, B, ctx, csa_idx_out=None):
    """Oracle check of a hybrid decode's outputs, per request."""
    t = ctx - 1
    if csa is not None:
        idx, out = csa_idx_out
        idx = idx.cpu().numpy()
        outs = to64(out)
        for b in range(B):
            r = oracle.csa_layer_decode(to64(csa["E"][b]), to64(csa["K_I"][b]), to64(csa["win"][b]),
                                        to64(csa["q"][b]), to64(csa["q_idx"][b]), csa["w_idx"][b].double().numpy(),
                                        t, m=s.m, topk=s.topk, n_win=s.n_win, scale=s.scale)
            check_topk_row(idx[b], r["idx"], r["scores"], s.topk, r["n_vis"])
            assert_norm_close(outs[b], r["O"], what=f"CSA decode request {b}")
    if hcad is not None:
        Eh, out = hcad["_gpu_Eh"], hcad["_out"]
        outs = to64(out)
        Eh64 = to64(Eh) if Eh is not None else None
        for b in range(B):
            if "block_cand" in hcad:
                r = oracle.hca_layer_decode(to64(hcad["E_h"][b]), to64(hcad["block_cand"][b]),
                                            to64(hcad["block_logits"][b]), to64(hcad["bias_hca"]),
                                            to64(hcad["win"][b]), to64(hcad["q"][b]), t, m_hca=s.m_hca,
                                            n_win=s.n_win, scale=s.scale)
                new64 = oracle.hca_compress(to64(hcad["block_cand"][b]), to64(hcad["block_logits"][b]),
                                            to64(hcad["bias_hca"]), s.m_hca)[0]
                assert_bf16_close(Eh64[b, -1], new64, f"new HCA entry {b}")
                o = r["O"]
            else:
                rows = np.concatenate([to64(hcad["E_h"][b]), to64(hcad["win"][b])])
                o = oracle.mqa_attend(to64(hcad["q"][b]), rows, s.scale)
            assert_norm_close(outs[b], o, what=f"HCA decode request {b}")


def _run_decode(hca, s, csa, hcad, B):
    dev = "cuda"
    cfg = hca.make_cfg(s)
    gc = to_dev(csa) if csa is not None else None
    gh = to_dev(hcad) if hcad is not None else None
    q_pos = (gc or gh)["q_pos"]
    idx = torch.empty((B, s.topk), dtype=torch.int32, device=dev) if csa is not None else None
    co = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device=dev) if csa is not None else None
    ho = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device=dev) if hcad is not None else None
    args, keep = hca.make_decode_args(B, q_pos, csa=gc, hca=gh, csa_topk_idx=idx, csa_out=co, hca_out=ho)
    hca.hybrid_attn_decode(cfg, args)
    torch.cuda.synchronize()
    return idx, co, (gh["E_h"] if gh is not None else None), ho


def test_csa_decode_b32_128k(hca):
    s = wl.PRO
    csa = wl.csa_decode_inputs(s, B=32, ctx=131072, seed=0, cache_std=1 / np.sqrt(512))
    idx, co, _, _ = _run_decode(hca, s, csa, None, 32)
    _decode_check(hca, s, csa, None, 32, 131072, (idx, co))


def test_hca_decode_b16_1m_with_block_compress(hca):
    s = wl.PRO
    h = wl.hca_decode_inputs(s, B=16, ctx=1048576, seed=0, cache_std=1 / np.sqrt(512))
    _, _, Eh, ho = _run_decode(hca, s, None, h, 16)
    h["_gpu_Eh"], h["_out"] = Eh, ho
    _decode_check(hca, s, None, h, 16, 1048576)


def test_hybrid_decode_b8_1m(hca):
    s = wl.PRO
    d = wl.hybrid_decode_inputs(s, B=8, ctx=1048576, seed=0, cache_std=1.0)
    idx, co, Eh, ho = _run_decode(hca, s, d["csa"], d["hca"], 8)
    d["hca"]["_gpu_Eh"], d["hca"]["_out"] = Eh, ho
    _decode_check(hca, s, d["csa"], d["hca"], 8, 1048576, (idx, co))


def test_decode_short_context_window_partial(hca):
    """Decode at t < n_win (window rows partly empty) and few compressed entries (< topk)."""
    s = wl.PRO
    ctx = 100
    d = wl.hybrid_decode_inputs(s, B=3, ctx=ctx, seed=5, cache_std=1.0)
    # hca cache at ctx=100 has 0 complete blocks: keep one dummy row, the kernel sees none
    d["hca"]["E_h"] = torch.zeros((3, 1, s.c), dtype=torch.bfloat16)
    idx, co, Eh, ho = _run_decode(hca, s, d["csa"], d["hca"], 3)
    t = ctx - 1
    idx = idx.cpu().numpy()
    for b in range(3):
        r = oracle.csa_layer_decode(to64(d["csa"]["E"][b]), to64(d["csa"]["K_I"][b]), to64(d["csa"]["win"][b]),
                                    to64(d["csa"]["q"][b]), to64(d["csa"]["q_idx"][b]),
                                    d["csa"]["w_idx"][b].double().numpy(), t, m=s.m, topk=s.topk, n_win=s.n_win,
                                    scale=s.scale)
        check_topk_row(idx[b], r["idx"], r["scores"], s.topk, r["n_vis"])
        assert_norm_close(to64(co[b]), r["O"], what="short CSA decode")
        o = oracle.mqa_attend(to64(d["hca"]["q"][b]), to64(d["hca"]["win"][b])[:ctx], s.scale)
        assert_norm_close(to64(ho[b]), o, what="short HCA decode (window only)")


def test_no_kernel_gave_up_waiting(hca):
    """After everything above, no kernel recorded an exhausted bounded wait."""
    assert hca.lib.hca_check_device() == 0, hca.last_error()
