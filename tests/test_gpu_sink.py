"""Attention sink (one learnable logit per head in the softmax denominator) on every
path where it enters: the tensor-core kernel's epilogue (a prefill query on one CTA),
the combine of split decode queries, the CUDA-core kernel (the tiny shape), and the
hybrid decode whose HCA layer runs on the side stream.  Against the oracle, which
adds exp(sink) to the denominator once per query.  Errors are normalised per
(query, head): a sink gives each head its own output scale, so one RMS per query
would let the bf16 rounding of its largest heads alone decide the verdict."""

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import assert_norm_close_per_head, check_topk_row, to64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hca():
    import long_context_attention_compress_b200 as h
    return h


def _sinks(H, seed, lo, hi):
    """Seeded per-head sink logits, uniform in [lo, hi): from a negligible share of
    the attention mass to most of it (the rows' logits here are O(1), over ~10^3 rows)."""
    g = torch.Generator().manual_seed(seed)
    return (lo + (hi - lo) * torch.rand(H, generator=g, dtype=torch.float64)).float()


def test_sparse_mqa_decode_split_with_sink(hca):
    """PRO shape, each query split over CTAs: the sink joins in the combine."""
    s = wl.PRO
    d = wl.csa_decode_inputs(s, B=4, ctx=4 * 16384, seed=13)
    g = to_dev(d)
    cfg = hca.make_cfg(s)
    N = d["E"].shape[1]
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(N, s.topk, replace=False) for _ in range(4)]).astype(np.int32)
    sink = _sinks(s.n_heads, 1, 0.0, 9.0)
    o = hca.sparse_mqa_attend(g["q"], g["E"], g["win"], g["q_pos"], cfg, idx=torch.from_numpy(idx).cuda(),
                              mode=hca.HCA_MODE_DECODE, sink=sink.cuda())
    torch.cuda.synchronize()
    for b in range(4):
        rows = np.concatenate([to64(d["E"][b])[idx[b]], to64(d["win"][b])])
        ref = oracle.mqa_attend(to64(d["q"][b]), rows, s.scale, sink.double().numpy())
        assert_norm_close_per_head(to64(o[b]), ref, what=f"split decode with sink, request {b}")
    # the sink does change the output (it is not silently ignored)
    o0 = hca.sparse_mqa_attend(g["q"], g["E"], g["win"], g["q_pos"], cfg, idx=torch.from_numpy(idx).cuda(),
                               mode=hca.HCA_MODE_DECODE)
    torch.cuda.synchronize()
    assert float((o.float() - o0.float()).abs().max()) > 0.1 * float(o0.float().abs().max())


class _Rows:
    """Float64 view of a bf16 tensor's rows, converted one row at a time."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, i):
        return self.t[i].float().numpy().astype(np.float64)


def test_prefill_pro_shape_with_sink(hca):
    """PRO shape prefill (one CTA per query on the tensor cores): the sink joins in
    the kernel's epilogue."""
    s = wl.PRO
    T = 3001
    d = wl.prefill_inputs(s, T=T, seed=6, with_hca=False)
    g = to_dev(d)
    dev = "cuda"
    Nc = T // s.m
    csa_kv = torch.empty((Nc, s.c), dtype=torch.bfloat16, device=dev)
    csa_k = torch.empty((Nc, s.d_idx), dtype=torch.bfloat16, device=dev)
    topk = torch.empty((T, s.topk), dtype=torch.int32, device=dev)
    out = torch.empty((T, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    sink = _sinks(s.n_heads, 2, -2.0, 8.0)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_prefill_args(g, csa_kv, csa_k, topk, out, csa_sink=sink.cuda())
    hca.hybrid_attn_prefill(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    f = lambda x: x.float().numpy().astype(np.float64)  # noqa: E731
    qs = [0, 1, 5, 127, 128, 1000, 2047, 3000]
    res = oracle.csa_layer_prefill(f(d["cand"]), f(d["logits"]), f(d["kidx_cand"]), f(d["bias_csa"]),
                                   _Rows(d["q_idx"]), d["w_idx"].double().numpy(), _Rows(d["q"]), m=s.m,
                                   topk=s.topk, d_idx=s.d_idx, n_win=s.n_win, scale=s.scale, queries=qs,
                                   sink=sink.double().numpy())
    ti = topk.cpu().numpy()
    o = out.cpu()
    for t in qs:
        check_topk_row(ti[t], res["idx"][t], res["scores"][t], s.topk, res["n_vis"][t])
        assert_norm_close_per_head(to64(o[t]), res["O"][t], what=f"prefill query {t} with sink")


def test_tiny_prefill_both_layers_with_sinks(hca):
    """The tiny shape runs on the CUDA-core attention kernel; both layers get sinks."""
    s = wl.TINY
    T = 1024
    d = wl.prefill_inputs(s, T=T, seed=7)
    g = to_dev(d)
    dev = "cuda"
    Nc, Nh = T // s.m, T // s.m_hca
    csa_kv = torch.empty((Nc, s.c), dtype=torch.bfloat16, device=dev)
    csa_k = torch.empty((Nc, s.d_idx), dtype=torch.bfloat16, device=dev)
    topk = torch.empty((T, s.topk), dtype=torch.int32, device=dev)
    csa_out = torch.empty((T, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    hca_kv = torch.empty((Nh, s.c), dtype=torch.bfloat16, device=dev)
    hca_out = torch.empty_like(csa_out)
    zc, zh = _sinks(s.n_heads, 3, -1.0, 4.0), _sinks(s.n_heads, 4, -1.0, 4.0)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_prefill_args(g, csa_kv, csa_k, topk, csa_out, hca_kv=hca_kv, hca_q=g["q"], hca_out=hca_out,
                                       csa_sink=zc.cuda(), hca_sink=zh.cuda())
    hca.hybrid_attn_prefill(cfg, args)
    torch.cuda.synchronize()
    n = {k: (to64(v) if v.is_floating_point() else v.numpy()) for k, v in d.items()}
    res = oracle.csa_layer_prefill(n["cand"], n["logits"], n["kidx_cand"], n["bias_csa"], n["q_idx"], n["w_idx"],
                                   n["q"], m=s.m, topk=s.topk, d_idx=s.d_idx, n_win=s.n_win, scale=s.scale,
                                   sink=zc.double().numpy())
    ti = topk.cpu().numpy()
    for t in range(T):
        check_topk_row(ti[t], res["idx"][t], res["scores"][t], s.topk, res["n_vis"][t])
    assert_norm_close_per_head(to64(csa_out), np.stack([res["O"][t] for t in range(T)]), what="CSA layer with sink")
    hres = oracle.hca_layer_prefill(n["cand"], n["logits"], n["bias_hca"], n["q"], m_hca=s.m_hca, n_win=s.n_win,
                                    scale=s.scale, sink=zh.double().numpy())
    assert_norm_close_per_head(to64(hca_out), np.stack([hres["O"][t] for t in range(T)]), what="HCA layer with sink")


def test_hybrid_decode_with_sinks(hca):
    """Both layers of a decode step, the HCA layer on the side stream, each with its sinks."""
    s = wl.PRO
    B, ctx = 3, 131072
    d = wl.hybrid_decode_inputs(s, B=B, ctx=ctx, seed=9, cache_std=1.0)
    gc, gh = to_dev(d["csa"]), to_dev(d["hca"])
    dev = "cuda"
    idx = torch.empty((B, s.topk), dtype=torch.int32, device=dev)
    co = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    ho = torch.empty_like(co)
    zc, zh = _sinks(s.n_heads, 5, 0.0, 12.0), _sinks(s.n_heads, 6, 0.0, 12.0)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_decode_args(B, gc["q_pos"], csa=gc, hca=gh, csa_topk_idx=idx, csa_out=co, hca_out=ho,
                                      csa_sink=zc.cuda(), hca_sink=zh.cuda())
    hca.hybrid_attn_decode(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    t = ctx - 1
    idx = idx.cpu().numpy()
    c, h = d["csa"], d["hca"]
    for b in range(B):
        r = oracle.csa_layer_decode(to64(c["E"][b]), to64(c["K_I"][b]), to64(c["win"][b]), to64(c["q"][b]),
                                    to64(c["q_idx"][b]), c["w_idx"][b].double().numpy(), t, m=s.m, topk=s.topk,
                                    n_win=s.n_win, scale=s.scale, sink=zc.double().numpy())
        check_topk_row(idx[b], r["idx"], r["scores"], s.topk, r["n_vis"])
        assert_norm_close_per_head(to64(co[b]), r["O"], what=f"CSA decode with sink, request {b}")
        nv = oracle.n_visible(t, s.m_hca, h["E_h"].shape[1])
        rows = np.concatenate([to64(h["E_h"][b])[:nv], to64(h["win"][b])])
        o = oracle.mqa_attend(to64(h["q"][b]), rows, s.scale, zh.double().numpy())
        assert_norm_close_per_head(to64(ho[b]), o, what=f"HCA decode with sink, request {b}")
