"""Edge shapes of the tensor-core paths at the PRO shape: very short prefills (no
compressed entry at all, one partial indexer tile, a handful of HCA blocks) with
both layers -- the HCA layer's dense prefill attention included -- checked on every
query, and a decode step of a single request (the one-request tensor-map strides)."""

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import assert_bf16_close, assert_norm_close, check_topk_row, to64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hca():
    import long_context_attention_compress_b200 as h
    return h


@pytest.mark.parametrize("T", [1, 130, 515])
def test_prefill_pro_shape_short_both_layers(hca, T):
    s = wl.PRO
    d = wl.prefill_inputs(s, T=T, seed=T)
    g = to_dev(d)
    dev = "cuda"
    Nc, Nh = T // s.m, T // s.m_hca
    csa_kv = torch.empty((max(Nc, 1), s.c), dtype=torch.bfloat16, device=dev)
    csa_k = torch.empty((max(Nc, 1), s.d_idx), dtype=torch.bfloat16, device=dev)
    topk = torch.empty((T, s.topk), dtype=torch.int32, device=dev)
    csa_out = torch.empty((T, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    hca_kv = torch.empty((max(Nh, 1), s.c), dtype=torch.bfloat16, device=dev)
    hca_out = torch.empty_like(csa_out)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_prefill_args(g, csa_kv, csa_k, topk, csa_out, hca_kv=hca_kv, hca_q=g["q"],
                                       hca_out=hca_out)
    hca.hybrid_attn_prefill(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    n = {k: (to64(v) if v.is_floating_point() else v.numpy()) for k, v in d.items()}
    res = oracle.csa_layer_prefill(n["cand"], n["logits"], n["kidx_cand"], n["bias_csa"], n["q_idx"], n["w_idx"],
                                   n["q"], m=s.m, topk=s.topk, d_idx=s.d_idx, n_win=s.n_win, scale=s.scale)
    if Nc:
        assert_bf16_close(to64(csa_kv[:Nc]), oracle.csa_compress(n["cand"], n["logits"], n["bias_csa"], s.m), "E")
    ti = topk.cpu().numpy()
    for t in range(T):
        check_topk_row(ti[t], res["idx"][t], res["scores"][t], s.topk, res["n_vis"][t])
    assert_norm_close(to64(csa_out), np.stack([res["O"][t] for t in range(T)]), what=f"CSA prefill T={T}")
    hres = oracle.hca_layer_prefill(n["cand"], n["logits"], n["bias_hca"], n["q"], m_hca=s.m_hca, n_win=s.n_win,
                                    scale=s.scale)
    if Nh:
        assert_bf16_close(to64(hca_kv[:Nh]), oracle.hca_compress(n["cand"], n["logits"], n["bias_hca"], s.m_hca),
                          "E_h")
    assert_norm_close(to64(hca_out), np.stack([hres["O"][t] for t in range(T)]), what=f"HCA prefill T={T}")


def test_decode_single_request_both_layers(hca):
    s = wl.PRO
    ctx = 65536
    d = wl.hybrid_decode_inputs(s, B=1, ctx=ctx, seed=21, cache_std=1.0)
    gc, gh = to_dev(d["csa"]), to_dev(d["hca"])
    dev = "cuda"
    idx = torch.empty((1, s.topk), dtype=torch.int32, device=dev)
    co = torch.empty((1, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    ho = torch.empty_like(co)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_decode_args(1, gc["q_pos"], csa=gc, hca=gh, csa_topk_idx=idx, csa_out=co, hca_out=ho)
    hca.hybrid_attn_decode(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    t = ctx - 1
    c, h = d["csa"], d["hca"]
    r = oracle.csa_layer_decode(to64(c["E"][0]), to64(c["K_I"][0]), to64(c["win"][0]), to64(c["q"][0]),
                                to64(c["q_idx"][0]), c["w_idx"][0].double().numpy(), t, m=s.m, topk=s.topk,
                                n_win=s.n_win, scale=s.scale)
    check_topk_row(idx[0].cpu().numpy(), r["idx"], r["scores"], s.topk, r["n_vis"])
    assert_norm_close(to64(co[0]), r["O"], what="single-request CSA decode")
    nv = oracle.n_visible(t, s.m_hca, h["E_h"].shape[1])
    rows = np.concatenate([to64(h["E_h"][0])[:nv], to64(h["win"][0])])
    assert_norm_close(to64(ho[0]), oracle.mqa_attend(to64(h["q"][0]), rows, s.scale), what="single-request HCA decode")
