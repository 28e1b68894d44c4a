"""GPU parity of the Q/KV RMSNorm + partial RoPE path against the oracle.

QbitAI write-up, "混合注意力機制" (Q/KV normalisation and partial-RoPE tricks);
"DeepSeek V4 Architecture Tricks", "Partial RoPE 和 Attention Sink".  Covered:
the normaliser alone (queries at positions up to 10^6, f32 input, in place,
both channel widths), the attention's output rotation on the tensor-core
path (split and unsplit) and on the CUDA-core path, and both layers with
normalisation in prefill and decode (the HCA entry compressed in the decode
step included).
"""

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


def _qkn(s, w):
    w = w.double().numpy()
    return oracle.QKNorm(w[0], w[1], eps=s.norm_eps, rope_dims=s.rope_dims, base=s.rope_base)


@pytest.mark.parametrize("shape", ["PRO", "TINY"])
def test_norm_rope_queries_at_large_positions(hca, shape):
    s = getattr(wl, shape)
    g = torch.Generator().manual_seed(11)
    Tq = 37
    q = (torch.randn((Tq, s.n_heads, s.c), generator=g) * 3).bfloat16()
    pos = torch.randint(0, 1_048_576, (Tq,), generator=g, dtype=torch.int32)
    pos[:3] = torch.tensor([0, 1, 1_048_575], dtype=torch.int32)
    w = wl.norm_weights(s, seed=1)
    cfg = hca.make_cfg(s)
    y = hca.rms_norm_rope(q.cuda(), w[0].cuda(), cfg, pos=pos.cuda())
    torch.cuda.synchronize()
    nrm = _qkn(s, w)
    ref = np.stack([oracle.norm_rope_rows(to64(q[t]), int(pos[t]), nrm.q_gamma, nrm) for t in range(Tq)])
    assert_bf16_close(to64(y), ref, "normalised queries")


def test_norm_rope_f32_entries_and_in_place(hca):
    s = wl.PRO
    g = torch.Generator().manual_seed(12)
    N, rate = 300, 4
    e = torch.randn((N, s.c), generator=g) * 0.02
    w = wl.norm_weights(s, seed=2)
    cfg = hca.make_cfg(s)
    nrm = _qkn(s, w)
    pos = oracle.entry_position(np.arange(N), rate)
    y = hca.rms_norm_rope(e.cuda(), w[1].cuda(), cfg, pos_add=rate - 1, pos_step=rate)
    ref = oracle.norm_rope_rows(e.double().numpy(), pos, nrm.kv_gamma, nrm)
    # in place on bf16 rows: a decode window block [B, n_win, c] ending at q_pos
    B = 3
    win = (torch.randn((B, s.n_win, s.c), generator=g)).bfloat16()
    qp = torch.tensor([5, 127, 900_000], dtype=torch.int32)
    wd = win.cuda()
    hca.rms_norm_rope(wd, w[1].cuda(), cfg, pos=qp.cuda(), pos_add=-(s.n_win - 1), pos_step=1, out=wd)
    torch.cuda.synchronize()
    assert_bf16_close(to64(y), ref, "normalised f32 entries")
    for b in range(B):
        wp = max(0, int(qp[b]) - s.n_win + 1) + np.arange(s.n_win)
        assert_bf16_close(to64(wd[b]), oracle.norm_rope_rows(to64(win[b]), wp, nrm.kv_gamma, nrm), f"window {b}")


@pytest.mark.parametrize("case", ["tc_decode_split", "tc_prefill", "cuda_cores_decode_split"])
def test_attention_output_rotation(hca, case):
    s = wl.TINY if case.startswith("cuda") else wl.PRO
    g = torch.Generator().manual_seed(13)
    cfg = hca.make_cfg(s)
    if case == "tc_prefill":
        T = 300
        q = torch.randn((T, s.n_heads, s.c), generator=g).bfloat16()
        raw = torch.randn((T, s.c), generator=g).bfloat16()
        N = T // s.m_hca
        E = torch.randn((N, s.c), generator=g).bfloat16()
        qp = torch.arange(T, dtype=torch.int32)
        out = hca.sparse_mqa_attend(q.cuda(), E.cuda(), raw.cuda(), qp.cuda(), cfg, rate=s.m_hca,
                                    mode=hca.HCA_MODE_PREFILL, rotate_out=True)
        torch.cuda.synchronize()
        for t in range(0, T, 7):
            nv = oracle.n_visible(t, s.m_hca, N)
            rows = np.concatenate([to64(E[:nv]), to64(raw[max(0, t - s.n_win + 1):t + 1])])
            ref = oracle.rope(oracle.mqa_attend(to64(q[t]), rows, s.scale), -t, s.rope_dims, s.rope_base)
            assert_norm_close(to64(out[t]), ref, what=f"{case} t={t}")
        return
    B, N = 3, (8192 if case.startswith("tc") else 2048)
    q = torch.randn((B, s.n_heads, s.c), generator=g).bfloat16()
    E = (torch.randn((B, N, s.c), generator=g) * (s.c ** -0.5)).bfloat16()
    win = torch.randn((B, s.n_win, s.c), generator=g).bfloat16()
    qp = torch.tensor([N * s.m_hca - 1, 777_777, N * s.m_hca + 5], dtype=torch.int32)
    out = hca.sparse_mqa_attend(q.cuda(), E.cuda(), win.cuda(), qp.cuda(), cfg, rate=s.m_hca,
                                mode=hca.HCA_MODE_DECODE, rotate_out=True)
    torch.cuda.synchronize()
    for b in range(B):
        t = int(qp[b])
        nv = oracle.n_visible(t, s.m_hca, N)
        rows = np.concatenate([to64(E[b, :nv]), to64(win[b, :min(s.n_win, t + 1)])])
        ref = oracle.rope(oracle.mqa_attend(to64(q[b]), rows, s.scale), -t, s.rope_dims, s.rope_base)
        assert_norm_close(to64(out[b]), ref, what=f"{case} request {b}")


def _prefill_with_norm(hca, s, T, seed):
    d = wl.prefill_inputs(s, T=T, seed=seed)
    g = to_dev(d)
    dev = "cuda"
    Nc, Nh = T // s.m, T // s.m_hca
    csa_kv = torch.empty((max(Nc, 1), s.c), dtype=torch.bfloat16, device=dev)
    csa_k = torch.empty((max(Nc, 1), s.d_idx), dtype=torch.bfloat16, device=dev)
    topk = torch.empty((T, s.topk), dtype=torch.int32, device=dev)
    csa_out = torch.empty((T, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    hca_kv = torch.empty((max(Nh, 1), s.c), dtype=torch.bfloat16, device=dev)
    hca_out = torch.empty_like(csa_out)
    wc, wh = wl.norm_weights(s, seed=seed), wl.norm_weights(s, seed=seed + 1)
    cfg = hca.make_cfg(s)
    # (temporaries on purpose: the args' keepalive must hold the weights)
    args, keep = hca.make_prefill_args(g, csa_kv, csa_k, topk, csa_out, hca_kv=hca_kv, hca_q=g["q"], hca_out=hca_out,
                                       csa_norm=wc.cuda(), hca_norm=wh.cuda())
    hca.hybrid_attn_prefill(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    n = {k: (to64(v) if v.is_floating_point() else v.numpy()) for k, v in d.items()}
    nc, nh = _qkn(s, wc), _qkn(s, wh)
    res = oracle.csa_layer_prefill(n["cand"], n["logits"], n["kidx_cand"], n["bias_csa"], n["q_idx"], n["w_idx"],
                                   n["q"], m=s.m, topk=s.topk, d_idx=s.d_idx, n_win=s.n_win, scale=s.scale, norm=nc)
    if Nc:
        E_exact = oracle.csa_compress(n["cand"], n["logits"], n["bias_csa"], s.m)
        assert_bf16_close(to64(csa_kv[:Nc]), oracle.norm_rope_rows(E_exact, oracle.entry_position(np.arange(Nc), s.m),
                                                                  nc.kv_gamma, nc), "normalised CSA entries")
    ti = topk.cpu().numpy()
    for t in range(T):
        check_topk_row(ti[t], res["idx"][t], res["scores"][t], s.topk, res["n_vis"][t])
    assert_norm_close(to64(csa_out), np.stack([res["O"][t] for t in range(T)]), what=f"CSA prefill T={T} with norm")
    hres = oracle.hca_layer_prefill(n["cand"], n["logits"], n["bias_hca"], n["q"], m_hca=s.m_hca, n_win=s.n_win,
                                    scale=s.scale, norm=nh)
    if Nh:
        E_exact = oracle.hca_compress(n["cand"], n["logits"], n["bias_hca"], s.m_hca)
        assert_bf16_close(to64(hca_kv[:Nh]),
                          oracle.norm_rope_rows(E_exact, oracle.entry_position(np.arange(Nh), s.m_hca), nh.kv_gamma, nh),
                          "normalised HCA entries")
    assert_norm_close(to64(hca_out), np.stack([hres["O"][t] for t in range(T)]), what=f"HCA prefill T={T} with norm")


def test_prefill_with_norm_tiny_cuda_cores(hca):
    _prefill_with_norm(hca, wl.TINY, 256, 31)


def test_prefill_with_norm_pro_tensor_cores(hca):
    _prefill_with_norm(hca, wl.PRO, 515, 32)


@pytest.mark.parametrize("ctx", [65536, 100])
def test_decode_with_norm_both_layers(hca, ctx):
    """Both layers in one step (overlapped HCA side stream at 64K), the HCA
    entry of the newest block normalised at its position; at ctx = 100 the
    window is partly empty and there is no HCA block yet (CSA layer only)."""
    s = wl.PRO
    B = 2
    csa = wl.csa_decode_inputs(s, B=B, ctx=ctx, seed=41, cache_std=1.0)
    hcad = wl.hca_decode_inputs(s, B=B, ctx=ctx, seed=42, cache_std=1.0) if ctx >= s.m_hca else None
    wc, wh = wl.norm_weights(s, seed=3), wl.norm_weights(s, seed=4)
    dev = "cuda"
    gc = to_dev(csa)
    gh = to_dev(hcad) if hcad is not None else None
    idx = torch.empty((B, s.topk), dtype=torch.int32, device=dev)
    co = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    ho = torch.empty_like(co) if hcad is not None else None
    cfg = hca.make_cfg(s)
    args, keep = hca.make_decode_args(B, gc["q_pos"], csa=gc, hca=gh, csa_topk_idx=idx, csa_out=co, hca_out=ho,
                                      csa_norm=wc.cuda(), hca_norm=wh.cuda() if hcad is not None else None)
    hca.hybrid_attn_decode(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    t = ctx - 1
    nc, nh = _qkn(s, wc), _qkn(s, wh)
    ii = idx.cpu().numpy()
    for b in range(B):
        r = oracle.csa_layer_decode(to64(csa["E"][b]), to64(csa["K_I"][b]), to64(csa["win"][b]), to64(csa["q"][b]),
                                    to64(csa["q_idx"][b]), csa["w_idx"][b].double().numpy(), t, m=s.m, topk=s.topk,
                                    n_win=s.n_win, scale=s.scale, norm=nc)
        check_topk_row(ii[b], r["idx"], r["scores"], s.topk, r["n_vis"])
        assert_norm_close(to64(co[b]), r["O"], what=f"CSA decode with norm, request {b}")
    if hcad is None:
        return
    Eh = to64(gh["E_h"])
    for b in range(B):
        r = oracle.hca_layer_decode(to64(hcad["E_h"][b]), to64(hcad["block_cand"][b]), to64(hcad["block_logits"][b]),
                                    to64(hcad["bias_hca"]), to64(hcad["win"][b]), to64(hcad["q"][b]), t,
                                    m_hca=s.m_hca, n_win=s.n_win, scale=s.scale, norm=nh)
        n_blk = (t + 1) // s.m_hca
        new_exact = oracle.hca_compress(to64(hcad["block_cand"][b]), to64(hcad["block_logits"][b]),
                                        to64(hcad["bias_hca"]), s.m_hca)
        assert_bf16_close(Eh[b, -1], oracle.norm_rope_rows(new_exact, oracle.entry_position(n_blk - 1, s.m_hca),
                                                           nh.kv_gamma, nh)[0], f"normalised new HCA entry {b}")
        assert_norm_close(to64(ho[b]), r["O"], what=f"HCA decode with norm, request {b}")
