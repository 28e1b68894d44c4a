"""The opt-in index check (HCA_DEBUG=1) of the attention kernels.

Selected entries reach the attention as plain integers; a wrong one (outside
[-1, N), or an entry whose last token lies after the query's position) would
silently change the output.  With HCA_DEBUG=1 the tensor-core and the CUDA-core
attention record such entries and hca_check_device reports them; the results
stay exactly those of the same call without the check, and an out-of-range
entry is skipped like an empty slot either way.  Every planted entry lies
inside the allocated cache or is skipped before any load, so no run reads
outside its buffers.  A whole hybrid prefill and decode under the check record
nothing: the indexer's top-k only ever selects visible entries.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import assert_norm_close, to64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hca():
    import long_context_attention_compress_b200 as h
    assert h.lib.hca_check_device() == 0, h.last_error()  # nothing pending from earlier tests
    return h


def _status(hca):
    st = hca.lib.hca_check_device()
    return st, hca.last_error()


def test_tensor_core_decode_flags_range_and_causal(hca, monkeypatch):
    s = wl.PRO
    B, ctx = 3, 16384
    d = wl.csa_decode_inputs(s, B=B, ctx=ctx, seed=31)
    N = d["E"].shape[1]
    q_pos = d["q_pos"].clone()
    q_pos[1] = 8191                          # request 1 sees entries [0, 2048) only
    d["q_pos"] = q_pos
    g = to_dev(d)
    cfg = hca.make_cfg(s)
    rng = np.random.default_rng(5)
    nvis = [oracle.n_visible(int(q_pos[b]), s.m, N) for b in range(B)]
    idx = np.stack([rng.choice(nvis[b], s.topk, replace=False) for b in range(B)]).astype(np.int32)
    idx[2, 17] = -1                          # an empty slot is acceptable

    def run(ix):
        o = hca.sparse_mqa_attend(g["q"], g["E"], g["win"], g["q_pos"], cfg, idx=torch.from_numpy(ix).cuda(),
                                  mode=hca.HCA_MODE_DECODE)
        torch.cuda.synchronize()
        return o

    ref_plain = run(idx)
    assert _status(hca)[0] == 0
    monkeypatch.setenv("HCA_DEBUG", "1")
    out_valid = run(idx)
    assert _status(hca) == (0, "")
    assert torch.equal(out_valid, ref_plain)  # the check changes no result

    bad = idx.copy()
    bad[0, 5] = N + 7                        # out of range
    bad[1, 9] = 3000                         # in the cache, after request 1's position
    out_bad = run(bad)
    st, msg = _status(hca)
    assert st == -5, (st, msg)               # HCA_ERR_DEVICE_CHECK
    assert "out of range" in msg and "not yet visible" in msg, msg
    assert "block-table" not in msg, msg
    assert _status(hca)[0] == 0              # reported once, then cleared

    monkeypatch.delenv("HCA_DEBUG")
    out_bad_plain = run(bad)
    assert _status(hca)[0] == 0              # nothing recorded without the check
    assert torch.equal(out_bad, out_bad_plain)
    # the out-of-range slot counts as empty
    E0, w0 = to64(d["E"][0]), to64(d["win"][0])
    keep = np.delete(bad[0], 5)
    ref0 = oracle.mqa_attend(to64(d["q"][0]), np.concatenate([E0[keep], w0]), s.scale)
    assert_norm_close(to64(out_bad[0]), ref0, what="out-of-range slot skipped")


def test_cuda_core_prefill_flags_range_and_causal(hca, monkeypatch):
    s = wl.TINY                              # c=64, 4 heads: the CUDA-core attention
    T = 256
    d = wl.prefill_inputs(s, T=T, seed=33, with_hca=False)
    Nc = T // s.m
    E = torch.randn((Nc, s.c), generator=torch.Generator().manual_seed(34)).bfloat16()
    rng = np.random.default_rng(6)
    idx = np.full((T, s.topk), -1, dtype=np.int32)
    for t in range(T):
        nv = oracle.n_visible(t, s.m, Nc)
        k = min(nv, s.topk)
        idx[t, :k] = rng.choice(nv, k, replace=False)
    g = to_dev(d)
    Eg = E.cuda()
    cfg = hca.make_cfg(s)

    def run(ix):
        o = hca.sparse_mqa_attend(g["q"], Eg, g["cand"], g["q_pos"], cfg, idx=torch.from_numpy(ix).cuda())
        torch.cuda.synchronize()
        return o

    monkeypatch.setenv("HCA_DEBUG", "1")
    run(idx)
    assert _status(hca) == (0, "")
    bad = idx.copy()
    bad[200, 3] = Nc + 3                     # out of range (skipped, never loaded)
    out_bad = run(bad)
    st, msg = _status(hca)
    assert st == -5 and "out of range" in msg and "not yet visible" not in msg, (st, msg)
    bad[10, 1] = 40                          # query 10 sees entries [0, 2) only
    run(bad)
    st, msg = _status(hca)
    assert st == -5 and "out of range" in msg and "not yet visible" in msg, (st, msg)
    monkeypatch.delenv("HCA_DEBUG")
    bad[10, 1] = idx[10, 1]
    assert torch.equal(run(bad), out_bad)
    assert _status(hca)[0] == 0
    # query 200 with the bad slot skipped
    t = 200
    keep = np.delete(bad[t], 3)
    keep = keep[keep >= 0]
    rows = np.concatenate([to64(E)[keep], to64(d["cand"])[oracle.window_rows(t, s.n_win)]])
    assert_norm_close(to64(out_bad[t:t + 1]), oracle.mqa_attend(to64(d["q"][t]), rows, s.scale)[None],
                      what="out-of-range slot skipped (CUDA cores)")


def test_whole_layers_record_nothing(hca, monkeypatch):
    """The indexer's selections are always in range and visible: a hybrid
    prefill (ragged length) and a hybrid decode with ragged positions pass the
    check."""
    monkeypatch.setenv("HCA_DEBUG", "1")
    s = wl.TINY
    T = 1001
    d = wl.prefill_inputs(s, T=T, seed=35)
    g = to_dev(d)
    Nc, Nh = T // s.m, T // s.m_hca
    dev = "cuda"
    csa_kv = torch.empty((Nc, s.c), dtype=torch.bfloat16, device=dev)
    csa_k = torch.empty((Nc, s.d_idx), dtype=torch.bfloat16, device=dev)
    topk = torch.empty((T, s.topk), dtype=torch.int32, device=dev)
    csa_out = torch.empty((T, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    hca_kv = torch.empty((Nh, s.c), dtype=torch.bfloat16, device=dev)
    hca_out = torch.empty_like(csa_out)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_prefill_args(g, csa_kv, csa_k, topk, csa_out, hca_kv=hca_kv, hca_q=g["q"],
                                       hca_out=hca_out)
    hca.hybrid_attn_prefill(cfg, args)
    assert _status(hca) == (0, "")

    s = wl.PRO
    B = 4
    dd = wl.hybrid_decode_inputs(s, B=B, ctx=65536, seed=36, cache_std=1.0)
    q_pos = dd["csa"]["q_pos"].clone()
    q_pos[:] = torch.tensor([65535, 40000, 9001, 511], dtype=q_pos.dtype)
    dd["csa"]["q_pos"] = q_pos
    dd["hca"]["q_pos"] = q_pos
    gc, gh = to_dev(dd["csa"]), to_dev(dd["hca"])
    idx = torch.empty((B, s.topk), dtype=torch.int32, device=dev)
    co = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
    ho = torch.empty_like(co)
    pcfg = hca.make_cfg(s)
    dargs, dkeep = hca.make_decode_args(B, gc["q_pos"], csa=gc, hca=gh, csa_topk_idx=idx, csa_out=co, hca_out=ho)
    hca.hybrid_attn_decode(pcfg, dargs)
    assert _status(hca) == (0, "")
    ii = idx.cpu().numpy()
    for b in range(B):
        nv = oracle.n_visible(int(q_pos[b]), s.m, dd["csa"]["E"].shape[1])
        sel = ii[b][ii[b] >= 0]
        assert len(sel) == min(nv, s.topk) and sel.max(initial=-1) < nv
