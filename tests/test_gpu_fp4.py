"""GPU parity of the FP4 indexer variant against the oracle.

"DeepSeek V4 Architecture Tricks", "FP4 / FP8 Quantization-Aware Training":
the indexer's QK path is cached, loaded and multiplied in FP4 and the index
scores are kept in BF16.  The quantiser must reproduce the oracle's MXFP4
codes and scales bit for bit.  The FP4 indexer's BF16 scores must pick the
oracle's top-k (oracle: MXFP4 values of the same bf16 inputs, float64 sums,
BF16 rounding) up to near-ties: a score formed in f32 and one formed in
float64 may round to neighbouring BF16 values, so an entry may swap in or out
only when its oracle score lies within two BF16 steps (2^-6 relative) of the
oracle's k-th score.  Its recall of the float64 top-k over the unquantised
keys is reported (not asserted: the write-ups' 99.7 % is a property of
trained activations, not of synthetic N(0, 1) data).
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import assert_norm_close, check_topk_row, to64

pytestmark = pytest.mark.gpu

FP4_BAND = 2.0 ** -6  # two BF16 steps of the k-th score


@pytest.fixture(scope="module")
def hca():
    import long_context_attention_compress_b200 as h
    return h


def _rows(rng, n, d):
    x = rng.normal(size=(n, d)) * 10.0 ** rng.uniform(-3, 3, size=(n, 1))
    x[0, :32] = 0.0                                   # an all-zero block
    x[1, :32] = [6, 3, -1.5, 0.25, 7, 0.75, -0.25, 1.25, 2.5, 5] + [0] * 22   # ties and saturation
    x[2, 32:64] = 1e-30                               # a tiny block
    x[3, 64:96] = -x[3, 64:96]
    return x


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_mxfp4_quantize_bit_exact(hca, dtype):
    rng = np.random.default_rng(0)
    x = torch.tensor(_rows(rng, 500, 128)).to(dtype)
    codes, scales = hca.mxfp4_quantize(x.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.mxfp4_quantize(to64(x))
    np.testing.assert_array_equal(scales.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(codes.cpu().numpy(), oracle.mxfp4_pack(c_ref))


def _fp4_keys(hca, K, s):
    """MXFP4 cache form of bf16 keys [B, N, d_I] on the device: codes [B, N, 64], scales [B, N, 4]."""
    B, N, _ = K.shape
    codes = torch.zeros((B, N, s.d_idx // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((B, N, s.d_idx // 32), dtype=torch.uint8, device="cuda")
    for b in range(B):
        hca.mxfp4_quantize(K[b].cuda(), codes=codes[b], scales=scales[b])
    return codes, scales


def _check_requests(idx, q, w, K, t, s, report=None):
    ii = idx.cpu().numpy()
    recalls = []
    for b in range(K.shape[0]):
        nv = oracle.n_visible(t, s.m, K.shape[1])
        Kb = to64(K[b])[:nv]
        sc = oracle.indexer_scores_fp4(to64(q[b]), w[b].double().numpy(), Kb)
        sel = oracle.topk_select(sc, s.topk)
        check_topk_row(ii[b], sel, sc, s.topk, nv, band=FP4_BAND)
        if report is not None:
            ref = oracle.topk_select(oracle.indexer_scores(to64(q[b]), w[b].double().numpy(), Kb), s.topk)
            recalls.append(oracle.topk_recall(ii[b][ii[b] >= 0], ref))
    if report is not None:
        report.append(recalls)


@pytest.mark.parametrize("B,N,t", [(4, 20000, 4 * 20000 - 1), (2, 100000, 4 * 100000 - 1),
                                   (3, 100000, 4 * 70001 + 2)])
def test_fp4_indexer_topk(hca, B, N, t):
    s = wl.PRO
    g = torch.Generator().manual_seed(N + t)
    K = torch.randn((B, N, s.d_idx), generator=g).bfloat16()
    q = torch.randn((B, s.n_idx_heads, s.d_idx), generator=g).bfloat16()
    w = torch.rand((B, s.n_idx_heads), generator=g)
    codes, scales = _fp4_keys(hca, K, s)
    q_pos = torch.full((B,), t, dtype=torch.int32)
    cfg = hca.make_cfg(s)
    idx = hca.csa_indexer_topk_fp4(q.cuda(), w.cuda(), codes, scales, q_pos.cuda(), cfg)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    _check_requests(idx, q, w, K, t, s)


def test_fp4_indexer_hybrid_1m_shape(hca):
    """The FP4 indexer inside hybrid_attn_decode at the 1M-context shape (8 requests x
    262,144 entries): top-k sets against the oracle, the CSA output against the oracle's
    attention over its own selection, and the recall of the float64 top-k reported."""
    s = wl.PRO
    B, ctx = 8, 1048576
    d = wl.hybrid_decode_inputs(s, B, ctx, seed=11)
    c = d["csa"]
    gc = {k: v.cuda() for k, v in c.items()}
    gh = {k: v.cuda() for k, v in d["hca"].items()}
    k4 = _fp4_keys(hca, c["K_I"], s)
    del gc["K_I"]
    idx = torch.empty((B, s.topk), dtype=torch.int32, device="cuda")
    oc = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device="cuda")
    oh = torch.empty_like(oc)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_decode_args(B, gc["q_pos"], csa=gc, hca=gh, csa_topk_idx=idx, csa_out=oc, hca_out=oh,
                                      csa_k4=k4)
    hca.hybrid_attn_decode(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    t = ctx - 1
    rec = []
    _check_requests(idx, c["q_idx"], c["w_idx"], c["K_I"], t, s, report=rec)
    print(f"FP4 + BF16-score recall of the float64 top-1024: per request {np.round(rec[0], 4).tolist()}")
    for b in range(2):  # end-to-end outputs of two requests, against the oracle's own selection
        sc = oracle.indexer_scores_fp4(to64(c["q_idx"][b]), c["w_idx"][b].double().numpy(), to64(c["K_I"][b]))
        sel = oracle.topk_select(sc, s.topk)
        rows = np.concatenate([to64(c["E"][b])[sel], to64(c["win"][b])])
        assert_norm_close(to64(oc[b].cpu()), oracle.mqa_attend(to64(c["q"][b]), rows, s.scale),
                          what=f"fp4 hybrid request {b}")
