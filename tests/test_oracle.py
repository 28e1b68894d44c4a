"""Pins of the CPU oracle against things other than itself.

Hand-worked values (tests/golden/hand_worked.json), closed forms, invariants,
special cases that reduce to a textbook result, and a pure-Python brute force
on tiny inputs.  Each test is chosen so that a plausible slip in the oracle
(a dropped term, a wrong sign or bias row, a transposed operand, ReLU applied
after the head sum, an off-by-one in causality) fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import brute_force as bf
import oracle
from long_context_attention_compress_b200 import workloads as wl

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))


def _np(t):
    return t.float().numpy().astype(np.float64)


# --------------------------------------------------------------------------
# hand-worked values
# --------------------------------------------------------------------------
def test_golden_hca_two_tokens():
    g = GOLD["hca_compress_two_tokens"]
    out = oracle.hca_compress(np.array(g["cand"]), np.array(g["logits"]), np.array(g["pos_bias"]), g["m_hca"])
    np.testing.assert_allclose(out, g["expected"], rtol=0, atol=1e-14)


def test_golden_csa_overlap():
    g = GOLD["csa_compress_overlap"]
    out = oracle.csa_compress(np.array(g["cand"]), np.array(g["logits"]), np.array(g["pos_bias"]), g["m"])
    np.testing.assert_allclose(out, g["expected"], rtol=0, atol=1e-14)


def test_golden_indexer_and_topk():
    g = GOLD["indexer_scores"]
    sc = oracle.indexer_scores(np.array(g["q_idx"]), np.array(g["w_idx"]), np.array(g["k_idx"]))
    np.testing.assert_allclose(sc, g["expected_scores"], rtol=0, atol=1e-14)
    assert oracle.topk_select(sc, g["topk"]).tolist() == g["expected_topk"]


def test_golden_topk_ties():
    g = GOLD["topk_ties"]
    assert oracle.topk_select(np.array(g["scores"]), g["topk"]).tolist() == g["expected_topk"]


def test_golden_mqa_two_rows():
    g = GOLD["mqa_two_rows"]
    o = oracle.mqa_attend(np.array(g["q"]), np.array(g["rows"]), g["scale"])
    np.testing.assert_allclose(o, g["expected"], rtol=0, atol=1e-15)


def test_golden_visibility_and_window():
    g = GOLD["visibility_m4"]
    got = [oracle.n_visible(t, g["m"], 10 ** 9) for t in g["t"]]
    assert got == g["expected_n_visible"]
    g = GOLD["window_n128"]
    for t, first, cnt in zip(g["t"], g["expected_first"], g["expected_count"]):
        w = oracle.window_rows(t, g["n_win"])
        assert w[0] == first and len(w) == cnt and w[-1] == t


def test_golden_bf16_rounding():
    g = GOLD["bf16_rounding"]
    assert oracle.round_bf16(np.array(g["x"])).tolist() == g["expected"]


def test_bf16_rounding_matches_torch_cast():
    # library routine: torch's float32 -> bfloat16 cast (round to nearest even)
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        1.0 + np.arange(256) * 2.0 ** -15]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(oracle.round_bf16(x), ref)


# --------------------------------------------------------------------------
# compressor: closed forms and invariants
# --------------------------------------------------------------------------
def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_compress_equal_logits_is_block_mean():
    rng = np.random.default_rng(2)
    T, c, m = 37, 5, 4
    C = _rand(rng, T, c)
    Z = np.full((T, c), 0.7)
    B = np.full((2 * m, c), -1.3)
    E = oracle.csa_compress(C, Z, B, m)
    for i in range(T // m):
        lo = max(0, (i - 1) * m)
        np.testing.assert_allclose(E[i], C[lo:(i + 1) * m].mean(0), atol=1e-13)
    Bh = np.full((8, c), 2.0)
    Eh = oracle.hca_compress(C, Z, Bh, 8)
    assert Eh.shape == (T // 8, c)
    for i in range(T // 8):
        np.testing.assert_allclose(Eh[i], C[8 * i:8 * i + 8].mean(0), atol=1e-13)


def test_hca_rate_one_is_identity():
    rng = np.random.default_rng(3)
    C, Z = _rand(rng, 9, 4), _rand(rng, 9, 4) * 5
    np.testing.assert_allclose(oracle.hca_compress(C, Z, _rand(rng, 1, 4), 1), C, atol=1e-15)


def test_csa_rate_one_one_hot_current_is_identity():
    rng = np.random.default_rng(4)
    C = _rand(rng, 11, 6)
    Z = np.zeros((11, 6))
    B = np.zeros((2, 6))
    B[1] = 30.0                     # bias row of the current block's token
    E = oracle.csa_compress(C, Z, B, 1)
    np.testing.assert_allclose(E, C, atol=1e-11)


def test_csa_previous_block_bias_rows():
    # bias row 0 (first token of the previous block) dominates: entry i >= 1
    # becomes token (i-1)m; entry 0 has no previous block and is a plain
    # softmax of its own block with bias rows m..2m-1 (zero here).
    rng = np.random.default_rng(5)
    T, c, m = 24, 3, 4
    C, Z = _rand(rng, T, c), _rand(rng, T, c) * 0.1
    B = np.zeros((2 * m, c))
    B[0] = 40.0
    E = oracle.csa_compress(C, Z, B, m)
    for i in range(1, T // m):
        np.testing.assert_allclose(E[i], C[(i - 1) * m], atol=1e-12)
    w = np.exp(Z[:m] - Z[:m].max(0))
    np.testing.assert_allclose(E[0], (w * C[:m]).sum(0) / w.sum(0), atol=1e-13)


def test_compress_two_token_sigmoid_closed_form():
    rng = np.random.default_rng(6)
    C, Z, B = _rand(rng, 2, 7), _rand(rng, 2, 7) * 3, _rand(rng, 2, 7)
    E = oracle.hca_compress(C, Z, B, 2)[0]
    x = (Z[0] + B[0]) - (Z[1] + B[1])
    sig = 1.0 / (1.0 + np.exp(-x))
    np.testing.assert_allclose(E, sig * C[0] + (1 - sig) * C[1], atol=1e-14)


@pytest.mark.parametrize("i", [0, 1, 5])
def test_compress_weights_sum_to_one(i):
    rng = np.random.default_rng(7)
    Z, B = _rand(rng, 32, 16) * 4, _rand(rng, 8, 16)
    w = oracle.compress_weights_csa(Z, B, 4, i)
    assert w.shape == ((4 if i == 0 else 8), 16)
    assert np.all(w > 0) and np.max(np.abs(w.sum(0) - 1.0)) < 1e-12
    wh = oracle.compress_weights_hca(Z, _rand(rng, 8, 16), 8, 2)
    assert np.max(np.abs(wh.sum(0) - 1.0)) < 1e-12


def test_trailing_incomplete_block_gives_no_entry():
    rng = np.random.default_rng(8)
    C, Z = _rand(rng, 10, 2), _rand(rng, 10, 2)
    assert oracle.csa_compress(C, Z, _rand(rng, 8, 2), 4).shape == (2, 2)
    assert oracle.hca_compress(C, Z, _rand(rng, 4, 2), 4).shape == (2, 2)


def test_compress_brute_force_tiny():
    rng = np.random.default_rng(9)
    T, c = 26, 3
    C, Z = _rand(rng, T, c), _rand(rng, T, c) * 2
    for m in (1, 2, 4):
        B = _rand(rng, 2 * m, c)
        np.testing.assert_allclose(oracle.csa_compress(C, Z, B, m),
                                   bf.csa_compress(C.tolist(), Z.tolist(), B.tolist(), m), atol=1e-13)
    Bh = _rand(rng, 8, c)
    np.testing.assert_allclose(oracle.hca_compress(C, Z, Bh, 8),
                               bf.hca_compress(C.tolist(), Z.tolist(), Bh.tolist(), 8), atol=1e-13)


# --------------------------------------------------------------------------
# indexer and top-k
# --------------------------------------------------------------------------
def test_indexer_single_head_aligned_query():
    rng = np.random.default_rng(10)
    K = _rand(rng, 5, 8)
    for s in range(5):
        q = np.zeros((3, 8))
        q[1] = 2.5 * K[s]
        w = np.array([0.0, 1.0, 0.0])
        assert abs(oracle.indexer_scores(q, w, K)[s] - 2.5 * K[s] @ K[s]) < 1e-12


def test_indexer_all_negative_dots_give_zero():
    rng = np.random.default_rng(11)
    K = np.abs(_rand(rng, 6, 4))
    q = -np.abs(_rand(rng, 3, 4))
    assert np.all(oracle.indexer_scores(q, np.ones(3), K) == 0.0)


def test_indexer_relu_is_per_head():
    # opposite-sign heads must not cancel: ReLU before the weighted head sum
    k = np.array([[1.0, 2.0]])
    q = np.array([[1.0, 2.0], [-1.0, -2.0]])
    assert oracle.indexer_scores(q, np.array([1.0, 1.0]), k)[0] == 5.0


def test_indexer_linear_in_weights():
    rng = np.random.default_rng(12)
    q, K = _rand(rng, 4, 6), _rand(rng, 9, 6)
    w1, w2 = rng.random(4), rng.random(4)
    np.testing.assert_allclose(oracle.indexer_scores(q, w1 + w2, K),
                               oracle.indexer_scores(q, w1, K) + oracle.indexer_scores(q, w2, K), atol=1e-12)


def test_indexer_brute_force_tiny():
    rng = np.random.default_rng(13)
    q, w, K = _rand(rng, 4, 8), rng.random(4), _rand(rng, 20, 8)
    ref = [bf.index_score(q.tolist(), w.tolist(), K[s].tolist()) for s in range(20)]
    np.testing.assert_allclose(oracle.indexer_scores(q, w, K), ref, atol=1e-12)


@pytest.mark.parametrize("k", [1, 7, 50, 64, 200])
def test_topk_matches_python_sort_and_threshold_property(k):
    rng = np.random.default_rng(14 + k)
    sc = np.round(rng.standard_normal(100) * 3)   # many exact ties
    sel = oracle.topk_select(sc, k)
    assert sel.tolist() == bf.topk(sc.tolist(), k)
    n = min(k, 100)
    assert len(set(sel.tolist())) == n
    rest = np.setdiff1d(np.arange(100), sel)
    if len(rest):
        thr = sc[sel].min()
        assert sc[rest].max() <= thr
        # among entries tied at the threshold, the selected ones have the lowest indices
        tied_out = rest[sc[rest] == thr]
        tied_in = sel[sc[sel] == thr]
        if len(tied_out):
            assert tied_in.max() < tied_out.min()


def test_topk_takes_all_when_fewer_than_k():
    assert sorted(oracle.topk_select(np.array([3.0, 1.0, 2.0]), 10).tolist()) == [0, 1, 2]
    assert oracle.topk_select(np.array([]), 4).tolist() == []


def test_visibility_brute_force():
    for rate in (1, 4, 32, 128):
        for t in list(range(0, 300)) + [4095, 4096, 65535]:
            assert oracle.n_visible(t, rate, 10 ** 9) == len(bf.visible(t, rate, 70000))
    assert oracle.n_visible(10 ** 6, 4, 17) == 17


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def test_attention_single_row_returns_it():
    rng = np.random.default_rng(15)
    q, r = _rand(rng, 3, 8), _rand(rng, 1, 8)
    np.testing.assert_allclose(oracle.mqa_attend(q, r, 0.3), np.repeat(r, 3, 0), atol=1e-15)


def test_attention_zero_query_is_mean():
    rng = np.random.default_rng(16)
    rows = _rand(rng, 13, 8)
    np.testing.assert_allclose(oracle.mqa_attend(np.zeros((2, 8)), rows, 1.0),
                               np.repeat(rows.mean(0, keepdims=True), 2, 0), atol=1e-14)


def test_attention_permutation_invariant():
    rng = np.random.default_rng(17)
    q, rows = _rand(rng, 4, 16), _rand(rng, 40, 16)
    p = rng.permutation(40)
    np.testing.assert_allclose(oracle.mqa_attend(q, rows, 0.25), oracle.mqa_attend(q, rows[p], 0.25), atol=1e-13)


def test_attention_two_rows_sigmoid():
    rng = np.random.default_rng(18)
    q, rows = _rand(rng, 3, 6), _rand(rng, 2, 6)
    s = 0.5 * q @ rows.T
    sig = 1.0 / (1.0 + np.exp(-(s[:, 0] - s[:, 1])))
    np.testing.assert_allclose(oracle.mqa_attend(q, rows, 0.5),
                               sig[:, None] * rows[0] + (1 - sig)[:, None] * rows[1], atol=1e-14)


def test_attention_brute_force_tiny():
    rng = np.random.default_rng(19)
    q, rows = _rand(rng, 3, 5), _rand(rng, 9, 5)
    np.testing.assert_allclose(oracle.mqa_attend(q, rows, 0.7), bf.attend(q.tolist(), rows.tolist(), 0.7),
                               atol=1e-13)


@pytest.mark.parametrize("cuts", [[5], [1, 2, 30], [10, 11, 12, 13]])
def test_split_combine_equals_unsplit(cuts):
    rng = np.random.default_rng(20)
    q, rows = _rand(rng, 4, 8) * 3, _rand(rng, 40, 8)
    bounds = [0] + cuts + [40]
    parts = [oracle.mqa_partial(q, rows[a:b], 0.5) for a, b in zip(bounds[:-1], bounds[1:])]
    np.testing.assert_allclose(oracle.combine_partials(parts), oracle.mqa_attend(q, rows, 0.5), atol=1e-13)


# --------------------------------------------------------------------------
# attention sink: one logit per head in the softmax denominator only
# ([QbitAI] "混合注意力機制", attention-sink paragraph; [Tricks] "Partial RoPE 和
# Attention Sink")
# --------------------------------------------------------------------------
def test_sink_at_minus_infinity_is_plain_attention():
    rng = np.random.default_rng(40)
    q, rows = _rand(rng, 4, 8), _rand(rng, 17, 8)
    np.testing.assert_array_equal(oracle.mqa_attend(q, rows, 0.5, sink=np.full(4, -np.inf)),
                                  oracle.mqa_attend(q, rows, 0.5))


def test_sink_with_one_row_is_a_sigmoid():
    from scipy.special import expit
    rng = np.random.default_rng(41)
    q, row = _rand(rng, 5, 8) * 2, _rand(rng, 1, 8)
    z = rng.standard_normal(5)
    s = 0.5 * (q @ row[0])
    np.testing.assert_allclose(oracle.mqa_attend(q, row, 0.5, sink=z), expit(s - z)[:, None] * row, atol=1e-14)


def test_sink_equals_an_extra_zero_valued_row():
    rng = np.random.default_rng(42)
    q, rows = _rand(rng, 3, 6) * 2, _rand(rng, 11, 6)
    z = rng.standard_normal(3) + 1.0
    np.testing.assert_allclose(oracle.mqa_attend(q, rows, 0.6, sink=z),
                               bf.attend_with_sink_row(q.tolist(), rows.tolist(), 0.6, z.tolist()), atol=1e-13)


@pytest.mark.parametrize("cuts", [[5], [1, 2, 30]])
def test_sink_split_combine_equals_unsplit(cuts):
    rng = np.random.default_rng(43)
    q, rows = _rand(rng, 4, 8) * 3, _rand(rng, 40, 8)
    z = rng.standard_normal(4) * 3
    bounds = [0] + cuts + [40]
    parts = [oracle.mqa_partial(q, rows[a:b], 0.5) for a, b in zip(bounds[:-1], bounds[1:])]
    np.testing.assert_allclose(oracle.combine_partials(parts, sink=z), oracle.mqa_attend(q, rows, 0.5, sink=z),
                               atol=1e-13)


def test_a_dominant_sink_silences_the_head():
    rng = np.random.default_rng(44)
    q, rows = _rand(rng, 2, 8), _rand(rng, 9, 8)
    o = oracle.mqa_attend(q, rows, 0.5, sink=np.array([500.0, -np.inf]))
    assert np.all(np.abs(o[0]) < 1e-200)
    np.testing.assert_array_equal(o[1], oracle.mqa_attend(q, rows, 0.5)[1])


# --------------------------------------------------------------------------
# whole layers on the tiny shape
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def tiny():
    d = wl.prefill_inputs(wl.TINY, T=256, seed=3)
    return {k: (_np(v) if v.is_floating_point() else v.numpy()) for k, v in d.items()}


def _csa(tiny, topk, queries):
    s = wl.TINY
    return oracle.csa_layer_prefill(tiny["cand"], tiny["logits"], tiny["kidx_cand"], tiny["bias_csa"],
                                    tiny["q_idx"], tiny["w_idx"], tiny["q"], m=s.m, topk=topk,
                                    d_idx=s.d_idx, n_win=s.n_win, scale=s.scale, queries=queries)


def test_csa_layer_with_k_at_least_visible_is_dense(tiny):
    s = wl.TINY
    qs = [0, 2, 3, 4, 63, 100, 255]
    res = _csa(tiny, topk=10 ** 6, queries=qs)
    E = res["E"]
    for t in qs:
        nv = oracle.n_visible(t, s.m, E.shape[0])
        assert sorted(res["idx"][t].tolist()) == list(range(nv))
        rows = np.concatenate([E[:nv], tiny["cand"][max(0, t - s.n_win + 1):t + 1]])
        np.testing.assert_allclose(res["O"][t], bf.attend(tiny["q"][t].tolist(), rows.tolist(), s.scale),
                                   atol=1e-12)


def test_csa_layer_brute_force_tiny(tiny):
    s = wl.TINY
    qs = [3, 40, 200, 255]
    res = _csa(tiny, topk=s.topk // 4, queries=qs)
    C, Z, KC, Bc = (tiny[k] for k in ("cand", "logits", "kidx_cand", "bias_csa"))
    E = oracle.round_bf16(np.array(bf.csa_compress(C.tolist(), Z.tolist(), Bc.tolist(), s.m)))
    KI = oracle.round_bf16(np.array(bf.csa_compress(KC.tolist(), Z[:, :s.d_idx].tolist(),
                                                    Bc[:, :s.d_idx].tolist(), s.m)))
    np.testing.assert_array_equal(res["E"], E)
    np.testing.assert_array_equal(res["K_I"], KI)
    for t in qs:
        vis = bf.visible(t, s.m, len(E))
        sc = [bf.index_score(tiny["q_idx"][t].tolist(), tiny["w_idx"][t].tolist(), KI[v].tolist()) for v in vis]
        sel = bf.topk(sc, s.topk // 4)
        assert res["idx"][t].tolist() == sel
        rows = [E[v].tolist() for v in sel] + [tiny["cand"][r].tolist() for r in range(max(0, t - s.n_win + 1), t + 1)]
        np.testing.assert_allclose(res["O"][t], bf.attend(tiny["q"][t].tolist(), rows, s.scale), atol=1e-12)


def test_hca_layer_brute_force_tiny(tiny):
    s = wl.TINY
    qs = [0, 30, 31, 32, 100, 255]
    res = oracle.hca_layer_prefill(tiny["cand"], tiny["logits"], tiny["bias_hca"], tiny["q"],
                                   m_hca=s.m_hca, n_win=s.n_win, scale=s.scale, queries=qs)
    E = oracle.round_bf16(np.array(bf.hca_compress(tiny["cand"].tolist(), tiny["logits"].tolist(),
                                                   tiny["bias_hca"].tolist(), s.m_hca)))
    np.testing.assert_array_equal(res["E"], E)
    for t in qs:
        vis = bf.visible(t, s.m_hca, len(E))
        rows = [E[v].tolist() for v in vis] + [tiny["cand"][r].tolist()
                                               for r in range(max(0, t - s.n_win + 1), t + 1)]
        np.testing.assert_allclose(res["O"][t], bf.attend(tiny["q"][t].tolist(), rows, s.scale), atol=1e-12)


def test_decode_entry_points_agree_with_prefill(tiny):
    s = wl.TINY
    t = 255
    res = _csa(tiny, topk=s.topk // 2, queries=[t])
    win = tiny["cand"][t - s.n_win + 1:t + 1]
    dec = oracle.csa_layer_decode(res["E"], res["K_I"], win[::-1], tiny["q"][t], tiny["q_idx"][t],
                                  tiny["w_idx"][t], t, m=s.m, topk=s.topk // 2, n_win=s.n_win, scale=s.scale)
    assert dec["idx"].tolist() == res["idx"][t].tolist()
    np.testing.assert_allclose(dec["O"], res["O"][t], atol=1e-13)
    hres = oracle.hca_layer_prefill(tiny["cand"], tiny["logits"], tiny["bias_hca"], tiny["q"],
                                    m_hca=s.m_hca, n_win=s.n_win, scale=s.scale, queries=[t])
    hdec = oracle.hca_layer_decode(hres["E"], tiny["cand"][t - s.m_hca + 1:t + 1], tiny["logits"][t - s.m_hca + 1:t + 1],
                                   tiny["bias_hca"], win, tiny["q"][t], t, m_hca=s.m_hca, n_win=s.n_win,
                                   scale=s.scale)
    np.testing.assert_array_equal(hdec["new_entry"], hres["E"][-1])
    np.testing.assert_allclose(hdec["O"], hres["O"][t], atol=1e-13)
