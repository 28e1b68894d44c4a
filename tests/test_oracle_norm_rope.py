"""Pins of the oracle's Q/KV RMSNorm, partial RoPE and output rotation.

What the pages fix (QbitAI write-up, "混合注意力機制": the Q/KV normalisation
and partial-RoPE tricks; "DeepSeek V4 Architecture Tricks", "Partial RoPE 和
Attention Sink"): queries and KV entries are RMS-normalised before core
attention, only the last 64 channels carry a rotary position, and the output is
rotated by -i so that only relative positions survive the shared K = V.  The
pins below are hand-worked values, rotation-group identities, the
relative-position property and the closed form of a one-row attention -- each
chosen so that a plausible slip (a missing weight, a swapped q/kv weight, a
rotation of the wrong channels or in the wrong sense, a forgotten or
same-sign output rotation, an off-by-one entry position) fails one of them.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from long_context_attention_compress_b200 import workloads as wl

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))


def _nrm(c, rng=None, rope_dims=64, eps=1e-6, gq=None, gkv=None, base=10000.0):
    rng = rng or np.random.default_rng(0)
    gq = rng.uniform(0.5, 1.5, c) if gq is None else gq
    gkv = rng.uniform(0.5, 1.5, c) if gkv is None else gkv
    return oracle.QKNorm(gq, gkv, eps=eps, rope_dims=rope_dims, base=base)


def test_rms_norm_hand_worked():
    g = GOLD["rms_norm_3_4"]
    for case in g["cases"]:
        y = oracle.rms_norm(np.array(g["x"]), np.array(case["gamma"]), case["eps"])
        np.testing.assert_allclose(y, case["expected"], rtol=0, atol=1e-15)


def test_rms_norm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(7, 512)) * rng.uniform(0.1, 30, size=(7, 1))
    y = oracle.rms_norm(x, np.ones(512), 0.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1) / math.sqrt(512), 1.0, atol=1e-14)
    np.testing.assert_allclose(oracle.rms_norm(3.7 * x, np.ones(512), 0.0), y, atol=1e-14)
    # eps keeps an all-zero row at zero
    assert np.all(oracle.rms_norm(np.zeros((1, 8)), np.ones(8), 1e-6) == 0.0)


def test_rope_hand_worked():
    g = GOLD["rope_pairs"]
    y = oracle.rope(np.array([g["x"]]), g["pos"], g["rope_dims"], g["base"])[0]
    np.testing.assert_array_equal(y[:2], g["untouched"])
    for j, a in enumerate(g["pair_angles"]):
        np.testing.assert_allclose(y[2 + 2 * j:4 + 2 * j], [math.cos(a), math.sin(a)], atol=1e-15)


def test_rope_theta_closed_form():
    th = oracle.rope_theta(64, 10000.0)
    assert th[0] == 1.0 and len(th) == 32
    np.testing.assert_allclose(th[16], 0.01, rtol=1e-14)   # 10000^(-32/64)
    np.testing.assert_allclose(th[1] / th[0], 10000.0 ** (-1 / 32), rtol=1e-14)


def test_rope_is_a_rotation_group():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(5, 512))
    a, b = 123.0, -4567.0
    np.testing.assert_allclose(oracle.rope(oracle.rope(x, a, 64, 1e4), b, 64, 1e4),
                               oracle.rope(x, a + b, 64, 1e4), atol=1e-12)
    np.testing.assert_array_equal(oracle.rope(x, 0.0, 64, 1e4), x)
    np.testing.assert_allclose(oracle.rope(oracle.rope(x, 99999.0, 64, 1e4), -99999.0, 64, 1e4), x, atol=1e-11)
    y = oracle.rope(x, 777.0, 64, 1e4)
    np.testing.assert_array_equal(y[:, :448], x[:, :448])
    pn = lambda z: z[:, 448::2] ** 2 + z[:, 449::2] ** 2  # noqa: E731
    np.testing.assert_allclose(pn(y), pn(x), rtol=1e-13)


def test_rope_dot_depends_only_on_offset():
    rng = np.random.default_rng(3)
    q, k = rng.normal(size=512), rng.normal(size=512)
    ref = oracle.rope(q, 1000, 64, 1e4) @ oracle.rope(k, 400, 64, 1e4)
    for s in (1, 17, 100000):
        got = oracle.rope(q, 1000 + s, 64, 1e4) @ oracle.rope(k, 400 + s, 64, 1e4)
        np.testing.assert_allclose(got, ref, rtol=1e-10)
    # ... and does depend on it
    assert abs(oracle.rope(q, 1001, 64, 1e4) @ oracle.rope(k, 400, 64, 1e4) - ref) > 1e-3


def test_entry_position_matches_causal_visibility():
    for m in (4, 128):
        for t in range(3 * m + 2):
            nv = oracle.n_visible(t, m, 10 ** 6)
            for s in range(4):
                assert (s < nv) == (oracle.entry_position(s, m) <= t)


def test_one_row_attention_is_the_row_turned_by_the_offset():
    """softmax over one row is 1: o = R(-t) R(j) norm(v) = R(j - t) norm(v)."""
    rng = np.random.default_rng(4)
    c = 512
    nrm = _nrm(c, rng)
    q, v = rng.normal(size=(8, c)), rng.normal(size=(1, c))
    t, j = 5000, 4321
    o = oracle.attend_norm_rope(q, t, v, [j], 1 / math.sqrt(c), nrm, bf16_operands=False)
    want = oracle.rope(oracle.rms_norm(v, nrm.kv_gamma, nrm.eps), j - t, 64, 1e4)[0]
    np.testing.assert_allclose(o, np.broadcast_to(want, o.shape), atol=1e-12)


def test_output_depends_only_on_relative_positions():
    rng = np.random.default_rng(5)
    c = 512
    nrm = _nrm(c, rng)
    q, rows = rng.normal(size=(8, c)), rng.normal(size=(40, c))
    pos = rng.integers(0, 3000, size=40)
    o = oracle.attend_norm_rope(q, 3000, rows, pos, 1 / math.sqrt(c), nrm, bf16_operands=False)
    for s in (1, 12345):
        np.testing.assert_allclose(oracle.attend_norm_rope(q, 3000 + s, rows, pos + s, 1 / math.sqrt(c), nrm,
                                                           bf16_operands=False), o, atol=1e-10)
    # without the output rotation the shift would show
    o_plain = oracle.mqa_attend(oracle.norm_rope_rows(q, 3000, nrm.q_gamma, nrm),
                                oracle.norm_rope_rows(rows, pos, nrm.kv_gamma, nrm), 1 / math.sqrt(c))
    assert np.max(np.abs(o_plain - o)) > 1e-2


def test_weights_act_on_their_own_side():
    """A query weight of 2 doubles the logits only; a KV weight of 2 doubles the
    logits and the values."""
    rng = np.random.default_rng(6)
    c, sc = 512, 1 / math.sqrt(512)
    q, rows = rng.normal(size=(8, c)), rng.normal(size=(30, c))
    pos, t = np.arange(30) * 7, 250
    one = np.ones(c)
    base = oracle.attend_norm_rope(q, t, rows, pos, 2 * sc, _nrm(c, gq=one, gkv=one))
    # (a weight of 2 scales by a power of two: the bf16 operands scale exactly too)
    np.testing.assert_allclose(oracle.attend_norm_rope(q, t, rows, pos, sc, _nrm(c, gq=2 * one, gkv=one)),
                               base, atol=1e-12)
    np.testing.assert_allclose(oracle.attend_norm_rope(q, t, rows, pos, sc, _nrm(c, gq=one, gkv=2 * one)),
                               2 * base, atol=1e-12)


def test_without_rope_unit_weights_it_is_attention_over_unit_rms_rows():
    rng = np.random.default_rng(7)
    c = 64
    q, rows = rng.normal(size=(4, c)) * 5, rng.normal(size=(9, c)) * 0.1
    nrm = _nrm(c, rope_dims=0, eps=0.0, gq=np.ones(c), gkv=np.ones(c))
    unit = lambda z: z / (np.linalg.norm(z, axis=1, keepdims=True) / math.sqrt(c))  # noqa: E731
    want = oracle.mqa_attend(unit(q), unit(rows), 0.125)
    np.testing.assert_allclose(oracle.attend_norm_rope(q, 77, rows, np.arange(9), 0.125, nrm, bf16_operands=False),
                               want, atol=1e-12)
    # with bf16 operands: the same attention over the rounded unit-RMS rows
    want16 = oracle.mqa_attend(oracle.round_bf16(unit(q)), oracle.round_bf16(unit(rows)), 0.125)
    np.testing.assert_allclose(oracle.attend_norm_rope(q, 77, rows, np.arange(9), 0.125, nrm), want16, atol=1e-12)


# --------------------------------------------------------------------------
# the layers with normalisation: entry points agree with one another
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def tiny():
    d = wl.prefill_inputs(wl.TINY, T=256, seed=3)
    return {k: (v.float().numpy().astype(np.float64) if v.is_floating_point() else v.numpy()) for k, v in d.items()}


def test_layers_with_norm_cache_and_decode_agree(tiny):
    s = wl.TINY
    nrm = _nrm(s.c, np.random.default_rng(8), rope_dims=16)
    t = 255
    res = oracle.csa_layer_prefill(tiny["cand"], tiny["logits"], tiny["kidx_cand"], tiny["bias_csa"],
                                   tiny["q_idx"], tiny["w_idx"], tiny["q"], m=s.m, topk=s.topk // 2,
                                   d_idx=s.d_idx, n_win=s.n_win, scale=s.scale, queries=[3, t], norm=nrm)
    E_exact = oracle.csa_compress(tiny["cand"], tiny["logits"], tiny["bias_csa"], s.m)
    pos = (np.arange(E_exact.shape[0]) + 1) * s.m - 1
    np.testing.assert_array_equal(res["E"], oracle.round_bf16(oracle.norm_rope_rows(E_exact, pos, nrm.kv_gamma, nrm)))
    # the indexer is untouched by the normalisation
    plain = oracle.csa_layer_prefill(tiny["cand"], tiny["logits"], tiny["kidx_cand"], tiny["bias_csa"],
                                     tiny["q_idx"], tiny["w_idx"], tiny["q"], m=s.m, topk=s.topk // 2,
                                     d_idx=s.d_idx, n_win=s.n_win, scale=s.scale, queries=[t])
    assert res["idx"][t].tolist() == plain["idx"][t].tolist()
    win = tiny["cand"][t - s.n_win + 1:t + 1]
    dec = oracle.csa_layer_decode(res["E"], res["K_I"], win, tiny["q"][t], tiny["q_idx"][t], tiny["w_idx"][t], t,
                                  m=s.m, topk=s.topk // 2, n_win=s.n_win, scale=s.scale, norm=nrm)
    np.testing.assert_allclose(dec["O"], res["O"][t], atol=1e-13)
    # a reversed window now matters: the rows carry their positions
    rev = oracle.csa_layer_decode(res["E"], res["K_I"], win[::-1], tiny["q"][t], tiny["q_idx"][t],
                                  tiny["w_idx"][t], t, m=s.m, topk=s.topk // 2, n_win=s.n_win, scale=s.scale,
                                  norm=nrm)
    assert np.max(np.abs(rev["O"] - dec["O"])) > 1e-3
    hres = oracle.hca_layer_prefill(tiny["cand"], tiny["logits"], tiny["bias_hca"], tiny["q"], m_hca=s.m_hca,
                                    n_win=s.n_win, scale=s.scale, queries=[t], norm=nrm)
    hdec = oracle.hca_layer_decode(hres["E"], tiny["cand"][t - s.m_hca + 1:t + 1],
                                   tiny["logits"][t - s.m_hca + 1:t + 1], tiny["bias_hca"], win, tiny["q"][t], t,
                                   m_hca=s.m_hca, n_win=s.n_win, scale=s.scale, norm=nrm)
    np.testing.assert_array_equal(hdec["new_entry"], hres["E"][-1])
    np.testing.assert_allclose(hdec["O"], hres["O"][t], atol=1e-13)


def test_early_query_window_positions(tiny):
    """A query at t < n_win - 1 sees tokens 0..t: the decode window's first t+1 rows."""
    s = wl.TINY
    nrm = _nrm(s.c, np.random.default_rng(9), rope_dims=16)
    t = 9
    hres = oracle.hca_layer_prefill(tiny["cand"], tiny["logits"], tiny["bias_hca"], tiny["q"], m_hca=s.m_hca,
                                    n_win=s.n_win, scale=s.scale, queries=[t], norm=nrm)
    win = np.concatenate([tiny["cand"][:t + 1], np.full((s.n_win - t - 1, s.c), 1e3)])
    want = oracle.attend_norm_rope(tiny["q"][t], t, win[:t + 1], np.arange(t + 1), s.scale, nrm)
    np.testing.assert_allclose(hres["O"][t], want, atol=1e-13)
