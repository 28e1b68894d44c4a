"""Pins of the oracle's FP4 indexer variant (MXFP4 quantisation, BF16 scores).

"DeepSeek V4 Architecture Tricks", "FP4 / FP8 Quantization-Aware Training":
the indexer's QK activations are cached, loaded and multiplied in FP4, the
index scores drop from FP32 to BF16, and FP4 values dequantise losslessly into
FP8 because FP8's exponent range absorbs the fine-grained scale.  The pins:
hand-worked blocks, the E2M1 grid, idempotence, the rounding-error bound,
exact absorption of power-of-two scalings (the property the lossless-FP8
remark rests on, checked against an E4M3 representability test), the nibble
order of the packed cache, and the BF16 scores.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))


def _block(g):
    x = np.zeros(g["pad_zeros_to"])
    x[:len(g["x"])] = g["x"]
    return x


@pytest.mark.parametrize("name", ["mxfp4_block", "mxfp4_small_block"])
def test_mxfp4_hand_worked(name):
    g = GOLD[name]
    codes, scales = oracle.mxfp4_quantize(_block(g)[None])
    assert int(scales[0, 0]) == g["scale_byte"]
    if "codes" in g:
        assert codes[0, :len(g["codes"])].tolist() == g["codes"]
    vals = oracle.mxfp4_dequantize(codes, scales)[0]
    np.testing.assert_array_equal(vals[:len(g["values"])], g["values"])
    assert np.all(vals[len(g["values"]):] == 0)


def test_e2m1_codes_and_grid():
    v = oracle.e2m1_value(np.arange(16))
    np.testing.assert_array_equal(v[:8], [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(v[8:], -v[:8])
    # a block holding every grid value (amax 6 -> scale 2^0) is stored exactly
    x = np.concatenate([v, v])[None]
    c, s = oracle.mxfp4_quantize(x)
    assert int(s[0, 0]) == 127
    np.testing.assert_array_equal(oracle.mxfp4_dequantize(c, s), x)


def test_mxfp4_idempotent_and_error_bound():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(50, 128)) * rng.uniform(1e-3, 1e3, size=(50, 1))
    c, s = oracle.mxfp4_quantize(x)
    y = oracle.mxfp4_dequantize(c, s)
    c2, s2 = oracle.mxfp4_quantize(y)
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_array_equal(s2, s)
    # |x - y| <= half the grid spacing at |x| / 2^X: 0.25 below 2, 0.5 below 4, 1 up to 6;
    # beyond 6 (saturation) the error is |x| - 6 2^X
    X = np.repeat(s.astype(np.float64) - 127, 32, axis=-1)
    a = np.abs(x) / np.exp2(X)
    half = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))
    bound = np.where(a <= 6, half, a - 6) * np.exp2(X)
    assert np.all(np.abs(x - y) <= bound * (1 + 1e-12))
    # every block's amax lands in [4, 8) after scaling
    amax = np.max(a.reshape(50, 4, 32), axis=-1)
    assert np.all((amax >= 4) & (amax < 8))


def test_power_of_two_scaling_is_absorbed_exactly():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(8, 64))
    c, s = oracle.mxfp4_quantize(x)
    for k in (-20, -3, 5, 40):
        ck, sk = oracle.mxfp4_quantize(x * 2.0 ** k)
        np.testing.assert_array_equal(ck, c)
        np.testing.assert_array_equal(sk.astype(int), s.astype(int) + k)


def _e4m3_exact(v: float) -> bool:
    """Is v exactly an FP8 E4M3 value (3 mantissa bits, normal exponents -6..8,
    subnormals down to 2^-9, max 448)?"""
    if v == 0:
        return True
    a = abs(v)
    if a > 448:
        return False
    e = max(math.floor(math.log2(a)), -6)
    q = a / 2.0 ** (e - 3)   # mantissa in units of the last bit
    return q == math.floor(q)


def test_fp4_values_dequantise_losslessly_into_fp8_for_moderate_scales():
    """The pages' lossless FP4 -> FP8 remark holds for MXFP4 values whose
    power-of-two scale keeps them in E4M3's range: every E2M1 value times 2^X,
    X in [-8, 6], is an exact E4M3 value."""
    grid = oracle.e2m1_value(np.arange(16))
    for X in range(-8, 7):
        for g in grid:
            assert _e4m3_exact(g * 2.0 ** X), (g, X)
    # ... and a scale that is not a power of two would not be absorbed
    assert not _e4m3_exact(1.5 * 1.3)


def test_pack_nibble_order_and_round_trip():
    codes = np.array([[1, 2, 15, 8]], dtype=np.uint8)
    packed = oracle.mxfp4_pack(codes)
    assert packed.tolist() == [[0x21, 0x8F]]
    rng = np.random.default_rng(2)
    c = rng.integers(0, 16, size=(5, 128)).astype(np.uint8)
    np.testing.assert_array_equal(oracle.mxfp4_unpack(oracle.mxfp4_pack(c)), c)


def test_fp4_scores_are_bf16_and_exact_for_representable_inputs():
    rng = np.random.default_rng(3)
    H, d, N = 8, 128, 40
    # inputs already on the MXFP4 grid: quantisation changes nothing
    q = oracle.mxfp4_dequantize(*oracle.mxfp4_quantize(rng.normal(size=(H, d))))
    k = oracle.mxfp4_dequantize(*oracle.mxfp4_quantize(rng.normal(size=(N, d))))
    w = rng.uniform(size=H)
    sc = oracle.indexer_scores_fp4(q, w, k)
    np.testing.assert_array_equal(sc, oracle.round_bf16(sc))
    np.testing.assert_array_equal(sc, oracle.round_bf16(oracle.indexer_scores(q, w, k)))


def test_recall():
    assert oracle.topk_recall(np.array([1, 2, 3]), np.array([3, 2, 9, 8])) == 0.5
    assert oracle.topk_recall(np.array([]), np.array([])) == 1.0
    # FP4 scores keep most of the FP32 selection on random inputs (a sanity bound, not the pages' figure)
    rng = np.random.default_rng(4)
    q, w, k = rng.normal(size=(64, 128)), rng.uniform(size=64), rng.normal(size=(4096, 128))
    ref = oracle.topk_select(oracle.indexer_scores(q, w, k), 256)
    got = oracle.topk_select(oracle.indexer_scores_fp4(q, w, k), 256)
    assert oracle.topk_recall(got, ref) > 0.5
