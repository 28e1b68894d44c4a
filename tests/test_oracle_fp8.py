"""Pins of the oracle's FP8 (E4M3) storage of the non-rotated KV channels.

"DeepSeek V4 Architecture Tricks", "Partial RoPE 和 Attention Sink": the RoPE
channels stay BF16 in the KV cache, the other KV channels use FP8.  The pins
decode every E4M3 code from the format's definition (sign, 4 exponent bits
with bias 7, 3 mantissa bits, exponent field 0 = subnormal, S.1111.111 = NaN)
and check the oracle's rounding against a brute-force nearest-grid search, plus
hand-worked ties, saturation, the per-group scale and the BF16 rope part.
"""

import numpy as np
import pytest

import oracle


def _e4m3_grid():
    """(value, code) of every finite E4M3 code, decoded from the format definition."""
    out = []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue  # NaN
        v = (m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        out.append((-v if s else v, code))
    return out


GRID = _e4m3_grid()
VALUES = np.array(sorted({v for v, _ in GRID}))


def test_grid_is_fixed_by_rounding():
    assert len(GRID) == 254 and VALUES.max() == 448.0 and VALUES[VALUES > 0].min() == 2.0 ** -9
    np.testing.assert_array_equal(oracle.round_e4m3(VALUES), VALUES)


def test_rounding_matches_brute_force_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(size=4000) * 10.0 ** rng.uniform(-3, 2.5, size=4000),
                        (VALUES[:-1] + VALUES[1:]) / 2])          # every midpoint, exactly
    x = x[np.abs(x) <= 448]
    codes = {v: c for v, c in GRID if not (v == 0 and c == 128)}  # +0 for zero
    got = oracle.round_e4m3(x)
    for xi, gi in zip(x, got):
        d = np.abs(VALUES - xi)
        cand = VALUES[d == d.min()]
        if len(cand) == 1:
            want = cand[0]
        else:  # a tie: the code with an even mantissa
            want = [v for v in cand if codes[v] % 2 == 0][0]
        assert gi == want, (xi, gi, want)


def test_hand_worked_ties_and_saturation():
    x = np.array([1.0625, 1.1875, -17.0, 232.0, 500.0, -1e9, 1.5 * 2 ** -9, 2.0 ** -10])
    want = [1.0, 1.25, -16.0, 224.0, 448.0, -448.0, 2.0 ** -8, 0.0]
    np.testing.assert_array_equal(oracle.round_e4m3(x), want)


def test_fp8_kv_rows():
    rng = np.random.default_rng(1)
    rows = rng.normal(size=(6, 512)) * rng.uniform(0.01, 10, size=(6, 1))
    codes, scales, rope = oracle.fp8_kv_quantize(rows, 64)
    assert codes.shape == (6, 448) and scales.shape == (6, 7) and rope.shape == (6, 64)
    np.testing.assert_array_equal(rope, oracle.round_bf16(rows[:, 448:]))
    np.testing.assert_array_equal(oracle.round_e4m3(codes), codes)          # on the grid
    assert np.all(np.abs(codes) <= 448) and np.all(np.max(np.abs(codes).reshape(6, 7, 64), -1) == 448)
    y = oracle.fp8_kv_dequantize(codes, scales, rope)
    body = rows[:, :448].reshape(6, 7, 64)
    err = np.abs(y[:, :448].reshape(6, 7, 64) - body)
    # half an E4M3 step at each value's magnitude (relative 2^-4), in units of the group's scale
    assert np.all(err <= np.abs(body) * 2.0 ** -4 + scales[..., None] * 2.0 ** -10)
    # a power-of-two scaling of a row moves only its scales
    c2, s2, _ = oracle.fp8_kv_quantize(rows * 2.0 ** 5, 64)
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(s2, scales * 32)


def test_all_zero_group_keeps_unit_scale():
    rows = np.zeros((1, 128))
    rows[0, 64:] = 3.0
    codes, scales, _ = oracle.fp8_kv_quantize(rows, 0)
    assert scales.tolist() == [[1.0, float(np.float32(3.0 / 448))]] and np.all(codes[0, :64] == 0)  # f32 scales
