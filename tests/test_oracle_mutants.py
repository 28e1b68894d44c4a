"""Planted mistakes in the oracle are caught by its pins (CPU only).

Each case replaces one oracle function with a plausible wrong version -- a
rotation in the wrong sense or over the wrong channels, a forgotten output
rotation, a dropped weight or epsilon, an entry placed at its block's start,
ties rounded away from even, a shared exponent rounded up, ReLU after the head
sum, a dropped positional bias or swapped bias rows, a missing logit scale, a
transposed page address, visibility off by one, a window without the query's
own token, top-k ties to the higher index, a combine without its max
rescaling or with the sink counted per part -- and checks that at least one
of the named pins then fails.  The
mistakes live only in this test, patched into the oracle module for its
duration.
"""

import numpy as np
import pytest

import oracle
import oracle.hca as H
import test_oracle as T0
import test_oracle_fp4 as TF
import test_oracle_fp8 as T8
import test_oracle_norm_rope as TN
import test_oracle_paged as TP

_rope, _rms, _code, _w_csa = H.rope, H.rms_norm, H._e2m1_code, H.compress_weights_csa


def _rope_wrong_sense(x, pos, d, base):
    return _rope(x, -np.asarray(pos, dtype=np.float64), d, base)


def _rope_first_channels(x, pos, d, base):
    x = np.array(x, dtype=np.float64, copy=True)
    if d == 0:
        return x
    ang = np.asarray(pos, dtype=np.float64)[..., None] * H.rope_theta(d, base)
    a, b = x[..., 0:d:2].copy(), x[..., 1:d:2].copy()
    x[..., 0:d:2] = a * np.cos(ang) - b * np.sin(ang)
    x[..., 1:d:2] = a * np.sin(ang) + b * np.cos(ang)
    return x


def _attend_without_output_rotation(q, t, rows, row_pos, scale, nrm, sink=None, rows_ready=None, bf16_operands=True):
    qn = H.norm_rope_rows(q, t, nrm.q_gamma, nrm)
    kv = H.norm_rope_rows(rows, np.asarray(row_pos), nrm.kv_gamma, nrm)
    if rows_ready is not None:
        kv = np.concatenate([np.asarray(rows_ready, dtype=np.float64), kv], axis=0)
    return H.mqa_attend(qn, kv, scale, sink)


def _rms_without_gamma(x, gamma, eps):
    return _rms(x, np.ones_like(np.asarray(gamma, dtype=np.float64)), eps)


def _rms_without_eps(x, gamma, eps):
    return _rms(x, gamma, 0.0)


def _entry_at_block_start(i, rate):
    return np.asarray(i) * rate


def _e2m1_ties_away(y):
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), 6.0)
    g = H.E2M1_GRID
    hi = np.searchsorted(g, a, side="left").clip(0, 7)
    lo = (hi - 1).clip(0, 7)
    mag = np.where(g[hi] - a <= a - g[lo], hi, lo)
    return (mag + 8 * ((y < 0) & (mag != 0))).astype(np.uint8)


def _mx_quantize_ceil(x):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    xb = x.reshape(x.shape[:-1] + (d // 32, 32))
    amax = np.max(np.abs(xb), axis=-1)
    X = np.clip(np.where(amax > 0, np.ceil(np.log2(np.where(amax > 0, amax, 1.0))) - 2, -127.0), -127, 127)
    codes = _code(xb / np.exp2(X)[..., None])
    return codes.reshape(x.shape).astype(np.uint8), (X + 127).astype(np.uint8)


def _indexer_relu_after_sum(q_idx, w_idx, k_idx):
    dots = np.asarray(k_idx, dtype=np.float64) @ np.asarray(q_idx, dtype=np.float64).T
    return np.maximum(dots @ np.asarray(w_idx, dtype=np.float64), 0.0)


def _weights_without_bias(logits, pos_bias, m, i):
    return _w_csa(logits, np.zeros_like(np.asarray(pos_bias, dtype=np.float64)), m, i)


_mqa_partial = H.mqa_partial


def _e4m3_ties_away(y):
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), H.E4M3_MAX)
    e = np.maximum(np.where(a > 0, np.floor(np.log2(np.where(a > 0, a, 1.0))), -6.0), -6.0)
    step = np.exp2(e - 3.0)
    r = np.floor(a / step + 0.5) * step
    return np.where(y < 0, -r, r)


def _paged_rows_transposed(pool, block_table, idx, rows_per_block):
    idx = np.asarray(idx, dtype=np.int64)
    bt = np.asarray(block_table, dtype=np.int64)
    return np.asarray(pool, dtype=np.float64)[bt[idx % rows_per_block], idx // rows_per_block]


_nvis, _wrows, _topk, _comb, _win = H.n_visible, H.window_rows, H.topk_select, H.combine_partials, H._csa_window


def _n_visible_off_by_one(t, rate, n_entries):
    return int(min(n_entries, t // rate))


def _window_without_t(t, n_win):
    return np.arange(max(0, t - n_win), t)


def _topk_ties_to_higher_index(scores, k):
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    return np.lexsort((-np.arange(n), -scores))[:min(k, n)].astype(np.int64)


def _combine_without_rescale(parts, sink=None):
    num = sum(p[2] for p in parts)
    den = sum(p[1] for p in parts)
    return num / den[:, None]


def _combine_sink_per_part(parts, sink=None):
    if sink is None:
        return _comb(parts)
    ms = np.stack([p[0] for p in parts])
    M = np.max(ms, axis=0)
    z = np.asarray(sink, dtype=np.float64)
    num = sum(np.exp(p[0] - M)[:, None] * p[2] for p in parts)
    den = sum(np.exp(p[0] - M) * p[1] + np.exp(z - M) for p in parts)
    return num / den[:, None]


def _csa_window_bias_swapped(i, m, T):
    lo, hi, b0 = _win(i, m, T)
    return lo, hi, (m - b0) if i > 0 else b0


CASES = {
    "visibility off by one": ({"n_visible": _n_visible_off_by_one},
                              [T0.test_golden_visibility_and_window, T0.test_visibility_brute_force]),
    "window misses the query's token": ({"window_rows": _window_without_t}, [T0.test_golden_visibility_and_window]),
    "top-k ties to the higher index": ({"topk_select": _topk_ties_to_higher_index}, [T0.test_golden_topk_ties]),
    "combine without max rescaling": ({"combine_partials": _combine_without_rescale},
                                      [lambda: T0.test_split_combine_equals_unsplit([13, 29])]),
    "sink counted once per part": ({"combine_partials": _combine_sink_per_part},
                                   [lambda: T0.test_sink_split_combine_equals_unsplit([13, 29])]),
    "CSA bias rows swapped": ({"_csa_window": _csa_window_bias_swapped},
                              [T0.test_golden_csa_overlap, T0.test_csa_previous_block_bias_rows]),
    "rope turns the wrong way": ({"rope": _rope_wrong_sense}, [TN.test_rope_hand_worked]),
    "rope on the first channels": ({"rope": _rope_first_channels},
                                   [TN.test_rope_hand_worked, TN.test_rope_is_a_rotation_group]),
    "no output rotation": ({"attend_norm_rope": _attend_without_output_rotation},
                           [TN.test_one_row_attention_is_the_row_turned_by_the_offset,
                            TN.test_output_depends_only_on_relative_positions]),
    "RMSNorm without its weights": ({"rms_norm": _rms_without_gamma}, [TN.test_rms_norm_hand_worked]),
    "RMSNorm without eps": ({"rms_norm": _rms_without_eps}, [TN.test_rms_norm_hand_worked]),
    "entry at its block's start": ({"entry_position": _entry_at_block_start},
                                   [TN.test_entry_position_matches_causal_visibility]),
    "E2M1 ties away from even": ({"_e2m1_code": _e2m1_ties_away},
                                 [lambda: TF.test_mxfp4_hand_worked("mxfp4_block")]),
    "shared exponent rounded up": ({"mxfp4_quantize": _mx_quantize_ceil},
                                   [lambda: TF.test_mxfp4_hand_worked("mxfp4_block"),
                                    TF.test_mxfp4_idempotent_and_error_bound]),
    "ReLU after the head sum": ({"indexer_scores": _indexer_relu_after_sum}, [T0.test_indexer_relu_is_per_head]),
    "no positional bias": ({"compress_weights_csa": _weights_without_bias}, [T0.test_csa_previous_block_bias_rows]),
    "no logit scale": ({"mqa_partial": lambda q, rows, scale: _mqa_partial(q, rows, 1.0)},
                       [T0.test_attention_two_rows_sigmoid]),
    "E4M3 ties away from even": ({"round_e4m3": _e4m3_ties_away}, [T8.test_hand_worked_ties_and_saturation]),
    "page address transposed": ({"paged_rows": _paged_rows_transposed}, [TP.test_paged_rows_identity_and_permuted]),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_planted_mistake_is_caught(monkeypatch, case):
    patches, pins = CASES[case]
    for name, fn in patches.items():
        monkeypatch.setattr(H, name, fn)
        if hasattr(oracle, name):
            monkeypatch.setattr(oracle, name, fn)
    caught = 0
    for pin in pins:
        try:
            pin()
        except Exception:  # a failed assertion, or a pin the mistake crashes (all pass unpatched: below)
            caught += 1
    assert caught > 0, f"no pin catches: {case}"


def test_pins_pass_on_the_oracle_itself():
    for _, pins in CASES.values():
        for pin in pins:
            pin()
