"""Helpers shared by the GPU parity tests: tensor conversion and the
acceptance rules.

Acceptance (floating point): bf16 inputs, f32 accumulation; an output
passes when max|gpu - oracle| / rms(oracle) <= 2e-2 over the compared
elements.  Compressor outputs get a stricter element-wise bound: the GPU's
bf16 value is within 2^-8 relative (one bf16 rounding of the f32 result plus
f32 arithmetic error) of the float64 oracle value.

Acceptance (top-k): the GPU's set has exactly min(k, n_visible) distinct,
visible entries (the rest -1); where it differs from the oracle's set, every
differing entry's oracle score lies within 1e-3 relative of the oracle's
k-th score (a near-tie that f32 accumulation may order either way).
"""

import numpy as np
import oracle
import torch

NORM_TOL = 2e-2
TOPK_BAND = 1e-3


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def to_dev(d, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def norm_err(gpu, ref) -> float:
    """max |gpu - ref| / rms(ref), each query normalised by its own output RMS.

    Arrays [Tq, H, c] (or [H, c] for one query): every query is its own
    attention problem, so its error is measured against its own output
    scale.  (One RMS over all queries would let the bf16 rounding of a query
    whose attention sits on a single row -- output values several times the
    global RMS -- exceed the tolerance by itself.)"""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.ndim < 3:
        gpu, ref = gpu[None], ref[None]
    ax = tuple(range(1, ref.ndim))
    rms = np.sqrt(np.mean(ref ** 2, axis=ax))
    err = np.max(np.abs(gpu - ref), axis=ax)
    return float(np.max(err / np.maximum(rms, 1e-30)))


def _per_query_norm_err(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.ndim < 3:
        gpu, ref = gpu[None], ref[None]
    ax = tuple(range(1, ref.ndim))
    rms = np.maximum(np.sqrt(np.mean(ref ** 2, axis=ax)), 1e-30)
    return np.max(np.abs(gpu - ref), axis=ax) / rms, ref, rms, ax


def assert_norm_close(gpu, ref, tol=NORM_TOL, what=""):
    """Per-query normalised max-abs error within `tol`, or -- for a query whose
    exact output cannot be stored in bf16 within `tol` at all -- within 1.5x the
    error of the correctly rounded exact output (the best any bf16 result can
    reach, plus room for the f32 accumulation).  That floor only matters for
    queries with few rows and a heavy-tailed output (short prefills), where one
    value many times the query's RMS carries a rounding error near 2^-9 of
    itself."""
    err, ref64, rms, ax = _per_query_norm_err(gpu, ref)
    floor = np.max(np.abs(oracle.round_bf16(ref64) - ref64), axis=ax) / rms
    bar = np.maximum(tol, 1.5 * floor)
    bad = np.nonzero(err > bar)[0]
    assert bad.size == 0, (f"{what}: normalised max-abs error {err[bad[0]]:.3e} > {bar[bad[0]]:.3e} "
                           f"at query {bad[0]} ({bad.size} queries over the bar)")
    return float(np.max(err))


def assert_norm_close_per_head(gpu, ref, tol=NORM_TOL, what=""):
    """max |gpu - ref| / rms(ref) over the c outputs of each (query, head).

    With attention-sink logits every head has its own output scale (the sink
    takes anything from none to nearly all of a head's mass), so one RMS per
    query would be set by its largest heads and the bf16 rounding of their
    largest elements alone could pass the bar; each head is held to its own."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    e = float(np.max(np.abs(gpu - ref) / np.maximum(rms, 1e-300)))
    assert e <= tol, f"{what}: per-head normalised max-abs error {e:.3e} > {tol}"
    return e


def assert_bf16_close(gpu, ref64, what=""):
    """gpu (bf16 values) within one bf16 rounding (half an ulp <= 2^-8 relative)
    of the unrounded float64 reference, plus f32 arithmetic slack."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref64 = np.asarray(ref64, dtype=np.float64)
    rms = np.sqrt(np.mean(ref64 ** 2)) if ref64.size else 0.0
    bound = 2.0 ** -8 * np.abs(ref64) + 2.0 ** -20 * rms
    excess = np.abs(gpu - ref64) - bound
    worst = float(np.max(excess)) if excess.size else -1.0
    assert worst <= 0.0, f"{what}: error exceeds one bf16 rounding by {worst:.3e}"
    return worst


def assert_bf16_ulps(a, b, ulps=1, what="", rms_slack=2.0 ** -20):
    """Two bf16-valued arrays agree to within `ulps` bf16 ulps element-wise, plus
    `rms_slack` times the RMS of b (for elements that come out of cancellation)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    rms = np.sqrt(np.mean(b ** 2)) if b.size else 0.0
    bound = ulps * 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + rms_slack * rms
    bad = np.abs(a - b) > bound
    assert not np.any(bad), f"{what}: {int(bad.sum())} elements differ by more than {ulps} bf16 ulp"


def check_topk_row(gpu_row, oracle_sel, oracle_scores, k, nvis, band=TOPK_BAND):
    """Returns the number of near-tie swaps; raises AssertionError on failure."""
    gpu_row = np.asarray(gpu_row)
    g = gpu_row[gpu_row >= 0]
    want = min(k, nvis)
    assert len(g) == want, f"selected {len(g)} entries, expected {want}"
    assert np.all(gpu_row[gpu_row < 0] == -1)
    assert len(np.unique(g)) == len(g), "duplicate entries"
    assert np.all((g >= 0) & (g < nvis)), "entry not visible"
    gs, os_ = set(g.tolist()), set(np.asarray(oracle_sel).tolist())
    if nvis <= k:
        assert gs == set(range(nvis))
        return 0
    diff = gs ^ os_
    if not diff:
        return 0
    kth = oracle_scores[oracle_sel[-1]]
    tol = band * abs(kth)
    bad = [s for s in diff if abs(oracle_scores[s] - kth) > tol]
    assert not bad, f"entries {bad[:5]} differ from the oracle outside the near-tie band (k-th score {kth})"
    return len(diff) // 2
