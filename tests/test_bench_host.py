"""bench.py's host-side rules (no GPU): which clock records force a re-measurement."""

import bench


def test_clock_rejection_rules():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 30}
    assert not bench.clock_rejected(ok)
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clock_rejected(dict(ok, reasons=[r]))
    # the power cap under a dense kernel is normal on a 1 kW part: kept
    assert not bench.clock_rejected(dict(ok, sm_mhz=1300.0, reasons=["sw_power_cap"]))
    # clocks far below the maximum with no reason: a leftover clock lock
    assert bench.clock_rejected(dict(ok, sm_mhz=1000.0))
    # no sampler (no nvidia-smi): nothing to judge by
    assert not bench.clock_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0})
