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


def test_clock_sampler_keeps_its_first_sample():
    """The sampler's first line (read before the timed region starts) is one of the
    samples: a short region must not come out with none."""
    first = "0, 1965, 1965, 300.5, 0x0, Not Active, Not Active, Not Active, Not Active\n"
    rest = "0, 1950, 1965, 640.1, 0x0, Not Active, Not Active, Not Active, Active\n"
    rows = bench.parse_clock_rows(first + rest)
    assert len(rows) == 2 and rows[0][1] == "1965"
    s = bench.ClockSampler(0)
    s.rows = rows
    summ = s.summary()
    assert summ["samples"] == 2 and summ["sm_mhz"] == 1957.5 and summ["reasons"] == ["sw_power_cap"]
