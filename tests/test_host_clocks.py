"""The clock record of the bench line (no GPU): bench.ClockSampler.summarize
turns nvidia-smi samples (index, clocks.sm, clocks.max.sm, power.draw, active
reasons, hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap)
into the median busy SM clock, the maximum clock and the throttle reasons seen,
which decide whether a run is kept (hw_slowdown, hw_thermal_slowdown and
sw_thermal_slowdown reject it; sw_power_cap is kept and noted)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def line(sm, mx=1965, hw="Not Active", hwt="Not Active", swt="Not Active", cap="Not Active"):
    return "0, %s, %s, 900.00, 0x0000000000000004, %s, %s, %s, %s" % (sm, mx, hw, hwt, swt, cap)


def test_median_of_busy_samples_and_reasons():
    lines = [line(345), line(1950), line(1920, cap="Active"), line(1935), line(210)]
    rec = bench.ClockSampler.summarize(lines)
    # the idle samples (below half the maximum clock) do not pull the median down
    assert rec == {"sm_mhz": 1935.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 5}


def test_every_reason_seen_active_is_reported():
    lines = [line(1900, hw="Active"), line(1900, hwt="Active"), line(1900, swt="Active")]
    rec = bench.ClockSampler.summarize(lines)
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_unusable_samples():
    assert bench.ClockSampler.summarize([]) is None
    assert bench.ClockSampler.summarize(["0, [N/A], 1965, 1, 0, a, b, c, d", "garbage"]) is None
    # a short or malformed line is skipped, the rest is used
    rec = bench.ClockSampler.summarize(["0, 1900", line(1800), "0, x, 1965, 1, 0, a, b, c, d"])
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1800.0


def test_all_idle_samples_still_give_a_clock():
    rec = bench.ClockSampler.summarize([line(300), line(500)])
    assert rec["sm_mhz"] == 400.0 and rec["samples"] == 2
