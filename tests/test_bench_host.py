"""Host-side logic of bench.py, without a GPU: the clock summary taken from nvidia-smi samples
during the timed region (median SM clock, highest max clock, throttle reasons seen active) and
the whole-job rate of N replicas."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_clock_summary_median_max_and_active_reasons():
    lines = ["1965, 1965, 700.1, Not Active, Not Active, Not Active, Not Active",
             "1830, 1965, 998.0, Not Active, Not Active, Not Active, Active",
             "1900, 1965, 990.0, Not Active, Not Active, Not Active, Active",
             "garbage",
             "[N/A], 1965, 1.0, Not Active, Not Active, Not Active, Not Active"]
    assert bench.ClockSampler.summarize(lines) == {
        "sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_reports_slowdowns():
    lines = ["1500, 1965, 500, Active, Not Active, Active, Not Active",
             "1490, 1965, 510, Not Active, Active, Not Active, Not Active"]
    c = bench.ClockSampler.summarize(lines)
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert c["sm_mhz"] == pytest.approx(1495.0)


def test_clock_summary_without_samples():
    assert bench.ClockSampler.summarize([]) == {
        "sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_replica_rate_is_the_whole_job():
    assert bench.replica_rate(1, 4, 10.0) == pytest.approx(400.0)
    assert bench.replica_rate(8, 4, 10.0) == pytest.approx(3200.0)  # 8 replicas, the max time
