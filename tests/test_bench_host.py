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


def test_captured_traffic_only_for_the_captured_sources(tmp_path, monkeypatch):
    """The bench reports a committed capture's DRAM bytes only while the kernel's sources
    hash to the value recorded with the capture; otherwise (or with no capture) null."""
    import hashlib
    import json
    csrc = tmp_path / "long_context_doc_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cu").write_text("kernel one\n")
    (csrc / "c.cuh").write_text("common\n")
    sha = hashlib.sha256(b"kernel one\n" + b"common\n").hexdigest()
    rec = {"kernel_src_sha256": sha, "dram_bytes_read": 1000, "dram_bytes_write": 24}
    (tmp_path / "profiles" / "cap.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic(("k.cu", "c.cuh"), "cap.json") == 1024
    assert bench.captured_traffic(("c.cuh", "k.cu"), "cap.json") is None  # order is part of it
    (csrc / "k.cu").write_text("kernel two\n")
    assert bench.captured_traffic(("k.cu", "c.cuh"), "cap.json") is None
    assert bench.captured_traffic(("k.cu",), "missing.json") is None


def test_committed_captures_name_their_sources():
    import json
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        if name.endswith("_dram.json"):
            with open(os.path.join(ROOT, "profiles", name)) as f:
                rec = json.load(f)
            assert len(rec["kernel_src_sha256"]) == 64, name
            assert int(rec["dram_bytes_read"]) > 0 and int(rec["dram_bytes_write"]) >= 0, name
