"""Host logic of bench.py that needs no GPU: the clock-sample summary (median SM clock,
throttle reasons) and the lookup of the committed DRAM-traffic figures."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_clock_summary_median_max_and_reasons():
    lines = [
        "1965, 1965, 812.3, Not Active, Not Active, Not Active, Not Active\n",
        "1942, 1965, 998.0, Not Active, Not Active, Not Active, Active\n",
        "1950, 1965, 1001.2, Not Active, Not Active, Not Active, Active\n",
        "19",                                              # partial last line: skipped
        "[N/A], 1965, 0, Not Active, Not Active, Not Active, Not Active\n",   # unparsable: skipped
    ]
    c = bench.ClockSampler.summarize(lines)
    assert c == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_reports_every_rejecting_reason_and_no_samples():
    lines = ["1200, 1965, 700, Active, Not Active, Active, Not Active\n"]
    c = bench.ClockSampler.summarize(lines)
    assert c["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"] and c["samples"] == 1
    assert bench.ClockSampler.summarize([]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_traffic_lookup_matches_the_committed_figures():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    assert bench.traffic_for("gemm_blockwise", "llama8b") == d["llama8b"]["gemm_blockwise"]
    assert bench.traffic_for("gemm_blockwise", "moe") is None      # no capture for that workload
    assert bench.traffic_for("quantize", "llama8b") is None
