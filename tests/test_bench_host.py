"""Host logic of bench.py that needs no GPU: the clock record of a timed
region and the rule that rules a number out, and the committed figures the
roofline line reads (DRAM traffic per launch, measured peaks)."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def sampler_with(lines):
    c = bench.ClockSampler(0)
    c.lines = list(lines)
    return c


# nvidia-smi --format=csv,noheader,nounits rows of ClockSampler.QUERY:
# index, clocks.sm, clocks.max.sm, power.draw, active mask, then the
# hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap flags.
CALM = "0, 1965, 1965, 640.2, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"
CAPPED = "0, 1335, 1965, 995.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active"
HOT = "0, 1500, 1965, 900.0, 0x0000000000000040, Not Active, Not Active, Active, Not Active"
LOCKED = "0, 1000, 1965, 400.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"


def test_summary_takes_the_median_clock_and_the_reasons_seen():
    s = sampler_with([CALM, CALM, CAPPED, "garbage", ""]).summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1965.0
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_summary_of_no_samples():
    s = sampler_with([]).summary()
    assert s == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    assert not bench.clocks_disqualify(s)


@pytest.mark.parametrize("lines,out", [
    ([CALM] * 5, False),                 # full clock, nothing active
    ([CAPPED] * 5, False),               # power capping is kept and noted
    ([CALM, HOT, CALM], True),           # a thermal slowdown in the region
    ([LOCKED] * 5, True),                # far below max with no reason: a clock lock
    ([LOCKED, LOCKED, CAPPED], False),   # low, but the power cap explains it
])
def test_clocks_disqualify(lines, out):
    assert bench.clocks_disqualify(sampler_with(lines).summary()) is out


def test_hardware_slowdown_disqualifies_whatever_the_clock():
    s = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown"], "samples": 4}
    assert bench.clocks_disqualify(s)


def test_traffic_figures_come_from_the_committed_summary():
    with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
        committed = json.load(f)
    for kernel, entry in committed.items():
        got = bench.load_traffic(kernel)
        assert got == entry["dram_bytes_per_launch"]
        # measured traffic is within a few per cent of the algorithmic bytes
        assert 0.8 < got / entry["algorithmic_bytes_per_launch"] < 1.1
    assert bench.load_traffic("no_such_kernel") is None


def test_peaks_are_the_measured_ones_when_present():
    p = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert p["source"] == "measured"
        assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    else:
        assert p["source"] == "fallback"
