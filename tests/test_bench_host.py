"""Host logic of bench.py that needs no GPU: the clock record of a timed
region and the rule that rules a number out, the committed figures the
roofline line reads (DRAM traffic per launch, measured peaks), and the JSON
line of the reference arm (the CPU oracle)."""
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
    """The committed ratio is the captured bytes over the algorithmic bytes
    of the captured launches, within a few per cent of 1, and the bench
    scales it by a launch's algorithmic bytes."""
    with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
        committed = json.load(f)
    for kernel, entry in committed.items():
        cap = sum(entry["captured_bytes"].values()) / len(entry["captured_bytes"])
        alg = sum(entry["algorithmic_bytes"].values()) / len(entry["algorithmic_bytes"])
        assert abs(entry["dram_over_algorithmic"] - cap / alg) < 0.02
        assert 0.9 < entry["dram_over_algorithmic"] < 1.1
        assert bench.load_traffic(kernel, 27678622) == round(entry["dram_over_algorithmic"] * 27678622)
    assert bench.load_traffic("no_such_kernel", 1000) is None


def test_peaks_are_the_measured_ones_when_present():
    p = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert p["source"] == "measured"
        assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    else:
        assert p["source"] == "fallback"


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """`bench.py --impl reference` prints one JSON line with the keys of the
    benchmark line.  The oracle's timing is replaced by a fixed sample here;
    the line's layout is what is checked."""
    calls = []

    def fake_sample(budget_s=12.0):
        calls.append(budget_s)
        return 1.25, 8, "21 Linears of the decode step, 2.0 s of CPU time"

    monkeypatch.setattr(bench, "oracle_decode_sample", fake_sample)
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    args = bench.argparse.Namespace(gpus=1, steps=4, warmup=3, impl="reference")
    bench.run_reference(args)
    line = capsys.readouterr().out.strip().splitlines()
    assert len(line) == 1
    out = json.loads(line[0])
    assert len(calls) == 7  # warm-up and timed steps
    assert out["impl"] == "reference" and out["value"] == 1.25 and out["steps"] == 4 and out["warmup"] == 3
    for key in ("metric", "unit", "n_gpus", "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in out
    assert out["cpu_baseline"] == {"value": 1.25, "unit": "GB/s", "cores": 8, "kind": "oracle",
                                   "sample": "21 Linears of the decode step, 2.0 s of CPU time"}
    assert out["e2e"] == {"value": 1.25, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in out["config"]


def test_reference_arm_is_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setattr(bench, "oracle_decode_sample", lambda budget_s=12.0: pytest.fail("rank 1 ran the oracle"))
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(bench.argparse.Namespace(gpus=2, steps=2, warmup=3, impl="reference"))
    assert capsys.readouterr().out == ""
