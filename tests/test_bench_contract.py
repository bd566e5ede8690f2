"""The benchmark's output contract, checked on the CPU: the reference arm
(the fp64 oracle on bounded samples) prints one JSON line with every key the
line must carry; the peak used for the roofline follows the sampled clocks;
every workload names itself and counts its FLOPs.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


@pytest.mark.parametrize("workload", ["tiny", "fp8_128"])
def test_reference_arm_line(workload):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", workload,
                        "--steps", "1", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    # the oracle's forward and backward seconds per (batch, head), and the whole workload extrapolated
    assert cb["fwd_s_per_head"] > 0 and cb["extrapolated_full_workload_s"] > cb["fwd_s_per_head"]
    assert (cb["bwd_s_per_head"] is None) == (not bench.WORKLOADS[workload]["bwd"])
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith(workload)


def test_peak_follows_the_sampled_clock():
    full = {"sm_mhz": 1965.0, "sm_min_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    dropped = {"sm_mhz": 1600.0, "sm_min_mhz": 1550.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert not bench.power_capped(full)      # the flag alone keeps the burst peak
    assert bench.power_capped(dropped)       # a clock below 95 % of max selects the sustained one
    assert not bench.power_capped(None)
    assert not bench.power_capped({"sm_mhz": None})


@pytest.mark.parametrize("name", sorted(bench.WORKLOADS))
def test_every_workload_describes_itself_and_counts_flops(name):
    w = bench.WORKLOADS[name]
    assert bench.describe(name, w).startswith(name + ":")
    kept = 52834 if w["sparse"] else None
    fwd, bwd = bench.workload_flops(w, kept)
    assert fwd > 0
    assert bwd == (2.5 * fwd if w["bwd"] else 0.0)
