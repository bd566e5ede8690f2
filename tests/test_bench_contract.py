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


def _prof(**ms_per_launch):
    # {kind: (ms summed over 10 steps, launches)} as the library reports it
    kinds = ("fwd", "bwd_pre", "bwd_main", "bwd_post", "bwd_dq", "fp8_quant", "fwd_fp8")
    launches = {"fp8_quant": 30}
    return {k: (ms_per_launch.get(k, 0.0) * launches.get(k, 10), launches.get(k, 10) if k in ms_per_launch else 0)
            for k in kinds}


FULL_CLOCK = {"sm_mhz": 1965.0, "sm_min_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}


def test_analyse_the_dsweep128_step():
    # per-launch times of the d = 128 sweep on one B200: forward 0.289 ms, backward main 0.772 ms
    w = bench.WORKLOADS["dsweep128"]
    fwd_f, bwd_f = bench.workload_flops(w)
    prof = _prof(fwd=0.289, bwd_pre=0.03, bwd_main=0.772, bwd_post=0.02)
    roof, kernels, split = bench.analyse(prof, w, "dsweep128", fwd_f, bwd_f, FULL_CLOCK, 10)
    burst = bench.peaks()[0]
    assert roof["kernel"] == "bwd_main" and roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert abs(roof["achieved"] - bwd_f / 0.772e-3 / 1e12) < 1e-6 and abs(roof["achieved"] - 890.3) < 1.0
    assert roof["peak"] == burst and abs(roof["frac"] - roof["achieved"] / burst) < 1e-12
    assert abs(split["fwd_tflops"] - 951.0) < 1.0
    assert abs(split["bwd_tflops"] - bwd_f / 0.822e-3 / 1e12) < 1e-6
    assert abs(sum(k["share"] for k in kernels.values()) - 1.0) < 1e-9
    assert kernels["bwd_main"]["launches"] == 10 and abs(kernels["bwd_main"]["ms_per_launch"] - 0.772) < 1e-12
    # a power-capped run (SM clock held below 95 % of max) is compared with the sustained figure
    capped = dict(FULL_CLOCK, sm_mhz=1500.0, sm_min_mhz=1400.0, reasons=["sw_power_cap"])
    roof2, _, split2 = bench.analyse(prof, w, "dsweep128", fwd_f, bwd_f, capped, 10)
    assert roof2["peak"] == bench.peaks()[1] and split2["peak_kind"].startswith("sustained")


def test_analyse_deterministic_and_fp8_steps():
    w = bench.WORKLOADS["det128"]
    fwd_f, bwd_f = bench.workload_flops(w)
    # the key-block kernel without dQ performs four of the five products, the dQ pass three
    roof, _, _ = bench.analyse(_prof(fwd=0.3, bwd_pre=0.03, bwd_main=0.513, bwd_dq=0.394), w, "det128",
                               fwd_f, bwd_f, FULL_CLOCK, 10)
    assert roof["kernel"] == "bwd_main" and abs(roof["achieved"] - 0.8 * bwd_f / 0.513e-3 / 1e12) < 1e-6
    roof, _, _ = bench.analyse(_prof(fwd=0.3, bwd_pre=0.03, bwd_main=0.3, bwd_dq=0.394), w, "det128",
                               fwd_f, bwd_f, FULL_CLOCK, 10)
    assert roof["kernel"] == "bwd_dq" and abs(roof["achieved"] - 0.6 * bwd_f / 0.394e-3 / 1e12) < 1e-6
    # FP8: the forward against twice the bf16 peak; the quantiser (three launches a step) against HBM
    w = bench.WORKLOADS["fp8_128"]
    fwd_f, bwd_f = bench.workload_flops(w)
    roof, _, split = bench.analyse(_prof(fwd_fp8=0.289, fp8_quant=0.04), w, "fp8_128", fwd_f, bwd_f, FULL_CLOCK, 10)
    # at d = 128 the exponentials (512 FLOPs each, 16 per clock per SM) cap E4M3 attention below twice
    # the bf16 rate: 16 x 148 x 1965 MHz x 512 = 2382 TFLOP/s
    assert roof["kernel"] == "fwd_fp8" and roof["bound"] == "alu" and abs(roof["peak"] - 2382.4) < 0.5
    assert roof["tensor_peak"] == 2 * bench.peaks()[0] and abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-12
    assert split["peak"] == 2 * bench.peaks()[0] and "bwd_tflops" not in split
    roof, _, _ = bench.analyse(_prof(fwd_fp8=0.05, fp8_quant=0.1), w, "fp8_128", fwd_f, bwd_f, FULL_CLOCK, 10)
    n = 4 * 16 * 4096 * 128
    assert roof["kernel"] == "fp8_quant" and roof["unit"] == "GB/s"
    assert abs(roof["achieved"] - 11 * n / (0.3e-3) / 1e9) < 1e-6     # 0.1 ms x 3 launches per step


def test_forward_roofline_takes_the_lower_ceiling():
    # d = 128 bf16: the exponential ceiling (2382) is above the tensor peak, which stays the roofline
    w = bench.WORKLOADS["long_fwd"]
    fwd_f, bwd_f = bench.workload_flops(w)
    roof, _, _ = bench.analyse(_prof(fwd=0.25), w, "long_fwd", fwd_f, bwd_f, FULL_CLOCK, 10)
    assert roof["bound"] == "tensor" and roof["peak"] == bench.peaks()[0] and "tensor_peak" not in roof
    # d = 64: 256 FLOPs per exponential cap the forward at 1191 TFLOP/s, below the tensor peak
    w = dict(bench.WORKLOADS["dsweep64"], bwd=False)
    fwd_f, bwd_f = bench.workload_flops(w)
    roof, _, split = bench.analyse(_prof(fwd=0.25), w, "dsweep64", fwd_f, bwd_f, FULL_CLOCK, 10)
    assert roof["bound"] == "alu" and abs(roof["peak"] - 1191.2) < 0.5 and roof["tensor_peak"] == bench.peaks()[0]
    assert abs(split["fwd_exp_ceiling"] - roof["peak"]) < 1e-9
    # the ceiling follows the sampled SM clock
    slow = dict(FULL_CLOCK, sm_mhz=1500.0)
    assert abs(bench.exp_ceiling_tflops(64, slow) - 1191.2 * 1500 / 1965) < 0.5


def test_clock_samples_are_summarised():
    lines = ["0, 1965, 1965, 650.1, Not Active, Not Active, Not Active, Not Active",
             "0, 1965, 1965, 998.0, Not Active, Not Active, Not Active, Active",
             "0, 1800, 1965, 1001.3, Not Active, Not Active, Not Active, Active",
             "0, [N/A], 1965, 10.0, Not Active, Not Active, Not Active, Not Active",   # unreadable: skipped
             "garbage"]
    c = bench.parse_clock_samples(lines)
    assert c["samples"] == 3 and c["sm_mhz"] == 1965.0 and c["sm_min_mhz"] == 1800.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert bench.power_capped(c)           # a sample at 1800 MHz is below 95 % of 1965
    hot = bench.parse_clock_samples(["0, 1400, 1965, 700, Active, Not Active, Active, Not Active"])
    assert hot["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.parse_clock_samples([])["sm_mhz"] is None


def test_nvml_clock_samples_are_summarised():
    # (SM MHz, NVML clock-event reason bits): 0x4 sw_power_cap, 0x8 hw_slowdown, 0x1 idle (ignored)
    c = bench.summarise_nvml([(1965, 0x1), (1965, 0x4), (1500, 0x4), (1965, 0)], 1965)
    assert c["samples"] == 4 and c["sm_mhz"] == 1965.0 and c["sm_min_mhz"] == 1500.0
    assert c["reasons"] == ["sw_power_cap"] and bench.power_capped(c)
    hot = bench.summarise_nvml([(1200, 0x8 | 0x40)], 1965)
    assert hot["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    none = bench.summarise_nvml([], 1965)
    assert none["sm_mhz"] is None and none["samples"] == 0


def test_packed_workload_flops_sum_over_sequences():
    from flash_fwd_b200 import accounting as acc
    w = bench.WORKLOADS["varlen128"]
    n = bench.varlen_lengths(w)
    assert len(n) == w["B"] and all(w["varlen"][0] <= x <= w["varlen"][1] for x in n)
    f, b = bench.workload_flops(w)
    assert f == sum(acc.fwd_flops(1, w["H"], x, w["d"], True) for x in n) and b == 2.5 * f
    per = [bench.head_flops(w, None, i) for i in range(w["B"] * w["H"])]
    assert abs(sum(per) - (f + b)) <= 1e-6 * (f + b)


def test_traffic_is_reported_only_for_unchanged_kernel_sources(tmp_path, monkeypatch):
    import json as _json
    sha = bench.kernel_source_sha()
    assert len(sha) == 16
    prof_dir = tmp_path / "profiles"
    prof_dir.mkdir()
    (prof_dir / "traffic.json").write_text(_json.dumps({
        "fwd": {"dsweep128": {"bytes_per_launch": 123, "source_sha": sha}},
        "bwd_main": {"dsweep128": {"bytes_per_launch": 456, "source_sha": "0" * 16}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: sha)
    assert bench.traffic_for("fwd", "dsweep128") == 123          # captured with these sources
    assert bench.traffic_for("bwd_main", "dsweep128") is None    # sources changed since the capture
    assert bench.traffic_for("fwd", "det128") is None            # never captured
    assert bench.traffic_for("fwd_fp8", "fp8_128") is None


def test_kernel_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    src = ('// header comment\n#include "x.cuh"\n/* block\n comment */ int f(int a) {  \n'
           '    const char *s = "// not a comment";   // trailing\n    char c = \'/\';\n\n    return a + 1;\n}\n')
    assert bench.strip_comments(src) == ('#include "x.cuh"\n  int f(int a) {\n'
                                         '    const char *s = "// not a comment";\n    char c = \'/\';\n    return a + 1;\n}')
    csrc = tmp_path / "flash_fwd_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "fa_api.cu").write_text(src)
    (csrc / "fa_common.cuh").write_text("int g;\n")
    (csrc / "fa_selftest.cu").write_text("int h;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha()
    (csrc / "fa_api.cu").write_text(src.replace("// trailing", "// another comment").replace("block", "other"))
    assert bench.kernel_source_sha() == h0                # comments only
    (csrc / "fa_selftest.cu").write_text("int h2;\n")
    assert bench.kernel_source_sha() == h0                # the failure self-test is not a measured kernel
    (csrc / "fa_api.cu").write_text(src.replace("a + 1", "a + 2"))
    assert bench.kernel_source_sha() != h0                # code
    (csrc / "fa_api.cu").write_text(src)
    (csrc / "fa_common.cuh").write_text("int g2;\n")
    assert bench.kernel_source_sha() != h0                # every header counts
