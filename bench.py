#!/usr/bin/env python
"""Benchmark of exact attention (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole path over one batch of synthetic input:
fa_fwd (O, LSE) then fa_bwd (dQ, dK, dV), called through the C ABI.
Throughput is TFLOP/s with the FLOP convention forward = 4*B*H*N^2*d (halved
for causal), backward = 2.5 x forward; block-sparse counts kept blocks only.

Default workload: B=4, H=16, N=4096, d=128, bf16, causal -- the shape on which
the forward >= 60% / backward >= 45% of dense bf16 peak targets are quoted.

With N > 1 (torchrun) every rank runs its own replica of the workload (weak
scaling; the path needs no exchange step), timed on the device, max over ranks.

Printed: one JSON line on rank 0 with value, roofline of the dominant kernel
(CUDA events around each launch, recorded by the library on the launching
stream), the CPU oracle baseline on a bounded sample (rank 0, N = 1 only), an
end-to-end figure through host buffers, the SM clocks sampled during the timed
region and the number of library kernel launches.

--impl reference times the fp64 CPU oracle (the reference arm; there is no
reference GPU code) on bounded samples of the same workload.
"""
import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOPs/s at N=1K–64K, d=64–256; % of B200 dense BF16 peak"
UNIT = "TFLOP/s"

WORKLOADS = {
    "dsweep128": dict(B=4, H=16, N=4096, d=128, dtype="bf16", causal=True, sparse=False, bwd=True),
    "dsweep64": dict(B=4, H=16, N=4096, d=64, dtype="bf16", causal=True, sparse=False, bwd=True),
    "dsweep256": dict(B=4, H=16, N=4096, d=256, dtype="bf16", causal=True, sparse=False, bwd=True),
    "gpt2s": dict(B=8, H=12, N=1024, d=64, dtype="bf16", causal=True, sparse=False, bwd=True),
    "long_fwd": dict(B=1, H=8, N=8192, d=128, dtype="f16", causal=False, sparse=False, bwd=False),
    "long_fwd_causal": dict(B=1, H=8, N=8192, d=128, dtype="f16", causal=True, sparse=False, bwd=False),
    "sparse64k": dict(B=1, H=4, N=65536, d=64, dtype="bf16", causal=False, sparse=True, bwd=True,
                      density=0.2),
    "tiny": dict(B=1, H=2, N=128, d=64, dtype="f16", causal=False, sparse=False, bwd=True),
    # the general entry points: a sliding window, a decoder chunk attending to
    # a longer context, ALiBi (causal), all at the d = 128 sweep's size
    "window128": dict(B=4, H=16, N=4096, d=128, dtype="bf16", causal=True, sparse=False, bwd=True,
                      window=(1024, 0)),
    "cross128": dict(B=4, H=16, N=1024, Nk=8192, d=128, dtype="bf16", causal=True, sparse=False, bwd=True),
    "alibi128": dict(B=4, H=16, N=4096, d=128, dtype="bf16", causal=True, sparse=False, bwd=True, alibi=True),
    # the deterministic backward (fa_bwd_deterministic) on the d = 128 sweep's shape
    "det128": dict(B=4, H=16, N=4096, d=128, dtype="bf16", causal=True, sparse=False, bwd=True,
                   deterministic=True),
    # the FP8 forward (block quantisation + incoherent processing) on the same shape:
    # a step quantises the bf16 Q, K, V and runs the E4M3 forward
    "fp8_128": dict(B=4, H=16, N=4096, d=128, dtype="bf16", causal=True, sparse=False, bwd=False, fp8=True),
    "fp8_64": dict(B=4, H=16, N=4096, d=64, dtype="bf16", causal=True, sparse=False, bwd=False, fp8=True),
    "fp8_256": dict(B=4, H=16, N=4096, d=256, dtype="bf16", causal=True, sparse=False, bwd=False, fp8=True),
    # a packed variable-length batch (fa_fwd_varlen / fa_bwd_varlen): 16
    # sequences with lengths drawn uniformly from [512, 4096] (seeded), N = the
    # bound of the lengths (max_seqlen)
    "varlen128": dict(B=16, H=16, N=4096, d=128, dtype="bf16", causal=True, sparse=False, bwd=True,
                      varlen=(512, 4096)),
}


def general(w):
    return "Nk" in w or "window" in w or w.get("alibi", False)


def varlen_lengths(w):
    """The sequence lengths of a packed workload (seed 0: every rank the same mix)."""
    from flash_fwd_b200 import inputs
    return inputs.varlen_lengths(w["B"], w["varlen"][0], w["varlen"][1], seed=0)


L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # the timed steps: a burst measurement (about 35 ms at the default
    # workload); --sustained-steps then times a region long enough to settle
    # under the 1000 W power cap, reported beside it
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--sustained-steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="dsweep128", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="wall-clock budget of the CPU oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p.get("bf16_tflops"), p.get("bf16_tflops_sustained"), p.get("hbm_gbs"), \
            "measured (MEASURED_PEAKS.json)"
    # the profiling recipe's figures for this pool, used only when the
    # measured file is absent; every line that uses them says so
    return 1590.0, 1400.0, 6650.0, "fallback (MEASURED_PEAKS.json absent)"


def workload_flops(w, kept_blocks=None):
    from flash_fwd_b200 import accounting as acc
    if w.get("varlen"):
        f = sum(acc.fwd_flops(1, w["H"], n, w["d"], w["causal"]) for n in varlen_lengths(w))
    elif w["sparse"]:
        f = acc.sparse_fwd_flops(w["B"], w["H"], w["d"], kept_blocks)
    elif "Nk" in w or "window" in w:
        f = acc.general_fwd_flops(w["B"], w["H"], w["N"], w.get("Nk", w["N"]), w["d"], w["causal"], w.get("window"))
    else:
        f = acc.fwd_flops(w["B"], w["H"], w["N"], w["d"], w["causal"])
    b = 2.5 * f if w["bwd"] else 0.0
    return f, b


def describe(name, w):
    s = f"{name}: B={w['B']} H={w['H']} N={w['N']} d={w['d']} {w['dtype']}"
    s += " causal" if w["causal"] else ""
    s += f" block-sparse(128x128, diag + Bernoulli {w['density']})" if w["sparse"] else ""
    s += f" Nk={w['Nk']}" if "Nk" in w else ""
    s += f" window={w['window']}" if "window" in w else ""
    s += " alibi" if w.get("alibi") else ""
    s += " fwd+bwd" if w["bwd"] else " fwd"
    s += " (deterministic backward)" if w.get("deterministic") else ""
    s += " (FP8 E4M3 with Hadamard rotation; step = quantise + forward)" if w.get("fp8") else ""
    if w.get("varlen"):
        n = varlen_lengths(w)
        s += (f" (packed variable-length batch: {len(n)} sequences, lengths uniform in "
              f"[{w['varlen'][0]}, {w['varlen'][1]}], {sum(n)} tokens, max_seqlen {max(n)})")
    return s


def device_info(index):
    """GPU name, driver and CUDA runtime of this rank's device."""
    import torch
    info = {"name": torch.cuda.get_device_name(index), "cuda_runtime": torch.version.cuda, "driver": None}
    try:
        r = subprocess.run(["nvidia-smi", "-i", str(index), "--query-gpu=driver_version", "--format=csv,noheader"],
                           capture_output=True, text=True, timeout=20)
        info["driver"] = r.stdout.strip() or None
    except (OSError, subprocess.SubprocessError):
        pass
    return info


def strip_comments(src):
    """C/C++ source without its comments, trailing blanks and empty lines
    (string and character literals kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def kernel_source_sha():
    """Hash of the code of the measured kernels and their launches (every
    header of the library and fa_api.cu, comments left out, so that a
    comment edit keeps the ncu counters taken on that code); the failure
    self-test of fa_selftest.cu is not part of it."""
    csrc = os.path.join(ROOT, "flash_fwd_b200", "csrc")
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(csrc, "*.cuh")) + [os.path.join(csrc, "fa_api.cu")]):
        with open(p, encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode("utf-8"))
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if the kernel
    sources are unchanged since it was taken (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel, {}).get(workload)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons sampled while the timed steps run.

    NVML is read from a thread every 2 ms (so that even a region of a few tens
    of milliseconds gets samples); where NVML is not available, nvidia-smi
    samples every 50 ms.  Only reads: no clock or other setting is changed."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.002

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None
        self.nvml = None
        self.thread = None
        self.samples = []

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.running = True
            self.thread = threading.Thread(target=self._nvml_loop, daemon=True)
            self.thread.start()
            return
        except Exception:   # no NVML here: nvidia-smi below
            self.nvml = None
        self._start_smi()

    def _nvml_loop(self):
        n = self.nvml
        reason = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or n.nvmlDeviceGetCurrentClocksThrottleReasons
        while self.running:
            try:
                self.samples.append((n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM), reason(self.handle)))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def _start_smi(self):
        """Starts nvidia-smi every 50 ms and returns once its first sample is
        in (at most 3 s), so that the samples fall inside the region timed next."""
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t0 = time.monotonic()
        while time.monotonic() - t0 < 3.0 and self.proc.poll() is None:
            if os.path.getsize(self.tmp.name) > 0:
                break
            time.sleep(0.01)
        # the first line may have been taken while the GPU idled: not a sample of the region
        self.skip = 1 if os.path.getsize(self.tmp.name) > 0 else 0

    def stop(self):
        if self.nvml is not None:
            self.running = False
            self.thread.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            return summarise_nvml(self.samples, self.max_mhz)
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        with open(self.tmp.name) as f:
            lines = [ln.strip() for ln in f if ln.strip()]
        os.unlink(self.tmp.name)
        out = parse_clock_samples(lines[getattr(self, "skip", 0):])
        out["source"] = "nvidia-smi, 50 ms"
        return out


# NVML clock-event reason bits (nvml.h)
NVML_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown"}


def summarise_nvml(samples, max_mhz):
    """Median, minimum and maximum SM clock of NVML samples [(MHz, reason bits)]
    and every reason seen active."""
    reasons = sorted({name for _, bits in samples for bit, name in NVML_REASONS.items() if bits & bit})
    if not samples:
        return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": reasons, "samples": 0, "source": "nvml, 2 ms"}
    sm = [float(c) for c, _ in samples]
    return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": float(max_mhz),
            "reasons": reasons, "samples": len(sm), "source": "nvml, 2 ms"}


def parse_clock_samples(lines):
    """Summary of nvidia-smi samples in ClockSampler.Q's column order (index,
    SM clock, max SM clock, power, then the four throttle reasons): median,
    minimum and maximum SM clock, and every reason seen active."""
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [x.strip() for x in ln.split(",")]
        if len(parts) < 8:
            continue
        try:
            sm.append(float(parts[1]))
            mx = float(parts[2])
        except ValueError:
            continue
        for n, v in zip(names, parts[4:8]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
    return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": mx,
            "reasons": sorted(reasons), "samples": len(sm)}


def power_capped(clocks):
    """True when the power cap actually slowed the timed region: SM clocks
    sampled below 95 % of their maximum.  The sw_power_cap flag alone, with
    the clock still at its maximum, keeps the burst peak."""
    if not clocks or clocks.get("sm_mhz") is None:
        return False
    mx = clocks.get("sm_max_mhz") or 0
    return bool(mx) and clocks.get("sm_min_mhz", mx) < 0.95 * mx


def make_inputs(w, seed, device):
    import torch

    from flash_fwd_b200 import inputs
    if w.get("varlen"):
        import flash_fwd_b200 as fa
        n = varlen_lengths(w)
        cu_q, cu_k, q, k, v, do = inputs.make_varlen(n, n, w["H"], w["d"], w["dtype"], seed=seed)
        host = dict(q=q, k=k, v=v, do=do, cu_q=cu_q, cu_k=cu_k, mask=None, slopes=None)
        dev = {x: (y.to(device) if y is not None else None) for x, y in host.items()}
        dev["o"] = torch.empty_like(dev["q"])
        dev["lse"] = torch.empty((w["H"], q.shape[0]), dtype=torch.float32, device=device)
        dev["dq"] = torch.empty_like(dev["q"])
        dev["dk"], dev["dv"] = torch.empty_like(dev["k"]), torch.empty_like(dev["v"])
        dev["ws"] = torch.empty(fa.fa_bwd_varlen_workspace_bytes(w["B"], w["H"], q.shape[0], max(n), w["d"]),
                                dtype=torch.uint8, device=device)
        dev["max_n"] = max(n)
        return host, dev
    if "Nk" in w:
        q, k, v, do = inputs.make_qkv_cross(w["B"], w["H"], w["N"], w["Nk"], w["d"], w["dtype"], seed=seed)
    else:
        q, k, v, do = inputs.make_qkv(w["B"], w["H"], w["N"], w["d"], w["dtype"], seed=seed, with_dout=w["bwd"])
    mask = inputs.make_block_mask(w["N"], 128, w.get("density", 0.2), seed=seed) if w["sparse"] else None
    slopes = inputs.alibi_slopes(w["H"]) if w.get("alibi") else None
    host = dict(q=q, k=k, v=v, do=do, mask=mask, slopes=slopes)
    dev = {n: (t.to(device) if t is not None else None) for n, t in host.items()}
    dev["o"] = torch.empty_like(dev["q"])
    dev["lse"] = torch.empty((w["B"], w["H"], w["N"]), dtype=torch.float32, device=device)
    if w.get("fp8"):
        dev["signs"] = inputs.hadamard_signs(w["d"], seed=seed).to(device)
    if w["bwd"]:
        import flash_fwd_b200 as fa
        dev["dq"] = torch.empty_like(dev["q"])
        dev["dk"], dev["dv"] = torch.empty_like(dev["k"]), torch.empty_like(dev["v"])
        ws_fn = fa.fa_bwd_deterministic_workspace_bytes if w.get("deterministic") else fa.fa_bwd_ex_workspace_bytes
        dev["ws"] = torch.empty(ws_fn(w["B"], w["H"], w["N"], w.get("Nk", w["N"]), w["d"]),
                                dtype=torch.uint8, device=device)
    return host, dev


def step(w, t, stream):
    import flash_fwd_b200 as fa
    scale = 1.0 / w["d"] ** 0.5
    if w.get("varlen"):
        fa.fa_fwd_varlen(t["q"], t["k"], t["v"], t["o"], t["lse"], t["cu_q"], t["cu_k"], t["max_n"], t["max_n"],
                         w["causal"], scale, stream=stream)
        fa.fa_bwd_varlen(t["q"], t["k"], t["v"], t["o"], t["do"], t["lse"], t["dq"], t["dk"], t["dv"], t["ws"],
                         t["cu_q"], t["cu_k"], t["max_n"], t["max_n"], w["causal"], scale, stream=stream)
    elif w.get("fp8"):
        q8, k8, v8, sq, sk, sv = fa.fa_fp8_quantize_qkv(t["q"], t["k"], t["v"], t["signs"], stream)
        fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, t["o"], t["lse"], w["causal"], scale, stream)
    elif w.get("deterministic"):
        fa.fa_fwd_ex(t["q"], t["k"], t["v"], t["o"], t["lse"], w["causal"], scale, w.get("window"), t["slopes"],
                     t["mask"], stream)
        fa.fa_bwd_deterministic(t["q"], t["k"], t["v"], t["o"], t["do"], t["lse"], t["dq"], t["dk"], t["dv"],
                                t["ws"], w["causal"], scale, w.get("window"), t["slopes"], t["mask"], stream)
    elif general(w):
        fa.fa_fwd_ex(t["q"], t["k"], t["v"], t["o"], t["lse"], w["causal"], scale, w.get("window"), t["slopes"],
                     t["mask"], stream)
        if w["bwd"]:
            fa.fa_bwd_ex(t["q"], t["k"], t["v"], t["o"], t["do"], t["lse"], t["dq"], t["dk"], t["dv"], t["ws"],
                         w["causal"], scale, w.get("window"), t["slopes"], t["mask"], stream)
    elif w["sparse"]:
        fa.fa_fwd_blocksparse(t["q"], t["k"], t["v"], t["o"], t["lse"], t["mask"], w["causal"], scale, stream)
        if w["bwd"]:
            fa.fa_bwd_blocksparse(t["q"], t["k"], t["v"], t["o"], t["do"], t["lse"], t["dq"], t["dk"], t["dv"],
                                  t["ws"], t["mask"], w["causal"], scale, stream)
    else:
        fa.fa_fwd(t["q"], t["k"], t["v"], t["o"], t["lse"], w["causal"], scale, stream)
        if w["bwd"]:
            fa.fa_bwd(t["q"], t["k"], t["v"], t["o"], t["do"], t["lse"], t["dq"], t["dk"], t["dv"], t["ws"],
                      w["causal"], scale, stream)


# --------------------------------------------------------------------------
# CPU oracle: the baseline leg and the reference arm
# --------------------------------------------------------------------------
def oracle_head_pass(host, w, head):
    """One (batch, head) of the workload through the fp64 oracle: forward on
    every row, dQ on every row, dK/dV on every key.  Returns the seconds of
    the forward and of the backward."""
    import numpy as np

    import oracle
    N, Nk, d = w["N"], w.get("Nk", w["N"]), w["d"]
    b, h = divmod(head, w["H"])
    sl = lambda t, n: t[b, h].reshape(1, n, d).double().numpy()  # noqa: E731
    if w.get("varlen"):
        # sequence b, head h of the packed batch: its own square problem
        c0, c1 = int(host["cu_q"][b]), int(host["cu_q"][b + 1])
        N = Nk = c1 - c0
        sl = lambda t, n: t[c0:c1, h].reshape(1, n, d).double().numpy()  # noqa: E731
    Q, K, V = sl(host["q"], N), sl(host["k"], Nk), sl(host["v"], Nk)
    flags = (oracle.CAUSAL if w["causal"] else 0) | (oracle.SPARSE if w["sparse"] else 0)
    mask = host["mask"].numpy() if w["sparse"] else None
    modes = dict(window=w.get("window"),
                 slopes=None if host.get("slopes") is None else host["slopes"][h:h + 1].double().numpy())
    rows = np.arange(N, dtype=np.int32)
    cols = np.arange(Nk, dtype=np.int32)
    if w.get("fp8"):
        from flash_fwd_b200 import inputs
        signs = inputs.hadamard_signs(d, seed=0).numpy()
        t0 = time.perf_counter()
        q8, sq = oracle.fp8_quantize(Q.astype(np.float32), 128, signs)
        k8, sk = oracle.fp8_quantize(K.astype(np.float32), 128, signs)
        v8, sv = oracle.fp8_quantize(V.astype(np.float32), N)
        oracle.fwd_fp8(q8, k8, v8, sq, sk, sv[:, 0], 1.0 / d ** 0.5, causal=w["causal"])
        return time.perf_counter() - t0, 0.0
    t0 = time.perf_counter()
    oracle.fwd_rows(Q, K, V, 1.0 / d ** 0.5, flags, mask, 128, rows, **modes)
    t1 = time.perf_counter()
    if w["bwd"]:
        DO = sl(host["do"], N)
        oracle.bwd_dq_rows(Q, K, V, DO, 1.0 / d ** 0.5, rows, flags, mask, 128, **modes)
        oracle.bwd_dkdv_cols(Q, K, V, DO, 1.0 / d ** 0.5, cols, flags, mask, 128, **modes)
    return t1 - t0, time.perf_counter() - t1


def per_head_flops(w, kept_blocks):
    f, b = workload_flops(w, kept_blocks)
    return (f + b) / (w["B"] * w["H"])


def head_flops(w, kept_blocks, head):
    """FLOPs of (batch, head) pair number `head` (a packed batch's sequences differ)."""
    if not w.get("varlen"):
        return per_head_flops(w, kept_blocks)
    from flash_fwd_b200 import accounting as acc
    n = varlen_lengths(w)[head // w["H"]]
    return (3.5 if w["bwd"] else 1.0) * acc.fwd_flops(1, 1, n, w["d"], w["causal"])


def cpu_sample(host, w, kept_blocks, budget_s, max_heads=None):
    """Whole (batch, head) passes of the oracle until the budget is spent (at
    least one).  Returns (heads, seconds, TFLOP/s, forward s, backward s)."""
    heads = w["B"] * w["H"] if max_heads is None else min(max_heads, w["B"] * w["H"])
    done, tf, tb, fl = 0, 0.0, 0.0, 0.0
    while done < heads and (tf + tb < budget_s or done == 0):
        f, b = oracle_head_pass(host, w, done)
        tf, tb = tf + f, tb + b
        fl += head_flops(w, kept_blocks, done)
        done += 1
    secs = tf + tb
    return done, secs, fl / secs / 1e12, tf, tb


def oracle_seconds(w, heads, tf, tb):
    """The oracle's forward and backward wall-clock seconds per (batch, head),
    and the whole workload's, extrapolated from the sampled heads."""
    per_f, per_b = tf / heads, tb / heads
    return {"fwd_s_per_head": per_f, "bwd_s_per_head": per_b if w["bwd"] else None,
            "extrapolated_full_workload_s": (per_f + per_b) * w["B"] * w["H"]}


def run_reference(args, w, name):
    from flash_fwd_b200 import dist as fdist
    rank, world, _ = fdist.env_ranks()
    if rank != 0:
        return
    host, _ = make_inputs_cpu(w)
    kept = int(host["mask"].sum()) if w["sparse"] else None
    for i in range(args.warmup):
        oracle_head_pass(host, w, i % (w["B"] * w["H"]))
    tf = tb = fl = 0.0
    for i in range(args.steps):
        head = (args.warmup + i) % (w["B"] * w["H"])
        f, b = oracle_head_pass(host, w, head)
        tf, tb = tf + f, tb + b
        fl += head_flops(w, kept, head)
    secs = tf + tb
    val = fl / secs / 1e12
    cores = os.cpu_count()
    what = ("E4M3 quantisation and the FP8 forward on all rows" if w.get("fp8") else
            "forward on all rows, dQ on all rows, dK/dV on all keys" if w["bwd"] else "forward on all rows")
    sample = f"one (batch, head) of the workload per step ({w['N']} rows): {what}"
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(name, w), "per_step": "one (batch, head)"},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                         **oracle_seconds(w, args.steps, tf, tb)},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def make_inputs_cpu(w):
    from flash_fwd_b200 import inputs
    if w.get("varlen"):
        n = varlen_lengths(w)
        cu_q, cu_k, q, k, v, do = inputs.make_varlen(n, n, w["H"], w["d"], w["dtype"], seed=0)
        return dict(q=q, k=k, v=v, do=do, cu_q=cu_q, cu_k=cu_k, mask=None, slopes=None), None
    if "Nk" in w:
        q, k, v, do = inputs.make_qkv_cross(w["B"], w["H"], w["N"], w["Nk"], w["d"], w["dtype"], seed=0)
    else:
        q, k, v, do = inputs.make_qkv(w["B"], w["H"], w["N"], w["d"], w["dtype"], seed=0, with_dout=w["bwd"])
    mask = inputs.make_block_mask(w["N"], 128, w.get("density", 0.2), seed=0) if w["sparse"] else None
    slopes = inputs.alibi_slopes(w["H"]) if w.get("alibi") else None
    return dict(q=q, k=k, v=v, do=do, mask=mask, slopes=slopes), None


SFU_EX2_PER_CLK_PER_SM = 16      # special-function unit, measured on B200 (one CTA per SM)
SMS = 148


def exp_ceiling_tflops(d, clocks):
    """The forward's ceiling set by the exponential: one ex2 per score, each
    score worth 4 d tensor FLOPs (S and P V), at the sampled SM clock (the
    maximum when none was sampled)."""
    mhz = (clocks or {}).get("sm_mhz") or (clocks or {}).get("sm_max_mhz") or 1965.0
    return SFU_EX2_PER_CLK_PER_SM * SMS * mhz * 1e6 * 4 * d / 1e12


def analyse(prof, w, name, fwd_f, bwd_f, clocks, steps):
    """From the library's per-kernel CUDA-event times ({kind: (ms summed over
    the timed steps, launches)}): the roofline of the dominant kernel, the
    per-kernel table and the forward / backward split.  fwd_f, bwd_f: the
    algorithmic FLOPs of one step's forward and backward."""
    dom = max(prof, key=lambda k: prof[k][0])
    dom_ms, dom_n = prof[dom]
    per_launch_ms = dom_ms / max(dom_n, 1)
    burst, sustained, hbm, src = peaks()
    # a run that hit the power cap is compared with the sustained GEMM figure
    # (cuBLAS under the same cap), a short one with the burst figure
    capped = power_capped(clocks)
    peak = sustained if capped and sustained else burst
    peak_kind = "sustained (power-capped run)" if capped and sustained else "burst"
    if dom == "fwd_fp8":
        # an E4M3 contraction: the measured bf16 GEMM peak x the nominal fp8 : bf16 ratio (2)
        achieved = fwd_f / (per_launch_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": 2 * peak, "unit": "TFLOP/s",
                "frac": achieved / (2 * peak),
                "peak_source": f"bf16 {peak_kind}, {src}, x 2, the nominal fp8 : bf16 ratio",
                "kernel": dom, "launch_ms": per_launch_ms}
    elif dom == "fp8_quant":
        # three launches per step: read Q, K, V and V again (16-bit), write three E4M3 tensors
        n = w["B"] * w["H"] * w["N"] * w["d"]
        alg_bytes = 4 * 2 * n + 3 * n
        step_ms = dom_ms / steps
        achieved = alg_bytes / (step_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_source": f"copy bandwidth, {src}", "kernel": dom, "step_ms": step_ms, "algorithmic_bytes": alg_bytes}
    elif dom in ("fwd", "bwd_main", "bwd_dq"):
        # tensor FLOPs the kernel performs: the backward's five products, of
        # which the deterministic backward's key-block kernel does four (no dQ)
        # and its dQ pass three (S and dP again, then dQ)
        det = w.get("deterministic", False)
        alg = {"fwd": fwd_f, "bwd_main": bwd_f * (0.8 if det else 1.0), "bwd_dq": bwd_f * 0.6}[dom]
        achieved = alg / (per_launch_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": f"bf16 {peak_kind}, {src}",
                "kernel": dom, "launch_ms": per_launch_ms}
    else:
        roof = {"bound": "hbm", "achieved": None, "peak": hbm, "unit": "GB/s", "frac": None, "kernel": dom}
    if dom in ("fwd", "fwd_fp8"):
        # a forward is also bounded by its exponentials: where that ceiling is
        # the lower one (d = 64; E4M3 products at d = 128) it is the roofline
        ceiling = exp_ceiling_tflops(w["d"], clocks)
        if ceiling < roof["peak"]:
            roof.update({"bound": "alu", "tensor_peak": roof["peak"], "tensor_frac": roof["frac"],
                         "tensor_peak_source": roof["peak_source"], "peak": ceiling,
                         "frac": roof["achieved"] / ceiling,
                         "peak_source": f"special-function unit: {SFU_EX2_PER_CLK_PER_SM} ex2 per clock per SM "
                                        f"x {SMS} SMs x the sampled SM clock x 4 d FLOPs per ex2 (derived)"})
    roof["traffic"] = traffic_for(dom, name)
    total = max(sum(x[0] for x in prof.values()), 1e-12)
    kernel_times = {k: {"ms_per_launch": (v[0] / v[1] if v[1] else 0.0), "launches": v[1], "share": v[0] / total}
                    for k, v in prof.items()}
    fkind = "fwd_fp8" if w.get("fp8") else "fwd"
    fwd_ms = prof[fkind][0] / max(prof[fkind][1], 1)
    fpeak = 2 * peak if w.get("fp8") else peak   # E4M3 products: twice the bf16 rate (nominal ratio)
    split = {"fwd_tflops": fwd_f / (fwd_ms / 1e3) / 1e12 if fwd_ms else None,
             "fwd_frac_of_peak": (fwd_f / (fwd_ms / 1e3) / 1e12) / fpeak if fwd_ms else None,
             "peak": fpeak, "peak_kind": peak_kind, "fwd_exp_ceiling": exp_ceiling_tflops(w["d"], clocks)}
    if w["bwd"]:
        bwd_ms = sum(prof[k][0] for k in ("bwd_pre", "bwd_main", "bwd_post", "bwd_dq")) / max(prof["bwd_main"][1], 1)
        split["bwd_tflops"] = bwd_f / (bwd_ms / 1e3) / 1e12
        split["bwd_frac_of_peak"] = split["bwd_tflops"] / peak
    return roof, kernel_times, split


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def run_ours(args, w, name):
    import torch

    import flash_fwd_b200 as fa
    from flash_fwd_b200 import dist as fdist

    rank, world, local = fdist.init("nccl" if args.gpus > 1 else "gloo")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    stream = torch.cuda.current_stream(device)
    host, t = make_inputs(w, seed=rank, device=device)
    kept = int(host["mask"].sum()) if w["sparse"] else None
    fwd_f, bwd_f = workload_flops(w, kept)
    flops = fwd_f + bwd_f

    for _ in range(args.warmup):
        step(w, t, stream)
    torch.cuda.synchronize(device)
    if fa.fa_last_device_status() != 0:
        raise RuntimeError("device status after warm-up is not ok")

    # ---------------- timed region: K steps on the device
    # Inputs smaller than L2 would stay resident from one step to the next:
    # then a buffer twice the size of L2 is written before every step, outside
    # the step's own event pair, and the K step times are summed.
    in_bytes = sum(x.numel() * x.element_size() for x in (t["q"], t["k"], t["v"]) + ((t["do"],) if w["bwd"] else ()))
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device) if in_bytes <= L2_BYTES else None
    sampler = ClockSampler(local)
    torch.cuda.reset_peak_memory_stats(device)
    base_bytes = torch.cuda.memory_allocated(device)
    fa.fa_profile_enable(True)
    fa.fa_profile_read()
    fdist.barrier(device)
    torch.cuda.synchronize(device)
    sampler.start()
    if flush is None:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step(w, t, stream)
        e1.record(stream)
        pairs = [(e0, e1)]
    else:
        pairs = []
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                step(w, t, stream)
                b.record(stream)
                pairs.append((a, b))
    torch.cuda.synchronize(device)
    fdist.barrier(device)
    clocks = sampler.stop()
    prof = fa.fa_profile_read()
    fa.fa_profile_enable(False)
    ms = sum(a.elapsed_time(b) for a, b in pairs)
    # device memory: what the steps held (inputs, outputs, workspace) against
    # one materialised N x N score matrix of the standard method
    from flash_fwd_b200 import accounting as acc
    memory = {"peak_allocated_bytes": torch.cuda.max_memory_allocated(device),
              "allocated_before_steps_bytes": base_bytes,
              "one_materialised_s_bytes": acc.s_matrix_bytes(w["B"], w["H"], w["N"], 2) * w.get("Nk", w["N"])
              // w["N"]}
    ms_max = fdist.max_over_ranks(ms, device if args.gpus > 1 else None)
    value = fdist.aggregate_throughput([flops * args.steps] * world, ms_max) / 1e12
    if fa.fa_last_device_status() != 0:
        raise RuntimeError("device status after the timed region is not ok")

    # ---------------- dominant kernel roofline, per-kernel times, forward/backward split
    roof, kernel_times, split = analyse(prof, w, name, fwd_f, bwd_f, clocks, args.steps)

    # ---------------- a sustained region: the same steps for about half a second or more
    sustained = None
    if args.sustained_steps > 0 and flush is None:
        fdist.barrier(device)
        torch.cuda.synchronize(device)
        sampler = ClockSampler(local)
        sampler.start()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.sustained_steps):
            step(w, t, stream)
        s1.record(stream)
        torch.cuda.synchronize(device)
        sclocks = sampler.stop()
        sms = fdist.max_over_ranks(s0.elapsed_time(s1), device if args.gpus > 1 else None)
        svalue = fdist.aggregate_throughput([flops * args.sustained_steps] * world, sms) / 1e12
        _, ssus, _, psrc = peaks()
        sustained = {"steps": args.sustained_steps, "ms_per_step": sms / args.sustained_steps, "value": svalue,
                     "unit": UNIT, "clocks": sclocks, "sustained_peak": ssus,
                     "peak_source": f"bf16 sustained, {psrc}"}
        if fa.fa_last_device_status() != 0:
            raise RuntimeError("device status after the sustained region is not ok")

    # ---------------- the same steps replayed from a CUDA graph (launch overhead removed)
    graph = None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step(w, t, side)                      # warm the capture stream once
        stream.wait_stream(side)
        torch.cuda.synchronize(device)
        with torch.cuda.graph(g):
            cap = torch.cuda.current_stream(device)
            for _ in range(args.steps):
                step(w, t, cap)
        torch.cuda.synchronize(device)
        g.replay()
        torch.cuda.synchronize(device)
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        g.replay()
        g1.record(stream)
        torch.cuda.synchronize(device)
        gms = g0.elapsed_time(g1)
        graph = {"ms_per_step": gms / args.steps, "value": flops * args.steps / (gms / 1e3) / 1e12, "unit": UNIT,
                 "steps_per_replay": args.steps}
        del g
        if fa.fa_last_device_status() != 0:
            raise RuntimeError("device status after the graph replay is not ok")
    except RuntimeError as e:   # capture refused or failed: reported, not fatal
        graph = {"error": str(e)[:200]}

    # ---------------- end to end through host buffers
    # Every step copies its inputs from pinned host memory and its outputs back
    # (PCIe: both directions at once).  Two device buffer sets alternate, so
    # that the input copy of step i + 1 and the output copy of step i - 1 run
    # beside the kernels of step i: inputs on one copy stream, outputs on
    # another, kernels on the compute stream, ordered by events (a buffer set
    # is refilled only after the kernels that read it, and its outputs are
    # overwritten only after they were copied out).  The timed region runs
    # from the first input copy to the last output copy.
    e2e = None
    if args.e2e_steps > 0:
        in_names = [n for n in ("q", "k", "v", "do", "cu_q", "cu_k") if host.get(n) is not None]
        out_names = ["o", "lse", "dq", "dk", "dv"] if w["bwd"] else ["o", "lse"]
        pin = {n: host[n].pin_memory() for n in in_names}
        outs = {n: torch.empty(t[n].shape, dtype=t[n].dtype, pin_memory=True) for n in out_names}
        h2d = sum(x.numel() * x.element_size() for x in pin.values())
        d2h = sum(x.numel() * x.element_size() for x in outs.values())
        sets = [t, dict(t)]
        for n in in_names + out_names:
            sets[1][n] = torch.empty_like(t[n])
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        read = [None, None]     # per buffer set: its last kernels completed (inputs free)
        drained = [None, None]  # per buffer set: its last outputs copied out
        fdist.barrier(device)
        torch.cuda.synchronize(device)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(s_in)
        for i in range(args.e2e_steps):
            b = sets[i % 2]
            if read[i % 2] is not None:
                s_in.wait_event(read[i % 2])
            with torch.cuda.stream(s_in):
                for n in in_names:
                    b[n].copy_(pin[n], non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
            stream.wait_event(landed)
            if drained[i % 2] is not None:
                stream.wait_event(drained[i % 2])
            step(w, b, stream)
            read[i % 2] = torch.cuda.Event()
            read[i % 2].record(stream)
            s_out.wait_event(read[i % 2])
            with torch.cuda.stream(s_out):
                for n in out_names:
                    outs[n].copy_(b[n], non_blocking=True)
            drained[i % 2] = torch.cuda.Event()
            drained[i % 2].record(s_out)
        a1.record(s_out)
        torch.cuda.synchronize(device)
        del sets
        e2e_ms = fdist.max_over_ranks(a0.elapsed_time(a1), device if args.gpus > 1 else None)
        e2e = {"value": fdist.aggregate_throughput([flops * args.e2e_steps] * world, e2e_ms) / 1e12,
               "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / args.e2e_steps}

    # ---------------- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads, secs, val, tf, tb = cpu_sample(host, w, kept, args.cpu_seconds)
        what = ("E4M3 quantisation of Q, K, V and the FP8 forward on all rows" if w.get("fp8") else
                "forward on all rows, dQ on all rows, dK/dV on all keys" if w["bwd"] else "forward on all rows")
        cpu = {"value": val, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
               "sample": f"{heads} of {w['B'] * w['H']} (batch, head) pairs, each: {what}; {secs:.1f} s",
               **oracle_seconds(w, heads, tf, tb)}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if w.get("fp8") else w["dtype"], "data": "synthetic",
        "config": {"workload": describe(name, w), "B": w["B"], "H": w["H"], "N": w["N"], "d": w["d"],
                   "causal": w["causal"], "block_sparse": w["sparse"],
                   "kept_blocks": kept, "parallelism": f"{world} independent replica(s), no collective",
                   "l2": ("inputs larger than L2, no flush" if flush is None else
                          f"inputs smaller than L2: {2 * L2_BYTES >> 20} MiB written before each timed step "
                          "(outside its events), step times summed; the graph replay is not flushed"),
                   "input_bytes": in_bytes},
        "split": split,
        "kernels": kernel_times,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clocks,
        "graph": graph,
        "sustained": sustained,
        "device": device_info(local),
        "gpu_launches": sum(v[1] for v in prof.values()),
        "memory": memory,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    fdist.shutdown()


def main():
    args = parse()
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w, args.workload)
    else:
        run_ours(args, w, args.workload)


if __name__ == "__main__":
    main()
