"""Benchmark: one training step of exact attention (forward + backward) per
GPU, through the C ABI, on synthetic inputs shaped like the long-sequence
workload B=4, H=16, N=8192, d=128 (non-causal), bf16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  The step is fa_fwd + fa_bwd (forward kernel,
D pre-pass, dK/dV kernel, dQ kernel).  FLOPs per step are counted as the
pages' dense attention work: forward 4*B*H*N^2*d, backward 2.5x forward
(five GEMMs), halved under a causal mask.  Several GPUs run independent
replicas (no collective: the (sequence, head) units share nothing).

--impl reference times the float64 CPU oracle (the reference arm: there is
no runnable reference implementation) on a bounded sample of the same
workload on the host cores.

--workload decode measures decode against a padded K/V cache
(fa_fwd_kvcache: B=16, H=16, one query per sequence, caches of 4096..8192
tokens in an 8192-row buffer, d=128) in GB/s of cache read against the HBM
roofline.

--workload fp8 measures the block-quantised FP8 forward on the training
shape (B=4, H=16, N=8192, d=128, non-causal, with the rotation): quantisation
of Q, K, V plus the FP8 forward kernel per step.  It is a separate,
lower-precision path, not exact attention.

--workload prefill_kv measures the cached-KV prefill forward instead
(fa_fwd_kvcache with the library's key split: B=4, H=16, 2048 new query
tokens after 6144 cached ones, so Nk=8192, d=128, causal aligned
bottom-right), with its own oracle sample.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "attention fwd/bwd TFLOPs/s (BF16, d=128) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = dict(B=4, H=16, N=8192, d=128, causal=False, window=0, seed=2)
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
# NVIDIA's dense BF16 tensor figure for an HGX B200 GPU (its published 2:4-sparse
# figure halved); reported beside the measured peak as a second denominator
NOMINAL_BF16_DENSE_TFLOPS = 2250.0

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# ncu captures.  Training step and FP8 forward: the B=2 H=16 N=8192 d=128
# non-causal case, scaled by 2 to the B=4 workload (each kernel's traffic grows
# with the number of heads it processes).  Decode and cached-KV prefill: those
# workloads themselves (the prefill figure is for the unsplit launch).  Valid only for
# the kernel sources a capture was taken on: each entry carries a hash of their
# comment-free text and is reported as null once that changes.
TRAFFIC = {
    "fwd": {"bytes_per_launch": 2 * (208.09e6 + 48.65e6), "workload": "train",
            "sources": ("fwd_kernel.cuh", "schedule.cuh", "sm100.cuh", "dead_rows.cuh"), "sha": "088330ef957fa172"},
    "dot": {"bytes_per_launch": 2 * (135.29e6 + 0.06e6), "workload": "train",
            "sources": ("bwd_kernels.cuh", "schedule.cuh", "sm100.cuh", "dead_rows.cuh"), "sha": "3ba12ef752ee6178"},
    "dkdv": {"bytes_per_launch": 2 * (274.15e6 + 104.73e6), "workload": "train",
             "sources": ("bwd_kernels.cuh", "schedule.cuh", "sm100.cuh", "dead_rows.cuh"), "sha": "3ba12ef752ee6178"},
    "dq": {"bytes_per_launch": 2 * (271.66e6 + 49.75e6), "workload": "train",
           "sources": ("bwd_kernels.cuh", "schedule.cuh", "sm100.cuh", "dead_rows.cuh"), "sha": "3ba12ef752ee6178"},
    "decode": {"bytes_per_launch": 792.83e6 + 4.23e6, "workload": "decode",
               "sources": ("decode_kernel.cuh", "sm100.cuh"), "sha": "5d5936e38ab0d8c6"},
    "fwd_kv": {"bytes_per_launch": 305.29e6 + 23.11e6, "workload": "prefill_kv",
               "sources": ("fwd_kernel.cuh", "schedule.cuh", "sm100.cuh", "dead_rows.cuh"),
               "sha": "088330ef957fa172"},
    "fwd_fp8": {"bytes_per_launch": 2 * (100.94e6 + 34.15e6), "workload": "fp8",
                "sources": ("fwd_kernel.cuh", "schedule.cuh", "sm100.cuh", "dead_rows.cuh"), "sha": "088330ef957fa172"},
}


def strip_comments(text):
    """C/C++ source without its comments and blank lines, trailing spaces
    removed: what the compiler sees, so that a comment edit does not count as
    a kernel change."""
    out, i, n = [], 0, len(text)
    in_str = False
    while i < n:
        c = text[i]
        if in_str:
            out.append(c)
            if c == "\\" and i + 1 < n:
                out.append(text[i + 1])
                i += 2
                continue
            if c == '"':
                in_str = False
            i += 1
        elif c == '"':
            in_str = True
            out.append(c)
            i += 1
        elif text.startswith("//", i):
            while i < n and text[i] != "\n":
                i += 1
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).split("\n"))
    return "\n".join(ln for ln in lines if ln)


def source_hash(files):
    """Hash of the comment-free text of kernel sources under csrc/, or None
    if one is missing."""
    import hashlib
    h = hashlib.sha256()
    try:
        for f in files:
            with open(os.path.join(ROOT, "io_aware_exact_21_b200", "csrc", f), encoding="utf-8") as fh:
                h.update(strip_comments(fh.read()).encode())
    except OSError:
        return None
    return h.hexdigest()[:16]


def traffic_for(kernel, workload="train"):
    """ncu traffic per launch if the kernel's sources still match the capture."""
    t = TRAFFIC.get(kernel)
    if not t or t["workload"] != workload:
        return None
    if source_hash(t["sources"]) != t["sha"]:
        return None
    if workload in ("train", "fp8"):
        w = WORKLOAD
        if (w["B"], w["H"], w["N"], w["d"], w["causal"]) != (4, 16, 8192, 128, False):
            return None
    return t["bytes_per_launch"]


PREFILL_KV = dict(B=4, H=16, Nq=2048, Nk=8192, d=128, causal=True, window=0, seed=5)


def flops_kv(B, H, Nq, Nk, d, causal):
    """Forward FLOPs of Nq queries against Nk keys: 4*d per (query, key) pair
    the mask keeps, with the causal triangle of the last Nq positions halved
    as in the self-attention count."""
    pairs = Nq * Nk - (0.5 * Nq * Nq if causal else 0.0)
    return 4.0 * B * H * pairs * d


def flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    if causal:
        f *= 0.5
    return f, 2.5 * f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(extra=None):
    w = WORKLOAD
    cfg = {"workload": "B%d H%d N%d d%d %s, forward+backward" % (
        w["B"], w["H"], w["N"], w["d"], "causal" if w["causal"] else "non-causal"),
        "B": w["B"], "H": w["H"], "N": w["N"], "d": w["d"], "causal": w["causal"],
        "window": w["window"], "seed": w["seed"],
        "l2": "inputs larger than L2 (Q, K, V, dO 128 MiB each); L2 not flushed"}
    if extra:
        cfg.update(extra)
    return cfg


# ------------------------------------------------- multi-rank helpers ---

def max_over_ranks(values, world, device=None):
    """Element-wise maximum of per-rank timings (every rank gets the result);
    the job is as slow as its slowest rank."""
    if world <= 1:
        return [float(v) for v in values]
    t = torch.tensor(values, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(step_flops, world, steps, elapsed_ms):
    """Whole-job TFLOP/s: the FLOPs all ranks processed over the max-over-ranks time."""
    return step_flops * world * steps / (elapsed_ms * 1e-3) / 1e12


# ------------------------------------------------------------ clocks ---

class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons every 100 ms."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device):
        self.proc = None
        self.lines = []
        self.t = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                 "-lms", "100"] + self.sel, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------- our arm ---

def make_inputs(device, seed):
    from io_aware_exact_21_b200.inputs import fixed_inputs
    w = WORKLOAD
    return fixed_inputs(w["B"], w["N"], w["H"], w["d"], seed=seed, with_dout=True)


def run_ours(args, rank, world, device):
    import io_aware_exact_21_b200 as fa
    w = WORKLOAD
    B, H, N, d, causal, window = w["B"], w["H"], w["N"], w["d"], w["causal"], w["window"]
    scale = 1.0 / math.sqrt(d)
    host = make_inputs(device, w["seed"] + rank)
    q, k, v, do = (host[n].to(device) for n in ("q", "k", "v", "dout"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d, 0), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        fa.forward(q, k, v, causal=causal, window=window, scale=scale, out=o, lse=lse, stream=stream)
        fa.backward(q, k, v, o, lse, do, causal=causal, window=window, scale=scale,
                    grads=(dq, dk, dv), workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    assert fa.fa_get_device_error() == 0

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---- device-resident timed region
    clocks = ClockSampler(device)
    clocks.start()
    barrier()
    torch.cuda.synchronize(device)
    fa.fa_profile_begin()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    elapsed = e0.elapsed_time(e1)
    prof = fa.fa_profile_end()
    fwd_balance, fwd_ctas = fa.fa_profile_cta_balance()
    clk = clocks.stop()
    assert fa.fa_get_device_error() == 0

    # ---- end to end: pinned host inputs in, results back to the host.  Every
    # step copies its Q, K, V, dO from pinned host memory and reads O, LSE, dQ,
    # dK, dV back, as a training loop would; with two device buffer sets and
    # separate copy streams, the copies of one step overlap the compute of the
    # neighbouring steps (stream events keep each buffer's uses in order).
    pin = {n: host[n].pin_memory() for n in ("q", "k", "v", "dout")}
    sets = []
    for b in range(2):
        dev_in = {n: torch.empty_like(q) for n in ("q", "k", "v", "dout")}
        dev_out = {"o": torch.empty_like(q), "lse": torch.empty_like(lse), "dq": torch.empty_like(q),
                   "dk": torch.empty_like(q), "dv": torch.empty_like(q)}
        host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in dev_out.items()}
        sets.append((dev_in, dev_out, host_out))
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in sets[0][2].values())
    s_h2d = torch.cuda.Stream(device)
    s_d2h = torch.cuda.Stream(device)
    comp_done = [torch.cuda.Event() for _ in range(2)]
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    for ev in comp_done + d2h_done:
        ev.record(stream)

    def e2e_step(i):
        dev_in, dev_out, host_out = sets[i % 2]
        b = i % 2
        s_h2d.wait_event(comp_done[b])                 # step i-2 has finished reading the inputs
        with torch.cuda.stream(s_h2d):
            for n in ("q", "k", "v", "dout"):
                dev_in[n].copy_(pin[n], non_blocking=True)
            h2d_done[b].record(s_h2d)
        stream.wait_event(h2d_done[b])
        stream.wait_event(d2h_done[b])                 # step i-2's results have left the device
        fa.forward(dev_in["q"], dev_in["k"], dev_in["v"], causal=causal, window=window, scale=scale,
                   out=dev_out["o"], lse=dev_out["lse"], stream=stream)
        fa.backward(dev_in["q"], dev_in["k"], dev_in["v"], dev_out["o"], dev_out["lse"], dev_in["dout"],
                    causal=causal, window=window, scale=scale,
                    grads=(dev_out["dq"], dev_out["dk"], dev_out["dv"]), workspace=ws, stream=stream)
        comp_done[b].record(stream)
        s_d2h.wait_event(comp_done[b])
        with torch.cuda.stream(s_d2h):
            for n, t in dev_out.items():
                host_out[n].copy_(t, non_blocking=True)
            d2h_done[b].record(s_d2h)

    e2e_steps = max(2, args.steps)
    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize(device)
    barrier()
    torch.cuda.synchronize(device)
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(s_h2d)
    for i in range(e2e_steps):
        e2e_step(i)
    e3.record(s_d2h)
    torch.cuda.synchronize(device)
    barrier()
    e2e_elapsed = e2.elapsed_time(e3)
    assert fa.fa_get_device_error() == 0

    elapsed, e2e_elapsed = max_over_ranks([elapsed, e2e_elapsed], world, device)
    configs = None
    fused = None
    if not args.no_configs:
        del sets, pin
        torch.cuda.empty_cache()
        configs = sweep_configs(device)
        if d == 128:
            fused = time_fused_backward(q, k, v, o, lse, do, causal, window, scale, device)
    if rank != 0:
        return None

    f_fwd, f_bwd = flops(B, H, N, d, causal)
    step_flops = f_fwd + f_bwd
    ms_step = elapsed / args.steps
    value = job_throughput(step_flops, world, args.steps, elapsed)
    e2e_value = job_throughput(step_flops, world, e2e_steps, e2e_elapsed)
    peaks, peak_src = load_peaks()
    per_kernel = {}
    for kind, (ms, cnt) in prof.items():
        per_kernel[kind] = {"ms_per_launch": ms / cnt if cnt else None, "launches": cnt}
    # Per-kernel rooflines.  Algorithmic FLOPs per launch are the GEMMs each
    # kernel executes: forward 4BHN^2d (S and PV); dK/dV kernel 4 GEMMs of
    # 2BHN^2d (S^T, dP^T, dV, dK); dQ kernel 3 (S, dP, dQ); halved under a causal
    # mask.  The pre-pass is HBM-bound: it reads dO, O and LSE and writes the
    # 8-byte statistics, 4d + 12 bytes per (row, head).  The kernels are timed
    # inside a sub-second loop, so the denominator is the measured burst peak.
    kernel_flops = {"fwd": f_fwd, "dkdv": 2.0 * f_fwd, "dq": 1.5 * f_fwd}
    peak_key = "bf16_tflops"
    peak = peaks.get(peak_key, FALLBACK_PEAKS[peak_key])
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    stats_bytes = float(B) * N * H * (4 * d + 12)
    rooflines = {}
    for kk in ("fwd", "dkdv", "dq", "dot"):
        ms = per_kernel[kk]["ms_per_launch"]
        if not ms:
            continue
        if kk == "dot":
            ach = stats_bytes / (ms * 1e-3) / 1e9
            rooflines[kk] = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm,
                             "unit": "GB/s", "frac": round(ach / hbm, 4),
                             "algorithmic": stats_bytes, "ms": round(ms, 4),
                             "traffic": traffic_for(kk)}
        else:
            ach = kernel_flops[kk] / (ms * 1e-3) / 1e12
            rooflines[kk] = {"bound": "tensor", "achieved": round(ach, 2), "peak": peak,
                             "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                             "algorithmic": kernel_flops[kk], "ms": round(ms, 4),
                             "traffic": traffic_for(kk)}
    # dominant kernel: the largest device time per step
    dom = max(("fwd", "dkdv", "dq"), key=lambda kk: prof[kk][0])
    achieved = rooflines[dom]["achieved"]
    t_fwd = per_kernel["fwd"]["ms_per_launch"]
    t_bwd = sum(per_kernel[kk]["ms_per_launch"] or 0.0 for kk in ("dot", "dkdv", "dq"))
    burst = peak
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: i.i.d. N(0,1) bf16 Q, K, V, dO (seeded), no dataset",
        "config": workload_config({"parallelism": "replicas" if world > 1 else "single GPU"}),
        "fwd": {"ms": round(t_fwd, 4), "tflops": round(f_fwd / (t_fwd * 1e-3) / 1e12, 2),
                "cta_balance": round(fwd_balance, 4),
                "frac_of_measured_burst_peak": round(f_fwd / (t_fwd * 1e-3) / 1e12 / burst, 4),
                "frac_of_nominal_dense_peak": round(f_fwd / (t_fwd * 1e-3) / 1e12
                                                    / NOMINAL_BF16_DENSE_TFLOPS, 4)},
        "bwd": {"ms": round(t_bwd, 4), "tflops": round(f_bwd / (t_bwd * 1e-3) / 1e12, 2),
                "frac_of_measured_burst_peak": round(f_bwd / (t_bwd * 1e-3) / 1e12 / burst, 4),
                "frac_of_nominal_dense_peak": round(f_bwd / (t_bwd * 1e-3) / 1e12
                                                    / NOMINAL_BF16_DENSE_TFLOPS, 4),
                "kernels_ms": {kk: round(per_kernel[kk]["ms_per_launch"] or 0.0, 4)
                               for kk in ("dot", "dkdv", "dq")}},
        "roofline": {"kernel": dom, "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4),
                     "peak_source": "%s %s (burst: kernels timed inside a sub-second loop)"
                                    % (peak_src, peak_key),
                     "traffic": traffic_for(dom),
                     "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "roofline_kernels": rooflines,
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "pinned host -> device copy of Q, K, V, dO and device -> host copy of O, LSE, "
                       "dQ, dK, dV every step, on copy streams overlapping the neighbouring steps' "
                       "compute (two device buffer sets)"},
        "gpu_launches": sum(c for (_, c) in prof.values()),
        "clocks": clk,
        "configs": configs,
        "bwd_fused_prototype": fused,
    }
    if fused:
        fused["tflops"] = round(f_bwd / (fused["ms"] * 1e-3) / 1e12, 2)
        fused["vs_two_kernel_backward"] = round(t_bwd / fused["ms"], 4)
    return out


# ------------------------------------------- the other parity workloads ---

# Device-timed throughput of the other workloads of the parity contract, on the
# same line as the headline: (label, workload name, mask override).
SWEEP = [
    ("2 training B4 H16 N2048 non-causal", "train"),
    ("2 training B4 H16 N2048 causal", "train_causal"),
    ("3a prefill B2 H16 N8192 causal", "prefill_b2_causal"),
    ("3b prefill B4 H16 N8192 causal", "prefill_b4_causal"),
    ("4 packed 16 seqs H32 causal", "varlen_causal"),
    ("4 packed 16 seqs H32 causal window 1024", "varlen_window"),
    ("5 backward B2 H16 N4096 causal", "bwd_causal"),
]


def allowed_pairs(n, causal, window):
    """(query, key) pairs the mask keeps in one sequence of n tokens.  Causal
    without a window uses n^2 / 2, the convention of the fixed-length count;
    a window counts the pairs exactly, sum over rows r of min(r + 1, W)."""
    n = int(n)
    if not causal:
        return float(n) * n
    if window <= 0:
        return 0.5 * n * n
    w = int(window)
    if n <= w:
        return n * (n + 1) / 2.0
    return w * (w + 1) / 2.0 + float(n - w) * w


def workload_flops(wl, lens):
    """Forward FLOPs (4d per allowed pair) and backward FLOPs (2.5x)."""
    pairs = sum(allowed_pairs(n, wl.causal, wl.window) for n in lens)
    f = 4.0 * wl.H * wl.d * pairs
    return f, 2.5 * f


def time_fused_backward(q, k, v, o, lse, do, causal, window, scale, device, reps=10, warmup=3):
    """The single-kernel backward (fa_bwd_fused) on the same inputs: pre-pass,
    fused kernel and dQ conversion, per-kernel CUDA events, mean over reps."""
    import io_aware_exact_21_b200 as fa
    stream = torch.cuda.current_stream(device)
    B, N, H, d = q.shape
    ws = torch.empty(fa.fa_bwd_fused_workspace_size(B, H, N, d, 0), dtype=torch.uint8, device=device)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))

    def step():
        fa.backward(q, k, v, o, lse, do, causal=causal, window=window, scale=scale, grads=grads,
                    workspace=ws, stream=stream, fused=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    fa.fa_profile_begin()
    for _ in range(reps):
        step()
    torch.cuda.synchronize(device)
    prof = fa.fa_profile_end()
    assert fa.fa_get_device_error() == 0
    ms = {kk: prof[kk][0] / prof[kk][1] for kk in ("dot", "bwd_fused", "dq_convert")}
    return {"ms": round(sum(ms.values()), 4), "kernels_ms": {kk: round(v, 4) for kk, v in ms.items()},
            "how": "fa_bwd_fused: pre-pass (statistics, zeroed fp32 dQ accumulator), one kernel for "
                   "dK, dV and the dQ parts (five GEMMs per tile pair, dQ parts added by bulk fp32 "
                   "reductions), dQ conversion; same inputs as the timed step"}


def sweep_configs(device, reps=10, warmup=3):
    """fwd and bwd TFLOP/s of each SWEEP workload: per-kernel CUDA events
    (fa_profile) around every launch, mean over `reps` calls after `warmup`."""
    import io_aware_exact_21_b200 as fa
    from io_aware_exact_21_b200.inputs import WORKLOADS, fixed_inputs, varlen_inputs
    peaks, _ = load_peaks()
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    stream = torch.cuda.current_stream(device)
    out = {}
    for label, name in SWEEP:
        wl = WORKLOADS[name]
        if wl.varlen is not None:
            nseq, lo, hi = wl.varlen
            host = varlen_inputs(nseq, lo, hi, wl.H, wl.d, wl.seed, with_dout=True)
            cu_h = host["cu_seqlens"]
            lens = [int(x) for x in (cu_h[1:] - cu_h[:-1])]
            cu = cu_h.to(device)
        else:
            host = fixed_inputs(wl.B, wl.N, wl.H, wl.d, wl.seed, with_dout=True)
            lens = [wl.N] * wl.B
            cu = None
        q, k, v, do = (host[n].to(device) for n in ("q", "k", "v", "dout"))
        o, lse = fa.forward(q, k, v, causal=wl.causal, window=wl.window, cu_seqlens=cu,
                            stream=stream)
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))

        def step():
            fa.forward(q, k, v, causal=wl.causal, window=wl.window, cu_seqlens=cu, out=o, lse=lse,
                       stream=stream)
            fa.backward(q, k, v, o, lse, do, causal=wl.causal, window=wl.window, cu_seqlens=cu,
                        grads=grads, stream=stream)

        for _ in range(warmup):
            step()
        torch.cuda.synchronize(device)
        fa.fa_profile_begin()
        for _ in range(reps):
            step()
        torch.cuda.synchronize(device)
        prof = fa.fa_profile_end()
        balance, ctas = fa.fa_profile_cta_balance()
        assert fa.fa_get_device_error() == 0
        ms = {kk: prof[kk][0] / prof[kk][1] for kk in ("fwd", "dot", "dkdv", "dq")}
        f_fwd, f_bwd = workload_flops(wl, lens)
        t_bwd = ms["dot"] + ms["dkdv"] + ms["dq"]
        tf_f = f_fwd / (ms["fwd"] * 1e-3) / 1e12
        tf_b = f_bwd / (t_bwd * 1e-3) / 1e12
        out[label] = {"fwd_ms": round(ms["fwd"], 4), "fwd_tflops": round(tf_f, 1),
                      "fwd_frac_of_measured_burst": round(tf_f / burst, 4),
                      "bwd_ms": round(t_bwd, 4), "bwd_tflops": round(tf_b, 1),
                      "bwd_frac_of_measured_burst": round(tf_b / burst, 4),
                      "kernels_ms": {kk: round(v, 4) for kk, v in ms.items()},
                      "fwd_cta_balance": round(balance, 4), "fwd_ctas": ctas,
                      "fwd_flops": f_fwd, "tokens": sum(lens)}
        del q, k, v, do, o, lse, grads, host
        torch.cuda.empty_cache()
    return out


# ------------------------------------------- cached-KV prefill arm ---

def prefill_kv_config(extra=None):
    w = PREFILL_KV
    cfg = {"workload": "cached-KV prefill B%d H%d Nq%d Nk%d d%d %s (bottom-right), forward only"
           % (w["B"], w["H"], w["Nq"], w["Nk"], w["d"], "causal" if w["causal"] else "non-causal"),
           "B": w["B"], "H": w["H"], "Nq": w["Nq"], "Nk": w["Nk"], "d": w["d"],
           "causal": w["causal"], "window": w["window"], "seed": w["seed"],
           "l2": "inputs larger than L2 (K, V 128 MiB each); L2 not flushed"}
    if extra:
        cfg.update(extra)
    return cfg


def run_prefill_kv(args, rank, world, device):
    import io_aware_exact_21_b200 as fa
    from io_aware_exact_21_b200.inputs import kv_inputs
    w = PREFILL_KV
    B, H, Nq, Nk, d = w["B"], w["H"], w["Nq"], w["Nk"], w["d"]
    causal, window = w["causal"], w["window"]
    scale = 1.0 / math.sqrt(d)
    host = kv_inputs(B, Nq, Nk, H, d, seed=w["seed"] + rank)
    q, k, v = (host[n].to(device) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    # through the cache interface, split along the keys as the library chooses
    ns = fa.fa_fwd_kvcache_num_splits(B, H, Nq, Nk, d)
    ws = torch.empty(max(16, fa.fa_fwd_kvcache_workspace_size(B, H, Nq, d, ns)), dtype=torch.uint8,
                     device=device)

    def step(qq, kk, vv, oo, ll):
        fa.forward_kvcache(qq, kk, vv, causal=causal, window=window, scale=scale, num_splits=ns,
                           out=oo, lse=ll, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step(q, k, v, o, lse)
    torch.cuda.synchronize(device)
    assert fa.fa_get_device_error() == 0

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    clocks = ClockSampler(device)
    clocks.start()
    barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(q, k, v, o, lse)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    elapsed = e0.elapsed_time(e1)
    clk = clocks.stop()
    # per-kernel times: the same steps once more with an event pair around
    # every launch, kept out of the timed region above (on a call of a tenth
    # of a millisecond the extra events would show in its time)
    fa.fa_profile_begin()
    for _ in range(args.steps):
        step(q, k, v, o, lse)
    torch.cuda.synchronize(device)
    prof = fa.fa_profile_end()
    assert fa.fa_get_device_error() == 0

    # end to end: the cached keys and values stay resident, as in serving;
    # each step copies the chunk's own inputs in from pinned host memory -- its
    # Nq queries and the keys and values of those Nq new tokens, the last Nq
    # rows of each sequence's cache slice (one contiguous copy per sequence) --
    # and O, LSE back, in order on one stream (no overlap between steps)
    pin_q = host["q"].pin_memory()
    pin_kv = {n: host[n][:, Nk - Nq:].contiguous().pin_memory() for n in ("k", "v")}
    dev_q = torch.empty_like(q)
    dev_kv = {n: t.clone() for n, t in (("k", k), ("v", v))}
    host_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    host_l = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = pin_q.numel() * pin_q.element_size() + sum(t.numel() * t.element_size() for t in pin_kv.values())
    d2h = host_o.numel() * host_o.element_size() + host_l.numel() * host_l.element_size()

    def e2e_step():
        dev_q.copy_(pin_q, non_blocking=True)
        for n in ("k", "v"):
            for b in range(B):
                dev_kv[n][b, Nk - Nq:].copy_(pin_kv[n][b], non_blocking=True)
        step(dev_q, dev_kv["k"], dev_kv["v"], o, lse)
        host_o.copy_(o, non_blocking=True)
        host_l.copy_(lse, non_blocking=True)

    e2e_steps = max(2, args.steps)
    e2e_step()
    torch.cuda.synchronize(device)
    barrier()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e3.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_elapsed = e2.elapsed_time(e3)
    assert fa.fa_get_device_error() == 0

    elapsed, e2e_elapsed = max_over_ranks([elapsed, e2e_elapsed], world, device)
    if rank != 0:
        return None
    f = flops_kv(B, H, Nq, Nk, d, causal)
    value = job_throughput(f, world, args.steps, elapsed)
    ms, cnt = prof["fwd"]
    kernel_ms = ms / cnt
    merge_ms = prof["combine"][0] / prof["combine"][1] if prof["combine"][1] else 0.0
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    achieved = f / (kernel_ms * 1e-3) / 1e12
    return {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(elapsed / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: i.i.d. N(0,1) bf16 Q, K, V (seeded), no dataset",
        "config": prefill_kv_config({"parallelism": "replicas" if world > 1 else "single GPU",
                                     "num_splits": ns, "api": "fa_fwd_kvcache"}),
        "kernels_ms": {"fwd": round(kernel_ms, 4), "merge": round(merge_ms, 4)},
        "roofline": {"kernel": "fwd", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": "%s bf16_tflops (burst: the kernel is timed alone)" % peak_src,
                     "traffic": traffic_for("fwd_kv", "prefill_kv") if ns == 1 else None,
                     "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "e2e": {"value": round(job_throughput(f, world, e2e_steps, e2e_elapsed), 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "cache resident; pinned host -> device copy of the chunk's queries and of "
                       "its new tokens' keys and values (the last Nq rows of each sequence's "
                       "cache slice) and device -> host copy of O, LSE every step, in order on "
                       "the compute stream"},
        "gpu_launches": sum(c for (_, c) in prof.values()),
        "clocks": clk,
    }


# ------------------------------------------------------------ decode arm ---

DECODE_UNIT = "GB/s"
DECODE_METRIC = "attention decode: K/V-cache bytes read per second (BF16, d=128), % of measured HBM bandwidth"


def decode_workload():
    from io_aware_exact_21_b200.inputs import WORKLOADS
    return WORKLOADS["decode"]


def decode_bytes(wl, lens):
    """Algorithmic HBM bytes of one decode call: the used K and V rows of every
    (sequence, head), plus Q read and O, LSE written."""
    kv = 2 * int(sum(int(n) for n in lens)) * wl.H * wl.d * 2
    qo = 2 * wl.B * wl.N * wl.H * wl.d * 2 + wl.B * wl.H * wl.N * 4
    return kv + qo


def decode_config(wl, extra=None):
    cfg = {"workload": "decode B%d H%d Nq%d cache %d..%d of %d rows d%d, bottom-right causal" % (
        wl.B, wl.H, wl.N, wl.cache_lens[0], wl.cache_lens[1], wl.Nk, wl.d),
        "B": wl.B, "H": wl.H, "Nq": wl.N, "Nk": wl.Nk, "cache_lens": list(wl.cache_lens),
        "d": wl.d, "causal": wl.causal, "seed": wl.seed,
        "l2": "cache larger than L2 (K, V about 400 MB each); L2 not flushed"}
    if extra:
        cfg.update(extra)
    return cfg


def run_decode(args, rank, world, device):
    import io_aware_exact_21_b200 as fa
    wl = decode_workload()
    host = wl.make()
    q, k, v = (host[n].to(device) for n in ("q", "k", "v"))
    lens = host["seqlens_k"].to(device)
    B, H, Nq, Nk, d = wl.B, wl.H, wl.N, wl.Nk, wl.d
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=device)
    ns = fa.fa_fwd_kvcache_num_splits(B, H, Nq, Nk, d)
    ws = torch.empty(max(16, fa.fa_fwd_kvcache_workspace_size(B, H, Nq, d, ns)), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.current_stream(device)

    def step(qq, ll, oo, ls):
        fa.forward_kvcache(qq, k, v, seqlens_k=ll, causal=wl.causal, window=wl.window,
                           num_splits=ns, out=oo, lse=ls, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step(q, lens, o, lse)
    torch.cuda.synchronize(device)
    assert fa.fa_get_device_error() == 0

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    clocks = ClockSampler(device)
    clocks.start()
    barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(q, lens, o, lse)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    elapsed = e0.elapsed_time(e1)
    clk = clocks.stop()
    # per-kernel times: the same steps once more with an event pair around
    # every launch, kept out of the timed region above (on a call of a tenth
    # of a millisecond the extra events would show in its time)
    fa.fa_profile_begin()
    for _ in range(args.steps):
        step(q, lens, o, lse)
    torch.cuda.synchronize(device)
    prof = fa.fa_profile_end()
    assert fa.fa_get_device_error() == 0

    # end to end: per step the new query and the cache lengths come from pinned
    # host memory and O, LSE go back (the cache stays resident, as in decoding)
    pin_q = host["q"].pin_memory()
    pin_l = host["seqlens_k"].pin_memory()
    dq_in = torch.empty_like(q)
    dl_in = torch.empty_like(lens)
    host_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    host_l = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = pin_q.numel() * pin_q.element_size() + pin_l.numel() * pin_l.element_size()
    d2h = host_o.numel() * host_o.element_size() + host_l.numel() * host_l.element_size()

    def e2e_step():
        dq_in.copy_(pin_q, non_blocking=True)
        dl_in.copy_(pin_l, non_blocking=True)
        step(dq_in, dl_in, o, lse)
        host_o.copy_(o, non_blocking=True)
        host_l.copy_(lse, non_blocking=True)

    e2e_steps = max(2, args.steps)
    e2e_step()
    torch.cuda.synchronize(device)
    barrier()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e3.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_elapsed = e2.elapsed_time(e3)
    assert fa.fa_get_device_error() == 0

    elapsed, e2e_elapsed = max_over_ranks([elapsed, e2e_elapsed], world, device)
    if rank != 0:
        return None
    nbytes = decode_bytes(wl, host["seqlens_k"].tolist())
    value = nbytes * world * args.steps / (elapsed * 1e-3) / 1e9
    e2e_value = nbytes * world * e2e_steps / (e2e_elapsed * 1e-3) / 1e9
    dec_ms, dec_n = prof["decode"]
    cmb_ms, cmb_n = prof["combine"]
    kernel_ms = dec_ms / dec_n
    peaks, peak_src = load_peaks()
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    # the decode kernel reads the K/V rows and Q; the merge kernel the partials
    dec_bytes = nbytes - B * H * Nq * (d * 2 + 4)
    achieved = dec_bytes / (kernel_ms * 1e-3) / 1e9
    return {
        "metric": DECODE_METRIC, "value": round(value, 1), "unit": DECODE_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(elapsed / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: i.i.d. N(0,1) bf16 Q, K/V cache (seeded), cache lengths seeded uniform",
        "config": decode_config(wl, {"parallelism": "replicas" if world > 1 else "single GPU",
                                     "num_splits": ns}),
        "kernels_ms": {"decode": round(kernel_ms, 5),
                       "merge": round(cmb_ms / cmb_n, 5) if cmb_n else None},
        "roofline": {"kernel": "decode", "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_source": "%s hbm_gbs (copy bandwidth)" % peak_src,
                     "traffic": traffic_for("decode", "decode"),
                     "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "e2e": {"value": round(e2e_value, 1), "unit": DECODE_UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "pinned host -> device copy of the new queries and cache lengths, device -> "
                       "host copy of O and LSE every step, in order on the compute stream; the "
                       "cache stays resident"},
        "gpu_launches": sum(c for (_, c) in prof.values()),
        "clocks": clk,
    }


def oracle_sample_decode(x=None):
    """The float64 oracle's decode on the whole decode workload (its inputs
    made here unless given)."""
    from oracle import oracle as orc
    wl = decode_workload()
    if x is None:
        x = wl.make()
    t0 = time.perf_counter()
    orc.fwd_kvcache(x["q"], x["k"], x["v"], wl.scale, seqlens_k=x["seqlens_k"],
                    causal=wl.causal, window=wl.window)
    secs = time.perf_counter() - t0
    nbytes = decode_bytes(wl, x["seqlens_k"].tolist())
    desc = ("decode of the whole workload (B%d H%d, caches %d..%d): %.2f s on %d threads"
            % (wl.B, wl.H, wl.cache_lens[0], wl.cache_lens[1], secs, orc.num_threads()))
    return nbytes / secs / 1e9, desc, orc.num_threads(), secs


# --------------------------------------------------------------- FP8 arm ---

FP8_METRIC = "attention FP8 (block-quantised e4m3) forward TFLOPs/s (d=128), % of B200 dense FP8 peak"


def fp8_config(extra=None):
    w = WORKLOAD
    cfg = {"workload": "FP8 forward B%d H%d N%d d%d non-causal, e4m3 with 128-row block scales and "
                       "the Hadamard rotation of Q and K; quantisation included" % (
                           w["B"], w["H"], w["N"], w["d"]),
           "B": w["B"], "H": w["H"], "N": w["N"], "d": w["d"], "causal": False, "seed": w["seed"],
           "l2": "inputs larger than L2 (Q, K, V 128 MiB each in bf16); L2 not flushed"}
    if extra:
        cfg.update(extra)
    return cfg


def run_fp8(args, rank, world, device):
    import io_aware_exact_21_b200 as fa
    from io_aware_exact_21_b200.inputs import fp8_signs
    w = WORKLOAD
    B, H, N, d = w["B"], w["H"], w["N"], w["d"]
    host = make_inputs(device, w["seed"] + rank)
    q, k, v = (host[n].to(device) for n in ("q", "k", "v"))
    signs = fp8_signs(1).to(device)
    stream = torch.cuda.current_stream(device)
    qz = fa.quantize_fp8(q, k, v, signs, stream=stream)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=device)

    def step(qq, kk, vv, oo, ll):
        fa.fa_quantize_fp8(qq, qz["q8"], qz["sq"], B, N, H, d, 0, signs, stream)
        fa.fa_quantize_fp8(kk, qz["k8"], qz["sk"], B, N, H, d, 0, signs, stream)
        fa.fa_quantize_fp8(vv, qz["vt8"], qz["sv"], B, N, H, d, 1, None, stream)
        fa.forward_fp8(qz, B, N, H, d, out=oo, lse=ll, stream=stream)

    for _ in range(args.warmup):
        step(q, k, v, o, lse)
    torch.cuda.synchronize(device)
    assert fa.fa_get_device_error() == 0

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    clocks = ClockSampler(device)
    clocks.start()
    barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(q, k, v, o, lse)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    elapsed = e0.elapsed_time(e1)
    clk = clocks.stop()
    # per-kernel times: the same steps once more with an event pair around
    # every launch, kept out of the timed region above (on a call of a tenth
    # of a millisecond the extra events would show in its time)
    fa.fa_profile_begin()
    for _ in range(args.steps):
        step(q, k, v, o, lse)
    torch.cuda.synchronize(device)
    prof = fa.fa_profile_end()
    assert fa.fa_get_device_error() == 0

    pin = {n: host[n].pin_memory() for n in ("q", "k", "v")}
    dev_in = {n: torch.empty_like(q) for n in pin}
    host_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    host_l = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = host_o.numel() * host_o.element_size() + host_l.numel() * host_l.element_size()

    def e2e_step():
        for n in ("q", "k", "v"):
            dev_in[n].copy_(pin[n], non_blocking=True)
        step(dev_in["q"], dev_in["k"], dev_in["v"], o, lse)
        host_o.copy_(o, non_blocking=True)
        host_l.copy_(lse, non_blocking=True)

    e2e_steps = max(2, args.steps)
    e2e_step()
    torch.cuda.synchronize(device)
    barrier()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e3.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_elapsed = e2.elapsed_time(e3)
    assert fa.fa_get_device_error() == 0

    elapsed, e2e_elapsed = max_over_ranks([elapsed, e2e_elapsed], world, device)
    if rank != 0:
        return None
    f, _ = flops(B, H, N, d, False)
    value = job_throughput(f, world, args.steps, elapsed)
    fwd_ms = prof["fwd_fp8"][0] / prof["fwd_fp8"][1]
    quant_ms = prof["quant_fp8"][0] / max(1, prof["quant_fp8"][1]) * 3
    peaks, peak_src = load_peaks()
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak = 2.0 * burst
    achieved = f / (fwd_ms * 1e-3) / 1e12
    return {
        "metric": FP8_METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(elapsed / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic: i.i.d. N(0,1) bf16 Q, K, V (seeded), no dataset",
        "config": fp8_config({"parallelism": "replicas" if world > 1 else "single GPU"}),
        "kernels_ms": {"quantise_q_k_v": round(quant_ms, 4), "fwd_fp8": round(fwd_ms, 4)},
        "roofline": {"kernel": "fwd_fp8", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": "%s bf16_tflops (burst) x 2, the nominal FP8:BF16 dense ratio"
                                    % peak_src,
                     "frac_of_nominal_dense_peak": round(achieved / (2.0 * NOMINAL_BF16_DENSE_TFLOPS), 4),
                     "traffic": traffic_for("fwd_fp8", "fp8"),
                     "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "e2e": {"value": round(job_throughput(f, world, e2e_steps, e2e_elapsed), 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "pinned host -> device copy of bf16 Q, K, V, quantisation, FP8 forward, "
                       "device -> host copy of O and LSE every step, in order on one stream"},
        "gpu_launches": sum(c for (_, c) in prof.values()),
        "clocks": clk,
    }


def oracle_sample_fp8(n_tokens=8192, seed=2):
    """The oracle's FP8 path (quantise Q, K, V with the rotation, then the
    block-quantised forward) on one (sequence, head) of the workload,
    truncated to n_tokens."""
    from oracle import oracle as orc
    from io_aware_exact_21_b200.inputs import fixed_inputs, fp8_signs
    d = WORKLOAD["d"]
    x = fixed_inputs(1, n_tokens, 1, d, seed=seed)
    signs = fp8_signs(1)
    t0 = time.perf_counter()
    qc, sq = orc.quantize_fp8(x["q"], signs)
    kc, sk = orc.quantize_fp8(x["k"], signs)
    vc, sv = orc.quantize_fp8(x["v"])
    orc.fwd_fp8(qc, kc, vc, sq, sk, sv, 1.0 / math.sqrt(d))
    secs = time.perf_counter() - t0
    f, _ = flops(1, 1, n_tokens, d, False)
    desc = ("FP8 path of one (sequence, head) of the workload truncated to %d tokens, d=%d: "
            "%.1f s on %d threads" % (n_tokens, d, secs, orc.num_threads()))
    return f / secs / 1e12, desc, orc.num_threads(), secs


def oracle_sample_kv(n_q=None, seed=5):
    """Time the float64 oracle's cached-KV forward on one (sequence, head) of
    the prefill workload, optionally with fewer queries (the key length and
    the queries' positions at its end are kept)."""
    from oracle import oracle as orc
    from io_aware_exact_21_b200.inputs import kv_inputs
    w = PREFILL_KV
    nq = n_q or w["Nq"]
    x = kv_inputs(1, nq, w["Nk"], 1, w["d"], seed=seed)
    t0 = time.perf_counter()
    orc.fwd_kv(x["q"], x["k"], x["v"], 1.0 / math.sqrt(w["d"]), causal=w["causal"],
               window=w["window"])
    secs = time.perf_counter() - t0
    f = flops_kv(1, 1, nq, w["Nk"], w["d"], w["causal"])
    desc = ("cached-KV forward of one (sequence, head) of the prefill workload: %d queries, "
            "%d keys, d=%d, %.1f s on %d threads" % (nq, w["Nk"], w["d"], secs, orc.num_threads()))
    return f / secs / 1e12, desc, orc.num_threads(), secs


# ------------------------------------------------- CPU oracle (sample) ---

def oracle_sample(n_tokens=None, seed=2):
    """Time the float64 oracle on a bounded sample of the workload: one
    (sequence, head) of the B4 H16 N8192 d128 problem -- its forward and
    backward (the oracle's backward recomputes the forward) -- optionally
    truncated to `n_tokens` tokens.  Returns (algorithmic TFLOP/s, sample
    description, threads, seconds)."""
    from oracle import oracle as orc
    from io_aware_exact_21_b200.inputs import fixed_inputs
    w = WORKLOAD
    d = w["d"]
    n = n_tokens or w["N"]
    scale = 1.0 / math.sqrt(d)
    x = fixed_inputs(1, n, 1, d, seed=seed, with_dout=True)
    t0 = time.perf_counter()
    orc.bwd(x["q"], x["k"], x["v"], x["dout"], scale, causal=w["causal"], window=w["window"])
    secs = time.perf_counter() - t0
    f_fwd, f_bwd = flops(1, 1, n, d, w["causal"])
    desc = ("forward + backward of one (sequence, head) of the workload%s: %d tokens, d=%d, "
            "%.1f s on %d threads" % ("" if n == w["N"] else " truncated", n, d, secs,
                                      orc.num_threads()))
    return (f_fwd + f_bwd) / secs / 1e12, desc, orc.num_threads(), secs


CPU_SAMPLE_MIN_S = 10.0


def cpu_baseline_sample(workload, min_secs=CPU_SAMPLE_MIN_S, max_reps=64):
    """The cpu_baseline leg: the workload's oracle sample, repeated (a new
    input seed each time, where the sample takes one) until at least
    min_secs of host time have been spent.  Returns (rate over all samples,
    description, threads)."""
    work = total = 0.0
    reps = 0
    first = threads = None
    dec_inputs = decode_workload().make() if workload == "decode" else None
    while reps < max_reps and (reps == 0 or total < min_secs):
        if workload == "train":
            val, desc, threads, secs = oracle_sample(seed=2 + reps)
        elif workload == "prefill_kv":
            val, desc, threads, secs = oracle_sample_kv(seed=5 + reps)
        elif workload == "fp8":
            val, desc, threads, secs = oracle_sample_fp8(seed=2 + reps)
        else:
            val, desc, threads, secs = oracle_sample_decode(dec_inputs)
        work += val * secs
        total += secs
        reps += 1
        first = first or desc
    desc = "%s; %d such sample%s%s, %.1f s in total" % (
        first, reps, "s" if reps > 1 else "",
        "" if workload == "decode" else " (input seed +1 each)", total)
    return work / total, desc, threads


def run_reference(args):
    """Reference arm: the float64 CPU oracle as it stands, timed on the host
    cores, one bounded sample of the workload per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    if args.workload == "decode":
        for _ in range(args.warmup):
            oracle_sample_decode()
        vals = []
        t0 = time.perf_counter()
        for _ in range(args.steps):
            val, desc, threads, _ = oracle_sample_decode()
            vals.append(val)
        elapsed = time.perf_counter() - t0
        value = statistics.mean(vals)
        return {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT,
                "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": elapsed * 1e3 / max(1, args.steps),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic: i.i.d. N(0,1) bf16 inputs upcast to float64",
                "config": decode_config(decode_workload(), {"parallelism": "host cores"}),
                "cpu_baseline": {"value": value, "unit": DECODE_UNIT, "cores": threads,
                                 "kind": "oracle", "sample": desc},
                "e2e": {"value": value, "unit": DECODE_UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    if args.workload == "fp8":
        for _ in range(args.warmup):
            oracle_sample_fp8(n_tokens=256)
        vals = []
        t0 = time.perf_counter()
        for _ in range(args.steps):
            val, desc, threads, _ = oracle_sample_fp8(n_tokens=1024)
            vals.append(val)
        elapsed = time.perf_counter() - t0
        value = statistics.mean(vals)
        return {"impl": "reference", "metric": FP8_METRIC, "value": value, "unit": UNIT,
                "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": elapsed * 1e3 / max(1, args.steps),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic: i.i.d. N(0,1) bf16 inputs; codes emulated in float32, "
                        "forward in float64",
                "config": fp8_config({"parallelism": "host cores"}),
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    kv = args.workload == "prefill_kv"
    for _ in range(args.warmup):
        if kv:
            oracle_sample_kv(n_q=16)
        else:
            oracle_sample(n_tokens=256)
    vals = []
    t0 = time.perf_counter()
    desc = threads = None
    for _ in range(args.steps):
        val, desc, threads, _ = oracle_sample_kv(n_q=256) if kv else oracle_sample(n_tokens=2048)
        vals.append(val)
    elapsed = time.perf_counter() - t0
    value = statistics.mean(vals)
    cfg = (prefill_kv_config if kv else workload_config)({"parallelism": "host cores"})
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed * 1e3 / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: i.i.d. N(0,1) bf16 inputs upcast to float64", "config": cfg,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing (used for profiling runs)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the sweep of the other parity workloads (train workload)")
    ap.add_argument("--shape", default=None,
                    help="B,H,N,d override of the workload (profiling of smaller cases)")
    ap.add_argument("--causal", action="store_true", help="causal mask (profiling)")
    ap.add_argument("--workload", choices=["train", "prefill_kv", "decode", "fp8"], default="train",
                    help="train: forward+backward step (default); prefill_kv: cached-KV "
                         "prefill forward; decode: decode against a K/V cache; fp8: the "
                         "block-quantised FP8 forward")
    args = ap.parse_args()
    if args.shape:
        B, H, N, d = (int(x) for x in args.shape.split(","))
        WORKLOAD.update(B=B, H=H, N=N, d=d)
    if args.causal:
        WORKLOAD.update(causal=True)
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        out = run_reference(args)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=device)
    runner = {"train": run_ours, "prefill_kv": run_prefill_kv, "decode": run_decode,
              "fp8": run_fp8}[args.workload]
    try:
        out = runner(args, rank, world, device)
        if out is not None:
            if not args.no_cpu_baseline and world == 1:
                val, desc, threads = cpu_baseline_sample(args.workload)
                out["cpu_baseline"] = {"value": val, "unit": out["unit"], "cores": threads,
                                       "kind": "oracle", "sample": desc}
            else:
                out["cpu_baseline"] = None
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
