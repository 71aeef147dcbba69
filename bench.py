"""Benchmark of the fused window-attention forward on B200.

One step = one pass of the whole hot path over one batch: the workload's
winattn_fwd call(s) (two calls, unshifted then shifted, for workloads that
alternate).  Default workload: the Swin-T stage-1 shape (B=64, 56x56 tokens,
3 heads of d=32, M=8 windows shifted by 4, bf16, learned 2D RoPE).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...      # the fp64 CPU oracle, bounded sample

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch (weak
scaling, no collective on the data path); the timed region is bracketed by a
barrier and the time is the max over ranks.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "window-attn fwd TFLOP/s & tokens/s on 1 B200 vs M; % of roofline"
L2_BYTES = 126 * 2**20
_CSRC = "windowed_attention_vision_b200/csrc/"
_COMMON = [_CSRC + "ptx.cuh", _CSRC + "geometry.cuh", _CSRC + "waits.cuh"]
# kernel id of winattn_launch_info -> (name used in profiles/, source files whose change voids a capture)
KERNELS = {0: ("tc", [_CSRC + "fwd_tc.cuh"] + _COMMON), 1: ("small", [_CSRC + "fwd_small.cuh"] + _COMMON),
           2: ("large", [_CSRC + "fwd_large.cuh"] + _COMMON), 3: ("simt", [_CSRC + "fwd_simt.cuh"] + _COMMON),
           4: ("pipe", [_CSRC + "fwd_pipe.cuh", _CSRC + "fwd_small.cuh"] + _COMMON),
           5: ("pipe16", [_CSRC + "fwd_pipe16.cuh", _CSRC + "fwd_pipe.cuh", _CSRC + "fwd_large.cuh",
                          _CSRC + "fwd_small.cuh"] + _COMMON)}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="swin")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-m", action="store_true", help="skip the per-M table (sweep, dense and SR calls)")
    return ap.parse_args()


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def kernel_source_hash(files) -> str:
    h = hashlib.sha256()
    for p in files:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def kernel_of(w):
    """(profile name, source files) of the kernel the library picks for the
    workload's last call."""
    from windowed_attention_vision_b200 import _lib
    dt = _lib.BF16 if w.dtype == "bf16" else _lib.FP32
    rc, info = _lib.launch_info(w.B, w.H, w.W, w.M, w.shifts[-1], w.heads, w.d, w.rank, dt)
    return KERNELS.get(info["kernel"], ("unknown", _COMMON)) if rc == 0 else ("unknown", _COMMON)


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def recorded_traffic(w):
    """DRAM bytes (read + write) per launch of the workload's kernel from the
    committed ncu summary ``profiles/winattn_fwd_<kernel>_<workload>.md``, or
    None when there is none or it was taken on a different kernel source."""
    name, files = kernel_of(w)
    path = os.path.join(ROOT, "profiles", f"winattn_fwd_{name}_{w.name}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    if not m_bytes or not m_hash or m_hash.group(1) != kernel_source_hash(files):
        return None
    return float(m_bytes.group(1))


# ----------------------------------------------------------------- clocks (NVML)

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, torch_device_index: int, period_s: float = 0.002):
        self.ok = False
        self.samples = []
        self.period = period_s
        self.marks = {}
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device_index)
            handle = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    handle = None
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.nvml, self.h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)

    def _reasons(self):
        try:
            return self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nvml.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(),
                                     self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM),
                                     self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def mark(self, name):
        self.marks[name] = time.perf_counter()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "NVML unavailable"}
        t0, t1 = self.marks.get("timed_start", 0), self.marks.get("timed_end", 1e30)
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        used = inside if inside else self.samples
        reasons = set()
        for _, _, r in used:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[1] for s in used]) if used else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(inside), "samples_window": "timed region" if inside else "warm-up + timed region"}


# ----------------------------------------------------------------- helpers

def workload_calls(w):
    """(shift) per call of one step."""
    return list(w.shifts)


def roofline(w, kernel_s, peaks, traffic):
    flops, nbytes = w.flops(), w.bytes()
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops / nbytes < ridge:
        achieved = nbytes / kernel_s / 1e9
        peak = peaks["hbm_gbs"]
        r = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s"}
    else:
        achieved = flops / kernel_s / 1e12
        peak = peaks["bf16_tflops"]
        r = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
             "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]}
    r["frac"] = r["achieved"] / r["peak"]
    r["traffic"] = traffic
    r["peak_source"] = peaks["source"]
    r["algorithmic_bytes_per_launch"] = nbytes
    r["algorithmic_flops_per_launch"] = flops
    return r


def oracle_sample_rate(w, target_s, base=0):
    """Time the fp64 oracle on a bounded sample of the workload's units on all
    host cores; returns (tokens/s extrapolated to the whole workload, sample
    description, cores)."""
    import numpy as np

    import oracle
    from windowed_attention_vision_b200 import inputs as I
    cores = cpu_cores()
    (qkv,), theta, bias = I.make_inputs(w, "cpu", base)
    args = [I.to_storage_numpy(t) for t in qkv]
    th = None if theta is None else theta.numpy()
    bs = I.to_storage_numpy(bias)
    orc = oracle.oracle()
    total_units = w.B * (w.H // w.M) * (w.W // w.M) * w.heads
    rng = np.random.default_rng(base)
    shift = w.shifts[-1]
    probe = min(total_units, cores)
    t0 = time.perf_counter()
    orc.fwd_units(*args, rng.choice(total_units, probe, replace=False), M=w.M, shift=shift, theta=th, bias=bs,
                  nthreads=cores)
    per_batch = time.perf_counter() - t0
    n = int(min(total_units, max(probe, probe * max(1.0, target_s / max(per_batch, 1e-6)))))
    units = rng.choice(total_units, n, replace=False)
    # when the whole call is faster than the target, repeat it (at most 100
    # times) so that the timed CPU work still lasts about target_s
    reps, dt = 0, 0.0
    t0 = time.perf_counter()
    while reps == 0 or (n == total_units and dt < target_s and reps < 100):
        orc.fwd_units(*args, units, M=w.M, shift=shift, theta=th, bias=bs, nthreads=cores)
        reps += 1
        dt = time.perf_counter() - t0
    calls = len(workload_calls(w))
    tokens_per_s = w.tokens * (n / total_units) * reps / dt
    sample = (f"{n} of {total_units} (window, head) units of one {w.name} call (shift {shift})"
              + (f", repeated {reps} times" if reps > 1 else "")
              + f", {dt:.1f} s on {cores} threads, extrapolated by unit count")
    return tokens_per_s, sample, cores, calls


# The metric is throughput against the window size M: besides the headline
# workload, one line per sweep point (shift M/2, both head dims) and the dense
# and SR calls, each timed with CUDA events over back-to-back calls.
# Device cycles of the spin that precedes the timed region (about 100 us at
# 2 GHz, well above the host's graph launch time).
SPIN_CYCLES = 200_000

PER_M = ([f"sweep_M{M}_d{d}_s{M // 2}" for M in (8, 16, 32, 64, 96) for d in (32, 64)]
         + ["dense", "sr", "flashswin_M16", "flashswin_M32"])


def per_m_table(dev, peaks, target_s=0.25):
    import torch

    import windowed_attention_vision_b200 as wa
    from windowed_attention_vision_b200 import _lib
    from windowed_attention_vision_b200 import inputs as I
    stream = torch.cuda.current_stream(dev)
    rows = []
    for name in PER_M:
        w = I.WORKLOADS[name]
        (qkv,), theta, bias = I.make_inputs(w, dev)
        out = torch.empty_like(qkv[0])
        calls = workload_calls(w)

        def one():
            for s in calls:
                wa.window_attention(*qkv, w.M, s, theta=theta, bias_feats=bias, out=out)

        one()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        one()
        torch.cuda.synchronize(dev)
        est = max(time.perf_counter() - t0, 1e-5)
        reps = int(max(3, min(200, target_s / est)))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            one()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        call_s = e0.elapsed_time(e1) / 1e3 / (reps * len(calls))
        r = roofline(w, call_s, peaks, None)
        rc, info = _lib.launch_info(w.B, w.H, w.W, w.M, calls[-1], w.heads, w.d, w.rank,
                                    _lib.BF16 if w.dtype == "bf16" else _lib.FP32)
        rows.append({"workload": name, "M": w.M, "d": w.d, "rank": w.rank, "shifts": list(calls),
                     "tokens": w.tokens, "kernel": KERNELS.get(info["kernel"], ("unknown",))[0],
                     "us_per_call": call_s * 1e6, "calls_timed": reps * len(calls),
                     "tflops": w.flops() / call_s / 1e12, "tokens_per_s": w.tokens / call_s,
                     "gbs": w.bytes() / call_s / 1e9, "bound": r["bound"], "achieved": r["achieved"],
                     "peak": r["peak"], "unit": r["unit"], "frac": r["frac"]})
        del qkv, out
        torch.cuda.empty_cache()
    return rows


# The backward pass (winattn_bwd) on the training shapes: algorithmic bytes
# read q, k, v, O, dO and the log-sum-exp once and write dq, dk, dv once;
# algorithmic flops are the five contractions per pair of a window (S^T, dP^T,
# dV, dK, dQ), masked pairs included.
BWD = ["swin", "dense", "flashswin_M32"]


def bwd_flops(w):
    return float(w.tokens) * w.heads * w.N * (6 * (w.d + w.rank) + 4 * w.d)


def bwd_bytes(w):
    return 8.0 * w.tokens * w.heads * w.d * w.elt + 4.0 * w.tokens * w.heads


def bwd_table(dev, peaks, target_s=0.25):
    import torch

    import windowed_attention_vision_b200 as wa
    from windowed_attention_vision_b200 import inputs as I
    stream = torch.cuda.current_stream(dev)
    rows = []
    for name in BWD:
        w = I.WORKLOADS[name]
        (qkv,), theta, bias = I.make_inputs(w, dev)
        s = w.shifts[-1]
        lse = torch.empty((w.B, w.H, w.W, w.heads), dtype=torch.float32, device=dev)
        out = wa.window_attention(*qkv, w.M, s, theta=theta, bias_feats=bias, lse=lse)
        dout = I.make_map(qkv[0].shape, "bf16", I.seed_for(w.name, "dout"), dev)

        def one():
            return wa.window_attention_backward(*qkv, out, dout, lse, w.M, s, theta=theta, bias_feats=bias)

        one()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        one()
        torch.cuda.synchronize(dev)
        reps = int(max(3, min(100, target_s / max(time.perf_counter() - t0, 1e-5))))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            one()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        call_s = e0.elapsed_time(e1) / 1e3 / reps
        flops, nbytes = bwd_flops(w), bwd_bytes(w)
        ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
        if flops / nbytes < ridge:
            bound, achieved, peak, unit = "hbm", nbytes / call_s / 1e9, peaks["hbm_gbs"], "GB/s"
        else:
            bound, achieved, peak, unit = "tensor", flops / call_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        rows.append({"workload": name, "M": w.M, "d": w.d, "shift": s, "us_per_call": call_s * 1e6,
                     "calls_timed": reps, "tflops": flops / call_s / 1e12, "tokens_per_s": w.tokens / call_s,
                     "gbs": nbytes / call_s / 1e9, "bound": bound, "achieved": achieved, "peak": peak,
                     "unit": unit, "frac": achieved / peak, "timing": "eager launches, CUDA events"})
        del qkv, out, dout, lse
        torch.cuda.empty_cache()
    return rows


def _time_calls(one, dev, target_s=0.25):
    """Seconds per call of `one` (eager launches, CUDA events, after one
    untimed call): enough calls to last about target_s."""
    import torch
    stream = torch.cuda.current_stream(dev)
    one()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    one()
    torch.cuda.synchronize(dev)
    reps = int(max(3, min(200, target_s / max(time.perf_counter() - t0, 1e-5))))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / 1e3 / reps, reps


def _roof(flops, nbytes, call_s, peaks):
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops / nbytes < ridge:
        return {"bound": "hbm", "achieved": nbytes / call_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": nbytes / call_s / 1e9 / peaks["hbm_gbs"]}
    return {"bound": "tensor", "achieved": flops / call_s / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": flops / call_s / 1e12 / peaks["bf16_tflops"]}


def extras_table(dev, peaks):
    """The rows around the attention: the gated-window residual (HSMLA) on
    30% of the windows, the RIB factor table and the attention with factors
    generated in the same call, and the CLA gate, each against its roofline
    (algorithmic bytes / flops stated per row)."""
    import math

    import numpy as np
    import torch

    import windowed_attention_vision_b200 as wa
    from windowed_attention_vision_b200 import inputs as I
    rows = []
    # gated residual: the listed windows' q, k, v read, out read and written;
    # two contractions per path (softmax and linear) over their pairs
    for name in ("swin", "dense"):
        w = I.WORKLOADS[name]
        (qkv,), theta, _ = I.make_inputs(w, dev)
        nwin = w.B * (w.H // w.M) * (w.W // w.M)
        wins = np.sort(np.random.default_rng(0).choice(nwin, int(round(0.3 * nwin)), replace=False))
        wt = torch.from_numpy(wins.astype(np.int32)).to(dev)
        frac = len(wins) / nwin
        o_lin = torch.randn_like(qkv[0].float()).to(torch.bfloat16)
        s = w.shifts[-1]
        call_s, reps = _time_calls(lambda: wa.window_attention_gated_residual(*qkv, o_lin, wt, w.M, s, theta=theta),
                                   dev)
        flops, nbytes = 2 * w.flops() * frac, 5.0 * w.tokens * w.heads * w.d * 2 * frac
        rows.append(dict({"row": "gated residual", "workload": name, "windows": f"{len(wins)} of {nwin}",
                          "us_per_call": call_s * 1e6, "calls_timed": reps,
                          "tokens_per_s": w.tokens * frac / call_s}, **_roof(flops, nbytes, call_s, peaks)))
        del qkv, o_lin
    # RIB factors (SR: M = 96, 6 heads, rank 16): the table alone, then the
    # attention with the table generated in the same call
    w = I.WORKLOADS["sr"]
    g = torch.Generator().manual_seed(0)
    w1 = (torch.randn((w.heads, 2, 32, 64), generator=g) / math.sqrt(32)).to(dev)
    w2 = (torch.randn((w.heads, 2, 64, w.rank), generator=g) / math.sqrt(64)).to(dev)
    table = torch.empty((w.heads, 2, w.N, w.rank), dtype=torch.bfloat16, device=dev)
    call_s, reps = _time_calls(lambda: wa.rib_features(w1, w2, w.M, table), dev)
    mlp_flops = w.heads * 2 * w.N * 2 * (32 * 64 + 64 * w.rank)
    rows.append({"row": "RIB factor table", "workload": "sr (M 96, 6 heads, rank 16)", "us_per_call": call_s * 1e6,
                 "calls_timed": reps, "mlp_gflops": mlp_flops / 1e9,
                 "note": "fp32 CUDA-core MLP, once per call; a few microseconds next to the attention"})
    (qkv,), _, _ = I.make_inputs(w, dev)
    out = torch.empty_like(qkv[0])
    call_s, reps = _time_calls(lambda: wa.window_attention_rib(*qkv, w.M, 0, w1, w2, out=out, table=table), dev)
    rows.append(dict({"row": "attention with generated RIB factors", "workload": "sr", "us_per_call": call_s * 1e6,
                      "calls_timed": reps, "tokens_per_s": w.tokens / call_s},
                     **_roof(w.flops(), w.bytes(), call_s, peaks)))
    del qkv, out
    # CLA gate: x and O read once, out written once; 2 C^2 flops per token
    for name, (B, H, W, C) in (("sr", (4, 192, 192, 192)), ("swin", (64, 56, 56, 96))):
        x = torch.randn((B, H, W, C), device=dev).to(torch.bfloat16)
        o = torch.randn_like(x)
        dw = torch.randn((C, 3, 3), device=dev) / 3
        dwb = torch.zeros(C, device=dev)
        pw = torch.randn((C, C), device=dev) / math.sqrt(C)
        pwb = torch.zeros(C, device=dev)
        out = torch.empty_like(x)
        call_s, reps = _time_calls(lambda: wa.cla_gate(x, o, dw, dwb, pw, pwb, out=out), dev)
        T = B * H * W
        rows.append(dict({"row": "CLA gate", "workload": f"{name} (B{B}, {H}x{W}, C {C})",
                          "us_per_call": call_s * 1e6, "calls_timed": reps, "tokens_per_s": T / call_s},
                         **_roof(2.0 * T * C * C, 3.0 * T * C * 2, call_s, peaks)))
        del x, o, out
    torch.cuda.empty_cache()
    return rows


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings over all ranks (every rank
    calls it at the same point; the job is as slow as its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tokens_per_s(w, calls_per_step, steps, world, elapsed_ms):
    """Whole-job throughput: every rank processes its own batch of the
    workload (weak scaling), so the job handles world times one rank's tokens
    in the slowest rank's time."""
    return w.tokens * calls_per_step * steps * world / (elapsed_ms / 1e3)


# ----------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from windowed_attention_vision_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    # the whole run stays within about 150 s of CPU time whatever K and W are
    per_step = max(0.2, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    rates = []
    for s in range(args.warmup + args.steps):
        rate, sample, cores, _ = oracle_sample_rate(w, per_step, base=s)
        if s >= args.warmup:
            rates.append(rate)
    value = statistics.median(rates)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.tokens / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def config_of(w, n):
    return {"workload": w.name, "B_per_gpu": w.B, "H": w.H, "W": w.W, "M": w.M, "shifts": list(w.shifts),
            "heads": w.heads, "d": w.d, "rank": w.rank, "rope": w.rope, "global_batch": w.B * n,
            "parallelism": f"replicas x{n} (independent batches)"}


# ----------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    import windowed_attention_vision_b200 as wa
    from windowed_attention_vision_b200 import _lib
    from windowed_attention_vision_b200 import inputs as I

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = I.WORKLOADS[args.workload]
    calls = workload_calls(w)
    map_bytes = w.tokens * w.heads * w.d * w.elt
    # rotate over enough input sets that one pass over them exceeds 2x L2
    copies = max(2, int((2 * L2_BYTES) // (4 * map_bytes)) + 1)
    sets, theta, bias = I.make_inputs(w, dev, base=rank, copies=copies)
    outs = [torch.empty_like(s[0]) for s in sets]
    stream = torch.cuda.current_stream(dev)

    def step(i):
        q, k, v = sets[i % copies]
        for s in calls:
            wa.window_attention(q, k, v, w.M, s, theta=theta, bias_feats=bias, out=outs[i % copies])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)

    def enqueue_steps():
        n = 0
        for i in range(args.steps):
            q, k, v = sets[i % copies]
            for s in calls:
                wa.window_attention(q, k, v, w.M, s, theta=theta, bias_feats=bias, out=outs[i % copies])
                n += 1
        return n

    # Eager launches first (reported, not the headline): the host time to
    # enqueue a call next to the device time per call.
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    h0 = time.perf_counter()
    n_eager = enqueue_steps()
    host_us = (time.perf_counter() - h0) / n_eager * 1e6
    e1.record(stream)
    torch.cuda.synchronize(dev)
    eager_ms = e0.elapsed_time(e1) / n_eager

    # The timed region: the K steps captured once as a CUDA graph (the same
    # launches, each a programmatic dependent of the previous one) and
    # replayed; the graph is replayed once untimed first.  The host then never
    # sits between two launches, so the device time is the kernels' own.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        n = enqueue_steps()
    graph.replay()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.01)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark("timed_start")
    # A short device-side spin (torch's, outside the timed region) keeps the
    # stream busy while the host records `start` and launches the graph, so
    # that `start` is taken when the device reaches the first step, not while
    # it waits for the host's graph launch.
    torch.cuda._sleep(SPIN_CYCLES)
    start.record(stream)
    graph.replay()
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark("timed_end")
    if world > 1:
        dist.barrier()
    time.sleep(0.01)
    clocks.stop()
    del graph
    status = wa.device_status(dev)
    elapsed_ms = start.elapsed_time(end)
    kernel_ms = elapsed_ms / n
    if world > 1:
        elapsed_ms, kernel_ms = max_over_ranks([elapsed_ms, kernel_ms], dev)

    value = job_tokens_per_s(w, len(calls), args.steps, world, elapsed_ms)
    tflops = w.flops() * len(calls) * args.steps * world / (elapsed_ms / 1e3) / 1e12

    # end to end through the C ABI on host buffers (pinned), copies inside the region
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv = (t.cpu().pin_memory() for t in sets[0])
        hout = torch.empty_like(hq).pin_memory()
        need = _lib.host_workspace_bytes(w.B, w.H, w.W, w.heads, w.d, _lib.BF16 if w.dtype == "bf16" else _lib.FP32)
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        for s in calls:
            wa.window_attention_host(hq, hk, hv, w.M, s, theta=theta, bias_feats=bias, out=hout, workspace=ws,
                                     device=dev, synchronize=False)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for s in calls:
                wa.window_attention_host(hq, hk, hv, w.M, s, theta=theta, bias_feats=bias, out=hout,
                                         workspace=ws, device=dev, synchronize=False)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1)
        if world > 1:
            (e2e_ms,) = max_over_ranks([e2e_ms], dev)
        e2e = {"value": w.tokens * len(calls) * args.e2e_steps * world / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": 3 * map_bytes * len(calls), "d2h_bytes_per_step": map_bytes * len(calls),
               "steps": args.e2e_steps, "api": "winattn_fwd_host (C ABI, pinned host buffers)"}

    if rank == 0:
        peaks = read_peaks()
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
                "config": dict(config_of(w, world),
                               l2=f"inputs larger than L2: {copies} rotating input sets of "
                                  f"{4 * map_bytes / 1e6:.0f} MB (q, k, v, out)"),
                "tflops": tflops, "kernel_ms_per_launch": kernel_ms,
                "timing": "CUDA events around one replay of a CUDA graph holding the K steps' launches, "
                          "the start event queued behind a short device spin so the graph launch is not timed",
                "eager": {"ms_per_launch": eager_ms, "host_us_per_call": host_us,
                          "note": "the same K steps launched one by one from Python (host time per call "
                                  "= wall time to enqueue them / K)"},
                "gpu_launches": args.steps * len(calls),
                "roofline": roofline(w, kernel_ms / 1e3, peaks, recorded_traffic(w)),
                "clocks": clocks.summary(), "e2e": e2e, "device_status": status}
        if not args.no_per_m:
            line["per_M"] = per_m_table(dev, peaks)
            line["backward"] = bwd_table(dev, peaks)
            line["extras"] = extras_table(dev, peaks)
        if world == 1 and not args.no_cpu_baseline:
            rate, sample, cores, _ = oracle_sample_rate(w, args.cpu_seconds)
            line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                    "sample": sample}
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
