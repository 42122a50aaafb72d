"""Throughput of the HSTU forward stack and of M-FALCON ranking on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one forward pass of the 8-layer, d=1024 HSTU stack over the
full-stack workload (128 users, Stochastic-Length-shortened lognormal
lengths, ~36k tokens), i.e. every step of the layer path: schedule, f1 +
SiLU, pointwise attention with relative bias, LayerNorm * U, f2 + residual.
M-FALCON ranking (32 users, 1024 candidates each, 3 layers) is timed the same
way and reported in the same line under "mfalcon"; Stochastic Length sampling
+ token embedding of the raw streams of a 128-user batch (1M-row content
table) under "stochastic_length", and those raw streams through Stochastic
Length, embedding and the 8-layer stack under "full_pipeline"; the stack
output's last row per user scored against the 1M-item catalog with top-100
selection under "retrieval"; one HSTU layer against one softmax-Transformer
layer on the long-history workload under "comparator".

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream with a 256 MB L2 flush between steps (outside the
events); barrier + synchronize around the timed region; max over ranks.
Under torchrun every rank runs its own replica batch (users are independent;
no collective on the data path) and `value` sums the tokens of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HSTU fwd tokens/s & M-FALCON candidates/s at 1 B200; % of bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_frac(tflops: float, peaks) -> dict:
    """Whole-step algorithmic TFLOP/s as a fraction of the measured bf16 GEMM
    rates (burst, sustained) and of the part's nominal dense bf16 rate."""
    return {"of_burst": round(tflops / float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])), 4),
            "of_sustained": round(tflops / float(peaks.get("bf16_tflops_sustained",
                                                           FALLBACK_PEAKS["bf16_tflops_sustained"])), 4),
            "of_nominal": round(tflops / 2250.0, 4)}


def ln_mode_text(mode: int, d_model: int) -> str:
    """Where LayerNorm * U runs for option `mode` at this layer width."""
    inside = mode == 1 or (mode == 2 and d_model <= 512)
    how = "inside f2's operand stage" if inside else "separate kernel, f2 reads Z"
    return how + (" (chosen by width)" if mode == 2 else "")


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ---------------------------------------------------------------- algorithmic work
def layer_flops(dims, lengths):
    d, h, dqk, dv = dims.d_model, dims.n_heads, dims.d_qk, dims.d_v
    F = 2 * h * (dqk + dv)
    n = np.asarray(lengths, np.float64)
    T = float(n.sum())
    pairs = float((n * (n + 1) / 2).sum())
    return dict(f1=2.0 * T * d * F, f2=2.0 * T * h * dv * d, attn=h * (2 * dqk + 2 * dv) * pairs)


def mfalcon_flops(dims, n_layers, hist_lens, cands):
    d, h, dqk, dv = dims.d_model, dims.n_heads, dims.d_qk, dims.d_v
    F = 2 * h * (dqk + dv)
    lf = layer_flops(dims, hist_lens)
    T = float(np.sum(hist_lens))
    hist = (n_layers - 1) * sum(lf.values()) + T * 2 * d * h * (dqk + dv)
    n = np.asarray(hist_lens, np.float64)
    m = np.asarray(cands, np.float64)
    cand = float((m * n_layers * (2 * d * F + 2 * h * dv * d + h * (2 * dqk + 2 * dv) * (n + 1))).sum()
                 + (2 * d * m).sum())
    return hist + cand


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled every ~2 ms while the timed
    region runs (NVML from a thread; nvidia-smi at 100 ms if NVML is absent).
    Samples also go to <HSTU_BENCH_OUT or bench_out>/clocks_rank<i>.csv."""

    NAMES = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
             "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
             "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
             "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
             "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, gpu_index: int, tag: str = ""):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.samples = []           # (sm_mhz, max_mhz, reason bitmask)
        out_dir = os.environ.get("HSTU_BENCH_OUT", os.path.join(ROOT, "bench_out"))
        self.path = os.path.join(out_dir, f"clocks_rank{gpu_index}{tag}.csv")

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:  # the CUDA device's own GPU, whatever CUDA_VISIBLE_DEVICES maps it to
            uid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            if not uid.startswith("GPU-"):
                uid = "GPU-" + uid
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self, nv, hdl):
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        mx = nv.nvmlDeviceGetMaxClockInfo(hdl, nv.NVML_CLOCK_SM)
        while not self.stop:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(hdl, nv.NVML_CLOCK_SM), mx, get_r(hdl)))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        import threading
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        self.stop = False
        try:
            nv, hdl = self._nvml_handle()
            self.nv = nv
            self.thread = threading.Thread(target=self._poll, args=(nv, hdl), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)
            with open(self.path, "w") as f:
                f.write("sm_mhz,max_sm_mhz,reasons_mask\n")
                for sm, mx, r in self.samples:
                    f.write(f"{sm},{mx},{r:#x}\n")
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.thread is not None:
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
            reasons = set()
            for _, _, r in self.samples:
                for nm, attr in self.NAMES.items():
                    bit = getattr(self.nv, attr, 0)
                    if bit and (r & bit):
                        reasons.add(nm)
            return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                    "sm_max_mhz": max(s[1] for s in self.samples),
                    "samples": len(self.samples), "source": "nvml", "reasons": sorted(reasons)}
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "source": "nvidia-smi", "reasons": sorted(reasons)}


# ---------------------------------------------------------------- traffic from ncu
# the source files each profiled kernel is built from (its own translation
# unit plus the shared device helpers and declarations)
KERNEL_SOURCES = {
    "gemm_f1_tc": ["gemm_tc.cu"], "gemm_f2_tc": ["gemm_tc.cu"], "attn_tc": ["attn_tc.cu"],
    "ln_gate": ["sched.cu"], "sl_select": ["sl.cu"], "sl_gather": ["sl.cu"],
}


def kernel_source_hash(kernel: str):
    csrc = os.path.join(ROOT, "hstu_sequential_transducer_layer_b200", "csrc")
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []) + ["ptx.cuh", "hstu_internal.h"]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if its
    recorded source hash matches the kernel's current sources (else null)."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash(kernel):
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU baseline (oracle)
def blas_cores() -> int:
    """Threads the oracle's BLAS calls use."""
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline_stack(w, budget_tokens: int):
    """Oracle on whole users of the workload (fixed seeded sample), tokens/s."""
    from oracle import hstu_oracle as O
    cores = blas_cores()
    order = np.random.default_rng(123).permutation(w.B)
    users, tok = [], 0
    for b in order:
        users.append(int(b))
        tok += int(w.lengths[b])
        if tok >= budget_tokens:
            break
    t0 = time.perf_counter()
    for b in users:
        s, e = int(w.offsets[b]), int(w.offsets[b + 1])
        O.stack_user(w.X[s:e], w.timestamps[s:e], w.weights, w.dims)
    dt = time.perf_counter() - t0
    return {"value": tok / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(users)} whole users ({tok} tokens) of the {w.name} workload, "
                      f"all {w.n_layers} layers, numpy float64",
            "seconds": dt}


# ---------------------------------------------------------------- end to end
def e2e_pipelined(torch, host_in, out_like, compute, steps, flush):
    """Steps through the public API from pinned host buffers, as a server
    runs them: step i+1's inputs go up (copy stream) and step i-1's result
    comes down (second copy stream) while step i computes; every step's
    copies are inside the timed region.  host_in: pinned host tensors;
    compute(dev_in, dev_out, stream) runs one step.  Returns ms per step."""
    s_c = torch.cuda.current_stream()
    s_up, s_dn = torch.cuda.Stream(), torch.cuda.Stream()
    d_in = [[torch.empty_like(h, device="cuda") for h in host_in] for _ in range(2)]
    d_out = [torch.empty_like(out_like) for _ in range(2)]
    h_out = [torch.empty(out_like.shape, dtype=out_like.dtype).pin_memory() for _ in range(2)]
    ev = lambda: torch.cuda.Event()
    up_done = [ev(), ev()]
    comp_done = [ev(), ev()]
    dn_done = [ev(), ev()]
    flush.zero_()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_c)
    s_up.wait_event(t0)
    s_dn.wait_event(t0)
    for i in range(steps + 2):
        if i < steps:                       # inputs of step i
            b = i % 2
            if i >= 2:
                s_up.wait_event(comp_done[b])   # step i-2 no longer reads them
            with torch.cuda.stream(s_up):
                for dst, src in zip(d_in[b], host_in):
                    dst.copy_(src, non_blocking=True)
            up_done[b].record(s_up)
        j = i - 1                            # compute of step i-1
        if 0 <= j < steps:
            b = j % 2
            s_c.wait_event(up_done[b])
            if j >= 2:
                s_c.wait_event(dn_done[b])      # step j-2's result has been read out
            compute(d_in[b], d_out[b], s_c)
            comp_done[b].record(s_c)
        k = i - 2                            # result of step i-2
        if 0 <= k < steps:
            b = k % 2
            s_dn.wait_event(comp_done[b])
            with torch.cuda.stream(s_dn):
                h_out[b].copy_(d_out[b], non_blocking=True)
            dn_done[b].record(s_dn)
    s_c.wait_stream(s_up)
    s_c.wait_stream(s_dn)
    t1.record(s_c)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def time_leg(fn, args, flush, stream):
    """Mean ms of one call of `fn` over args.steps timed calls (CUDA events on
    `stream`, L2 flushed between calls, after args.warmup untimed ones), and
    the library's per-kernel mean launch times from a second, traced pass."""
    import torch
    import hstu_sequential_transducer_layer_b200 as H
    for _ in range(args.warmup):
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    H.hstu_trace_enable(args.steps * 256 + 256)
    for _ in range(args.steps):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    tr = H.hstu_trace_read()
    H.hstu_trace_enable(0)
    ker = {}
    for kid, t in tr:
        e = ker.setdefault(H.hstu_kernel_name(kid), [0, 0.0])
        e[0] += 1
        e[1] += t
    return (sum(a.elapsed_time(b) for a, b in evs) / len(evs),
            {k: round(v[1] / v[0], 4) for k, v in ker.items()})


def cpu_baseline_extrapolated(w, budget_tokens: int, shortest: bool = False):
    """The oracle on whole users of a one-layer workload (a seeded random
    sample up to `budget_tokens`, or only the shortest user), its algorithmic
    GFLOP/s, and the workload's tokens/s at that rate (the workload's FLOPs
    divided by the oracle's FLOP rate): long users cost more per token, so
    the sample's own tokens/s would not stand for the workload."""
    from oracle import hstu_oracle as O
    if shortest:
        users = [int(np.argmin(w.lengths))]
    else:
        users, tok = [], 0
        for b in np.random.default_rng(123).permutation(w.B):
            users.append(int(b))
            tok += int(w.lengths[b])
            if tok >= budget_tokens:
                break
    lens = w.lengths[users]
    t0 = time.perf_counter()
    for b in users:
        s, e = int(w.offsets[b]), int(w.offsets[b + 1])
        O.stack_user(w.X[s:e], w.timestamps[s:e], w.weights, w.dims)
    dt = time.perf_counter() - t0
    f_sample = w.n_layers * sum(layer_flops(w.dims, lens).values())
    f_all = w.n_layers * sum(layer_flops(w.dims, w.lengths).values())
    rate = f_sample / dt
    return {"value": w.T / (f_all / rate), "unit": "tokens/s", "cores": blas_cores(),
            "kind": "oracle", "gflops": round(rate / 1e9, 3), "seconds": round(dt, 2),
            "sample": f"{len(users)} whole user(s) ({int(lens.sum())} tokens) of the {w.name} "
                      f"workload, numpy float64; tokens/s of the whole workload at the sample's "
                      f"algorithmic FLOP rate"}


# ---------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import hstu_workloads as hw
    import hstu_sequential_transducer_layer_b200 as H
    from hstu_sequential_transducer_layer_b200.build import build

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if rank == 0 or world == 1:
        build()
    if world > 1:
        torch.distributed.barrier()
    peaks, peak_src = load_peaks()
    H.hstu_set_option("ln_fusion", args.ln_fusion)

    # ---------------- inputs (a replica batch per rank)
    w = hw.full_stack(seed=args.seed + rank)
    r = H.HSTURunner(hw.dims_dict(w.dims), w.weights, dev)
    off = r.to_device(w.offsets, "i64")
    X = r.to_device(w.X, "act")
    ts = r.to_device(w.timestamps, "i64")
    out = torch.empty_like(X)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flops = layer_flops(w.dims, w.lengths)
    T = w.T

    def step():
        r.stack(off, X, ts, w.max_len, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if r.status() != 0:
        raise RuntimeError(f"device status {r.status()} after warm-up")

    # the same steps with no per-launch event pairs, just before the timed
    # region (those pairs add a little to its steps; this is the step time
    # without them)
    u_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    for a, b in u_evs:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    untraced_ms = sum(a.elapsed_time(b) for a, b in u_evs) / len(u_evs)

    # ---------------- timed region: an event pair around every launch of the
    # dominant kernel (the f1 GEMM: 47 % of the step's device time in the ncu
    # launch list) gives its per-launch device time for the roofline; the
    # other kernels run without event pairs (their split comes from a
    # separate traced pass below)
    f1_id = next(i for i in range(64) if H.hstu_kernel_name(i) == "gemm_f1_tc")
    n_launch0 = H.hstu_launch_count()
    H.hstu_trace_only(f1_id)
    H.hstu_trace_enable(args.steps * 8 + 64)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    n_launch = H.hstu_launch_count() - n_launch0
    f1_trace = H.hstu_trace_read()
    H.hstu_trace_enable(0)
    H.hstu_trace_only(-1)
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = sum(step_ms) / len(step_ms)
    if r.status() != 0:
        raise RuntimeError(f"device status {r.status()} after timing")

    # per-kernel device time of every kernel, from a separate traced pass of
    # the same steps (outside the timed region)
    H.hstu_trace_enable(args.steps * 8 * 6 + 64)
    for _ in range(args.steps):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    trace = H.hstu_trace_read()
    H.hstu_trace_enable(0)
    per_kernel = {}
    for kid, t in trace:
        nm = H.hstu_kernel_name(kid)
        a = per_kernel.setdefault(nm, [0, 0.0])
        a[0] += 1
        a[1] += t
    dominant = max(per_kernel.items(), key=lambda kv: kv[1][1])[0] if per_kernel else None
    kflops = {"gemm_f1_tc": flops["f1"], "gemm_f2_tc": flops["f2"], "attn_tc": flops["attn"]}
    roofline = None
    if dominant == "gemm_f1_tc" and f1_trace:
        # the dominant kernel's launches inside the timed region
        n, tot = len(f1_trace), sum(t for _, t in f1_trace)
        avg_s = tot / n / 1e3
        achieved = kflops[dominant] / avg_s / 1e12
        # the timed region is a burst of well under a second at full clocks,
        # so the denominator is the measured burst GEMM rate
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        roofline = {"bound": "tensor", "kernel": dominant, "achieved": round(achieved, 1),
                    "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "peak_source": f"bf16_tflops, burst ({peak_src})",
                    "traffic": ncu_traffic(dominant, w.name),
                    "avg_launch_ms": round(tot / n, 4),
                    # the same achieved rate against the sustained figure and
                    # the nominal dense bf16 rate of the part (2.25 PFLOP/s)
                    "frac_sustained": round(achieved / float(peaks.get(
                        "bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])), 4),
                    "frac_nominal": round(achieved / 2250.0, 4)}
    step_flops = args_layers = w.n_layers * sum(flops.values())
    del args_layers

    # ---------------- end to end through the public API, host buffers
    Xh = X.cpu().pin_memory()
    offh = off.cpu().pin_memory()
    tsh = ts.cpu().pin_memory()
    Yh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(max(3, args.steps // 2))]
    Xd, offd, tsd = torch.empty_like(X), torch.empty_like(off), torch.empty_like(ts)
    for a, b in e_evs:
        flush.zero_()
        a.record(stream)
        Xd.copy_(Xh, non_blocking=True)
        offd.copy_(offh, non_blocking=True)
        tsd.copy_(tsh, non_blocking=True)
        r.stack(offd, Xd, tsd, w.max_len, out=out)
        Yh.copy_(out, non_blocking=True)
        b.record(stream)
    torch.cuda.synchronize()
    e2e_serial_ms = sum(a.elapsed_time(b) for a, b in e_evs) / len(e_evs)
    h2d = Xh.numel() * Xh.element_size() + offh.numel() * 8 + tsh.numel() * 8
    d2h = Yh.numel() * Yh.element_size()
    e2e_ms = e2e_pipelined(
        torch, [Xh, offh, tsh], out,
        lambda di, do, st: r.stack(di[1], di[0], di[2], w.max_len, out=do, stream=st),
        max(4, args.steps), flush)

    # ---------------- M-FALCON
    mf = None
    if not args.no_mfalcon:
        wm = hw.mfalcon(seed=args.seed + rank)
        rm = H.HSTURunner(hw.dims_dict(wm.dims), wm.weights, dev)
        ins = dict(ho=rm.to_device(wm.offsets, "i64"), hx=rm.to_device(wm.X),
                   ht=rm.to_device(wm.timestamps, "i64"), co=rm.to_device(wm.cand_offsets, "i64"),
                   cx=rm.to_device(wm.candidates), hv=rm.to_device(wm.head_vec))
        scores = torch.empty(wm.candidates.shape[0], dtype=torch.float32, device=dev)

        def mstep():
            rm.rank(ins["ho"], ins["hx"], ins["ht"], ins["co"], ins["cx"], None, wm.microbatch,
                    ins["hv"], wm.max_len, wm.max_cands, scores=scores)
        for _ in range(args.warmup):
            mstep()
        torch.cuda.synchronize()
        m_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a, b in m_evs:
            flush.zero_()
            a.record(stream)
            mstep()
            b.record(stream)
        torch.cuda.synchronize()
        if rm.status() != 0:
            raise RuntimeError(f"M-FALCON device status {rm.status()}")
        m_ms = sum(a.elapsed_time(b) for a, b in m_evs) / len(m_evs)
        C = wm.candidates.shape[0]
        mflop = mfalcon_flops(wm.dims, wm.n_layers, wm.lengths, np.diff(wm.cand_offsets))
        # (the line's last characters: the candidates/s half of the metric)
        mf = {"config": {"workload": "mfalcon: M-FALCON ranking, 3-layer stack (d=512, 4 heads, "
                                     "head dim 128), 32 users with 512-4096 history tokens, 1024 "
                                     "candidates per user in microbatches of 256",
                         "users": wm.B, "candidates_per_user": wm.max_cands,
                         "microbatch": wm.microbatch, "layers": wm.n_layers, "d_model": 512,
                         "heads": 4, "head_dim": 128, "history_tokens": wm.T},
              "tflops": round(mflop / (m_ms / 1e3) / 1e12, 1),
              "tensor_frac": tensor_frac(mflop / (m_ms / 1e3) / 1e12, peaks),
              "ms_per_step": round(m_ms, 4),
              "value": C / (m_ms / 1e3), "unit": "candidates/s"}

    # ---------------- Stochastic Length + token embedding (raw streams of the
    # same 128-user batch, 1M-row content table on the device)
    sl = None
    if not args.no_sl:
        rs = hw.full_stack_raw(args.seed + rank)
        ctab = hw.device_embedding_table(args.seed + rank, 0, rs.n_content, rs.d_model, dev)
        atab = hw.device_embedding_table(args.seed + rank, 1, rs.n_actions, rs.d_model, dev)
        s_in = [torch.from_numpy(a).to(dev) for a in (rs.raw_offsets, rs.raw_ids, rs.raw_timestamps)]
        s_off = torch.empty(rs.B + 1, dtype=torch.int64, device=dev)
        s_X = torch.empty(rs.R, rs.d_model, dtype=torch.bfloat16, device=dev)
        s_ts = torch.empty(rs.R, dtype=torch.int64, device=dev)
        s_ws = torch.empty(H.hstu_sl_embed_workspace_size(), dtype=torch.uint8, device=dev)

        def sstep():
            H.hstu_sl_embed(rs.B, rs.R, rs.max_raw_len, *s_in, rs.sl_seed, ctab, atab, s_off, s_X,
                            s_ts, s_ws)
        for _ in range(args.warmup):
            sstep()
        s_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a, b in s_evs:
            flush.zero_()
            a.record(stream)
            sstep()
            b.record(stream)
        torch.cuda.synchronize()
        # per-kernel times from a second, traced pass (an event pair around
        # each of three short kernels would inflate the step timed above)
        H.hstu_trace_enable(args.steps * 3 + 8)
        for _ in range(args.steps):
            flush.zero_()
            sstep()
        torch.cuda.synchronize()
        s_trace = H.hstu_trace_read()
        H.hstu_trace_enable(0)
        s_kern = {}
        for kid, t in s_trace:
            e = s_kern.setdefault(H.hstu_kernel_name(kid), [0, 0.0])
            e[0] += 1
            e[1] += t
        if H.hstu_read_status(s_ws) != 0:
            raise RuntimeError(f"Stochastic Length device status {H.hstu_read_status(s_ws)}")
        s_ms = sum(a.elapsed_time(b) for a, b in s_evs) / len(s_evs)
        kept = int(s_off[-1])
        # algorithmic bytes: raw offsets in, kept offsets out, and per kept
        # token its id and timestamp in, its timestamp and embedding row out
        # plus the row read from the table (keys are computed, not read)
        s_bytes = 16 * (rs.B + 1) + kept * (24 + 4 * rs.d_model)
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        s_gbs = s_bytes / (s_ms / 1e3) / 1e9
        # the gather kernel moves all of those bytes except the offsets
        g_n, g_ms = s_kern.get("sl_gather", [1, float("nan")])
        g_bytes = kept * (24 + 4 * rs.d_model)
        g_gbs = g_bytes / (g_ms / g_n / 1e3) / 1e9
        sl = {"value": rs.R / (s_ms / 1e3), "unit": "raw tokens/s",
              "kept_tokens_per_s": kept / (s_ms / 1e3), "ms_per_step": round(s_ms, 4),
              "step_hbm": {"achieved": round(s_gbs, 1), "frac": round(s_gbs / hbm, 4),
                           "bytes_per_step": int(s_bytes)},
              "roofline": {"bound": "hbm", "kernel": "sl_gather", "achieved": round(g_gbs, 1),
                           "peak": hbm, "unit": "GB/s", "frac": round(g_gbs / hbm, 4),
                           "peak_source": f"hbm_gbs ({peak_src})", "bytes_per_launch": int(g_bytes),
                           "avg_launch_ms": round(g_ms / g_n, 4),
                           "traffic": ncu_traffic("sl_gather", rs.name)},
              "kernels": {k: {"launches": v[0], "avg_ms": round(v[1] / v[0], 4)}
                          for k, v in s_kern.items()},
              "config": {"workload": rs.name, "users": rs.B, "raw_tokens": rs.R,
                         "kept_tokens": kept, "d_model": rs.d_model,
                         "content_rows": rs.n_content, "action_rows": rs.n_actions}}

    # ---------------- the whole path from raw streams: Stochastic Length +
    # embedding, then the 8-layer stack (same weights as the main step)
    pipe = None
    if sl is not None:
        raw_len = np.diff(rs.raw_offsets)
        kept_sz = r.kept_sizes(raw_len)
        p_T = kept_sz[0]
        p_out = torch.empty(p_T, rs.d_model, dtype=torch.bfloat16, device=dev)

        def pstep(ins):
            r.stack_raw(raw_len, *ins, rs.sl_seed, ctab, atab, rs.max_raw_len, out=p_out,
                        kept=kept_sz)
        for _ in range(args.warmup):
            pstep(s_in)
        p_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a, b in p_evs:
            flush.zero_()
            a.record(stream)
            pstep(s_in)
            b.record(stream)
        torch.cuda.synchronize()
        if r.sl_status() != 0 or r.status() != 0:
            raise RuntimeError(f"pipeline device status {r.sl_status()} / {r.status()}")
        p_ms = sum(a.elapsed_time(b) for a, b in p_evs) / len(p_evs)
        # end to end: the raw streams come from pinned host memory every step
        # (embedding tables and weights stay resident) and Y goes back
        h_in = [torch.from_numpy(a).pin_memory() for a in (rs.raw_offsets, rs.raw_ids,
                                                          rs.raw_timestamps)]
        d_in = [torch.empty_like(x, device=dev) for x in h_in]
        p_Yh = torch.empty(p_out.shape, dtype=p_out.dtype).pin_memory()
        pe_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(max(3, args.steps // 2))]
        for a, b in pe_evs:
            flush.zero_()
            a.record(stream)
            for x, y in zip(d_in, h_in):
                x.copy_(y, non_blocking=True)
            pstep(d_in)
            p_Yh.copy_(p_out, non_blocking=True)
            b.record(stream)
        torch.cuda.synchronize()
        pe_serial_ms = sum(a.elapsed_time(b) for a, b in pe_evs) / len(pe_evs)
        pe_ms = e2e_pipelined(
            torch, h_in, p_out,
            lambda di, do, st: r.stack_raw(raw_len, *di, rs.sl_seed, ctab, atab, rs.max_raw_len,
                                           out=do, stream=st, kept=kept_sz),
            max(4, args.steps), flush)
        kept_len = np.array([H.hstu_sl_keep_count(int(n)) for n in raw_len])
        pf = layer_flops(w.dims, kept_len)
        p_flops = w.n_layers * sum(pf.values())
        pipe = {"value": p_T / (p_ms / 1e3), "unit": "tokens/s", "ms_per_step": round(p_ms, 4),
                "tflops": round(p_flops / (p_ms / 1e3) / 1e12, 1),
                "tensor_frac": tensor_frac(p_flops / (p_ms / 1e3) / 1e12, peaks),
                "e2e": {"value": p_T / (pe_ms / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": int(sum(x.numel() * 8 for x in h_in)),
                        "d2h_bytes_per_step": int(p_Yh.numel() * p_Yh.element_size()),
                        "ms_per_step": round(pe_ms, 4), "mode": "pipelined",
                        "serial_ms_per_step": round(pe_serial_ms, 4)},
                "config": {"workload": "full_stack_raw -> Stochastic Length -> 8-layer stack",
                           "users": rs.B, "raw_tokens": rs.R, "tokens": p_T,
                           "max_len": kept_sz[1]}}

    # ---------------- full-catalog retrieval: the stack output's last row per
    # user scored against the 1M-row content table, top 100
    ret = None
    if not args.no_retrieval:
        r_E = ctab if sl is not None else hw.device_embedding_table(args.seed + rank, 0, 1_000_000,
                                                                    w.dims.d_model, dev)
        r_M, r_d, r_K, r_U = int(r_E.shape[0]), int(r_E.shape[1]), 100, w.B
        r_ws = torch.empty(H.hstu_retrieval_workspace_size(r_U, r_M, r_d, r_K, True),
                           dtype=torch.uint8, device=dev)
        r_s = torch.empty((r_U, r_K), dtype=torch.float32, device=dev)
        r_i = torch.empty((r_U, r_K), dtype=torch.int64, device=dev)

        def rstep():
            H.hstu_retrieval_topk(out, r_E, r_K, r_s, r_i, r_ws, user_offsets=off, n_users=r_U)
        for _ in range(args.warmup):
            rstep()
        r_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a, b in r_evs:
            flush.zero_()
            a.record(stream)
            rstep()
            b.record(stream)
        torch.cuda.synchronize()
        H.hstu_trace_enable(args.steps * 4 + 8)
        for _ in range(args.steps):
            flush.zero_()
            rstep()
        torch.cuda.synchronize()
        r_trace = H.hstu_trace_read()
        H.hstu_trace_enable(0)
        if H.hstu_read_status(r_ws) != 0:
            raise RuntimeError(f"retrieval device status {H.hstu_read_status(r_ws)}")
        r_fallback = H.hstu_retrieval_fallback_taken(r_ws)
        r_ms = sum(a.elapsed_time(b) for a, b in r_evs) / len(r_evs)
        r_kern = {}
        for kid, t in r_trace:
            e = r_kern.setdefault(H.hstu_kernel_name(kid), [0, 0.0])
            e[0] += 1
            e[1] += t
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        # algorithmic minimum: the catalog read once, the user rows and results
        r_bytes = r_M * r_d * 2 + r_U * r_d * 2 + r_U * r_K * 12
        # the GEMM that scores the whole catalog: the filtering one, or on the
        # direct path the scoring one (on the filtering path "gemm_scores_tc"
        # is the 1-in-16 sample pass)
        g_n, g_ms = r_kern.get("gemm_scores_tc" if r_fallback else "gemm_filter_tc",
                               [1, float("nan")])
        r_flops = 2.0 * r_U * r_M * r_d
        ret = {"value": r_U * r_M / (r_ms / 1e3), "unit": "user-item scores/s",
               "ms_per_step": round(r_ms, 4),
               "roofline": {"bound": "hbm", "achieved": round(r_bytes / (r_ms / 1e3) / 1e9, 1),
                            "peak": hbm, "unit": "GB/s",
                            "frac": round(r_bytes / (r_ms / 1e3) / 1e9 / hbm, 4),
                            "peak_source": f"hbm_gbs ({peak_src})",
                            "bytes_per_step": int(r_bytes),
                            "note": "whole step against the catalog read once (the filtering "
                                    "pass reads it once more after a 1-in-16 sample pass)"},
               "path": ("direct (fallback: every score written)" if r_fallback else
                        "sample threshold + filtering GEMM epilogue (no score matrix)"),
               "tflops": round(r_flops / (r_ms / 1e3) / 1e12, 1),
               "gemm_tflops": round(r_flops / (g_ms / g_n / 1e3) / 1e12, 1),
               "kernels": {k: {"launches": v[0], "avg_ms": round(v[1] / v[0], 4)}
                           for k, v in r_kern.items()},
               "config": {"workload": "full_stack output x 1M-item catalog", "users": r_U,
                          "items": r_M, "d_model": r_d, "K": r_K}}

    # ---------------- the softmax-Transformer comparator: one HSTU layer and one
    # pre-LN Transformer layer (d_ff = 2048) on the long-history workload
    # (16 users of 2,048-8,192 tokens, d = 512, 8 heads, head dim 64)
    cmp_ = None
    if not args.no_comparator:
        wl = hw.long_history(seed=args.seed + rank)
        rh = H.HSTURunner(hw.dims_dict(wl.dims), wl.weights, dev)
        c_off = rh.to_device(wl.offsets, "i64")
        c_x = rh.to_device(wl.X, "act")
        c_ts = rh.to_device(wl.timestamps, "i64")
        c_yh = torch.empty_like(c_x)
        c_yt = torch.empty_like(c_x)
        rt = H.TransformerRunner(512, 8, 2048, hw.transformer_weights(args.seed + rank, 512, 2048),
                                 device=dev)

        h_ms, h_k = time_leg(lambda: rh.stack(c_off, c_x, c_ts, wl.max_len, out=c_yh), args,
                             flush, stream)
        t_ms, t_k = time_leg(lambda: rt.layer(c_off, c_x, wl.max_len, out=c_yt), args, flush,
                             stream)
        if rh.status() != 0 or rt.status() != 0:
            raise RuntimeError(f"comparator device status {rh.status()} / {rt.status()}")
        pairs = float((wl.lengths * (wl.lengths + 1) // 2).sum())
        attn_flops = 4.0 * 64 * 8 * pairs   # Q.K and P.V, 2 flops per multiply-add
        sa_ms = t_k.get("tf_softmax_attn_tc", float("nan"))
        cmp_ = {"workload": "long_history (16 users, 2048-8192 tokens, d=512, 8 heads, dh=64)",
                "tokens": wl.T, "hstu_layer_ms": round(h_ms, 4),
                "transformer_layer_ms": round(t_ms, 4),
                "hstu_speedup": round(t_ms / h_ms, 3),
                "hstu_kernels_ms": h_k, "transformer_kernels_ms": t_k,
                "softmax_attention_tflops": round(attn_flops / (sa_ms / 1e3) / 1e12, 1),
                "hstu_attention_tflops": round(attn_flops / (h_k.get("attn_tc", float("nan")) / 1e3)
                                               / 1e12, 1),
                "note": "one layer each; the Transformer layer has an FFN (4d) and no rab"}

    # ---------------- backward pass (training): hstu_stack_bwd over the same
    # 8-layer full-stack batch, a bf16 output gradient resident in HBM
    bwd = None
    if not args.no_backward:
        dYb = torch.randn(X.shape, generator=torch.Generator(device=dev).manual_seed(7),
                          device=dev, dtype=torch.float32).to(torch.bfloat16)
        b_dX = torch.empty_like(X)
        b_grads = None

        def bstep():
            nonlocal b_grads
            _, b_grads = r.stack_bwd(off, X, ts, dYb, w.max_len, dX=b_dX, grads=b_grads)
        b_ms, b_k = time_leg(bstep, args, flush, stream)
        if r.bwd_status() != 0:
            raise RuntimeError(f"backward device status {r.bwd_status()}")
        # algorithmic work of the gradients: twice the forward's products (the
        # input-gradient and weight-gradient products of f1 and f2; dA, dV, dK
        # and dQ against S and P.V in attention); the forward pass the call runs
        # first is not counted
        b_flops = 2.0 * step_flops
        b_tf = b_flops / (b_ms / 1e3) / 1e12
        bwd = {"value": T / (b_ms / 1e3), "unit": "tokens/s", "ms_per_step": round(b_ms, 4),
               "tflops": round(b_tf, 1), "tensor_frac": tensor_frac(b_tf, peaks),
               "kernels_ms": b_k,
               "note": "gradients of every parameter and of the input, 8 layers; the stack's "
                       "forward runs inside the call first (not counted in tflops)",
               "config": {"workload": "full_stack backward", "layers": w.n_layers,
                          "tokens": T}}

    # ---------------- one-layer legs: the single-layer workload (64 users,
    # lognormal lengths capped at 1024, d = 256, 4 heads, head dim 64) and the
    # long-history workload as a layer on its own (16 users of 2,048-8,192
    # tokens, d = 512, 8 heads, head dim 64)
    legs = None
    if not args.no_layer_legs:
        legs = {}
        for name, make, shortest in (("single_layer", hw.single_layer, False),
                                     ("long_history", hw.long_history, True)):
            wl = make(seed=args.seed + rank)
            rl = H.HSTURunner(hw.dims_dict(wl.dims), wl.weights, dev)
            l_in = (rl.to_device(wl.offsets, "i64"), rl.to_device(wl.X, "act"),
                    rl.to_device(wl.timestamps, "i64"))
            l_out = torch.empty_like(l_in[1])
            l_ms, l_k = time_leg(lambda: rl.stack(l_in[0], l_in[1], l_in[2], wl.max_len,
                                                  out=l_out), args, flush, stream)
            if rl.status() != 0:
                raise RuntimeError(f"{name} device status {rl.status()}")
            lf = layer_flops(wl.dims, wl.lengths)
            l_tf = sum(lf.values()) / (l_ms / 1e3) / 1e12
            att = l_k.get("attn_tc")
            legs[name] = {
                "value": wl.T / (l_ms / 1e3), "unit": "tokens/s", "ms_per_step": round(l_ms, 4),
                "tflops": round(l_tf, 1), "tensor_frac": tensor_frac(l_tf, peaks),
                "attention_tflops": (round(lf["attn"] / (att / 1e3) / 1e12, 1) if att else None),
                "kernels_ms": l_k,
                "cpu_baseline": (None if (world > 1 or args.no_cpu_baseline) else
                                 cpu_baseline_extrapolated(wl, args.cpu_tokens, shortest)),
                "config": {"workload": name, "users": wl.B, "tokens": wl.T,
                           "layernorm_u": ln_mode_text(args.ln_fusion, wl.dims.d_model),
                           "d_model": wl.dims.d_model, "heads": wl.dims.n_heads,
                           "head_dim": wl.dims.d_qk, "max_len": wl.max_len}}
            del rl, l_in, l_out

    # ---------------- reduce over ranks
    tokens = float(T)
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms, e2e_ms, e2e_serial_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, e2e_ms, e2e_serial_ms = float(t[0]), float(t[1]), float(t[2])
        s = torch.tensor([tokens], dtype=torch.float64, device=dev)
        dist.all_reduce(s, op=dist.ReduceOp.SUM)
        tokens = float(s[0])
        if mf is not None:
            t = torch.tensor([mf["ms_per_step"]], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            mf["value"] = wm.candidates.shape[0] * world / (float(t[0]) / 1e3)
            mf["ms_per_step"] = float(t[0])
        if pipe is not None:
            t = torch.tensor([pipe["ms_per_step"], pipe["e2e"]["ms_per_step"]],
                             dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            s = torch.tensor([p_T], dtype=torch.float64, device=dev)
            dist.all_reduce(s, op=dist.ReduceOp.SUM)
            pipe["ms_per_step"], pipe["e2e"]["ms_per_step"] = float(t[0]), float(t[1])
            pipe["value"] = float(s[0]) / (float(t[0]) / 1e3)
            pipe["e2e"]["value"] = float(s[0]) / (float(t[1]) / 1e3)
        if ret is not None:
            t = torch.tensor([ret["ms_per_step"]], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ret["ms_per_step"] = float(t[0])
            ret["value"] = world * ret["config"]["users"] * ret["config"]["items"] / (float(t[0]) / 1e3)
        if bwd is not None:
            t = torch.tensor([bwd["ms_per_step"]], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            bwd["ms_per_step"] = float(t[0])
            bwd["value"] = world * T / (float(t[0]) / 1e3)
        for leg in (legs or {}).values():
            t = torch.tensor([leg["ms_per_step"]], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            leg["ms_per_step"] = float(t[0])
            leg["value"] = world * leg["config"]["tokens"] / (float(t[0]) / 1e3)
        if sl is not None:
            t = torch.tensor([sl["ms_per_step"], rs.R, sl["config"]["kept_tokens"]],
                             dtype=torch.float64, device=dev)
            dist.all_reduce(t[:1], op=dist.ReduceOp.MAX)
            dist.all_reduce(t[1:], op=dist.ReduceOp.SUM)
            sl["ms_per_step"] = float(t[0])
            sl["value"] = float(t[1]) / (float(t[0]) / 1e3)
            sl["kept_tokens_per_s"] = float(t[2]) / (float(t[0]) / 1e3)

    line = None
    if rank == 0:
        cpu = None if (world > 1 or args.no_cpu_baseline) else cpu_baseline_stack(w, args.cpu_tokens)
        if cpu is not None:
            # the same oracle on one BLAS thread, on a smaller sample
            try:
                import threadpoolctl
                with threadpoolctl.threadpool_limits(1):
                    one = cpu_baseline_stack(w, max(1, args.cpu_tokens // 4))
                cpu["one_thread"] = {"value": one["value"], "unit": "tokens/s", "cores": 1,
                                     "sample": one["sample"]}
            except Exception as exc:  # threadpoolctl absent: say so
                cpu["one_thread"] = {"value": None, "note": f"not measured: {exc}"}
        line = {
            "metric": METRIC, "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
            "data": "synthetic (seeded; random-init weights)",
            "config": {"workload": "full_stack",
                       "layernorm_u": ln_mode_text(args.ln_fusion, w.dims.d_model),
                       "layers": w.n_layers, "d_model": w.dims.d_model,
                       "heads": w.dims.n_heads, "head_dim": w.dims.d_qk, "users_per_gpu": w.B,
                       "tokens_per_gpu": T, "max_len": w.max_len,
                       "l2": "256 MB flush between timed steps",
                       "precision": "tensor-core operands fp16 (layer 0's f1 bf16), fp32 "
                                    "accumulation; input and output bf16",
                       "parallelism": f"replicas x{world} (users independent, no collective)"},
            "tflops": round(step_flops / (ms / 1e3) / 1e12, 1),
            "tensor_frac": tensor_frac(step_flops / (ms / 1e3) / 1e12, peaks),
            "roofline": roofline,
            # per-kernel split of the step's device time (a traced pass of the
            # same steps after the timed region)
            "kernels": {k: {"launches": v[0], "ms": round(v[1], 3),
                            "share": round(v[1] / max(1e-9, sum(x[1] for x in per_kernel.values())), 4)}
                        for k, v in sorted(per_kernel.items(), key=lambda kv: -kv[1][1])},
            "cpu_baseline": cpu,
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": round(e2e_ms, 4),
                    "mode": "pipelined: step i+1's upload and step i-1's download overlap "
                            "step i's compute (separate copy streams)",
                    "serial_ms_per_step": round(e2e_serial_ms, 4),
                    "serial_value": tokens / (e2e_serial_ms / 1e3)},
            "gpu_launches": int(n_launch),
            "untraced_ms_per_step": round(untraced_ms, 4),
            "untraced_value": tokens / (untraced_ms / 1e3),
            "clocks": clk.summary(),
            "stochastic_length": sl,
            "full_pipeline": pipe,
            "retrieval": ret,
            "comparator": cmp_,
            "layer_legs": legs,
            "backward": bwd,
            # last key: the second half of the metric (candidates/s)
            "mfalcon": mf,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return line


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import hstu_workloads as hw
    w = hw.full_stack(seed=args.seed)
    base = cpu_baseline_stack(w, 1)  # warm caches / BLAS threads
    del base
    vals = []
    sample_tokens = args.ref_tokens
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline_stack(w, sample_tokens)
        if i >= args.warmup:
            vals.append(cb)
    v = sum(c["value"] for c in vals) / len(vals)
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded; random-init weights)", "impl": "reference",
            "config": {"workload": "full_stack", "sample": vals[0]["sample"]},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": vals[0]["cores"],
                             "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return line


def run_leg(args):
    """One workload alone, W untimed and K timed calls, for profilers: prints
    one small JSON line (not the bench line).  Legs: full_stack (the 8-layer
    stack), long_history / single_layer (one layer), mfalcon (ranking),
    backward (the 8-layer stack's backward pass), comparator (the
    softmax-Transformer layer on the long-history workload)."""
    import torch
    import hstu_workloads as hw
    import hstu_sequential_transducer_layer_b200 as H
    from hstu_sequential_transducer_layer_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    make = {"full_stack": hw.full_stack, "long_history": hw.long_history,
            "single_layer": hw.single_layer, "mfalcon": hw.mfalcon,
            "backward": hw.full_stack, "comparator": hw.long_history}[args.leg]
    H.hstu_set_option("ln_fusion", args.ln_fusion)
    w = make(seed=args.seed)
    r = H.HSTURunner(hw.dims_dict(w.dims), w.weights, dev)
    off, X, ts = r.to_device(w.offsets, "i64"), r.to_device(w.X), r.to_device(w.timestamps, "i64")
    out = torch.empty_like(X)
    if args.leg == "mfalcon":
        co, cx, hv = r.to_device(w.cand_offsets, "i64"), r.to_device(w.candidates), r.to_device(w.head_vec)
        sc = torch.empty(w.candidates.shape[0], dtype=torch.float32, device=dev)
        fn = lambda: r.rank(off, X, ts, co, cx, None, w.microbatch, hv, w.max_len, w.max_cands,
                            scores=sc)
    elif args.leg == "backward":
        dY = torch.randn(X.shape, device=dev).to(torch.bfloat16)
        fn = lambda: r.stack_bwd(off, X, ts, dY, w.max_len)
    elif args.leg == "comparator":
        rt = H.TransformerRunner(512, 8, 2048, hw.transformer_weights(args.seed, 512, 2048),
                                 device=dev)
        fn = lambda: rt.layer(off, X, w.max_len, out=out)
        r = rt
    else:
        fn = lambda: r.stack(off, X, ts, w.max_len, out=out)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    # one more call with an event pair around every launch: per-kernel
    # launches and device time of one call
    H.hstu_trace_enable(8192)
    fn()
    torch.cuda.synchronize()
    tr = H.hstu_trace_read()
    H.hstu_trace_enable(0)
    ker = {}
    for kid, t in tr:
        e = ker.setdefault(H.hstu_kernel_name(kid), [0, 0.0])
        e[0] += 1
        e[1] += t
    st = r.bwd_status() if args.leg == "backward" else r.status()
    print(json.dumps({"leg": args.leg, "ms_per_call": ms, "status": st,
                      "kernels_per_call": {k: [v[0], round(v[1], 4)] for k, v in
                                           sorted(ker.items(), key=lambda kv: -kv[1][1])}}),
          flush=True)
    if st != 0:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-mfalcon", action="store_true")
    ap.add_argument("--no-sl", action="store_true")
    ap.add_argument("--no-retrieval", action="store_true")
    ap.add_argument("--no-comparator", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-layer-legs", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--ln-fusion", type=int, default=2, choices=[0, 1, 2],
                    help="1: LayerNorm * U formed inside f2's operand stage; 0: a separate "
                         "kernel; 2: by layer width (inside f2 when d_model <= 512)")
    ap.add_argument("--cpu-tokens", type=int, default=4000)
    ap.add_argument("--ref-tokens", type=int, default=2000,
                    help="reference arm: whole users per step, drawn like the CPU baseline's, "
                         "until this many tokens")
    ap.add_argument("--leg", default=None,
                    choices=["full_stack", "long_history", "single_layer", "mfalcon", "backward",
                             "comparator"],
                    help="run one workload alone (for profilers) instead of the bench line")
    args = ap.parse_args()
    if args.leg:
        run_leg(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
