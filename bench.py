"""Benchmark of the DART mixer forward (chunk states + SSD scan + SMA + gated combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one dart_layer_fwd over the Mamba-2-370M-shaped workload (batch 4,
32 heads, L=8192, S=256, N=128, P=64, G=1, bf16, per-head gate), inputs resident
in HBM, L2 flushed (a 256 MiB write) before every step outside the timed span.
Timing: CUDA events around every step on the launching stream, barrier + device
synchronize on both sides of the timed region, max over ranks. Prints one JSON
line on rank 0. For N > 1 (torchrun) every rank runs its own batch (weak
scaling); the only collectives are the barrier and the max of the times.

``--impl reference`` times the float64 CPU oracle (the one reference this
method has) on a bounded sample of the same workload and prints its line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from typing import Optional

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "DART mixer fwd tokens/s at L=8192 (1 B200); % bf16 tensor peak / % HBM BW"
WORKLOAD = W.M370M_BF16
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(w: W.LayerWorkload) -> str:
    return (f"{w.name}: batch {w.batch}, {w.nheads} heads, L={w.seqlen}, S={w.chunk}, N={w.dstate}, "
            f"P={w.headdim}, G={w.ngroups}, {w.dtype}, gate {w.gate}")


def sma_pairs(w: W.LayerWorkload) -> int:
    """(token, historical chunk) pairs of one forward: sum over tokens of chunk(t), per (b, h)."""
    per_bh = sum(min(w.chunk, w.seqlen - i * w.chunk) * i for i in range(w.nchunks))
    return w.batch * w.nheads * per_bh


def sma_flops(w: W.LayerWorkload) -> float:
    """Algorithmic MMA flops of SMA: per pair 2NP for Q dH plus 2NP for C dH (eq 12)."""
    return float(sma_pairs(w)) * 4.0 * w.dstate * w.headdim


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples nvidia-smi SM clock and throttle reasons every 200 ms in the background.

    Each sample is timestamped on arrival; summary() keeps the samples that fall in
    the window marked by mark_start() / mark_end() (widened by one sampling period).
    """

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.2

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.t_start = None
        self.t_end = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(int(self.PERIOD_S * 1000))], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t0 = time.monotonic()
            while not self.lines and time.monotonic() - t0 < 5.0:  # wait for the sampler to be running
                time.sleep(0.02)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark_start(self):
        self.t_start = time.monotonic()

    def mark_end(self):
        self.t_end = time.monotonic()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(self.PERIOD_S * 1.5)  # let one more sample land after the window
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lo = (self.t_start or 0.0) - self.PERIOD_S
        hi = (self.t_end or float("inf")) + self.PERIOD_S
        for t, line in self.lines:
            if not (lo <= t <= hi):
                continue
            parts = [q.strip() for q in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() in ("active", "1"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def source_digest(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, digest: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on this exact kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_digest") != digest:
        return None
    return rec.get("bytes_per_launch_full_size")


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; only barrier and max of times)
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(value: float, dist, device) -> float:
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        import torch

        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def weak_scaling_value(tokens_per_rank: int, world: int, max_total_s: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / max_total_s


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_gpu(args, world, rank, local):
    import torch

    import ssm_state_memory_b200 as dart
    from ssm_state_memory_b200 import _lib

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    w = WORKLOAD
    inp = W.make_layer_inputs(w, seed=W.BASE_SEED + w.index + 1000 * rank)

    def dev(x):
        if isinstance(x, W.Stored):
            if x.dtype == "bf16":
                return torch.from_numpy(x.storage.view(np.int16)).view(torch.bfloat16).to(device)
            return torch.from_numpy(x.storage).to(device)
        return torch.from_numpy(np.ascontiguousarray(x)).to(device)

    names = ("X", "B", "C", "Q", "E", "logA", "g")
    d_in = {k: dev(inp[k]) for k in names}
    d = dart.dims_from(d_in["X"], d_in["B"], w.chunk)
    out = torch.empty(d_in["X"].shape, dtype=torch.float32, device=device)
    dH = torch.empty((w.batch, w.nheads, w.nchunks, w.dstate, w.headdim), dtype=d_in["X"].dtype, device=device)
    lse = torch.empty((w.batch, w.nheads, w.seqlen), dtype=torch.float32, device=device)
    ws = dart.workspace(dart.OP_LAYER_FWD, d, d_in["X"].dtype, device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        dart.dart_layer_fwd(d, d_in["X"], d_in["B"], d_in["C"], d_in["Q"], d_in["E"], d_in["logA"], d_in["g"],
                            inp["g_strides"], out, dH, lse, ws)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        for _ in range(args.warmup):
            flush.fill_(1)
            step()
        torch.cuda.synchronize()
        dart.dart_profile_reset()
        barrier(dist, device)
        torch.cuda.synchronize()
        launches0 = dart.dart_kernel_launches()
        clocks.mark_start()
        for i in range(args.steps):
            flush.fill_(1)  # evict L2 (126 MB) between steps, outside the timed span
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
    barrier(dist, device)
    launches = dart.dart_kernel_launches() - launches0
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    # Per-kernel split and the dominant kernel's launch duration: the same K steps again, timed by the
    # library's launch events (an event before and after every kernel). They are kept out of the pass
    # above because the events between kernels take GPU time of their own (about 15 us per step).
    barrier(dist, device)
    torch.cuda.synchronize()
    dart.dart_profile_enable(True)
    for i in range(args.steps):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    dart.dart_profile_enable(False)
    kern = {k: v for k, v in dart.profile_table().items() if v[1] > 0}
    dart.dart_profile_reset()
    max_ms = max_over_ranks(total_ms, dist, device)
    tokens = w.batch * w.seqlen
    value = weak_scaling_value(tokens * args.steps, world, max_ms / 1e3)

    # roofline of the dominant kernel (SMA)
    peaks, peak_src = load_peaks()
    tc = "sma_fwd_tc" in kern
    sma_name = "sma_fwd_tc" if tc else "sma_fwd"
    sma_ms, sma_n = kern.get(sma_name, (float("nan"), 0))
    sma_avg_s = sma_ms / max(sma_n, 1) / 1e3
    flops = sma_flops(w)
    achieved = flops / sma_avg_s / 1e12
    if tc:
        bound, peak = "tensor", float(peaks["bf16_tflops"])
        peak_note = f"dense bf16 cuBLAS burst, {peak_src}"
        digest = source_digest(["ssm_state_memory_b200/csrc/k_sm100.cu", "ssm_state_memory_b200/csrc/sm100_ptx.cuh"])
    else:
        # fp32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 flop x max SM clock
        bound = "alu"
        peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
        peak_note = "fp32 FMA peak from 148 SMs x 128 lanes x 2 flop x max SM clock"
        digest = source_digest(["ssm_state_memory_b200/csrc/k_simt.cu"])
    traffic = recorded_traffic(sma_name, digest)

    # end to end through the public API: pinned host inputs -> device -> layer -> host output
    pinned = {k: (torch.from_numpy(inp[k].storage.view(np.int16)).view(torch.bfloat16) if isinstance(inp[k], W.Stored)
                  and inp[k].dtype == "bf16" else torch.from_numpy(np.ascontiguousarray(
                      inp[k].storage if isinstance(inp[k], W.Stored) else inp[k]))).pin_memory() for k in names}
    host_outs = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = host_outs[0].numel() * host_outs[0].element_size()
    # Steps are pipelined as a streaming user would run them: step k + 1's inputs copy in (its own stream)
    # while step k computes and step k - 1's output copies out (a third stream), with two device sets of
    # inputs and outputs. Every step still moves all of its inputs in and all of its output out; the
    # timed span runs from the first input copy to the last output copy. Up to 32 steps, so that the
    # pipeline's fill and drain (one input copy and one output copy) weigh little against the steady state.
    e2e_steps = max(1, min(args.steps, 32))
    sets = [(d_in, out), ({k: torch.empty_like(v) for k, v in d_in.items()}, torch.empty_like(out))]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of set j have landed
    ev_done = [torch.cuda.Event() for _ in range(2)]  # the step on set j has finished (inputs free, output ready)
    ev_out = [torch.cuda.Event() for _ in range(2)]   # output of set j has been copied out
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(e2e_steps):
        j = i % 2
        di, do = sets[j]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[j])
            for k in names:
                di[k].copy_(pinned[k], non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if i >= 2:
            stream.wait_event(ev_out[j])
        flush.fill_(1)
        dart.dart_layer_fwd(d, di["X"], di["B"], di["C"], di["Q"], di["E"], di["logA"], di["g"], inp["g_strides"], do,
                            dH, lse, ws)
        ev_done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[j])
            host_outs[j].copy_(do, non_blocking=True)
            ev_out[j].record(s_out)
    s_out.wait_event(ev_out[(e2e_steps - 1) % 2])
    s_out.wait_stream(s_in)
    t1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), dist, device)
    e2e_value = weak_scaling_value(tokens * e2e_steps, world, e2e_ms / 1e3)
    barrier(dist, device)

    sma_alone = run_sma_standalone(d, d_in, dH, flush, stream, peaks, flops) if args.sma_variants else None
    barrier(dist, device)
    bwd = (run_sma_backward(w, d, d_in, dH, flush, stream, peaks, flops,
                            norm_eps=1e-6 if args.sma_variants else None) if args.backward else None)
    barrier(dist, device)
    decode = run_decode(max(10, min(args.steps, 50)), 3, device, args.decode_batch) if args.decode else None
    barrier(dist, device)

    result = None
    if rank == 0:
        result = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; the paper's value distributions)",
            "config": {"workload": workload_desc(w), "tokens_per_step_per_gpu": tokens,
                       "l2": "flushed (256 MiB write) before every step, outside the timed span",
                       "parallelism": f"dp{world} (independent batches per GPU, no data-path collective)"},
            "roofline": {"bound": bound, "kernel": sma_name, "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_flops_per_launch": flops, "avg_launch_ms": sma_avg_s * 1e3,
                         "peak_source": peak_note},
            "kernels_ms_per_step": {k: v[0] / args.steps for k, v in kern.items()},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                    "overlap": "step k+1's inputs copy in and step k-1's output copies out while step k "
                               "computes (three streams, two device sets)"},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
        }
        if decode is not None:
            result["decode"] = decode
        if sma_alone is not None:
            result["sma_standalone"] = sma_alone
        if bwd is not None:
            result["sma_backward"] = bwd
    if dist is not None:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return result, inp, {"d": d, "d_in": d_in, "dH": dH}


# ---------------------------------------------------------------------------
# SMA on its own: the plain score branch and the normalised one (App. B.1)
# ---------------------------------------------------------------------------

def run_sma_standalone(d, d_in, dH, flush, stream, peaks, flops, eps: float = 1e-6, steps: int = 3):
    """Time dart_sma_fwd, dart_sma_fwd_norm_ws (key factors r in a pass of their own) and dart_sma_fwd_norm
    (r computed by the SMA kernel's scaler warps) on the layer's own inputs and the chunk memories the
    timed layer steps left in dH (L2 flushed before each call, CUDA events on the launching stream)."""
    import torch

    import ssm_state_memory_b200 as dart

    R = torch.empty(d_in["E"].shape, dtype=torch.float32, device=d_in["E"].device)
    lse = torch.empty((d.batch, d.nheads, d.seqlen), dtype=torch.float32, device=R.device)
    args = (d, d_in["Q"], d_in["C"], d_in["E"], dH, R, lse)
    ws = dart.workspace(dart.OP_SMA_FWD_NORM, d, d_in["Q"].dtype, R.device)
    calls = {"plain": lambda: dart.dart_sma_fwd(*args),
             "normalised": lambda: dart.dart_sma_fwd_norm_ws(*args, eps, ws),
             "normalised_in_kernel": lambda: dart.dart_sma_fwd_norm(*args, eps)}
    out = {"flops_per_call": flops, "peak_tflops": float(peaks["bf16_tflops"]), "eps": eps, "steps": steps}
    for name, call in calls.items():
        flush.fill_(1)
        call()  # warm-up
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in ev:
            flush.fill_(1)
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in ev) / steps
        # per-kernel split from one more call with the library's launch events on (kept out of the timed
        # calls: the events' host work delays the launch behind the flush)
        flush.fill_(1)
        dart.dart_profile_reset()
        dart.dart_profile_enable(True)
        call()
        torch.cuda.synchronize()
        dart.dart_profile_enable(False)
        kern = {k: v[0] for k, v in dart.profile_table().items() if v[1] > 0}
        dart.dart_profile_reset()
        tf = flops / (ms / 1e3) / 1e12
        out[name] = {"ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / out["peak_tflops"], "kernels_ms": kern}
    return out


# ---------------------------------------------------------------------------
# SMA backward by recomputation (dart_sma_bwd)
# ---------------------------------------------------------------------------

def run_sma_backward(w, d, d_in, dH, flush, stream, peaks, fwd_flops, steps: int = 3,
                     norm_eps: Optional[float] = None):
    """Time dart_sma_bwd on the layer's inputs, the chunk memories the timed steps left in dH, R and lse
    from dart_sma_fwd, and a seeded dR (L2 flushed before each call, CUDA events on the stream).

    Algorithmic MMA flops: per (token, chunk) pair 12NP = the recomputed Q dH and C dH (4NP), dQ and dC
    (4NP) and the two contractions of ddH (4NP), i.e. 3x the forward's."""
    import torch

    import ssm_state_memory_b200 as dart

    dev = d_in["E"].device
    R = torch.empty(d_in["E"].shape, dtype=torch.float32, device=dev)
    lse = torch.empty((d.batch, d.nheads, d.seqlen), dtype=torch.float32, device=dev)
    dart.dart_sma_fwd(d, d_in["Q"], d_in["C"], d_in["E"], dH, R, lse)
    dR = torch.from_numpy(W.make_readout_grad(w)).to(dev)
    dQ = torch.empty(d_in["Q"].shape, dtype=torch.float32, device=dev)
    dC = torch.empty_like(dQ)
    dE = torch.empty(d_in["E"].shape, dtype=torch.float32, device=dev)
    ddH = torch.empty(dH.shape, dtype=torch.float32, device=dev)
    ws = dart.workspace(dart.OP_SMA_BWD, d, d_in["Q"].dtype, dev)

    def call():
        dart.dart_sma_bwd(d, d_in["Q"], d_in["C"], d_in["E"], dH, R, lse, dR, dQ, dC, dE, ddH, ws)

    flush.fill_(1)
    call()  # warm-up
    torch.cuda.synchronize()
    dart.dart_profile_reset()
    dart.dart_profile_enable(True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush.fill_(1)
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    dart.dart_profile_enable(False)
    kern = {k: v[0] / steps for k, v in dart.profile_table().items() if v[1] > 0}
    dart.dart_profile_reset()
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    flops = 3.0 * fwd_flops
    tf = flops / (ms / 1e3) / 1e12
    out = {"ms": ms, "algorithmic_flops": flops, "tflops": tf, "frac_of_bf16_peak": tf / float(peaks["bf16_tflops"]),
           "kernels_ms": kern, "steps": steps}
    if norm_eps is not None:
        # the normalised branch's backward (tensor cores: logits from the key rows as bf16 hi + lo pairs,
        # recomputed softmax statistics, gradient products in fp16), one warm-up call, then `steps` timed
        # calls with L2 flushed before each
        wsn = dart.workspace(dart.OP_SMA_BWD_NORM, d, d_in["Q"].dtype, dev)

        def call_norm():
            dart.dart_sma_bwd_norm(d, norm_eps, d_in["Q"], d_in["C"], d_in["E"], dH, R, lse, dR, dQ, dC, dE, ddH, wsn)

        flush.fill_(1)
        call_norm()
        torch.cuda.synchronize()
        dart.dart_profile_reset()
        dart.dart_profile_enable(True)
        evn = []
        for _ in range(steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush.fill_(1)
            a.record(stream)
            call_norm()
            b.record(stream)
            evn.append((a, b))
        torch.cuda.synchronize()
        dart.dart_profile_enable(False)
        kern_n = {k: v[0] / steps for k, v in dart.profile_table().items() if v[1] > 0}
        dart.dart_profile_reset()
        msn = sum(a.elapsed_time(b) for a, b in evn) / steps
        out["normalised"] = {"ms": msn, "eps": norm_eps, "tflops": flops / (msn / 1e3) / 1e12,
                             "frac_of_bf16_peak": flops / (msn / 1e3) / 1e12 / float(peaks["bf16_tflops"]),
                             "kernels_ms": kern_n, "steps": steps,
                             "engine": "tensor cores (logits from bf16 hi + lo key rows; gradient products in fp16)"}
    return out


# ---------------------------------------------------------------------------
# single-token decode over the cached chunk memories (bandwidth-bound)
# ---------------------------------------------------------------------------

def run_decode(steps: int, warmup: int, device, batch: int = 0):
    """Time dart_sma_decode on the decode workload (64 x 32 heads, 256 cached chunks, 8.6 GB cache)."""
    import torch

    import ssm_state_memory_b200 as dart
    import workloads.device as WD

    w = W.DECODE_BF16 if not batch else W.DECODE_BF16.with_(batch=batch)
    inp = W.make_decode_inputs(w)

    def dev(x):
        return torch.from_numpy(x.storage.view(np.int16)).view(torch.bfloat16).to(device)

    Q, C, E, Y = (dev(inp[k]) for k in ("Q", "C", "E", "Y"))
    g = torch.from_numpy(inp["g"]).to(device)
    cache = torch.empty((w.batch, w.nheads, w.n_chunks, w.dstate, w.headdim), dtype=torch.bfloat16, device=device)
    WD.fill_cache(cache, w, inp["key"])
    out = torch.empty(Y.shape, dtype=torch.float32, device=device)
    lse = torch.empty((w.batch, w.nheads), dtype=torch.float32, device=device)
    nbytes = dart.dart_decode_workspace_size(w.batch, w.nheads, w.dstate, w.headdim, w.n_chunks, dart.DART_BF16)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)

    def step():
        dart.dart_sma_decode(w.n_chunks, Q, C, E, Y, g, inp["g_strides"], cache, out, lse, ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    dart.dart_profile_reset()
    dart.dart_profile_enable(True)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):  # the 8.6 GB cache is 68x the L2, so every step streams it from HBM
        step()
    b.record(stream)
    torch.cuda.synchronize()
    dart.dart_profile_enable(False)
    kern = {k: v for k, v in dart.profile_table().items() if v[1] > 0}
    dart.dart_profile_reset()
    ms = a.elapsed_time(b) / steps
    cache_bytes = cache.numel() * cache.element_size()
    vec_bytes = sum(t.numel() * t.element_size() for t in (Q, C, E, Y, out, lse))
    k_ms, k_n = kern.get("sma_decode", (float("nan"), 1))
    peaks, src = load_peaks()
    gbs_kernel = cache_bytes / (k_ms / k_n / 1e3) / 1e9
    # the whole decode step: state update (state, open chunk memory), readout over the cached memories
    # before the token's chunk, combine; a step that closes no chunk (the common case: one in S closes)
    Xd, Bd = dev(inp["X"]), dev(inp["B"])
    logA = torch.from_numpy(inp["logA"]).to(device)
    state = torch.zeros((w.batch, w.nheads, w.dstate, w.headdim), dtype=torch.float32, device=device)
    acc = torch.zeros_like(state)
    n_hist = w.n_chunks - 1
    nb2 = dart.dart_decode_step_workspace_size(w.batch, w.nheads, w.dstate, w.headdim, n_hist, dart.DART_BF16)
    ws2 = torch.empty(max(nb2, 256), dtype=torch.uint8, device=device)

    def full_step():
        dart.dart_decode_step(n_hist, False, Xd, Bd, C, Q, E, logA, g, inp["g_strides"], state, acc, cache, out, lse,
                              ws2)

    for _ in range(warmup):
        full_step()
    torch.cuda.synchronize()
    dart.dart_profile_reset()
    dart.dart_profile_enable(True)
    a.record(stream)
    for _ in range(steps):
        full_step()
    b.record(stream)
    torch.cuda.synchronize()
    dart.dart_profile_enable(False)
    kern2 = {k: v for k, v in dart.profile_table().items() if v[1] > 0}
    dart.dart_profile_reset()
    ms2 = a.elapsed_time(b) / steps
    state_bytes = 4 * state.numel() * state.element_size()  # state and open memory, each read and written
    step2_bytes = cache_bytes * n_hist // w.n_chunks + state_bytes + vec_bytes
    del cache, state, acc
    torch.cuda.empty_cache()
    return {
        "workload": (f"{w.name}: batch {w.batch}, {w.nheads} heads, {w.n_chunks} cached chunk memories "
                     f"(N={w.dstate}, P={w.headdim}, bf16, {cache_bytes / 1e9:.2f} GB), one new token per row"),
        "tokens_per_s": w.batch * 1e3 / ms, "ms_per_step": ms, "steps": steps,
        "roofline": {"bound": "hbm", "kernel": "sma_decode", "achieved": gbs_kernel,
                     "peak": float(peaks["hbm_gbs"]), "unit": "GB/s", "frac": gbs_kernel / float(peaks["hbm_gbs"]),
                     "algorithmic_bytes_per_launch": cache_bytes, "avg_launch_ms": k_ms / k_n,
                     "peak_source": f"STREAM-style copy, {src}"},
        "step_bytes": cache_bytes + vec_bytes,
        "kernels_ms_per_step": {k: v[0] / steps for k, v in kern.items()},
        "full_step": {
            "what": (f"dart_decode_step: state and open chunk memory (fp32) updated, readout over {n_hist} "
                     f"cached memories, combine; no chunk closes in the timed steps"),
            "tokens_per_s": w.batch * 1e3 / ms2, "ms_per_step": ms2, "bytes_per_step": step2_bytes,
            "gbs": step2_bytes / (ms2 / 1e3) / 1e9,
            "kernels_ms_per_step": {k: v[0] / steps for k, v in kern2.items()},
        },
    }


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline on the GPU line, and the --impl reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w: W.LayerWorkload, inp, heads, threads, rows=(0,)):
    """Time the float64 oracle on the given batch rows and heads (full sequence each). Returns seconds;
    the conversion of each row's inputs to float64 is outside the timed span."""
    import oracle

    orc = oracle.get()
    hs = list(heads)
    gd = W.gate_dense(inp["g"], inp["g_strides"], w.batch, w.seqlen, w.nheads)
    secs = 0.0
    for b in rows:
        def part(st, head_axis=True):
            a = st.storage[b:b + 1]
            if head_axis:
                a = a[:, :, hs]
            return W.Stored(np.ascontiguousarray(a), st.dtype).f64

        X, E = part(inp["X"]), part(inp["E"])
        B, C, Q = part(inp["B"], False), part(inp["C"], False), part(inp["Q"], False)
        logA = np.ascontiguousarray(inp["logA"][b:b + 1][:, :, hs])
        g = np.ascontiguousarray(gd[b:b + 1][:, :, hs])
        t0 = time.perf_counter()
        orc.layer(X, B, C, Q, E, logA, g, (w.seqlen * len(hs), len(hs), 1), w.chunk, threads=threads)
        secs += time.perf_counter() - t0
    return secs


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def norm_sampled_error(w: W.LayerWorkload, inp, ctx, eps: float = 1e-6, n_tokens: int = 64):
    """Accuracy of the normalised SMA forward (dart_sma_fwd_norm_ws, the timed call) at the bench workload:
    the float64 oracle's chunk memories of two (batch row, heads) samples, rounded once to bf16, replace the
    GPU's in those heads; the oracle then computes the normalised readout at sampled tokens of chunks >= 1,
    and the result is max |R_gpu - R_ref| / rms(R_ref) over the samples."""
    import torch

    import oracle
    import ssm_state_memory_b200 as dart

    t0 = time.perf_counter()
    orc = oracle.get()
    d, d_in = ctx["d"], ctx["d_in"]
    dH = ctx["dH"].clone()
    S, L = w.chunk, w.seqlen
    rng = np.random.default_rng(w.index + 11)
    tok = np.sort(rng.choice(np.arange(S, L), size=min(n_tokens, L - S), replace=False))

    def part(st, b, heads=None):
        a = st.storage[b:b + 1]
        if heads is not None:
            a = a[:, :, list(heads)]
        return W.Stored(np.ascontiguousarray(a), st.dtype).f64

    samples = [(0, [0, min(13, w.nheads - 1)]), (w.batch - 1, [min(7, w.nheads - 1), w.nheads - 1])]
    refs = []
    for b, hs in samples:
        dH_o = orc.chunk_states(part(inp["X"], b, hs), part(inp["B"], b),
                                np.ascontiguousarray(inp["logA"][b:b + 1][:, :, hs]), S)
        st = W.store(dH_o, w.dtype)
        dH[b, hs] = torch.from_numpy(st.storage.view(np.int16)).view(torch.bfloat16).to(dH.device)[0]
        refs.append((b, hs, st.f64))
    R = torch.empty(d_in["E"].shape, dtype=torch.float32, device=dH.device)
    lse = torch.empty((w.batch, w.nheads, w.seqlen), dtype=torch.float32, device=dH.device)
    ws = dart.workspace(dart.OP_SMA_FWD_NORM, d, d_in["Q"].dtype, dH.device)
    dart.dart_sma_fwd_norm_ws(d, d_in["Q"], d_in["C"], d_in["E"], dH, R, lse, eps, ws)
    torch.cuda.synchronize()
    tok_t = torch.as_tensor(tok, device=R.device)
    worst = 0.0
    for b, hs, dH64 in refs:
        R_ref, _ = orc.sma(part(inp["Q"], b), part(inp["C"], b), part(inp["E"], b, hs), dH64, S, tokens=tok,
                           norm_eps=eps)
        got = R[b][tok_t][:, hs].double().cpu().numpy()
        worst = max(worst, float(np.abs(got - R_ref[0]).max() / np.sqrt((R_ref[0] ** 2).mean())))
    return {"max_abs_err_over_rms": worst, "eps": eps,
            "sample": (f"{len(tok)} tokens of chunks >= 1 x heads {samples[0][1]} of batch row {samples[0][0]} and "
                       f"{samples[1][1]} of row {samples[1][0]}; float64 oracle on its own chunk memories "
                       f"(rounded once to bf16, the GPU reading the same)"),
            "seconds": time.perf_counter() - t0}


def cpu_baseline(w: W.LayerWorkload, inp, n_heads: int, n_rows: int):
    threads = cpu_threads()
    heads = range(n_heads)
    n_rows = max(1, min(n_rows, w.batch))
    secs = oracle_sample(w, inp, heads, threads, rows=range(n_rows))
    frac = n_heads * n_rows / (w.batch * w.nheads)  # share of the (batch, head) work the sample covers
    value = w.batch * w.seqlen * frac / secs
    return {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": (f"float64 oracle (recurrence + direct-sum chunk memories + explicit-loop SMA + combine) on "
                       f"batch rows 0..{n_rows - 1}, heads 0..{n_heads - 1}, all {w.seqlen} tokens = {frac:.4f} "
                       f"of one step; {secs:.2f} s; CPU {cpu_model()}"),
            "seconds": secs}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = WORKLOAD
    inp = W.make_layer_inputs(w)
    cores = cpu_threads()
    # size each step's sample so that the whole run stays within about 150 s of oracle time
    t_one = oracle_sample(w, inp, range(1), cores)
    budget = 150.0 / max(1, args.steps + args.warmup)
    n_heads = int(max(1, min(args.ref_heads, budget // max(t_one, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample(w, inp, range(n_heads), cores)
    secs = [oracle_sample(w, inp, range(n_heads), cores) for _ in range(args.steps)]
    frac = n_heads / (w.batch * w.nheads)
    total = sum(secs)
    value = w.batch * w.seqlen * frac * args.steps / total
    sample = (f"each step: float64 oracle on batch row 0, heads 0..{n_heads - 1}, all {w.seqlen} tokens "
              f"({frac:.4f} of the workload); CPU {cpu_model()}")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3 / frac,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; the paper's value distributions)",
        "config": {"workload": workload_desc(w), "tokens_per_step_per_gpu": w.batch * w.seqlen},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-heads", type=int, default=32, help="heads per batch row in the cpu_baseline sample")
    ap.add_argument("--cpu-rows", type=int, default=4, help="batch rows in the cpu_baseline sample")
    ap.add_argument("--ref-heads", type=int, default=8, help="max (batch, head) pairs per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", dest="decode", action="store_false",
                    help="skip the single-token decode measurement that is reported under 'decode'")
    ap.add_argument("--no-backward", dest="backward", action="store_false",
                    help="skip the SMA backward timing")
    ap.add_argument("--no-sma-variants", dest="sma_variants", action="store_false",
                    help="skip the standalone SMA timings (plain and normalised score branch)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="batch rows of the decode measurement (default: the decode workload's 64)")
    ap.add_argument("--batch", type=int, default=0,
                    help="batch rows of the layer workload (default: its 4); a smaller case for profiling")
    args = ap.parse_args(argv)
    global WORKLOAD
    if args.batch:
        WORKLOAD = W.M370M_BF16.with_(batch=args.batch)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("run N > 1 under torchrun (one process per GPU)")
    if args.impl == "reference":
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    res, inp, ctx = run_gpu(args, world, rank, local)
    if rank == 0 and res is not None:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(WORKLOAD, inp, args.cpu_heads, args.cpu_rows)
            if "sma_standalone" in res:  # the oracle's sampled check of the timed normalised call
                res["sma_standalone"]["normalised"]["sampled_error"] = norm_sampled_error(WORKLOAD, inp, ctx)
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
