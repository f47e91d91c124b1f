#!/usr/bin/env python3
"""Benchmark of silu_dot_fwd_bwd_quant_fuse on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sdq|reference]
                    [--workload NAME|INDEX] [--no-per-workload] [--no-cpu-baseline]

One step = one call of the fused op over one synthetic batch of the
workload (default: M=16384 tokens, K=7168 channels, the bandwidth-roofline
case and the largest of the five workloads).  Prints ONE JSON line on rank 0;
besides the headline it carries a per_workload list timing all five
workloads (skipped with --no-per-workload).

Timing: W untimed warm-up calls (one eager, W-1 replayed from a CUDA graph
just before the timed region), then EXACTLY K calls replayed from CUDA
graphs, bracketed by a barrier and a device synchronize and timed with CUDA
events on the launching stream; the maximum over ranks is taken.  Between
consecutive calls the inputs and outputs rotate through at least three buffer
sets, and enough to exceed 3x the L2 cache, so no call finds its data in L2:
even where one call moves more than L2 holds (1.07 GB on the default
workload), lines that a call leaves behind in L2 would otherwise serve a
small part of the next call's reads.  The per_workload entries
time each workload for at least about 50 ms of calls.

value = algorithmic bytes of all ranks / time (GB/s); the algorithmic bytes
are 6 B read + 3 B written per (token, channel) plus the fp32 scales.
e2e   = the same metric through the host-buffer entry point (sdq_fuse_host):
        pinned host inputs -> device -> kernel -> all four outputs back to
        pinned host memory, every step inside the timed region.
cpu_baseline / --impl reference = the CPU oracle (single thread) timed on
        bounded samples of the same workload.
with_y / int8_grad_y = side measurements on the same workload: the call that
        also writes the bf16 y, and the call with grad_y as INT8 codes + fp32
        scales (skipped with --no-variants).

Multi-GPU (torchrun): each rank runs an independent replica of the workload
(the op has no exchange step; weak scaling); NCCL carries only the barrier
and the max-over-ranks of the timings.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = W.WORKLOADS[4].name
METRIC = "µs/call and achieved HBM GB/s (fraction of B200 roofline) per (M,K)"
FALLBACK_HBM_GBS = 6650.0
FWD_SOURCES = ["swiglu_backward_int8_b200/csrc/fwd_kernel.cuh",
               "swiglu_backward_int8_b200/csrc/fwd_api.cu",
               "swiglu_backward_int8_b200/csrc/sdq_ptx.cuh"]
KERNEL_SOURCES = ["swiglu_backward_int8_b200/csrc/sdq_kernel.cuh",
                  "swiglu_backward_int8_b200/csrc/sdq_ptx.cuh",
                  "swiglu_backward_int8_b200/csrc/sdq_api.cu"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["sdq", "reference"], default="sdq")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--group-size", type=int, default=128, choices=[32, 64, 128, 256],
                    help="the page's group_size argument for the timed calls (default 128)")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the per_workload list (every workload timed after the headline)")
    ap.add_argument("--per-workload-ms", type=float, default=50.0,
                    help="timed calls per workload: enough for about this many ms")
    ap.add_argument("--per-call", type=int, default=50, metavar="N",
                    help="per_workload entries also time N single calls, each after a write of "
                         "2x L2, for their median / p10 / p90 (0: skip)")
    ap.add_argument("--traffic-probe", type=int, default=0, metavar="N",
                    help="no timing: N rounds of (read a 512 MB buffer, one call, read it again) "
                         "on one buffer set, for an ncu capture of the call's DRAM bytes including "
                         "the write-backs of its outputs that the second read forces")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=0, help="0 = min(steps, 50)")
    ap.add_argument("--codes", choices=["int8", "e4m3"], default="int8",
                    help="code format of the timed calls (the page's: int8)")
    ap.add_argument("--scales", choices=["fp32", "e8m0"], default="fp32",
                    help="scale format of the timed calls (the page's: fp32)")
    ap.add_argument("--y-scale-layout", choices=["k_mg", "mg_k"], default="k_mg")
    ap.add_argument("--op", choices=["fuse", "swiglu_q8_1"], default="fuse",
                    help="fuse: the backward op (the headline); swiglu_q8_1: the forward-side "
                         "SwiGLU + q8_1 rows on the workload's gate and up (rows = M, inter = K)")
    ap.add_argument("--limit", type=float, default=0.0, help="swiglu_q8_1: the clamp (0: none)")
    ap.add_argument("--int8-grad-y", action="store_true",
                    help="also time the call with grad_y given as INT8 codes + fp32 scales "
                         "(on by default; see --no-variants)")
    ap.add_argument("--with-y", action="store_true",
                    help="also time the call with the optional bf16 y output (on by default; "
                         "see --no-variants)")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the side measurements of the y output and the INT8 grad_y input "
                         "unless asked for by --with-y / --int8-grad-y")
    ap.add_argument("--all-formats", action="store_true",
                    help="also time every output format on the workload and add a per_format list")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be at least 3")
    if a.steps < 1:
        ap.error("--steps must be at least 1")
    return a


def pick_workload(name: str) -> W.Workload:
    if name.isdigit():
        return W.WORKLOADS[int(name)]
    return W.BY_NAME[name]


def _code_only(text: str) -> str:
    """C/CUDA source without comments and blank-line or trailing-space
    differences (no string literal in these sources holds a comment marker)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_sha(sources=None) -> str:
    """Digest of a kernel's sources, comments excluded: a profile recorded
    under it stays valid across comment-only edits and lapses with any code
    change."""
    h = hashlib.sha256()
    for f in (sources or KERNEL_SOURCES):
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(workload: str, sources=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current sources of that kernel (else None): bytes read, bytes
    written during the launch and, where recorded, the write-backs of its
    outputs still dirty in L2 when it ends (forced out by a following read
    of a buffer larger than L2)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = kernel_sha(sources)
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == workload and parts[1] == sha:
            return sum(int(v) for v in parts[2:5])
    return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (every 200 ms) of this GPU's clocks and reasons."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", gpu_uuid],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                self.samples.append({
                    "t": time.time(), "sm": float(parts[1]), "max": float(parts[2]),
                    "active": parts[4], "hw_slowdown": parts[5] == "Active",
                    "hw_thermal_slowdown": parts[6] == "Active",
                    "sw_thermal_slowdown": parts[7] == "Active",
                    "sw_power_cap": parts[8] == "Active"})
            except ValueError:
                continue

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        inside = [s for s in self.samples if t0 <= s["t"] <= t1]
        window = "timed region"
        if not inside:  # region shorter than the sampling period: nearest samples
            inside = [s for s in self.samples if t0 - 0.5 <= s["t"] <= t1 + 0.5] or self.samples[-3:]
            window = "within 0.5 s of the timed region"
        reasons = set()
        for s in inside:
            for k in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"):
                if s[k]:
                    reasons.add(k)
        return {"sm_mhz": statistics.median(s["sm"] for s in inside),
                "sm_max_mhz": max(s["max"] for s in inside), "reasons": sorted(reasons),
                "samples": len(inside), "window": window}


# ---------------------------------------------------------------- distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    return world, rank, local


def workload_config(w: W.Workload, fmt=None, world: int = 1) -> dict:
    """The line's `config`, the same in both arms: the workload, its formats,
    the parallel layout and how L2 is kept out of the timing."""
    fmt = fmt or PAGE_FORMAT
    return {"workload": w.name, "M": w.M, "K": w.K, "group_size": w.group_size,
            "io": "bf16 x, grad_y in; " + {"int8": "int8", "e4m3": "fp8 e4m3"}[fmt[0]]
                  + " codes + " + fmt[1] + " scales out, y_s_t " + fmt[2],
            "parallelism": f"replicas x{world} (no exchange)",
            "l2": "inputs+outputs rotate over at least 3 buffer sets and enough to exceed "
                  "3x L2, so consecutive calls never share buffers"}


# ---------------------------------------------------------------- CPU oracle timing

def time_oracle(w: W.Workload, x, gy, min_seconds=10.0, max_rows=None):
    """Time the CPU oracle (single thread) on a bounded sample of the
    workload: its first R token rows, repeated until min_seconds pass."""
    import oracle
    rows = w.M if max_rows is None else min(w.M, max_rows)
    xs, gys = x[:rows], gy[:rows]
    sw = W.Workload(w.name + "_sample", rows, w.K, w.sigma_x, w.sigma_grad_y, w.seed)
    oracle.silu_dot_fwd_bwd_quant_fuse(xs[:1], gys[:1])  # build/load outside the clock
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.silu_dot_fwd_bwd_quant_fuse(xs, gys)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    gbs = sw.algorithmic_bytes() * reps / el / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {rows} of {w.M} token rows x K={w.K}, {reps} repetitions "
                      f"in {el:.1f} s (single-threaded C++ oracle, fp64)"}


def run_reference(args):
    """--impl reference: the CPU oracle as it stands, on host cores, each step a
    bounded sample (one 128-token group x all K channels, cycling through the
    workload)."""
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    w = pick_workload(args.workload)
    if args.group_size != w.group_size:   # same inputs, another group size
        w = W.Workload(w.name, w.M, w.K, w.sigma_x, w.sigma_grad_y, w.seed, args.group_size,
                       w.outlier_frac, w.outlier_mult, w.zero_group_every)
    x, gy = W.make_inputs(w)
    import oracle
    G = w.group_size
    Mg = w.Mg

    def step(s):
        i = s % Mg
        r0, r1 = i * G, min(w.M, i * G + G)
        oracle.silu_dot_fwd_bwd_quant_fuse(x[r0:r1], gy[r0:r1], G)
        return W.Workload("s", r1 - r0, w.K, 1, 1, 0, G).algorithmic_bytes()

    for s in range(args.warmup):
        step(s)
    total, t0 = 0, time.perf_counter()
    for s in range(args.steps):
        total += step(args.warmup + s)
    el = time.perf_counter() - t0
    gbs = total / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, None, args.gpus),
        "step": f"one {G}-token group x all K channels of the workload (a bounded sample), "
                "cycling through its token groups",
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{args.steps} steps of one {G}-token group x K={w.K}"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU timing

def buffer_sets(bytes_per_call: int, l2_bytes: int) -> int:
    """How many input/output sets the timed calls rotate over: enough that
    the sets together exceed 3x L2, and never fewer than three.  Even where
    one call moves more than L2 holds, consecutive calls over the same
    buffers ran 8 % faster on M=16384 K=7168 (188 against 203-207 us, same
    DRAM bytes within 1 %) and found 0.7 % of their reads in L2; a backward
    pass never hands the op the previous call's buffers."""
    return max(3, -(-3 * l2_bytes // bytes_per_call))


def _to_device_bf16(a_u16, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).view(torch.bfloat16).to(device)


PAGE_FORMAT = ("int8", "fp32", "k_mg")


def format_name(fmt) -> str:
    return "-".join(fmt)


def scale_bytes(fmt) -> int:
    return 1 if fmt[1] == "e8m0" else 4


def int8_grad_y_bytes(w: W.Workload) -> int:
    """Algorithmic bytes of one call with grad_y as INT8 codes + fp32 scales."""
    return w.algorithmic_bytes() - 2 * w.M * w.K + w.M * w.K + 4 * w.M * (w.K // 128)


def measure_device(w: W.Workload, x_np, gy_np, steps: int, warmup: int, device, fmt=PAGE_FORMAT,
                   with_y: bool = False, int8_grad_y=None):
    """int8_grad_y: None, or (codes, scales) numpy arrays used in place of gy_np."""
    import torch
    import swiglu_backward_int8_b200 as sdq
    M, K = w.M, w.K
    codes, scales, layout = fmt
    footprint = w.algorithmic_bytes(scale_bytes(fmt)) + (2 * M * K if with_y else 0)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nsets = buffer_sets(footprint, l2)
    x0 = _to_device_bf16(x_np, device)
    if int8_grad_y is None:
        g0, gs0 = _to_device_bf16(gy_np, device), None
    else:
        g0 = torch.from_numpy(int8_grad_y[0]).to(device)
        gs0 = torch.from_numpy(int8_grad_y[1]).to(device)
    sets = []
    for s in range(nsets):
        xs = x0 if s == 0 else x0.clone()
        gs = g0 if s == 0 else g0.clone()
        gss = gs0 if (s == 0 or gs0 is None) else gs0.clone()
        sets.append((xs, gs, gss, sdq.allocate_outputs(M, K, device, group_size=w.group_size, codes=codes,
                                                       scales=scales, y_scale_layout=layout),
                     torch.empty(M, K, dtype=torch.bfloat16, device=device) if with_y else None))
    stream = torch.cuda.current_stream(device)

    def call(k):
        xs, gs, gss, outs, ys = sets[k % nsets]
        sdq.silu_dot_fwd_bwd_quant_fuse(xs, gs, *outs, w.group_size, codes=codes, scales=scales,
                                        y_scale_layout=layout, y=ys, grad_y_s=gss)

    # W untimed warm-up calls: the first eager (it sets up the library on the
    # device), the other W-1 replayed from a graph right before the timed
    # region, so the GPU is not left idle while the graphs are captured.
    call(0)
    torch.cuda.synchronize(device)

    def capture(first: int, count: int):
        """CUDA graphs of `count` calls from call index `first` (chunks of at most 1000)."""
        out, done = [], 0
        while done < count:
            n = min(1000, count - done)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=torch.cuda.Stream(device)):
                for k in range(n):
                    call(first + done + k)
            out.append(g)
            done += n
        return out

    warm = capture(1, warmup - 1)
    graphs = capture(warmup, steps)
    from swiglu_backward_int8_b200 import parallel
    torch.cuda.synchronize(device)
    for g in warm:
        g.replay()
    torch.cuda.synchronize(device)
    parallel.barrier(device)
    torch.cuda.synchronize(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    ev0.record(stream)
    for g in graphs:
        g.replay()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    t1 = time.time()
    parallel.barrier(device)
    ms = ev0.elapsed_time(ev1)
    st = sdq.sdq_device_status(stream.cuda_stream)
    if st != 0:
        raise RuntimeError(f"device status {sdq.status_string(st)}")
    del graphs, warm
    return ms, (t0, t1), nsets


def measure_per_call(w: W.Workload, x_np, gy_np, calls: int, device, warmup: int = 10) -> dict:
    """Single calls, each after a write of 2x L2 (so it finds none of its data
    in L2) and timed alone by CUDA events around it on the launching stream:
    the latency of one cold call, launch included, as a median and p10/p90.
    The graph-replayed figures time back-to-back calls instead."""
    import torch
    import swiglu_backward_int8_b200 as sdq
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=device)
    x = _to_device_bf16(x_np, device)
    g = _to_device_bf16(gy_np, device)
    outs = sdq.allocate_outputs(w.M, w.K, device, group_size=w.group_size)
    stream = torch.cuda.current_stream(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(calls)]
    for k in range(warmup + calls):
        flush.fill_(k & 0xFF)
        if k >= warmup:
            evs[k - warmup][0].record(stream)
        sdq.silu_dot_fwd_bwd_quant_fuse(x, g, *outs, w.group_size)
        if k >= warmup:
            evs[k - warmup][1].record(stream)
    torch.cuda.synchronize(device)
    st = sdq.sdq_device_status(stream.cuda_stream)
    if st != 0:
        raise RuntimeError(f"device status {sdq.status_string(st)}")
    us = np.array([a.elapsed_time(b) * 1e3 for a, b in evs])
    p10, p50, p90 = np.percentile(us, [10, 50, 90])
    return {"median": float(p50), "p10": float(p10), "p90": float(p90), "calls": calls,
            "l2_flush_bytes": 2 * l2}


def measure_e2e(w: W.Workload, x_np, gy_np, steps: int, device):
    import torch
    import swiglu_backward_int8_b200 as sdq
    M, K = w.M, w.K
    xh = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    gyh = torch.from_numpy(gy_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    outs = [t.pin_memory() for t in sdq.allocate_outputs(M, K, "cpu")]
    ws = torch.empty(sdq.sdq_fuse_host_workspace_bytes(M, K, 0), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    for _ in range(3):
        sdq.silu_dot_fwd_bwd_quant_fuse_host(xh, gyh, *outs, workspace=ws, synchronize=False)
    torch.cuda.synchronize(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        sdq.silu_dot_fwd_bwd_quant_fuse_host(xh, gyh, *outs, workspace=ws, synchronize=False)
    ev1.record(stream)
    torch.cuda.synchronize(device)
    ms = ev0.elapsed_time(ev1) / steps
    h2d = xh.numel() * 2 + gyh.numel() * 2
    d2h = sum(t.numel() * t.element_size() for t in outs)
    return {"value": w.algorithmic_bytes() / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": steps, "path": "sdq_fuse_host (C ABI, pinned host buffers, chunked "
                                    "H2D/kernel/D2H overlap)"}


def run_sdq(args):
    world, rank, local = dist_setup(args)
    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import swiglu_backward_int8_b200 as sdq  # fails loudly if the CUDA library is missing
    from swiglu_backward_int8_b200 import parallel
    parallel.init_from_env("nccl", timeout_s=120.0, device=device)

    w = pick_workload(args.workload)
    if args.group_size != w.group_size:   # same inputs, another group size
        w = W.Workload(w.name, w.M, w.K, w.sigma_x, w.sigma_grad_y, w.seed, args.group_size,
                       w.outlier_frac, w.outlier_mult, w.zero_group_every)
    # Each rank its own replica (seed offset by rank): weak scaling, no exchange.
    wr = W.Workload(w.name, w.M, w.K, w.sigma_x, w.sigma_grad_y, w.seed + 1000 * rank,
                    w.group_size, w.outlier_frac, w.outlier_mult, w.zero_group_every)
    x_np, gy_np = W.make_inputs(wr)
    peak, peak_kind = measured_peaks()

    uuid = str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    time.sleep(0.3)
    fmt = (args.codes, args.scales, args.y_scale_layout)
    ms, (t0, t1), nsets = measure_device(wr, x_np, gy_np, args.steps, args.warmup, device, fmt)
    clocks = sampler.summary(t0, t1)
    ms_max = parallel.max_over_ranks(ms, device)
    per_step_ms = ms_max / args.steps
    bytes_step = w.algorithmic_bytes(scale_bytes(fmt))
    value = parallel.aggregate_gbs(bytes_step * args.steps, world, ms_max)
    achieved = bytes_step / (per_step_ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e and fmt != PAGE_FORMAT:
        e2e = {"unavailable": "the host-buffer entry points write the page's format only"}
    elif not args.no_e2e:
        e2e_steps = args.e2e_steps or min(args.steps, 50)
        e = measure_e2e(wr, x_np, gy_np, e2e_steps, device)
        e_ms = parallel.max_over_ranks(e["ms_per_step"], device)
        e["value"] = parallel.aggregate_gbs(bytes_step, world, e_ms)
        e2e = e

    per = None
    if not args.no_per_workload:
        per = []
        cache = {w.name: (wr, x_np, gy_np)} if rank == 0 or world == 1 else {}
        for ow in W.WORKLOADS:
            if ow.name in cache:
                ow_r, ox, og = cache[ow.name]
            else:
                ow_r = W.Workload(ow.name, ow.M, ow.K, ow.sigma_x, ow.sigma_grad_y,
                                  ow.seed + 1000 * rank, ow.group_size, ow.outlier_frac,
                                  ow.outlier_mult, ow.zero_group_every)
                ox, og = W.make_inputs(ow_r)
            # enough calls for about per_workload_ms at a first guess of 4 TB/s (small
            # workloads are launch-bound, so they run longer than that)
            guess_us = max(5.0, ow.algorithmic_bytes() / 4e3 / 1e3)
            osteps = int(min(10000, max(args.steps, args.per_workload_ms * 1e3 / guess_us)))
            oms, (o0, o1), ons = measure_device(ow_r, ox, og, osteps, args.warmup, device)
            oms = parallel.max_over_ranks(oms, device)
            us = oms / osteps * 1e3
            gbs = ow.algorithmic_bytes() / (us * 1e-6) / 1e9
            entry = {"workload": ow.name, "M": ow.M, "K": ow.K, "us_per_call": us,
                     "GB_s": gbs, "frac_of_measured_hbm": gbs / peak, "frac_of_8TBs": gbs / 8000,
                     "algorithmic_bytes_per_launch": ow.algorithmic_bytes(),
                     "steps": osteps, "buffer_sets": ons,
                     "clocks_sm_mhz": sampler.summary(o0, o1).get("sm_mhz")}
            if args.per_call > 0:   # this rank's own device only: no collective
                try:
                    entry["per_call_us"] = measure_per_call(ow_r, ox, og, args.per_call, device)
                except Exception as exc:   # a side measurement never costs the line
                    entry["per_call_us"] = {"error": f"{type(exc).__name__}: {exc}"[:200]}
            per.append(entry)
            del ox, og

    per_fmt = None
    if args.all_formats:
        per_fmt = []
        for c in ("int8", "e4m3"):
            for sc in ("fp32", "e8m0"):
                for lay in ("k_mg", "mg_k"):
                    f = (c, sc, lay)
                    fms, _, _ = measure_device(wr, x_np, gy_np, args.steps, args.warmup, device, f)
                    fms = parallel.max_over_ranks(fms, device)
                    us = fms / args.steps * 1e3
                    fb = w.algorithmic_bytes(scale_bytes(f))
                    gbs = fb / (us * 1e-6) / 1e9
                    per_fmt.append({"format": format_name(f), "us_per_call": us, "GB_s": gbs,
                                    "frac_of_measured_hbm": gbs / peak,
                                    "algorithmic_bytes_per_launch": fb})

    with_y = None
    if args.with_y or not args.no_variants:   # the same call also writing the optional bf16 y
        yms, _, _ = measure_device(wr, x_np, gy_np, args.steps, args.warmup, device, with_y=True)
        yms = parallel.max_over_ranks(yms, device)
        us = yms / args.steps * 1e3
        yb = w.algorithmic_bytes() + 2 * w.M * w.K
        gbs = yb / (us * 1e-6) / 1e9
        with_y = {"us_per_call": us, "GB_s": gbs, "frac_of_measured_hbm": gbs / peak,
                  "algorithmic_bytes_per_launch": yb, "format": format_name(PAGE_FORMAT)}

    int8_gy = None
    if args.int8_grad_y or not args.no_variants:   # grad_y handed over as INT8 codes + fp32 scales
        qgy = W.quantized_grad_y(wr)
        qms, _, _ = measure_device(wr, x_np, gy_np, args.steps, args.warmup, device,
                                   int8_grad_y=qgy)
        qms = parallel.max_over_ranks(qms, device)
        us = qms / args.steps * 1e3
        qb = int8_grad_y_bytes(w)
        gbs = qb / (us * 1e-6) / 1e9
        int8_gy = {"us_per_call": us, "GB_s": gbs, "frac_of_measured_hbm": gbs / peak,
                   "algorithmic_bytes_per_launch": qb, "format": format_name(PAGE_FORMAT)}

    sampler.stop()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle(w, x_np, gy_np, min_seconds=10.0, max_rows=1024)

    if rank == 0:
        traffic = recorded_traffic(w.name) if fmt == PAGE_FORMAT else None
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_ms,
            "us_per_call": per_step_ms * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(w, fmt, world),
            "buffer_sets": nsets,
            "timing": "K calls replayed from CUDA graphs, CUDA events on the launching stream",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "frac_of_8TBs": achieved / 8000.0,
                         "traffic": traffic, "algorithmic_bytes_per_launch": bytes_step,
                         "kernel": "sdq::fuse_kernel"},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps, "clocks": clocks,
            "kernel_sources_sha": kernel_sha(),
        }
        if per is not None:
            line["per_workload"] = per
            for e in per:   # per_workload runs the page's format at group size 128
                if (e["workload"] == w.name and "per_call_us" in e and fmt == PAGE_FORMAT
                        and w.group_size == 128):
                    line["per_call_us"] = e["per_call_us"]
        if per_fmt is not None:
            line["per_format"] = per_fmt
        if with_y is not None:
            line["with_y"] = with_y
        if int8_gy is not None:
            line["int8_grad_y"] = int8_gy
        print(json.dumps(line), flush=True)
    import torch.distributed as tdist
    if tdist.is_initialized():
        parallel.barrier(device)
        tdist.destroy_process_group()
    return 0


FWD_METRIC = "µs/call and achieved HBM GB/s (fraction of B200 roofline): SwiGLU forward + q8_1 rows"


def fwd_bytes(rows: int, inter: int, with_w: bool = True) -> int:
    """Algorithmic bytes of the forward op: read gate and up (4 B per element)
    and the row weights, write h (2 B) and the q8_1 blocks (36 B per 32)."""
    return rows * inter * 6 + rows * (inter // 32) * 36 + (4 * rows if with_w else 0)


def run_fwd(args):
    """The forward-side neighbour on one GPU: device-timed like the backward
    op (CUDA-graph replay, buffers rotating through >= 3x L2)."""
    import torch
    world, rank, local = dist_setup(args)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import swiglu_backward_int8_b200 as sdq  # fails loudly if the CUDA library is missing
    from swiglu_backward_int8_b200 import parallel
    parallel.init_from_env("nccl", timeout_s=120.0, device=device)
    w = pick_workload(args.workload)
    rows, inter = w.M, w.K
    g_np, u_np, wt_np = W.fwd_inputs(W.Workload(w.name, w.M, w.K, w.sigma_x, w.sigma_grad_y,
                                                w.seed + 1000 * rank, w.group_size, w.outlier_frac,
                                                w.outlier_mult, w.zero_group_every))
    peak, peak_kind = measured_peaks()
    nbytes = fwd_bytes(rows, inter)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nsets = buffer_sets(nbytes, l2)
    x0 = _to_device_bf16(np.concatenate([g_np, u_np], axis=1), device)
    wt0 = torch.from_numpy(wt_np).to(device)
    sets = []
    for k in range(nsets):
        xs = x0 if k == 0 else x0.clone()
        sets.append((xs, wt0 if k == 0 else wt0.clone(),
                     torch.empty((rows, inter), dtype=torch.bfloat16, device=device),
                     torch.empty((rows, inter // 32, 36), dtype=torch.uint8, device=device)))

    def call(k):
        xs, wt, h, q8 = sets[k % nsets]
        sdq.swiglu_q8_1(xs[:, :inter], xs[:, inter:], wt, args.limit, h, q8)

    call(0)   # warm-up 1 of W, eager: sets the library up on the device
    torch.cuda.synchronize(device)

    def capture(first: int, count: int):
        out, done = [], 0
        while done < count:
            n = min(1000, count - done)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=torch.cuda.Stream(device)):
                for k in range(n):
                    call(first + done + k)
            out.append(g)
            done += n
        return out

    warm = capture(1, args.warmup - 1)   # warm-up 2..W, replayed right before the timed region
    graphs = capture(args.warmup, args.steps)
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    time.sleep(0.3)
    stream = torch.cuda.current_stream(device)
    for g in warm:
        g.replay()
    torch.cuda.synchronize(device)
    parallel.barrier(device)
    torch.cuda.synchronize(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    ev0.record(stream)
    for g in graphs:
        g.replay()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    t1 = time.time()
    clocks = sampler.summary(t0, t1)
    sampler.stop()
    ms = parallel.max_over_ranks(ev0.elapsed_time(ev1), device)
    per_ms = ms / args.steps
    achieved = nbytes / (per_ms * 1e-3) / 1e9
    value = parallel.aggregate_gbs(nbytes * args.steps, world, ms)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        r = min(rows, 512)
        gs, us, ws = (np.ascontiguousarray(g_np[:r]), np.ascontiguousarray(u_np[:r]), wt_np[:r])
        oracle.swiglu_q8_1_rows(gs[:1], us[:1], ws[:1])
        reps, c0 = 0, time.perf_counter()
        while time.perf_counter() - c0 < 10.0:
            oracle.swiglu_q8_1_rows(gs, us, ws, args.limit)
            reps += 1
        el = time.perf_counter() - c0
        cpu = {"value": fwd_bytes(r, inter) * reps / el / 1e9, "unit": "GB/s", "cores": 1,
               "kind": "oracle", "sample": f"first {r} of {rows} rows x inter={inter}, {reps} "
                                           f"repetitions in {el:.1f} s (single-threaded C++ oracle, fp64)"}
    if rank == 0:
        print(json.dumps({
            "metric": FWD_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_ms, "us_per_call": per_ms * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": w.name + "_swiglu_q8_1", "rows": rows, "inter": inter,
                       "limit": args.limit, "row_weights": "uniform (0, 1]",
                       "io": "bf16 gate, up, fp32 w in; bf16 h + q8_1 blocks out",
                       "parallelism": f"replicas x{world} (no exchange)",
                       "l2": f"inputs+outputs rotate over {nsets} buffer sets (>= 3, >= 3x L2)",
                       "timing": "K calls replayed from CUDA graphs, CUDA events"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "traffic": recorded_traffic(w.name + "_swiglu_q8_1", FWD_SOURCES),
                         "algorithmic_bytes_per_launch": nbytes, "kernel": "sdq::fwd::swiglu_q8_1_kernel"},
            "cpu_baseline": cpu,
            "e2e": {"unavailable": "the forward op has a device entry point only"},
            "gpu_launches": args.steps, "clocks": clocks, "kernel_sources_sha": kernel_sha(FWD_SOURCES),
        }), flush=True)
    del graphs, warm
    import torch.distributed as tdist
    if tdist.is_initialized():
        parallel.barrier(device)
        tdist.destroy_process_group()
    return 0


def run_traffic_probe(args):
    """No timing: N rounds of (read a 512 MB buffer, one call of the op, read
    the buffer again) on one GPU and one buffer set.  The first read leaves
    only clean lines in L2, so the call's own DRAM writes are what ncu counts
    for it; the second read evicts the outputs the call left dirty in L2, so
    its DRAM writes are the call's remaining write-backs.  Capture with
    ncu --cache-control none, kernels matching fuse_kernel|reduce_kernel,
    skipping the first round (its first read also writes back the buffer's
    initial fill)."""
    import torch
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    import swiglu_backward_int8_b200 as sdq  # fails loudly if the CUDA library is missing
    w = pick_workload(args.workload)
    x_np, gy_np = W.make_inputs(w)
    xs, gs = _to_device_bf16(x_np, device), _to_device_bf16(gy_np, device)
    outs = sdq.allocate_outputs(w.M, w.K, device)
    flush = torch.ones(512 << 20, dtype=torch.uint8, device=device)
    torch.cuda.synchronize(device)
    for _ in range(args.traffic_probe):
        flush.amax()
        sdq.silu_dot_fwd_bwd_quant_fuse(xs, gs, *outs)
        flush.amax()
    torch.cuda.synchronize(device)
    st = sdq.sdq_device_status()
    if st != 0:
        raise RuntimeError(f"device status {sdq.status_string(st)}")
    print(json.dumps({"traffic_probe": w.name, "rounds": args.traffic_probe,
                      "algorithmic_bytes_per_launch": w.algorithmic_bytes(),
                      "kernel_sources_sha": kernel_sha()}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.traffic_probe:
        return run_traffic_probe(args)
    if args.op == "swiglu_q8_1":
        return run_fwd(args)
    return run_sdq(args)


if __name__ == "__main__":
    sys.exit(main())
