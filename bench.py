#!/usr/bin/env python3
"""Throughput of the exact-attention hot path on B200: one step = forward +
backward of the fused kernels over one batch of synthetic input.

Workload (default): B=4, H=16, N=4096, d=128, causal, bf16 Q/K/V/dO i.i.d.
N(0,1) with Q and K doubled (softmax range stress) -- the forward+backward
workload at N >= 4096, d = 128 on which the performance target is stated.
Metric: attention TFLOP/s of forward + backward, with the algorithmic FLOP
count 4 B H N^2 d for the forward (halved for causal) and 2.5x that for the
backward.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronize, timed with CUDA events on the launching stream; multi-GPU
runs report the max over ranks.  The inputs (256 MiB of bf16) are larger than
the 126 MB L2, so no flush is needed between steps.  SM clocks and throttle
reasons are sampled with nvidia-smi during the timed region.

Lines printed: one JSON object (rank 0).  `--impl reference` times the fp64
CPU oracle instead (the slow baseline), on a bounded sample of the same
workload.  `--sweep` instead times every call of every workload the path is
specified on (one GPU): 10 warm-up calls, then >= 30 calls each bracketed by
CUDA events, reported as min / median / p90 with one JSON line per
(workload, mode, direction).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import (DECODE_WORKLOADS, WORKLOADS, make_decode, make_dense, make_fp8_dense,  # noqa: E402
                       make_workload)

WORKLOAD = "fwd_bwd_causal_b4_h16_n4096_d128_qk2x"
METRIC = "attention TFLOP/s fwd+bwd (bf16), fraction of B200 dense BF16 peak"
UNIT = "TFLOP/s"


def fwd_flops(B, N, H, d, causal):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"bf16_tflops": float(p["bf16_tflops"]), "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]),
                "hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def kernel_source_sha() -> str:
    """Hash of every file the library is compiled from (the build's own list)."""
    from exact_io_aware_95_b200 import build as fabuild
    h = hashlib.sha256()
    for f in fabuild.deps():
        with open(f, "rb") as fh:
            h.update(os.path.relpath(f, ROOT).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.md")
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha()
    for line in open(path):
        m = re.match(r"\|\s*(\S+)\s*\|\s*(\S+)\s*\|\s*([0-9.eE+]+)\s*\|", line)
        if m and m.group(1) == kernel and m.group(2) == sha:
            return float(m.group(3))
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.tmp = None
        self.dev = device_index

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.tmp, stderr=subprocess.DEVNULL)
            time.sleep(0.5)  # let the sampler start producing before the timed region
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.tmp.name)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        busy = [x for x in sm if x > 500] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None,
                "power_w_max": max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit()),
                "samples": len(rows), "reasons": sorted(reasons)}


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def host_info() -> dict:
    """The host the oracle runs on: logical CPUs, the BLAS library's thread
    count (its matrix products use them all) and the CPU model."""
    info = {"logical_cpus": os.cpu_count()}
    try:
        from threadpoolctl import threadpool_info
        blas = [p for p in threadpool_info() if p.get("user_api") == "blas"]
        info["blas_threads"] = max(p["num_threads"] for p in blas) if blas else None
        info["blas"] = blas[0].get("internal_api") if blas else None
    except Exception:
        info["blas_threads"] = None
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    info["cpu_model"] = model
    return info


_SAMPLE_CACHE = {}


def oracle_sample(w, n_heads: int, seed: int = 0):
    """Time the fp64 oracle (as it stands) on `n_heads` (b, h) heads of the
    workload, forward + backward.  Returns (TFLOP/s, seconds, description)."""
    import numpy as np
    import oracle  # test infrastructure: only this baseline leg calls it

    # n_heads (b, h) pairs spread evenly over the B * H heads of the workload
    nbh = w.B * w.H
    heads = [divmod((i * nbh) // n_heads, w.H) for i in range(n_heads)]
    key = (w.name, n_heads, seed)
    if key not in _SAMPLE_CACHE:
        x = make_dense(w.B, w.N, w.H, w.d, seed=seed, qk_scale_factor=w.qk_scale_factor)
        # the sampled heads only, as [1, N, n, d] float64 arrays
        _SAMPLE_CACHE[key] = {k: np.stack([v[b, :, h].float().numpy() for b, h in heads], axis=1)[None]
                              .astype(np.float64) for k, v in x.items()}
    a = _SAMPLE_CACHE[key]
    causal = True in w.causal
    scale = 1.0 / math.sqrt(w.d)
    t0 = time.perf_counter()
    oracle.attn_fwd_ref(a["q"], a["k"], a["v"], scale, causal)
    oracle.attn_bwd_ref(a["q"], a["k"], a["v"], a["do"], scale, causal)
    dt = time.perf_counter() - t0
    flops = 3.5 * fwd_flops(1, w.N, 1, w.d, causal) * len(heads)
    return flops / dt / 1e12, dt, f"oracle fwd+bwd on {len(heads)} of {w.B * w.H} (b,h) heads, N={w.N}, d={w.d}"


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate_tflops(flops_per_rank_step: float, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: the work all ranks did per step over the slowest
    rank's step time (weak scaling: every rank runs its own shard of equal size)."""
    return flops_per_rank_step * world / (ms_per_step_max * 1e-3) / 1e12


def allmax(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle timed on the host cores."""
    if rank != 0:
        return None
    w = WORKLOADS[WORKLOAD]
    vals = []
    for i in range(args.warmup + args.steps):
        v, dt, desc = oracle_sample(w, 1)
        if i >= args.warmup:
            vals.append((v, dt))
    value = statistics.mean(v for v, _ in vals)
    ms = statistics.mean(dt for _, dt in vals) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": w.B, "N": w.N, "H": w.H, "d": w.d, "causal": True},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "sample": desc + " per step", **host_info()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


def run_gpu(args, world, rank, local):
    import exact_io_aware_95_b200 as fa

    w = WORKLOADS[WORKLOAD]
    B, N, H, d = w.B, w.N, w.H, w.d
    causal = True
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda", local)
    host = make_dense(B, N, H, d, seed=args.seed + rank, qk_scale_factor=w.qk_scale_factor)
    g = {k: v.to(dev) for k, v in host.items()}
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])
    ws = torch.empty(fa.workspace_size(B, N, H, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.fwd(g["q"], g["k"], g["v"], causal=causal, scale=scale, out=o, lse=lse)
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=causal, scale=scale, workspace=ws, dq=dq, dk=dk, dv=dv)

    for _ in range(args.warmup):
        step()
    fa.check_device_error()
    torch.cuda.synchronize(dev)

    # ---- timed region: whole steps, plus per-kernel events for the roofline.
    # ev[i][0..1] bracket the forward kernel; the library itself records
    # kev[i][0..3] on the same stream around the three launches of fa_bwd
    # (preprocess, fused main kernel, dQ conversion).
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e in (x for row in ev + kev for x in row):
        e.record(stream)  # torch creates events lazily; the library needs live handles
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        fa.fwd(g["q"], g["k"], g["v"], causal=causal, scale=scale, out=o, lse=lse)
        ev[i][1].record(stream)
        fa.record_launch_events(kev[i])
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=causal, scale=scale, workspace=ws, dq=dq, dk=dk, dv=dv)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    fa.check_device_error()
    total_ms = allmax(t_start.elapsed_time(t_end), world)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    bwd_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in kev)
    bwd_stage_ms = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in kev) for j in range(3)]
    bwd_main_ms = bwd_stage_ms[1]
    ms_step = total_ms / args.steps

    ff = fwd_flops(B, N, H, d, causal)
    bf = 2.5 * ff
    value = aggregate_tflops(ff + bf, world, ms_step)
    fwd_tflops = ff / (fwd_ms * 1e-3) / 1e12
    bwd_tflops = bf / (bwd_ms * 1e-3) / 1e12
    bwd_main_tflops = bf / (bwd_main_ms * 1e-3) / 1e12
    peaks = load_peaks()

    # ---- end to end through the public API with pinned host buffers.  Every
    # step copies its inputs host -> device and its results device -> host
    # inside the timed region; three streams overlap the copies of one step
    # with the compute of its neighbours (the host link is full duplex), with
    # two device buffer sets so a step's copies never touch buffers in use.
    pin = {k: v.pin_memory() for k, v in host.items()}
    outs = (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))
    out_h = [{n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in outs} for _ in range(2)]
    dev_in = [{k: torch.empty_like(v) for k, v in g.items()} for _ in range(2)]
    dev_out = [{n: torch.empty_like(t) for n, t in outs} for _ in range(2)]
    ws2 = [ws, ws]  # the compute stream runs one step at a time
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in out_h[0].values())
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_ready, cmp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in cmp_done + out_done:
        e.record(stream)

    def e2e_step(i):
        k = i & 1
        with torch.cuda.stream(s_in):
            s_in.wait_event(cmp_done[k])          # step i-2 finished reading these inputs
            for n, t in pin.items():
                dev_in[k][n].copy_(t, non_blocking=True)
            in_ready[k].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_ready[k])
            s_cmp.wait_event(out_done[k])         # step i-2's results have left these buffers
            x, y = dev_in[k], dev_out[k]
            fa.fwd(x["q"], x["k"], x["v"], causal=causal, scale=scale, out=y["o"], lse=y["lse"])
            fa.bwd(x["q"], x["k"], x["v"], y["o"], y["lse"], x["do"], causal=causal, scale=scale, workspace=ws2[k],
                   dq=y["dq"], dk=y["dk"], dv=y["dv"])
            cmp_done[k].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[k])
            for n, _ in outs:
                out_h[k][n].copy_(dev_out[k][n], non_blocking=True)
            out_done[k].record(s_out)

    for i in range(max(2, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e_steps = max(2, min(args.steps, 20))
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    s0.record(s_in)
    for i in range(e_steps):
        e2e_step(i)
    s_in.wait_stream(s_out)
    s1.record(s_in)
    torch.cuda.synchronize(dev)
    barrier(world)
    fa.check_device_error()
    e2e_ms = allmax(s0.elapsed_time(s1), world) / e_steps
    e2e_value = aggregate_tflops(ff + bf, world, e2e_ms)

    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "N": N, "H": H, "d": d, "causal": causal,
                   "qk_scale_factor": w.qk_scale_factor, "per_gpu_batch": B, "global_batch": B * world,
                   "parallelism": f"replicas x{world} (independent (batch, head) shards)",
                   "l2": "inputs (256 MiB bf16) larger than the 126 MB L2; no flush"},
        "fwd_tflops": fwd_tflops, "bwd_tflops": bwd_tflops, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
        "frac_of_peak": {"step_vs_burst": value / world / peaks["bf16_tflops"],
                         "fwd_vs_burst": fwd_tflops / peaks["bf16_tflops"],
                         "bwd_vs_burst": bwd_tflops / peaks["bf16_tflops"],
                         "peak_source": peaks["source"]},
        "bwd_kernel_ms": {"fa_bwd_preprocess_kernel": bwd_stage_ms[0], "fa_bwd_kernel": bwd_stage_ms[1],
                          "fa_bwd_dq_convert_kernel": bwd_stage_ms[2]},
        "roofline": {"kernel": "fa_bwd_kernel", "bound": "tensor",
                     "achieved": bwd_main_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": bwd_main_tflops / peaks["bf16_tflops"],
                     "peak_kind": f"burst bf16 GEMM ({peaks['source']})",
                     "how": "687.2 GFLOP (2.5 x the causal forward) per launch / mean CUDA-event duration of the "
                            "fa_bwd_kernel launch alone, events recorded by the library on the launch stream",
                     "frac_of_sustained": bwd_main_tflops / peaks["bf16_tflops_sustained"],
                     "traffic": recorded_traffic("fa_bwd_kernel")},
        "roofline_bwd_call": {"kernels": "fa_bwd call: preprocess + fa_bwd_kernel + dq_convert", "bound": "tensor",
                              "achieved": bwd_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": bwd_tflops / peaks["bf16_tflops"]},
        "roofline_fwd": {"kernel": "fa_fwd_kernel", "bound": "tensor", "achieved": fwd_tflops,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": fwd_tflops / peaks["bf16_tflops"],
                         "frac_of_sustained": fwd_tflops / peaks["bf16_tflops_sustained"],
                         "traffic": recorded_traffic("fa_fwd_kernel")},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "steps": e_steps,
                "how": "pinned host inputs copied in and all outputs copied out every step; copies of neighbouring steps overlap compute on separate streams"},
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        v, dt, desc = oracle_sample(w, 16)  # about 10 s of fp64 work on the host
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle", "sample": desc,
                                "seconds": dt, **host_info()}
    return line


DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense bf16, vendor datasheet (context only)


def _pct(xs, q):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, int(math.ceil(q * len(xs))) - 1)]


def run_sweep(args):
    """Per-call timing of each workload, mode and direction on one GPU."""
    import exact_io_aware_95_b200 as fa

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    iters = max(30, args.calls)
    # a buffer larger than L2, written between calls for the flushed variant
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    names = [args.only] if args.only else list(WORKLOADS) + list(DECODE_WORKLOADS)
    for name in names:
        if name in DECODE_WORKLOADS:
            _sweep_decode(fa, DECODE_WORKLOADS[name], args, dev, stream, peaks, iters)
            continue
        w = WORKLOADS[name]
        x = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in make_workload(w, seed=args.seed).items()}
        scale = 1.0 / math.sqrt(w.d)
        flush_variants = (False, True) if w.N and w.N <= 128 else (False,)
        for causal in w.causal:
            if w.varlen_total:
                lens = x["lengths"]
                ff = sum(4.0 * w.H * L * L * w.d for L in lens) / (2 if causal else 1)
                mx = max(lens)

                def f():
                    return fa.varlen_fwd(x["q"], x["k"], x["v"], x["cu_seqlens"], mx, causal=causal, scale=scale,
                                         out=o, lse=lse)

                def b(det=False):
                    fa.varlen_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], x["cu_seqlens"], mx, causal=causal,
                                  scale=scale, workspace=ws, dq=dq, dk=dk, dv=dv, deterministic=det)
                o = torch.empty_like(x["q"])
                lse = torch.empty((w.H, w.varlen_total), dtype=torch.float32, device=dev)
                ws = torch.empty(fa.workspace_size(1, w.varlen_total, w.H, w.d), dtype=torch.uint8, device=dev)
                shape = {"total": w.varlen_total, "nseq": len(lens), "H": w.H, "d": w.d, "lengths": lens}
            else:
                ff = fwd_flops(w.B, w.N, w.H, w.d, causal)

                def f():
                    return fa.fwd(x["q"], x["k"], x["v"], causal=causal, scale=scale, out=o, lse=lse)

                def b(det=False):
                    fa.bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal, scale=scale, workspace=ws,
                           dq=dq, dk=dk, dv=dv, deterministic=det)
                o = torch.empty_like(x["q"])
                lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
                ws = torch.empty(fa.workspace_size(w.B, w.N, w.H, w.d), dtype=torch.uint8, device=dev)
                shape = {"B": w.B, "N": w.N, "H": w.H, "d": w.d}
            dq, dk, dv = (torch.empty_like(x["q"]) for _ in range(3))
            f()
            # the deterministic backward is credited with the same algorithmic
            # FLOPs (2.5x forward); its recomputation of S and dP is not counted
            dirs = [("fwd", f, ff)] + ([("bwd", b, 2.5 * ff), ("bwd_deterministic", lambda: b(True), 2.5 * ff)]
                                       if w.backward else [])
            if not w.varlen_total and w.d == 128:
                # the 8-bit forward on the same draws, quantized per tensor
                x8, sc = make_fp8_dense(w.B, w.N, w.H, w.d, seed=args.seed, qk_scale_factor=w.qk_scale_factor)
                x8 = {n: t.to(dev) for n, t in x8.items()}
                ws8 = torch.empty(fa.fwd_fp8_workspace_size(w.B, w.N, w.H, w.d), dtype=torch.uint8, device=dev)

                def f8():
                    fa.fwd_fp8(x8["q"], x8["k"], x8["v"], sc["q"], sc["k"], sc["v"], causal=causal, scale=scale,
                               out=o, lse=lse, workspace=ws8)
                dirs.append(("fwd_fp8", f8, ff))
            for direction, fn, flops in dirs:
                for flush in flush_variants:
                    for _ in range(10):
                        fn()
                    fa.check_device_error()
                    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                           for _ in range(iters)]
                    clocks = ClockSampler(0)
                    torch.cuda.synchronize(dev)
                    clocks.start()
                    for e0, e1 in evs:
                        if flush:
                            flush_buf.fill_(1)
                        e0.record(stream)
                        fn()
                        e1.record(stream)
                    torch.cuda.synchronize(dev)
                    clk = clocks.stop()
                    fa.check_device_error()
                    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
                    med = statistics.median(ms)
                    tf = flops / (med * 1e-3) / 1e12
                    print(json.dumps({
                        "sweep": name, "causal": causal, "direction": direction, "calls": iters, "warmup": 10,
                        "l2": "flushed before each call" if flush else "not flushed",
                        "shape": shape, "gflop": flops / 1e9,
                        "ms": {"min": min(ms), "median": med, "p90": _pct(ms, 0.9)},
                        "tflops_at_median": tf,
                        "frac": {"measured_burst": tf / peaks["bf16_tflops"],
                                 "measured_sustained": tf / peaks["bf16_tflops_sustained"],
                                 "datasheet_2250": tf / DATASHEET_BF16_TFLOPS, "peak_source": peaks["source"]},
                        "clocks": clk}), flush=True)
        del x


def run_oracle_timings(args):
    """The fp64 oracle timed on the host cores, per workload, mode and
    direction: full runs where they take seconds to a minute (the tiny, d = 64
    and Q,K-doubled workloads), else heads {0, H/2, H-1} timed and the time
    scaled by H/3, labelled as such.  One JSON line each, with the host's
    cores, BLAS threads and CPU model."""
    import numpy as np
    import oracle  # test infrastructure: only the baseline legs call it

    info = host_info()
    for name, w in WORKLOADS.items():
        full = (w.varlen_total == 0 and w.N <= 4096)
        heads = list(range(w.H)) if full else sorted({0, w.H // 2, w.H - 1})
        x = make_workload(w, seed=args.seed)
        a = {k: x[k].float().numpy().astype(np.float64) for k in ("q", "k", "v", "do") if k in x}
        scale = 1.0 / math.sqrt(w.d)
        for causal in w.causal:
            if w.varlen_total:
                lens = x["lengths"]
                cu = x["cu_seqlens"].numpy()
                ff = sum(4.0 * w.H * L * L * w.d for L in lens) / (2 if causal else 1)
                fwd = lambda: oracle.attn_varlen_fwd_ref(a["q"], a["k"], a["v"], cu, scale, causal, heads=heads)
                bwd = lambda: oracle.attn_varlen_bwd_ref(a["q"], a["k"], a["v"], a["do"], cu, scale, causal,
                                                         heads=heads)
                nh = w.H
            else:
                ff = fwd_flops(w.B, w.N, w.H, w.d, causal)
                pairs = [(b, h) for b in range(w.B) for h in heads]
                fwd = lambda: oracle.attn_fwd_ref(a["q"], a["k"], a["v"], scale, causal, heads=pairs)
                bwd = lambda: oracle.attn_bwd_ref(a["q"], a["k"], a["v"], a["do"], scale, causal, heads=pairs)
                nh = w.H
            dirs = [("fwd", fwd, ff)] + ([("bwd", bwd, 2.5 * ff)] if w.backward else [])
            for direction, fn, flops in dirs:
                t0 = time.perf_counter()
                fn()
                dt = time.perf_counter() - t0
                scaled = dt * nh / len(heads)
                print(json.dumps({
                    "oracle_timing": name, "causal": causal, "direction": direction,
                    "heads_timed": len(heads), "heads_total": nh,
                    "measured_s": dt, "whole_workload_s": scaled,
                    "kind": "full run" if len(heads) == nh else f"measured on {len(heads)} heads, x{nh}/{len(heads)} extrapolated",
                    "tflops": flops / scaled / 1e12, "gflop": flops / 1e9, "cores": cpu_cores(), **info}), flush=True)


def _sweep_decode(fa, w, args, dev, stream, peaks, iters):
    """Decode lines: HBM-bound, reported as GB/s of the bytes the call must
    move (the valid K and V cache rows, q, o and lse) against the measured
    copy bandwidth."""
    x = {k: v.to(dev) for k, v in make_decode(w.B, w.Nq, w.Nk, w.H, w.d, w.lo, w.hi, seed=args.seed).items()}
    lens = x["seqlens"].tolist()
    o = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    nws = fa.decode_workspace_size(w.B, w.Nq, w.Nk, w.H, w.d)
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=dev)
    nbytes = sum(lens) * w.H * w.d * 2 * 2 + 2 * w.B * w.Nq * w.H * w.d * 2 + w.B * w.H * w.Nq * 4

    def fn():
        fa.decode_fwd(x["q"], x["k"], x["v"], x["seqlens"], causal=True, out=o, lse=lse, workspace=ws)
    for _ in range(10):
        fn()
    fa.check_device_error()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    clocks = ClockSampler(0)
    torch.cuda.synchronize(dev)
    clocks.start()
    for e0, e1 in evs:
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    fa.check_device_error()
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    med = statistics.median(ms)
    gbs = nbytes / (med * 1e-3) / 1e9
    print(json.dumps({
        "sweep": w.name, "causal": True, "direction": "decode_fwd", "calls": iters, "warmup": 10,
        "l2": f"cache ({nbytes / 2**30:.2f} GiB) larger than the 126 MB L2; not flushed",
        "shape": {"B": w.B, "Nq": w.Nq, "Nk": w.Nk, "H": w.H, "d": w.d, "seqlens_sum": sum(lens)},
        "bytes": nbytes, "ms": {"min": min(ms), "median": med, "p90": _pct(ms, 0.9)},
        "gbs_at_median": gbs, "frac": {"measured_hbm": gbs / peaks["hbm_gbs"], "peak_source": peaks["source"]},
        "clocks": clk}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="per-call timing of every workload (one GPU)")
    ap.add_argument("--only", default=None, help="with --sweep: one workload by name")
    ap.add_argument("--calls", type=int, default=30, help="with --sweep: timed calls per line (>= 30)")
    ap.add_argument("--oracle-timings", action="store_true",
                    help="time the fp64 oracle on the host cores for every workload (no GPU)")
    args = ap.parse_args()
    if args.oracle_timings:
        run_oracle_timings(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        line = run_reference(args, world, rank) if args.impl == "reference" else run_gpu(args, world, rank, local)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
