"""Multi-rank plumbing of the bench, on CPU with the gloo backend.

The attention path shards into independent (batch entry, head) problems with
no exchange step, so N GPUs run N independent shards (weak scaling) and the
only collectives are a barrier and the max-over-ranks reduction of the step
time.  These tests run that host logic with world size 2 on CPU: the barrier,
the max reduction, the aggregation of throughput, and the bench's reference
arm under torch.distributed.run, where rank 0 alone works and prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    w, r, _ = bench.dist_setup(None)
    assert (w, r) == (world, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    mx = bench.allmax(1.5 + rank, w)   # ranks report 1.5 ms and 2.5 ms
    val = bench.aggregate_tflops(1e12, w, mx)
    q.put((rank, mx, val))
    dist.destroy_process_group()


def test_two_gloo_ranks_barrier_max_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
    assert all(p.exitcode == 0 for p in ps), [p.exitcode for p in ps]
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, mx, val in res:
        assert mx == 2.5                          # the slowest rank's time
        assert abs(val - 2 * 1.0 / 2.5e-3 / 1e0) < 1e-9  # 2 ranks x 1 TFLOP each per 2.5 ms -> 800 TFLOP/s


def test_reference_arm_under_torchrun_rank0_only():
    port = free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
