"""A device pipeline wait that runs out is reported, not hung on.

Every mbarrier wait in the kernels is bounded (FA_WAIT_TIMEOUT_NS of global
time); an expired wait sets the device error word, raises the CTA's abort
flag so its other warps leave, and the kernel frees its tensor memory and
returns.  Here a test-only build of the library (the same sources with a
20 ms bound, plus tests/wait_probe/fa_wait_probe.cu) runs a one-CTA kernel
that waits on an mbarrier nothing ever arrives on.  Checked: the kernel
returns; fa_get_device_error() reports FA_ERR_TIMEOUT once and FA_OK on the
next call; the second warp left through the abort flag before its own limit;
and the same library then computes a forward and backward pass in the same
context that match the oracle.  Nothing here faults or hangs the GPU: the
wait is bounded by construction."""
import ctypes
import math
import os

import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from exact_io_aware_95_b200 import build as fabuild
from tests.common import GRAD_RTOL_FRO, LSE_ATOL, O_ATOL, f64, max_abs, rel_fro
from workloads import make_dense

HERE = os.path.dirname(os.path.abspath(__file__))
PROBE_SRC = os.path.join(HERE, "wait_probe", "fa_wait_probe.cu")
PROBE_LIB = os.path.join(os.path.dirname(fabuild.LIB_PATH), "libfa_b200_waitprobe.so")
LIMIT_NS = 20_000_000


def build_probe():
    return fabuild.build(out=PROBE_LIB, defines=[f"FA_WAIT_TIMEOUT_NS={LIMIT_NS}ull"], sources=[PROBE_SRC])


def load_probe():
    L = fa.lib(path=build_probe())  # a separate handle: its own device error word
    L.fa_wait_probe.restype = ctypes.c_int
    L.fa_wait_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    L.fa_wait_probe_limit_ns.restype = ctypes.c_ulonglong
    L.fa_wait_probe_delay_ns.restype = ctypes.c_ulonglong
    return L


def test_probe_library_builds_and_exports():
    """CPU: the test build compiles, carries the short limit and exports the
    library's entry points next to the probe."""
    L = load_probe()
    assert L.fa_wait_probe_limit_ns() == LIMIT_NS
    assert L.fa_wait_probe_delay_ns() < LIMIT_NS
    for name in fa.EXPORTS:
        assert hasattr(L, name), name


@pytest.mark.gpu
def test_expired_wait_is_reported_and_the_context_stays_usable():
    L = load_probe()
    s = torch.cuda.current_stream().cuda_stream
    assert L.fa_get_device_error(s) == fa.FA_OK
    rec = torch.full((5,), -1, dtype=torch.int64, device="cuda")
    assert L.fa_wait_probe(rec.data_ptr(), s) == fa.FA_OK
    assert L.fa_get_device_error(s) == fa.FA_ERR_TIMEOUT  # synchronises: the kernel returned
    assert L.fa_get_device_error(s) == fa.FA_OK           # the word was read and cleared
    ok0, t0, ok1, t1, abort_seen = rec.cpu().tolist()
    delay = L.fa_wait_probe_delay_ns()
    assert ok0 == 0 and t0 >= LIMIT_NS, (ok0, t0)                    # gave up at the limit
    assert ok1 == 0 and abort_seen == 1, (ok1, abort_seen)           # left through the abort flag
    assert t1 < delay + LIMIT_NS, (t1, delay)                        # before its own limit
    # the main library's error word is separate and untouched
    assert fa.lib().fa_get_device_error(s) == fa.FA_OK

    # the same library, in the same context, afterwards: forward + backward
    B, N, H, d = 1, 300, 2, 128
    x = make_dense(B, N, H, d, seed=3)
    g = {k: v.cuda() for k, v in x.items()}
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    scale = 1.0 / math.sqrt(d)
    assert L.fa_fwd(g["q"].data_ptr(), g["k"].data_ptr(), g["v"].data_ptr(), o.data_ptr(), lse.data_ptr(),
                    B, N, H, d, scale, 1, s) == fa.FA_OK
    dq, dk, dv = (torch.empty_like(g["q"]) for _ in range(3))
    ws = torch.empty(fa.workspace_size(B, N, H, d), dtype=torch.uint8, device="cuda")
    assert L.fa_bwd(g["q"].data_ptr(), g["k"].data_ptr(), g["v"].data_ptr(), o.data_ptr(), lse.data_ptr(),
                    g["do"].data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel(),
                    B, N, H, d, scale, 1, s) == fa.FA_OK
    assert L.fa_get_device_error(s) == fa.FA_OK
    a = [f64(x[n]) for n in ("q", "k", "v", "do")]
    O, LS = oracle.attn_fwd_ref(*a[:3], scale, True)
    assert max_abs(f64(o), O) <= O_ATOL and max_abs(f64(lse), LS) <= LSE_ATOL
    G = oracle.attn_bwd_ref(*a, scale, True)
    assert max(rel_fro(f64(t), r) for t, r in zip((dq, dk, dv), G)) <= GRAD_RTOL_FRO
