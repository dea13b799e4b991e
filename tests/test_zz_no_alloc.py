"""fa_bwd_noalloc: the backward pass for callers that cannot allocate.

Some callers may not allocate device memory at the point where they run the
backward pass -- code running inside an allocator or memory-pool callback, or
a runtime working within a fixed, pre-planned memory budget.  fa_bwd_noalloc
serves them: it takes the same inputs and outputs as fa_bwd but no workspace,
and uses a static scratch array carried in the library's device image.

Checked here, through the C ABI, on two calls in a row with a different
problem in between: dK and dV are bitwise equal to those of fa_bwd (which
takes a caller-allocated workspace; the same kernels compute them in a fixed
order), dQ agrees with fa_bwd's to 1e-2 relative Frobenius error (its fp32
atomic sums may be added in another order), and the gradients match the
fp64 oracle directly.  Repeated calls leave the device's free memory
unchanged, and a problem needing more scratch than the array holds is
refused before anything runs.  Named so that pytest collects it last.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import GRAD_RTOL_FRO, f64, rel_fro
from workloads import make_dense

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 64 << 20  # FA_STATIC_SCRATCH_BYTES in include/fa.h
DQ_RTOL_VS_WORKSPACE_CALL = 1e-2


def noalloc_into(x, o, lse, causal, out):
    B, N, H, d = x["q"].shape
    st = fa.lib().fa_bwd_noalloc(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), x["do"].data_ptr(), out[0].data_ptr(), out[1].data_ptr(),
                                 out[2].data_ptr(), B, N, H, d, 1.0 / math.sqrt(d), int(causal),
                                 torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.status_string(st)
    fa.check_device_error()
    return out


def noalloc(x, o, lse, causal):
    return noalloc_into(x, o, lse, causal, [torch.full_like(x["q"], float("nan")) for _ in range(3)])


def problem(B, N, H, d, causal, seed):
    x = {k: v.cuda() for k, v in make_dense(B, N, H, d, seed=seed).items()}
    o, lse = fa.fwd(x["q"], x["k"], x["v"], causal=causal)
    ref = fa.bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal)  # caller-allocated workspace
    fa.check_device_error()
    return x, o, lse, ref


def agrees_with_workspace_call(got, ref):
    dq, dk, dv = got
    assert all(torch.isfinite(t).all() for t in got)
    assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    assert rel_fro(f64(dq), f64(ref[0])) <= DQ_RTOL_VS_WORKSPACE_CALL


@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_matches_workspace_entry_point_twice(causal):
    x, o, lse, ref = problem(2, 333, 3, 128, causal, seed=21)
    first = noalloc(x, o, lse, causal)
    # a different problem in between leaves other contents in the shared array
    y, oy, ly, refy = problem(1, 700, 2, 64, causal, seed=22)
    mid = noalloc(y, oy, ly, causal)
    second = noalloc(x, o, lse, causal)
    agrees_with_workspace_call(first, ref)
    agrees_with_workspace_call(mid, refy)
    agrees_with_workspace_call(second, ref)


def test_noalloc_matches_the_oracle():
    causal = True
    x, o, lse, _ = problem(1, 515, 2, 64, causal, seed=23)
    got = noalloc(x, o, lse, causal)
    G = oracle.attn_bwd_ref(*(f64(x[n]) for n in ("q", "k", "v", "do")), 1 / math.sqrt(64), causal)
    for t, r in zip(got, G):
        assert rel_fro(f64(t), r) <= GRAD_RTOL_FRO


def test_noalloc_allocates_nothing_on_repeated_calls():
    causal = False
    x, o, lse, ref = problem(1, 384, 2, 128, causal, seed=24)
    out = [torch.empty_like(x["q"]) for _ in range(3)]
    noalloc_into(x, o, lse, causal, out)  # the first call may load the module and resolve the array
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    noalloc_into(x, o, lse, causal, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    noalloc_into(x, o, lse, causal, out)
    torch.cuda.synchronize()
    free2, _ = torch.cuda.mem_get_info()
    assert free0 == free1 == free2, (free0, free1, free2)
    agrees_with_workspace_call(out, ref)


def test_noalloc_refuses_problems_larger_than_the_static_scratch():
    B, N, H, d = 8, 4096, 16, 128
    assert fa.workspace_size(B, N, H, d) > STATIC_SCRATCH_BYTES
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    # refused on the host before any pointer is used or anything is launched
    st = fa.lib().fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, N, H, d, 0.1, 1,
                                 torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_ERR_WORKSPACE
