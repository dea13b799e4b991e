"""fa_bwd_noalloc: the backward pass for callers that cannot allocate.

Some callers may not allocate device memory at the point where they run the
backward pass -- code running inside an allocator or memory-pool callback, or
a runtime working within a fixed, pre-planned memory budget.  fa_bwd_noalloc
serves them: it takes the same inputs and outputs as fa_bwd but no workspace,
and uses a static scratch array carried in the library's device image.

This file checks, through the C ABI, that its gradients agree with those of
fa_bwd (which takes a caller-allocated workspace) within the gradient
tolerance the parity tests use, on two calls in a row with a different
problem in between, and that a problem needing more scratch than the array
holds is refused before anything runs.  It is named so that pytest collects
it last.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
from tests.common import GRAD_RTOL_FRO, f64, rel_fro
from workloads import make_dense

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 64 << 20  # FA_STATIC_SCRATCH_BYTES in include/fa.h


def noalloc(x, o, lse, causal):
    B, N, H, d = x["q"].shape
    out = [torch.full_like(x["q"], float("nan")) for _ in range(3)]
    st = fa.lib().fa_bwd_noalloc(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), x["do"].data_ptr(), out[0].data_ptr(), out[1].data_ptr(),
                                 out[2].data_ptr(), B, N, H, d, 1.0 / math.sqrt(d), int(causal),
                                 torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.status_string(st)
    fa.check_device_error()
    return out


def problem(B, N, H, d, causal, seed):
    x = {k: v.cuda() for k, v in make_dense(B, N, H, d, seed=seed).items()}
    o, lse = fa.fwd(x["q"], x["k"], x["v"], causal=causal)
    ref = fa.bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal)  # caller-allocated workspace
    fa.check_device_error()
    return x, o, lse, ref


@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_matches_workspace_entry_point_twice(causal):
    x, o, lse, ref = problem(2, 333, 3, 128, causal, seed=21)
    first = noalloc(x, o, lse, causal)
    # a different problem in between leaves other contents in the shared array
    y, oy, ly, refy = problem(1, 700, 2, 64, causal, seed=22)
    mid = noalloc(y, oy, ly, causal)
    second = noalloc(x, o, lse, causal)
    for got in (first, second):
        for g, r in zip(got, ref):
            g64, r64 = f64(g), f64(r)
            assert np.isfinite(g64).all()
            assert rel_fro(g64, r64) <= GRAD_RTOL_FRO
    for g, r in zip(mid, refy):
        assert rel_fro(f64(g), f64(r)) <= GRAD_RTOL_FRO


def test_noalloc_refuses_problems_larger_than_the_static_scratch():
    B, N, H, d = 8, 4096, 16, 128
    assert fa.workspace_size(B, N, H, d) > STATIC_SCRATCH_BYTES
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    # refused on the host before any pointer is used or anything is launched
    st = fa.lib().fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, N, H, d, 0.1, 1,
                                 torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_ERR_WORKSPACE
