"""Backward parity: dQ, dK, dV from the CUDA path against the fp64 oracle's
textbook softmax-Jacobian gradients.  Bar: relative Frobenius error <= 5e-2
per tensor (and per (batch, head) where sampled)."""
import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import GRAD_RTOL_FRO, O_ATOL, LSE_ATOL, f64, max_abs, rel_fro, scale_of
from workloads import WORKLOADS, make_dense

pytestmark = pytest.mark.gpu


def run_bwd(x, causal, heads=None):
    B, N, H, d = x["q"].shape
    scale = scale_of(d)
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fwd(g["q"], g["k"], g["v"], causal=causal)
    dq, dk, dv = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=causal)
    fa.check_device_error()
    args = [f64(x[n]) for n in ("q", "k", "v", "do")]
    G = oracle.attn_bwd_ref(*args, scale, causal, heads=heads)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    errs = []
    for got, ref in zip((dq, dk, dv), G):
        got = f64(got)
        assert np.isfinite(got).all()
        a = np.stack([got[b, :, h] for b, h in pairs])
        r = np.stack([ref[b, :, h] for b, h in pairs])
        errs.append(rel_fro(a, r))
    return errs


SMALL = [(2, 333, 3), (1, 1, 1), (1, 2, 1), (1, 127, 2), (1, 128, 1), (1, 129, 1), (1, 256, 2), (2, 515, 2)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H", SMALL)
def test_small_full(B, N, H, d, causal):
    x = make_dense(B, N, H, d, seed=B * 7 + N + H)
    errs = run_bwd(x, causal)
    assert max(errs) <= GRAD_RTOL_FRO, errs


def test_tiny_fwd_bwd_b1_h2_n128_d64():
    w = WORKLOADS["tiny_fwd_bwd_b1_h2_n128_d64"]
    x = make_dense(w.B, w.N, w.H, w.d, seed=0)
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fwd(g["q"], g["k"], g["v"], causal=False)
    O, L = oracle.attn_fwd_ref(f64(x["q"]), f64(x["k"]), f64(x["v"]), scale_of(w.d), False)
    assert max_abs(f64(o), O) <= O_ATOL and max_abs(f64(lse), L) <= LSE_ATOL
    errs = run_bwd(x, False)
    assert max(errs) <= GRAD_RTOL_FRO, errs


def test_range_stress_b4_h16_n4096_d128_sampled():
    w = WORKLOADS["fwd_bwd_causal_b4_h16_n4096_d128_qk2x"]
    x = make_dense(w.B, w.N, w.H, w.d, seed=0, qk_scale_factor=2.0)
    errs = run_bwd(x, True, heads=[(0, 0), (1, 5), (3, 15)])
    assert max(errs) <= GRAD_RTOL_FRO, errs


def test_workspace_too_small_raises():
    x = {k: v.cuda() for k, v in make_dense(1, 64, 1, 64, seed=1).items()}
    o, lse = fa.fwd(x["q"], x["k"], x["v"])
    ws = torch.empty(fa.workspace_size(1, 64, 1, 64) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.bwd(x["q"], x["k"], x["v"], o, lse, x["do"], workspace=ws)
    assert e.value.status == fa.FA_ERR_WORKSPACE


@pytest.mark.parametrize("d", [64, 128])
def test_repeated_runs_all_within_tolerance(d):
    """Twenty backward passes of one problem: an ordering race between the
    warp roles would show up as an occasional wrong result."""
    x = make_dense(2, 600, 2, d, seed=31)
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fwd(g["q"], g["k"], g["v"], causal=True)
    G = oracle.attn_bwd_ref(*(f64(x[n]) for n in ("q", "k", "v", "do")), scale_of(d), True)
    for _ in range(20):
        dq, dk, dv = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=True)
        fa.check_device_error()
        errs = [rel_fro(f64(t), r) for t, r in zip((dq, dk, dv), G)]
        assert max(errs) <= GRAD_RTOL_FRO, errs
