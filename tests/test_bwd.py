"""Backward parity: dQ, dK, dV from the CUDA path against the fp64 oracle's
textbook softmax-Jacobian gradients.  Bar: relative Frobenius error <= 5e-2
per tensor (and per (batch, head) where sampled)."""
import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import GRAD_RTOL_FRO, O_ATOL, LSE_ATOL, Agg, f64, max_abs, nan_like, oracle_per_head, rel_fro, scale_of
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


def fwd_bwd_all_heads(x, causal, heads=None):
    """Forward and backward at full size with NaN-prefilled outputs (every
    element must be written) and the oracle on every listed (b, h) head
    (default: all of them).  Returns the aggregated errors."""
    B, N, H, d = x["q"].shape
    scale = scale_of(d)
    g = {k: v.cuda() for k, v in x.items()}
    o = nan_like(g["q"])
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    fa.fwd(g["q"], g["k"], g["v"], causal=causal, out=o, lse=lse)
    dq, dk, dv = nan_like(g["q"]), nan_like(g["k"]), nan_like(g["v"])
    fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=causal, dq=dq, dk=dk, dv=dv)
    fa.check_device_error()
    for t in (o, lse, dq, dk, dv):
        assert torch.isfinite(t).all()
    o, lse, dq, dk, dv = (f64(t) for t in (o, lse, dq, dk, dv))
    del g
    a = {n: f64(x[n]) for n in ("q", "k", "v", "do")}
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    items = [((b, h),) + tuple(a[n][b, :, h] for n in ("q", "k", "v", "do")) for b, h in pairs]
    ref = oracle_per_head(items, scale, causal, grads=True)
    agg = Agg()
    for (b, h), (O, L, gq, gk, gv) in ref.items():
        agg.fwd(o[b, :, h], O, lse[b, h], L)
        agg.bwd((dq[b, :, h], dk[b, :, h], dv[b, :, h]), (gq, gk, gv))
    return agg


def test_range_stress_b4_h16_n4096_d128_all_heads():
    """The forward+backward workload (Q, K doubled), all 64 heads: O, LSE and
    dQ, dK, dV against the oracle on every head (the heads run in several
    scheduling groups at this size)."""
    w = WORKLOADS["fwd_bwd_causal_b4_h16_n4096_d128_qk2x"]
    x = make_dense(w.B, w.N, w.H, w.d, seed=0, qk_scale_factor=2.0)
    agg = fwd_bwd_all_heads(x, True)
    assert agg.eo <= O_ATOL and agg.el <= LSE_ATOL, (agg.eo, agg.el)
    assert max(agg.grads()) <= GRAD_RTOL_FRO, agg.grads()
    assert max(agg.worst_head) <= GRAD_RTOL_FRO, agg.worst_head


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


def test_launch_events_time_the_three_backward_kernels():
    """The measurement hook: the library records the caller's events around
    its three launches; the stage times are positive and add up to the call."""
    x = make_dense(2, 1024, 4, 128, seed=41)
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fwd(g["q"], g["k"], g["v"], causal=True)
    s = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:
        e.record(s)
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    outer[0].record(s)
    fa.record_launch_events(ev)
    fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=True)
    outer[1].record(s)
    torch.cuda.synchronize()
    fa.check_device_error()
    stages = [ev[j].elapsed_time(ev[j + 1]) for j in range(3)]
    assert all(t > 0 for t in stages), stages
    assert sum(stages) <= outer[0].elapsed_time(outer[1]) + 1e-3
    assert stages[1] > stages[0] and stages[1] > stages[2]  # the fused kernel dominates
    # the hook is cleared after one call: the next call records nothing more
    before = ev[3].elapsed_time(ev[0])
    fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=True)
    torch.cuda.synchronize()
    assert ev[3].elapsed_time(ev[0]) == before
