"""Deterministic backward (fa_bwd_deterministic / fa_varlen_bwd_deterministic).

The pages call the method exact and deterministic ("FlashAttention-2 (PT)",
section "Desempenho e eficiencia").  These entry points give gradients that
are bitwise identical from run to run: dK and dV come from the fused pass
(without its dQ product), dQ from a pass that sums the key tiles of each
query tile in a fixed order.  Checked here: parity with the fp64 oracle
(the same tolerance as the default backward), bitwise reproducibility over
repeated runs, and bitwise equality of dK and dV with the default backward
(the same pass computes them)."""
import math

import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import GRAD_RTOL_FRO, Agg, f64, nan_like, oracle_per_head, rel_fro
from workloads import make_dense, make_varlen

pytestmark = pytest.mark.gpu


def _dense(B, N, H, d, causal, seed, qk=1.0):
    x = make_dense(B, N, H, d, seed=seed, qk_scale_factor=qk)
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fwd(g["q"], g["k"], g["v"], causal=causal)
    return x, g, o, lse


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 128, 300, 513])
def test_dense_matches_oracle_and_is_bitwise_reproducible(N, causal, d):
    x, g, o, lse = _dense(2, N, 2, d, causal, seed=60 + N)
    runs = [fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=causal, deterministic=True) for _ in range(3)]
    ref = oracle.attn_bwd_ref(*(f64(x[n]) for n in ("q", "k", "v", "do")), 1 / math.sqrt(d), causal)
    for t, r in zip(runs[0], ref):
        assert rel_fro(f64(t), r) <= GRAD_RTOL_FRO
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a, b)
    fa.check_device_error()


@pytest.mark.parametrize("causal", [False, True])
def test_dk_dv_equal_the_default_backward_bitwise(causal):
    x, g, o, lse = _dense(2, 700, 3, 128, causal, seed=71, qk=2.0)
    dq_a, dk_a, dv_a = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=causal)
    dq_d, dk_d, dv_d = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=causal, deterministic=True)
    assert torch.equal(dk_a, dk_d) and torch.equal(dv_a, dv_d)
    assert rel_fro(f64(dq_d), f64(dq_a)) <= 1e-2


def test_varlen_matches_oracle_and_is_bitwise_reproducible():
    x = make_varlen([70, 1, 200, 129, 384], 2, 128, seed=72)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    mx = max(x["lengths"])
    o, lse = fa.varlen_fwd(g["q"], g["k"], g["v"], g["cu_seqlens"], mx, causal=True)
    runs = [fa.varlen_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], g["cu_seqlens"], mx, causal=True,
                          deterministic=True) for _ in range(3)]
    ref = oracle.attn_varlen_bwd_ref(*(f64(x[n]) for n in ("q", "k", "v", "do")), x["cu_seqlens"].numpy(),
                                     1 / math.sqrt(128), True)
    for t, r in zip(runs[0], ref):
        assert rel_fro(f64(t), r) <= GRAD_RTOL_FRO
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a, b)


def test_bench_shape_every_head_and_reproducible():
    """B4 H16 N4096 d128 causal, Q,K x2: two full runs bitwise equal, the
    outputs NaN-prefilled, and every (b, h) head against the oracle."""
    B, N, H, d = 4, 4096, 16, 128
    x, g, o, lse = _dense(B, N, H, d, True, seed=0, qk=2.0)
    bufs = [nan_like(g["q"]) for _ in range(3)]
    r1 = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=True, deterministic=True,
                dq=bufs[0], dk=bufs[1], dv=bufs[2])
    r2 = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=True, deterministic=True)
    fa.check_device_error()
    for a, b in zip(r1, r2):
        assert torch.isfinite(a).all()
        assert torch.equal(a, b)
    got = [f64(t) for t in r1]
    a = {n: f64(x[n]) for n in ("q", "k", "v", "do")}
    items = [((b_, h_),) + tuple(a[n][b_, :, h_] for n in ("q", "k", "v", "do")) for b_ in range(B) for h_ in range(H)]
    agg = Agg()
    for (b_, h_), (_, _, gq, gk, gv) in oracle_per_head(items, 1 / math.sqrt(d), True, grads=True).items():
        agg.bwd(tuple(t[b_, :, h_] for t in got), (gq, gk, gv))
    assert max(agg.grads()) <= GRAD_RTOL_FRO, agg.grads()
    assert max(agg.worst_head) <= GRAD_RTOL_FRO, agg.worst_head


def test_autograd_deterministic_flag():
    x = make_dense(1, 257, 2, 64, seed=73)
    grads = []
    for _ in range(2):
        q, k, v = (x[n].cuda().requires_grad_(True) for n in ("q", "k", "v"))
        fa.attention(q, k, v, causal=True, deterministic=True).backward(x["do"].cuda())
        grads.append((q.grad, k.grad, v.grad))
    for a, b in zip(*grads):
        assert torch.equal(a, b)
