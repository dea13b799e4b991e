"""Forward parity: the CUDA kernel (through the C ABI) against the fp64 oracle
on the same seeded bf16 inputs.  Bar: O max-abs <= 2e-2, LSE max-abs <= 1e-3."""
import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import LSE_ATOL, O_ATOL, Agg, f64, max_abs, nan_like, oracle_per_head, scale_of
from workloads import WORKLOADS, make_dense

pytestmark = pytest.mark.gpu


def run_and_compare(x, causal, heads=None, scale=None):
    B, N, H, d = x["q"].shape
    scale = scale_of(d) if scale is None else scale
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fwd(g["q"], g["k"], g["v"], causal=causal, scale=scale)
    fa.check_device_error()
    O, L = oracle.attn_fwd_ref(f64(x["q"]), f64(x["k"]), f64(x["v"]), scale, causal, heads=heads)
    o, lse = f64(o), f64(lse)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    eo = max(max_abs(o[b, :, h], O[b, :, h]) for b, h in pairs)
    el = max(max_abs(lse[b, h], L[b, h]) for b, h in pairs)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    return eo, el


SMALL = [(2, 333, 3), (1, 1, 1), (1, 2, 2), (1, 127, 1), (1, 128, 1), (1, 129, 2), (1, 255, 1), (1, 256, 1),
         (1, 257, 1), (2, 700, 2)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H", SMALL)
def test_small_full(B, N, H, d, causal):
    x = make_dense(B, N, H, d, seed=B * 1000 + N + H, with_grad=False)
    eo, el = run_and_compare(x, causal)
    assert eo <= O_ATOL and el <= LSE_ATOL, (eo, el)


@pytest.mark.parametrize("d", [64, 128])
def test_deterministic_bitwise(d):
    x = {k: v.cuda() for k, v in make_dense(2, 1000, 4, d, seed=5, with_grad=False).items()}
    a = fa.fwd(x["q"], x["k"], x["v"], causal=True)
    b = fa.fwd(x["q"], x["k"], x["v"], causal=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def fwd_all_heads(x, causal, scale=None):
    """Forward at full size with NaN-prefilled outputs: every element must be
    written, and every (batch entry, head) is compared with the oracle."""
    B, N, H, d = x["q"].shape
    scale = scale_of(d) if scale is None else scale
    g = {k: v.cuda() for k, v in x.items()}
    o = nan_like(g["q"])
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    fa.fwd(g["q"], g["k"], g["v"], causal=causal, scale=scale, out=o, lse=lse)
    fa.check_device_error()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    o, lse = f64(o), f64(lse)
    a = {n: f64(x[n]) for n in ("q", "k", "v")}
    items = [((b, h), a["q"][b, :, h], a["k"][b, :, h], a["v"][b, :, h], None) for b in range(B) for h in range(H)]
    ref = oracle_per_head(items, scale, causal, grads=False)
    agg = Agg()
    for (b, h), (O, L, *_) in ref.items():
        agg.fwd(o[b, :, h], O, lse[b, h], L)
    return agg


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_b8_h16_n2048_d64_all_heads(causal):
    """The d = 64 forward workload, all 128 heads (several scheduling groups of
    heads at this size, the last one partial)."""
    w = WORKLOADS["fwd_b8_h16_n2048_d64"]
    x = make_dense(w.B, w.N, w.H, w.d, seed=0, with_grad=False)
    agg = fwd_all_heads(x, causal)
    assert agg.eo <= O_ATOL and agg.el <= LSE_ATOL, (agg.eo, agg.el)


@pytest.mark.parametrize("step", [1 / 64, 1 / 16, 1 / 4])
@pytest.mark.parametrize("causal", [False, True])
def test_running_max_moves_every_tile(step, causal):
    """Scores grow with the key index, so the row max rises in every key tile
    (by less than, and by more than, the rescale threshold)."""
    N, d = 900, 64
    q = torch.zeros(1, N, 1, d)
    q[..., 0] = 1.0
    k = torch.zeros(1, N, 1, d)
    k[0, :, 0, 0] = torch.arange(N, dtype=torch.float32) * step
    v = torch.randn(1, N, 1, d, generator=torch.Generator().manual_seed(3))
    x = {"q": q.bfloat16(), "k": k.bfloat16(), "v": v.bfloat16()}
    eo, el = run_and_compare(x, causal, scale=1.0)
    assert eo <= O_ATOL and el <= LSE_ATOL, (eo, el)


def test_all_scores_equal_gives_mean():
    N, d = 300, 128
    x = make_dense(1, N, 2, d, seed=9, with_grad=False)
    x["q"] = torch.zeros_like(x["q"])
    eo, el = run_and_compare(x, False)
    assert eo <= O_ATOL and el <= LSE_ATOL
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fwd(g["q"], g["k"], g["v"])
    mean = f64(x["v"]).mean(axis=1, keepdims=True)
    assert max_abs(f64(o), np.broadcast_to(mean, o.shape)) <= O_ATOL
    assert max_abs(f64(lse), np.full(lse.shape, np.log(N))) <= LSE_ATOL


def test_outputs_fully_written_and_nothing_else():
    """Pre-poisoned outputs inside guard regions: every element written, no canary touched."""
    B, N, H, d = 2, 333, 3, 128
    x = {k: v.cuda() for k, v in make_dense(B, N, H, d, seed=11, with_grad=False).items()}
    n_o, n_l, pad = B * N * H * d, B * H * N, 4096
    obuf = torch.full((n_o + 2 * pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((n_l + 2 * pad,), float("nan"), dtype=torch.float32, device="cuda")
    obuf[:pad] = 7.0
    obuf[-pad:] = 7.0
    lbuf[:pad] = 7.0
    lbuf[-pad:] = 7.0
    o = obuf[pad:pad + n_o].view(B, N, H, d)
    l = lbuf[pad:pad + n_l].view(B, H, N)
    fa.fwd(x["q"], x["k"], x["v"], causal=True, out=o, lse=l)
    fa.check_device_error()
    assert torch.isfinite(o).all() and torch.isfinite(l).all()
    assert (obuf[:pad] == 7).all() and (obuf[-pad:] == 7).all()
    assert (lbuf[:pad] == 7).all() and (lbuf[-pad:] == 7).all()


def test_bad_arguments_raise():
    x = {k: v.cuda() for k, v in make_dense(1, 64, 1, 64, seed=1, with_grad=False).items()}
    with pytest.raises(TypeError):
        fa.fwd(x["q"].float(), x["k"], x["v"])
    q96 = torch.zeros(1, 64, 1, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fwd(q96, q96, q96)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
