"""Packed variable-length batches: every sequence attends only to itself.
Parity against the oracle run sequence by sequence, plus the bitwise check
that a sequence gives the same forward output packed or alone."""
import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import GRAD_RTOL_FRO, LSE_ATOL, O_ATOL, Agg, f64, max_abs, nan_like, oracle_per_head, rel_fro, scale_of
from workloads import WORKLOADS, make_varlen, varlen_lengths

pytestmark = pytest.mark.gpu

LENS = [1, 64, 65, 300, 128, 129, 7, 513]


def run(x, H, d, causal, seqs=None):
    scale = scale_of(d)
    cu = x["cu_seqlens"].cuda()
    g = {k: x[k].cuda() for k in ("q", "k", "v", "do")}
    mx = max(x["lengths"])
    o, lse = fa.varlen_fwd(g["q"], g["k"], g["v"], cu, mx, causal=causal)
    dq, dk, dv = fa.varlen_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], cu, mx, causal=causal)
    fa.check_device_error()
    a = [f64(x[n]) for n in ("q", "k", "v", "do")]
    O, L = oracle.attn_varlen_fwd_ref(*a[:3], x["cu_seqlens"].numpy(), scale, causal, seqs=seqs)
    G = oracle.attn_varlen_bwd_ref(*a, x["cu_seqlens"].numpy(), scale, causal, seqs=seqs)
    cu_h = x["cu_seqlens"].tolist()
    idx = np.concatenate([np.arange(cu_h[s], cu_h[s + 1]) for s in (seqs or range(len(cu_h) - 1))])
    o, lse = f64(o), f64(lse)
    eo = max_abs(o[idx], O[idx])
    el = max_abs(lse[:, idx], L[:, idx])
    eg = [rel_fro(f64(t)[idx], r[idx]) for t, r in zip((dq, dk, dv), G)]
    return eo, el, eg


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_small_packed(d, causal):
    x = make_varlen(LENS, 3, d, seed=4)
    eo, el, eg = run(x, 3, d, causal)
    assert eo <= O_ATOL and el <= LSE_ATOL and max(eg) <= GRAD_RTOL_FRO, (eo, el, eg)


@pytest.mark.parametrize("d", [64, 128])
def test_single_sequence(d):
    x = make_varlen([777], 2, d, seed=6)
    eo, el, eg = run(x, 2, d, True)
    assert eo <= O_ATOL and el <= LSE_ATOL and max(eg) <= GRAD_RTOL_FRO, (eo, el, eg)


@pytest.mark.parametrize("causal", [False, True])
def test_packed_equals_alone_bitwise(causal):
    d, H = 128, 2
    x = make_varlen(LENS, H, d, seed=8, with_grad=False)
    cu = x["cu_seqlens"].cuda()
    g = {k: x[k].cuda() for k in ("q", "k", "v")}
    o, lse = fa.varlen_fwd(g["q"], g["k"], g["v"], cu, max(LENS), causal=causal)
    cu_h = x["cu_seqlens"].tolist()
    for s in range(len(LENS)):
        a, e = cu_h[s], cu_h[s + 1]
        oa, la = fa.fwd(*(g[n][a:e].unsqueeze(0).contiguous() for n in ("q", "k", "v")), causal=causal)
        assert torch.equal(oa[0], o[a:e]), s
        assert torch.equal(la[0], lse[:, a:e]), s


def test_varlen_total32768_h32_d128_all_sequences():
    """The packed workload at full size: NaN-prefilled outputs must come back
    finite, and every sequence of every head is compared with the oracle."""
    w = WORKLOADS["varlen_total32768_h32_d128"]
    lens = varlen_lengths(w.varlen_total, w.varlen_lo, w.varlen_hi, 0)
    x = make_varlen(lens, w.H, w.d, seed=0)
    scale = scale_of(w.d)
    cu = x["cu_seqlens"].cuda()
    g = {k: x[k].cuda() for k in ("q", "k", "v", "do")}
    mx = max(lens)
    o = nan_like(g["q"])
    lse = torch.full((w.H, w.varlen_total), float("nan"), dtype=torch.float32, device="cuda")
    fa.varlen_fwd(g["q"], g["k"], g["v"], cu, mx, causal=True, out=o, lse=lse)
    dq, dk, dv = nan_like(g["q"]), nan_like(g["k"]), nan_like(g["v"])
    fa.varlen_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], cu, mx, causal=True, dq=dq, dk=dk, dv=dv)
    fa.check_device_error()
    for t in (o, lse, dq, dk, dv):
        assert torch.isfinite(t).all()
    o, lse, dq, dk, dv = (f64(t) for t in (o, lse, dq, dk, dv))
    a = {n: f64(x[n]) for n in ("q", "k", "v", "do")}
    cu_h = x["cu_seqlens"].tolist()
    items = [((s, h),) + tuple(a[n][cu_h[s]:cu_h[s + 1], h] for n in ("q", "k", "v", "do"))
             for s in range(len(lens)) for h in range(w.H)]
    ref = oracle_per_head(items, scale, True, grads=True)
    agg = Agg()
    for (s, h), (O, L, gq, gk, gv) in ref.items():
        r = slice(cu_h[s], cu_h[s + 1])
        agg.fwd(o[r, h], O, lse[h, r], L)
        agg.bwd((dq[r, h], dk[r, h], dv[r, h]), (gq, gk, gv))
    assert agg.eo <= O_ATOL and agg.el <= LSE_ATOL, (agg.eo, agg.el)
    assert max(agg.grads()) <= GRAD_RTOL_FRO, agg.grads()
    assert max(agg.worst_head) <= GRAD_RTOL_FRO, agg.worst_head


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_items_past_sequence_ends(d, causal):
    """The backward takes (key tile, sequence, head) items from a grid sized by
    max_seqlen; with max_seqlen well above most lengths most items lie past
    their sequence's end and must be skipped, while the CTAs that run go on
    through several real items each.  NaN-prefilled gradients must come back
    finite, and every sequence and head must match the oracle."""
    lens = [3, 130, 1, 256, 257, 40, 900, 17, 128, 1100, 5, 384]
    H = 5
    x = make_varlen(lens, H, d, seed=12)
    scale = scale_of(d)
    cu = x["cu_seqlens"].cuda()
    g = {k: x[k].cuda() for k in ("q", "k", "v", "do")}
    mx = 2048  # an upper bound, not the true maximum (1100): extra empty key tiles
    o, lse = fa.varlen_fwd(g["q"], g["k"], g["v"], cu, mx, causal=causal)
    dq, dk, dv = nan_like(g["q"]), nan_like(g["k"]), nan_like(g["v"])
    fa.varlen_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], cu, mx, causal=causal, dq=dq, dk=dk, dv=dv)
    fa.check_device_error()
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
    a = [f64(x[n]) for n in ("q", "k", "v", "do")]
    G = oracle.attn_varlen_bwd_ref(*a, x["cu_seqlens"].numpy(), scale, causal)
    cu_h = x["cu_seqlens"].tolist()
    for s in range(len(lens)):
        r = slice(cu_h[s], cu_h[s + 1])
        eg = [rel_fro(f64(t)[r], ref[r]) for t, ref in zip((dq, dk, dv), G)]
        assert max(eg) <= GRAD_RTOL_FRO, (s, lens[s], eg)
