"""Decode-shaped forward (fa_decode_fwd): few queries against a KV cache.

GPU parity with the fp64 decode oracle (O max-abs 2e-2, LSE max-abs 1e-3,
as for the forward pass) over query counts 1..16, both head dims, both
modes, ragged cache lengths (0, 1, < Nq, exact tile multiples, ragged
tails), one and several key ranges, garbage past the valid rows, the
serving-size workloads on every head, the KV-cache identity against the
dense causal forward, and device-side rejection of bad lengths."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import LSE_ATOL, O_ATOL, f64, max_abs
from workloads import DECODE_WORKLOADS, make_decode, make_dense


def _check(x, o, lse, causal, heads=None):
    d = x["q"].shape[-1]
    O, L = oracle.attn_decode_ref(f64(x["q"]), f64(x["k"]), f64(x["v"]), x["seqlens"].numpy(), 1 / math.sqrt(d),
                                  causal, heads=heads)
    o64, l64 = f64(o), lse.double().cpu().numpy()
    if heads is not None:
        sel = tuple(zip(*heads))
        O, L = O.transpose(0, 2, 1, 3)[sel], L[sel]
        o64, l64 = o64.transpose(0, 2, 1, 3)[sel], l64[sel]
    fin = np.isfinite(L)
    assert np.array_equal(fin, np.isfinite(l64)), "fully masked rows differ"
    assert np.all(np.isneginf(l64[~fin]))
    assert max_abs(o64, O) <= O_ATOL
    assert np.max(np.abs(l64[fin] - L[fin]), initial=0.0) <= LSE_ATOL


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq", [1, 3, 16])
def test_ragged_lengths_match_oracle(nq, causal, d):
    x = make_decode(6, nq, 700, 3, d, 0, 700, seed=80 + nq)
    x["seqlens"] = torch.tensor([700, 0, 1, 2, 128, 513], dtype=torch.int32)
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.decode_fwd(g["q"], g["k"], g["v"], g["seqlens"], causal=causal)
    fa.check_device_error()
    _check(x, o, lse, causal)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,Nk", [(1, 1, 16384), (2, 4, 5000), (64, 16, 300)])
def test_one_and_many_key_ranges(B, H, Nk):
    """(1, 1, 16384) splits the cache into many ranges; (64, 16, 300) into one."""
    x = make_decode(B, 1, Nk, H, 128, 1, Nk, seed=81)
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.decode_fwd(g["q"], g["k"], g["v"], g["seqlens"], causal=True)
    fa.check_device_error()
    _check(x, o, lse, True)


@pytest.mark.gpu
def test_no_seqlens_means_full_cache_and_garbage_is_ignored():
    x = make_decode(3, 2, 333, 2, 128, 333, 333, seed=82)
    g = {k: v.cuda() for k, v in x.items()}
    o_full, l_full = fa.decode_fwd(g["q"], g["k"], g["v"], None, causal=False)
    _check(x, o_full, l_full, False)
    lens = torch.tensor([333, 100, 7], dtype=torch.int32)
    o1, l1 = fa.decode_fwd(g["q"], g["k"], g["v"], lens.cuda(), causal=False)
    k2, v2 = g["k"].clone(), g["v"].clone()
    for b, L in enumerate(lens.tolist()):
        k2[b, L:] = float("nan")
        v2[b, L:] = float("inf")
    o2, l2 = fa.decode_fwd(g["q"], k2, v2, lens.cuda(), causal=False)
    fa.check_device_error()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(DECODE_WORKLOADS))
def test_serving_workload_every_head(name):
    """The serving-size workloads: every head of every entry, outputs
    NaN-prefilled (a fully masked row is the only place -inf may appear)."""
    w = DECODE_WORKLOADS[name]
    x = make_decode(w.B, w.Nq, w.Nk, w.H, w.d, w.lo, w.hi, seed=0)
    g = {k: v.cuda() for k, v in x.items()}
    o = torch.full_like(g["q"], float("nan"))
    lse = torch.full((w.B, w.H, w.Nq), float("nan"), dtype=torch.float32, device="cuda")
    fa.decode_fwd(g["q"], g["k"], g["v"], g["seqlens"], causal=True, out=o, lse=lse)
    fa.check_device_error()
    assert torch.isfinite(o).all() and not torch.isnan(lse).any()
    _check(x, o, lse, True)


@pytest.mark.gpu
def test_kv_cache_identity_with_dense_forward():
    """The last nq rows of the causal forward over a sequence equal decoding
    those nq tokens against the cache of the whole sequence."""
    nq, L = 4, 1000
    x = make_dense(1, L, 2, 128, seed=83)
    g = {k: v.cuda() for k, v in x.items()}
    o_full, lse_full = fa.fwd(g["q"], g["k"], g["v"], causal=True)
    o, lse = fa.decode_fwd(g["q"][:, L - nq:].contiguous(), g["k"], g["v"], None, causal=True)
    assert (o.float() - o_full[:, L - nq:].float()).abs().max().item() <= 2 * O_ATOL
    assert (lse - lse_full[:, :, L - nq:]).abs().max().item() <= 2 * LSE_ATOL


@pytest.mark.gpu
def test_length_beyond_cache_is_reported():
    x = make_decode(2, 1, 256, 1, 64, 256, 256, seed=84)
    g = {k: v.cuda() for k, v in x.items()}
    bad = torch.tensor([256, 257], dtype=torch.int32, device="cuda")
    fa.decode_fwd(g["q"], g["k"], g["v"], bad)
    with pytest.raises(fa.FaError) as e:
        fa.check_device_error()
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    fa.check_device_error()  # the word was cleared


def test_decode_recipe_is_seeded():
    a = make_decode(2, 1, 64, 2, 64, 10, 64, seed=5)
    b = make_decode(2, 1, 64, 2, 64, 10, 64, seed=5)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert a["q"].dtype == torch.bfloat16 and a["seqlens"].dtype == torch.int32
    assert int(a["seqlens"].min()) >= 10 and int(a["seqlens"].max()) <= 64
