"""The differentiable entry points (attention, varlen_attention) and the
packing helpers.  Packing logic runs on the CPU; the autograd round trip
through the CUDA library is checked against the oracle on the GPU."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import GRAD_RTOL_FRO, O_ATOL, f64, max_abs, rel_fro
from workloads import make_dense, make_varlen


def test_pack_unpack_roundtrip_cpu():
    seqs = [torch.randn(L, 2, 8) for L in (3, 0, 5, 1)]
    packed, cu, mx = fa.pack(seqs)
    assert packed.shape == (9, 2, 8) and cu.tolist() == [0, 3, 3, 8, 9] and cu.dtype == torch.int32 and mx == 5
    back = fa.unpack(packed, cu)
    assert len(back) == 4
    for a, b in zip(seqs, back):
        assert torch.equal(a, b)


def test_pack_rejects_mismatched_shapes():
    with pytest.raises(ValueError):
        fa.pack([torch.randn(3, 2, 8), torch.randn(3, 4, 8)])
    with pytest.raises(ValueError):
        fa.pack([])


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_attention_autograd_matches_oracle(causal):
    x = make_dense(2, 300, 2, 64, seed=41)
    q, k, v = (x[n].cuda().requires_grad_(True) for n in ("q", "k", "v"))
    o = fa.attention(q, k, v, causal=causal)
    o.backward(x["do"].cuda())
    scale = 1 / math.sqrt(64)
    O, _ = oracle.attn_fwd_ref(f64(x["q"]), f64(x["k"]), f64(x["v"]), scale, causal)
    G = oracle.attn_bwd_ref(*(f64(x[n]) for n in ("q", "k", "v", "do")), scale, causal)
    assert max_abs(f64(o), O) <= O_ATOL
    for t, r in zip((q.grad, k.grad, v.grad), G):
        assert rel_fro(f64(t), r) <= GRAD_RTOL_FRO


@pytest.mark.gpu
def test_varlen_attention_autograd_matches_oracle():
    x = make_varlen([70, 1, 200, 129], 2, 128, seed=42)
    q, k, v = (x[n].cuda().requires_grad_(True) for n in ("q", "k", "v"))
    cu = x["cu_seqlens"].cuda()
    o = fa.varlen_attention(q, k, v, cu, max(x["lengths"]), causal=True)
    o.backward(x["do"].cuda())
    scale = 1 / math.sqrt(128)
    a = [f64(x[n]) for n in ("q", "k", "v", "do")]
    O, _ = oracle.attn_varlen_fwd_ref(*a[:3], x["cu_seqlens"].numpy(), scale, True)
    G = oracle.attn_varlen_bwd_ref(*a, x["cu_seqlens"].numpy(), scale, True)
    assert max_abs(f64(o), O) <= O_ATOL
    for t, r in zip((q.grad, k.grad, v.grad), G):
        assert rel_fro(f64(t), r) <= GRAD_RTOL_FRO


@pytest.mark.gpu
def test_packed_helper_feeds_varlen_attention():
    seqs = [make_dense(1, L, 2, 64, seed=50 + L, with_grad=False)["q"][0].cuda() for L in (5, 130, 64)]
    packed, cu, mx = fa.pack(seqs)
    o = fa.varlen_attention(packed, packed, packed, cu, mx, causal=True)
    for s, part in zip(seqs, fa.unpack(o, cu)):
        ref = fa.attention(s[None], s[None], s[None], causal=True)[0]
        assert torch.equal(part, ref)


@pytest.mark.gpu
def test_calls_from_a_new_host_thread():
    """A thread that has never touched CUDA (as the autograd engine's worker
    threads may be) gets the same results as the thread that set up the data."""
    import threading
    x = make_dense(1, 257, 2, 128, seed=43)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, causal=True)
    dq, dk, dv = fa.bwd(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    got = {}

    def work():
        try:
            o2, lse2 = fa.fwd(q, k, v, causal=True)
            got["g"] = (o2, lse2) + fa.bwd(q, k, v, o2, lse2, do, causal=True)
            torch.cuda.synchronize()
        except Exception as e:  # reported on the main thread
            got["err"] = e

    t = threading.Thread(target=work)
    t.start()
    t.join()
    assert "err" not in got, got.get("err")
    o2, lse2, dq2, dk2, dv2 = got["g"]
    assert torch.equal(o2, o) and torch.equal(lse2, lse)
    assert torch.equal(dk2, dk) and torch.equal(dv2, dv)
    assert rel_fro(f64(dq2), f64(dq)) <= 1e-2  # dQ sums tiles with atomics: order may differ
