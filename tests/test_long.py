"""Long sequence: B=1, H=16, N=16384, d=128, causal and non-causal, forward and
backward.  Parity on sampled heads against the fp64 oracle, and the memory
claim of the method -- memory linear in N, no N x N buffer ("FlashAttention-2
(PT)", section "Pre-requisitos"; "FlashAttention: Fast and Memory-Efficient
Exact Attention with IO-Awareness", section "Resultados"): the device memory
high-water mark rises by exactly the outputs and the workspace, all allocated
by the caller, while one fp32 N x N score block per head would be 1 GiB."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import GRAD_RTOL_FRO, LSE_ATOL, O_ATOL, f64, max_abs, rel_fro
from workloads import WORKLOADS, make_dense

pytestmark = pytest.mark.gpu

W = WORKLOADS["long_b1_h16_n16384_d128"]


@pytest.fixture(scope="module")
def inputs():
    return make_dense(W.B, W.N, W.H, W.d, seed=0)


def _heads(x, heads):
    return {k: v[:, :, [h for _, h in heads]].contiguous() for k, v in x.items()}


@pytest.mark.parametrize("causal", [False, True])
def test_long_forward_sampled_heads_and_linear_memory(inputs, causal):
    x = inputs
    g = {k: v.cuda() for k, v in x.items()}
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    o, lse = fa.fwd(g["q"], g["k"], g["v"], causal=causal)
    fa.check_device_error()
    peak = torch.cuda.max_memory_allocated() - base
    out_bytes = o.numel() * o.element_size() + lse.numel() * lse.element_size()
    assert peak <= out_bytes + (1 << 20), (peak, out_bytes)   # allocator rounding only
    assert peak < W.N * W.N * 4                                # far below one N x N fp32 block
    heads = [(0, 0), (0, W.H - 1)]
    sub = _heads(x, heads)
    O, L = oracle.attn_fwd_ref(f64(sub["q"]), f64(sub["k"]), f64(sub["v"]), 1 / math.sqrt(W.d), causal)
    on, ln = f64(o), f64(lse)
    for i, (_, h) in enumerate(heads):
        assert max_abs(on[0, :, h], O[0, :, i]) <= O_ATOL
        assert max_abs(ln[0, h], L[0, i]) <= LSE_ATOL


@pytest.mark.parametrize("causal", [False, True])
def test_long_backward_sampled_head_and_linear_memory(inputs, causal):
    x = inputs
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fwd(g["q"], g["k"], g["v"], causal=causal)
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    dq, dk, dv = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], causal=causal)
    fa.check_device_error()
    peak = torch.cuda.max_memory_allocated() - base
    need = 3 * dq.numel() * dq.element_size() + fa.workspace_size(W.B, W.N, W.H, W.d)
    assert peak <= need + (1 << 20), (peak, need)
    heads = [(0, W.H // 2)]
    sub = _heads(x, heads)
    G = oracle.attn_bwd_ref(*(f64(sub[n]) for n in ("q", "k", "v", "do")), 1 / math.sqrt(W.d), causal)
    h = heads[0][1]
    for got, ref in zip((dq, dk, dv), G):
        assert rel_fro(f64(got)[0, :, h], ref[0, :, 0]) <= GRAD_RTOL_FRO
