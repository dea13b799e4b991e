"""Long sequence: B=1, H=16, N=16384, d=128, causal and non-causal, forward and
backward.  Every output element is checked to be written (NaN-prefilled
outputs must come back finite); parity against the fp64 oracle on one head
from every scheduling group of heads; and the memory
claim of the method -- memory linear in N, no N x N buffer ("FlashAttention-2
(PT)", section "Pre-requisitos"; "FlashAttention: Fast and Memory-Efficient
Exact Attention with IO-Awareness", section "Resultados"): the device memory
high-water mark rises by exactly the outputs and the workspace, all allocated
by the caller, while one fp32 N x N score block per head would be 1 GiB."""
import pytest
import torch

import exact_io_aware_95_b200 as fa
from tests.common import GRAD_RTOL_FRO, LSE_ATOL, O_ATOL
from tests.test_bwd import fwd_bwd_all_heads
from workloads import WORKLOADS, make_dense

pytestmark = pytest.mark.gpu

W = WORKLOADS["long_b1_h16_n16384_d128"]


@pytest.fixture(scope="module")
def inputs():
    return make_dense(W.B, W.N, W.H, W.d, seed=0)


@pytest.mark.parametrize("causal", [False, True])
def test_long_forward_linear_memory(inputs, causal):
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


@pytest.mark.parametrize("causal", [False, True])
def test_long_backward_linear_memory(inputs, causal):
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


# The host schedules the heads of this workload in groups sized to keep their
# streamed operands in L2: 6 heads per forward group ([0-5], [6-11], [12-15])
# and 3 per backward group ([0-2], ..., [12-14], [15]).  These heads take one
# from each group of both, the partial last ones included.
GROUP_HEADS = [(0, 2), (0, 5), (0, 8), (0, 11), (0, 14), (0, 15)]


@pytest.mark.parametrize("causal", [False, True])
def test_long_every_element_written_and_one_head_per_group(inputs, causal):
    agg = fwd_bwd_all_heads(inputs, causal, heads=GROUP_HEADS)
    assert agg.eo <= O_ATOL and agg.el <= LSE_ATOL, (agg.eo, agg.el)
    assert max(agg.grads()) <= GRAD_RTOL_FRO, agg.grads()
    assert max(agg.worst_head) <= GRAD_RTOL_FRO, agg.worst_head
