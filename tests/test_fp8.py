"""FP8 (e4m3) forward (fa_fwd_fp8), checked against the fp64 oracle on the
dequantized inputs.

Tolerance, from the arithmetic of the kernel.  The scores are exact
products of 8-bit values summed in fp32, so S, the row maxima and the row
sums (which add the unrounded P) match the exact attention of the
dequantized inputs up to fp32 rounding: LSE keeps the 1e-3 bound of the
bf16 path.  The one large error is P rounded to e4m3 before the P V
product.  With E_ij = exp(S_ij - max_j S_ij) and l_i = sum_j E_ij, the
kernel rounds E_ij * 2^k (0 <= k <= 8, its reference max) to e4m3: a
relative error <= 2^-4 for values >= 2^-6 (3 mantissa bits) and an absolute
error <= min(value, 2^-10) below (subnormal spacing 2^-9).  Dividing by the
row sum, which scales by the same 2^k, the error of an output element is at
most
    bound_ic = sum_j max(2^-4 E_ij, min(E_ij, 2^-10)) |V_jc| / l_i
(largest at k = 0), plus the bf16 rounding of the output (<= 2^-9 |O|,
taken as 2^-8 |O|) and 1e-4 for fp32 accumulation.  Every element is
checked against its own bound."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
import oracle
from tests.common import LSE_ATOL
from workloads import make_fp8_dense, quantize_e4m3


def e4m3_value(code: int) -> float:
    """The OCP FP8 E4M3 format: sign, 4 exponent bits (bias 7), 3 mantissa
    bits, subnormals at exponent 0, no infinities, S.1111.111 is NaN."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def test_e4m3_decoding_matches_the_format_definition():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    got = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    want = np.array([e4m3_value(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert np.nanmax(want) == 448.0 and np.nanmin(np.abs(want[want != 0])) == 2.0 ** -9


def test_quantization_recipe_is_seeded_and_in_range():
    a, sa = make_fp8_dense(1, 64, 2, 128, seed=3)
    b, sb = make_fp8_dense(1, 64, 2, 128, seed=3)
    for n in ("q", "k", "v"):
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)) and sa[n] == sb[n]
        assert float(a[n].to(torch.float32).abs().max()) <= 448.0
    x = torch.tensor([0.5, -3.0, 1e-3])
    q, s = quantize_e4m3(x)
    assert s == 3.0 / 448.0 and float(q[1].to(torch.float32)) == -448.0


def _deq(x8, s):
    return x8.to(torch.float64).numpy() * s


def _check_head(q, k, v, o, lse, b, h, scale, causal):
    Q, K, V = q[b, :, h], k[b, :, h], v[b, :, h]
    O_ref, lse_ref, P = oracle.attn_head_fwd(Q, K, V, scale, causal)
    S = oracle.scores(Q, K, scale, causal)
    E = np.exp(S - np.max(S, axis=-1, keepdims=True))
    l = E.sum(axis=-1, keepdims=True)
    err = np.maximum(2.0 ** -4 * E, np.minimum(E, 2.0 ** -10))
    bound = (err @ np.abs(V)) / l + 2.0 ** -8 * np.abs(O_ref) + 1e-4
    got = o[b, :, h].double().cpu().numpy()
    excess = np.abs(got - O_ref) - bound
    assert np.max(excess) <= 0, f"head {(b, h)}: bound exceeded by {np.max(excess)}"
    assert np.max(np.abs(lse[b, h].double().cpu().numpy() - lse_ref)) <= LSE_ATOL


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 130, 300, 1000])
def test_matches_oracle_within_the_derived_bound(N, causal):
    x8, sc = make_fp8_dense(2, N, 2, 128, seed=90 + N)
    g = {n: t.cuda() for n, t in x8.items()}
    scale = 1 / math.sqrt(128)
    o, lse = fa.fwd_fp8(g["q"], g["k"], g["v"], sc["q"], sc["k"], sc["v"], causal=causal, scale=scale)
    fa.check_device_error()
    q, k, v = (_deq(x8[n], sc[n]) for n in ("q", "k", "v"))
    for b in range(2):
        for h in range(2):
            _check_head(q, k, v, o, lse, b, h, scale, causal)


@pytest.mark.gpu
def test_bench_shape_every_head():
    """B4 H16 N4096 d128 causal with Q, K doubled before quantization: every
    output element written (NaN-prefilled buffers come back finite) and every
    (b, h) head within its bound."""
    from concurrent.futures import ThreadPoolExecutor

    from tests.common import oracle_workers
    B, N, H, d = 4, 4096, 16, 128
    x8, sc = make_fp8_dense(B, N, H, d, seed=0, qk_scale_factor=2.0)
    g = {n: t.cuda() for n, t in x8.items()}
    scale = 1 / math.sqrt(d)
    o = torch.full((B, N, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    fa.fwd_fp8(g["q"], g["k"], g["v"], sc["q"], sc["k"], sc["v"], causal=True, scale=scale, out=o, lse=lse)
    fa.check_device_error()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    q, k, v = (_deq(x8[n], sc[n]) for n in ("q", "k", "v"))
    o, lse = o.cpu(), lse.cpu()
    pairs = [(b, h) for b in range(B) for h in range(H)]
    with ThreadPoolExecutor(oracle_workers(len(pairs), 10.0 * N * N * 8)) as ex:
        list(ex.map(lambda bh: _check_head(q, k, v, o, lse, bh[0], bh[1], scale, True), pairs))


@pytest.mark.gpu
def test_deterministic_and_close_to_bf16_path():
    """Repeated calls are bitwise equal; the result is close to the bf16
    forward run on the same inputs.  The scales are powers of two, so every
    dequantized value (3 mantissa bits) is exactly a bf16 value and both
    paths see identical inputs."""
    from workloads import make_dense
    x = make_dense(1, 777, 3, 128, seed=91, with_grad=False)
    x8, sc = {}, {}
    for n in ("q", "k", "v"):
        s2 = 2.0 ** math.ceil(math.log2(float(x[n].float().abs().max()) / 448.0))
        x8[n], sc[n] = (x[n].float() / s2).to(torch.float8_e4m3fn), s2
    g = {n: t.cuda() for n, t in x8.items()}
    r1 = fa.fwd_fp8(g["q"], g["k"], g["v"], sc["q"], sc["k"], sc["v"], causal=True)
    r2 = fa.fwd_fp8(g["q"], g["k"], g["v"], sc["q"], sc["k"], sc["v"], causal=True)
    assert torch.equal(r1[0], r2[0]) and torch.equal(r1[1], r2[1])
    bf = {n: (g[n].to(torch.float32) * sc[n]).to(torch.bfloat16) for n in g}
    o_bf, lse_bf = fa.fwd(bf["q"], bf["k"], bf["v"], causal=True)
    assert (r1[1] - lse_bf).abs().max().item() <= LSE_ATOL
    assert (r1[0].float() - o_bf.float()).abs().mean().item() <= 2e-2


def test_host_validation_without_gpu():
    L = fa.lib()
    P = 4096
    ws = fa.fwd_fp8_workspace_size(1, 100, 1, 128)
    assert ws == 128 * 112 + (256 - (128 * 112) % 256) % 256
    assert fa.fwd_fp8_workspace_size(1, 100, 1, 64) == 0
    assert L.fa_fwd_fp8(P, P, P, 1.0, 1.0, 1.0, P, P, P * 64, ws, 1, 100, 1, 64, 1.0, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_fwd_fp8(P, P, P, 0.0, 1.0, 1.0, P, P, P * 64, ws, 1, 100, 1, 128, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd_fp8(P, P, P, 1.0, 1.0, 1.0, P, P, P * 64, ws - 1, 1, 100, 1, 128, 1.0, 0, None) == \
        fa.FA_ERR_WORKSPACE
    assert L.fa_fwd_fp8(P, P, P, 1.0, 1.0, 1.0, P, P, P + 16, ws, 1, 100, 1, 128, 1.0, 0, None) == \
        fa.FA_ERR_INVALID_ARG
