"""Pins for the fp64 oracle, against things other than the oracle itself.

Each pin is chosen so that a plausible slip in the oracle -- a dropped scale,
a wrong sign, a transposed operand, an off-by-one in the causal mask, a
missing Jacobian term -- fails at least one of them:

* closed forms: a two-token problem solved by hand; identical keys; uniform V;
  causal row 0; the causal prefix mean;
* invariants: rows of P sum to 1; shifting every key by u shifts LSE_i by
  scale q_i.u and leaves P alone; permuting keys with values leaves the
  non-causal output alone; P_i . dP_i = dO_i . O_i;
* finite differences of the loss sum(dO * O) (fp64, central, tiny shapes);
* a library special case: torch's float64 CPU scaled_dot_product_attention
  (math path) and its autograd gradients;
* brute force: scalar Python loops with math.exp on tiny inputs;
* packing: the packed result equals the per-sequence dense result, and equals
  a dense problem over the concatenation under a block-diagonal mask.

The method's defining property -- attention computed exactly, identical to the
standard computation ("FlashAttention: Fast and Memory-Efficient Exact
Attention with IO-Awareness", section "En pocas palabras") -- is why the oracle
is the plain definition and why these pins are about the definition.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import make_dense, make_varlen, varlen_lengths, cu_seqlens_of, WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- closed forms

def test_two_token_closed_form_forward_and_backward():
    """d = 1, scale = 1, q = [ln 3, 0], k = [1, 0], v = [4, 8], dO = [1, 0].

    Row 0 scores [ln 3, 0] -> P = [3/4, 1/4], O = 5, LSE = ln 4.
    Row 1 scores [0, 0]    -> P = [1/2, 1/2], O = 6, LSE = ln 2.
    Loss = O_0 = (4 e^q + 8) / (e^q + 1) at q = ln 3, so dQ_0 = -4 e^q/(e^q+1)^2 = -3/4;
    dV = P_0 = [3/4, 1/4]; dS_0 = P_0 * (dP_0 - P_0.dP_0) = [-3/4, 3/4];
    dK = dS_0 * q_0 = [-3/4 ln 3, 3/4 ln 3].
    Causal: row 0 sees key 0 only -> O_0 = 4, LSE_0 = ln 3; row 1 unchanged.
    """
    q = np.array([[math.log(3.0)], [0.0]])
    k = np.array([[1.0], [0.0]])
    v = np.array([[4.0], [8.0]])
    do = np.array([[1.0], [0.0]])
    O, lse, P = oracle.attn_head_fwd(q, k, v, 1.0, False)
    np.testing.assert_allclose(P, [[0.75, 0.25], [0.5, 0.5]], atol=1e-15)
    np.testing.assert_allclose(O[:, 0], [5.0, 6.0], atol=1e-14)
    np.testing.assert_allclose(lse, [math.log(4.0), math.log(2.0)], atol=1e-15)
    dq, dk, dv = oracle.attn_head_bwd(q, k, v, do, 1.0, False)
    np.testing.assert_allclose(dq[:, 0], [-0.75, 0.0], atol=1e-14)
    np.testing.assert_allclose(dv[:, 0], [0.75, 0.25], atol=1e-14)
    np.testing.assert_allclose(dk[:, 0], [-0.75 * math.log(3.0), 0.75 * math.log(3.0)], atol=1e-14)
    Oc, lsec, _ = oracle.attn_head_fwd(q, k, v, 1.0, True)
    np.testing.assert_allclose(Oc[:, 0], [4.0, 6.0], atol=1e-14)
    np.testing.assert_allclose(lsec, [math.log(3.0), math.log(2.0)], atol=1e-15)


def test_pages_score_count_golden():
    """The worked size on the aiunderstanding page: 4000 tokens -> 16 million scores."""
    with open(os.path.join(GOLDEN, "score_count_n4000.json")) as f:
        g = json.load(f)
    N = g["tokens"]
    S = oracle.scores(np.zeros((N, 1)), np.zeros((N, 1)), 1.0, False)
    assert S.size == g["scores"]


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_values_give_that_value(causal):
    r = rng(1)
    N, d = 37, 8
    q, k = r.standard_normal((N, d)), r.standard_normal((N, d))
    row = r.standard_normal(d)
    v = np.tile(row, (N, 1))
    O, _, _ = oracle.attn_head_fwd(q, k, v, 1 / math.sqrt(d), causal)
    np.testing.assert_allclose(O, v, atol=1e-13)


def test_identical_keys_noncausal_mean_and_lse():
    r = rng(2)
    N, d = 29, 16
    scale = 1 / math.sqrt(d)
    q = r.standard_normal((N, d))
    kr = r.standard_normal(d)
    k = np.tile(kr, (N, 1))
    v = r.standard_normal((N, d))
    O, lse, _ = oracle.attn_head_fwd(q, k, v, scale, False)
    np.testing.assert_allclose(O, np.tile(v.mean(0), (N, 1)), atol=1e-13)
    np.testing.assert_allclose(lse, scale * (q @ kr) + math.log(N), atol=1e-12)


def test_identical_keys_causal_prefix_mean():
    r = rng(3)
    N, d = 23, 4
    q = r.standard_normal((N, d))
    k = np.tile(r.standard_normal(d), (N, 1))
    v = r.standard_normal((N, d))
    O, lse, _ = oracle.attn_head_fwd(q, k, v, 0.5, True)
    for i in range(N):
        np.testing.assert_allclose(O[i], v[: i + 1].mean(0), atol=1e-13)
        assert abs(lse[i] - (0.5 * q[i] @ k[0] + math.log(i + 1))) < 1e-12


def test_causal_row_zero():
    r = rng(4)
    N, d = 17, 8
    scale = 1 / math.sqrt(d)
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    O, lse, _ = oracle.attn_head_fwd(q, k, v, scale, True)
    np.testing.assert_allclose(O[0], v[0], atol=1e-14)
    assert abs(lse[0] - scale * q[0] @ k[0]) < 1e-13


# ----------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    r = rng(5)
    q, k = r.standard_normal((50, 32)) * 3, r.standard_normal((50, 32)) * 3
    S = oracle.scores(q, k, 0.2, causal)
    P, _ = oracle.softmax_rows(S)
    assert np.max(np.abs(P.sum(-1) - 1.0)) <= 1e-12
    if causal:
        assert np.all(P[np.triu_indices(50, 1)] == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_shifts_lse_only(causal):
    r = rng(6)
    N, d = 31, 8
    scale = 0.3
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    u = r.standard_normal(d)
    O1, l1, P1 = oracle.attn_head_fwd(q, k, v, scale, causal)
    O2, l2, P2 = oracle.attn_head_fwd(q, k + u, v, scale, causal)
    np.testing.assert_allclose(P2, P1, atol=1e-13)
    np.testing.assert_allclose(O2, O1, atol=1e-12)
    np.testing.assert_allclose(l2 - l1, scale * (q @ u), atol=1e-12)


def test_key_value_permutation_invariance():
    r = rng(7)
    N, d = 40, 8
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    perm = r.permutation(N)
    O1, l1, _ = oracle.attn_head_fwd(q, k, v, 0.35, False)
    O2, l2, _ = oracle.attn_head_fwd(q, k[perm], v[perm], 0.35, False)
    np.testing.assert_allclose(O2, O1, atol=1e-12)
    np.testing.assert_allclose(l2, l1, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_p_dot_dp_equals_do_dot_o(causal):
    r = rng(8)
    N, d = 33, 16
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    O, _, P = oracle.attn_head_fwd(q, k, v, 0.25, causal)
    dP = do @ v.T
    np.testing.assert_allclose(np.sum(P * dP, -1), np.sum(do * O, -1), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_explicit_jacobian_matches_rowwise(causal):
    r = rng(9)
    N, d = 9, 3
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    a = oracle.attn_head_bwd(q, k, v, do, 0.7, causal, explicit_jacobian=True)
    b = oracle.attn_head_bwd(q, k, v, do, 0.7, causal, explicit_jacobian=False)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-13)


def test_jacobian_is_derivative_of_softmax():
    r = rng(10)
    s = r.standard_normal(6)
    h = 1e-6
    J = oracle.softmax_jacobian(oracle.softmax_rows(s[None])[0][0])
    for j in range(6):
        e = np.zeros(6)
        e[j] = h
        fd = (oracle.softmax_rows((s + e)[None])[0][0] - oracle.softmax_rows((s - e)[None])[0][0]) / (2 * h)
        np.testing.assert_allclose(J[:, j], fd, atol=1e-9)


# ----------------------------------------------------------- finite differences

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(5, 3), (8, 4), (1, 2)])
def test_finite_differences(causal, shape):
    N, d = shape
    r = rng(11 + N)
    scale = 1 / math.sqrt(d)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))

    def loss(q_, k_, v_):
        O, _, _ = oracle.attn_head_fwd(q_, k_, v_, scale, causal)
        return float(np.sum(do * O))

    dq, dk, dv = oracle.attn_head_bwd(q, k, v, do, scale, causal)
    h = 1e-6
    for which, g in ((0, dq), (1, dk), (2, dv)):
        fd = np.zeros_like(g)
        for idx in np.ndindex(*g.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        denom = max(np.linalg.norm(fd), 1e-12)
        assert np.linalg.norm(fd - g) / denom <= 1e-6, (which, np.linalg.norm(fd - g) / denom)


# ------------------------------------------------------- library special case

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H,d", [(1, 128, 2, 64), (2, 96, 3, 32)])
def test_matches_torch_sdpa_float64(causal, B, N, H, d):
    r = rng(12)
    scale = 1 / math.sqrt(d)
    q, k, v, do = (r.standard_normal((B, N, H, d)) for _ in range(4))
    O, L = oracle.attn_fwd_ref(q, k, v, scale, causal)
    dQ, dK, dV = oracle.attn_bwd_ref(q, k, v, do, scale, causal)

    tq, tk, tv = (torch.tensor(x).permute(0, 2, 1, 3).contiguous().requires_grad_(True) for x in (q, k, v))
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    to.backward(torch.tensor(do).permute(0, 2, 1, 3))
    np.testing.assert_allclose(O, to.detach().permute(0, 2, 1, 3).numpy(), atol=1e-10)
    np.testing.assert_allclose(dQ, tq.grad.permute(0, 2, 1, 3).numpy(), atol=1e-10)
    np.testing.assert_allclose(dK, tk.grad.permute(0, 2, 1, 3).numpy(), atol=1e-10)
    np.testing.assert_allclose(dV, tv.grad.permute(0, 2, 1, 3).numpy(), atol=1e-10)
    # torch's own logsumexp over its own masked scores, as an independent LSE check
    s = torch.einsum("bhnd,bhmd->bhnm", tq.detach(), tk.detach()) * scale
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(L, torch.logsumexp(s, -1).numpy(), atol=1e-10)


# --------------------------------------------------------------- brute force

def _brute(q, k, v, do, scale, causal):
    N, d = len(q), len(q[0])
    O, L, P = [], [], []
    for i in range(N):
        js = [j for j in range(N) if (not causal or j <= i)]
        s = {j: scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in js}
        m = max(s.values())
        e = {j: math.exp(s[j] - m) for j in js}
        z = sum(e.values())
        p = [e[j] / z if j in e else 0.0 for j in range(N)]
        P.append(p)
        O.append([sum(p[j] * v[j][c] for j in range(N)) for c in range(d)])
        L.append(m + math.log(z))
    dV = [[sum(P[i][j] * do[i][c] for i in range(N)) for c in range(d)] for j in range(N)]
    dP = [[sum(do[i][c] * v[j][c] for c in range(d)) for j in range(N)] for i in range(N)]
    dS = []
    for i in range(N):
        # J_i dP_i with J_i[j][t] = P_ij (delta_jt - P_it)
        dS.append([sum(P[i][j] * ((1.0 if j == t else 0.0) - P[i][t]) * dP[i][t] for t in range(N))
                   for j in range(N)])
    dQ = [[scale * sum(dS[i][j] * k[j][c] for j in range(N)) for c in range(d)] for i in range(N)]
    dK = [[scale * sum(dS[i][j] * q[i][c] for i in range(N)) for c in range(d)] for j in range(N)]
    return O, L, dQ, dK, dV


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 1), (3, 2), (7, 5), (16, 4)])
def test_brute_force_loops(causal, N, d):
    r = rng(13 + N)
    scale = 1 / math.sqrt(d)
    q, k, v, do = (r.standard_normal((N, d)) * 1.5 for _ in range(4))
    O, L, dQ, dK, dV = _brute(q.tolist(), k.tolist(), v.tolist(), do.tolist(), scale, causal)
    o, l, _ = oracle.attn_head_fwd(q, k, v, scale, causal)
    gq, gk, gv = oracle.attn_head_bwd(q, k, v, do, scale, causal)
    np.testing.assert_allclose(o, O, atol=1e-12)
    np.testing.assert_allclose(l, L, atol=1e-12)
    np.testing.assert_allclose(gq, dQ, atol=1e-12)
    np.testing.assert_allclose(gk, dK, atol=1e-12)
    np.testing.assert_allclose(gv, dV, atol=1e-12)


# -------------------------------------------------------------------- packing

@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_per_sequence_dense(causal):
    r = rng(14)
    lens = [5, 1, 17, 9]
    H, d = 3, 8
    total = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, do = (r.standard_normal((total, H, d)) for _ in range(4))
    O, L = oracle.attn_varlen_fwd_ref(q, k, v, cu, 0.3, causal)
    G = oracle.attn_varlen_bwd_ref(q, k, v, do, cu, 0.3, causal)
    for s in range(len(lens)):
        a, e = cu[s], cu[s + 1]
        o, l = oracle.attn_fwd_ref(q[None, a:e], k[None, a:e], v[None, a:e], 0.3, causal)
        g = oracle.attn_bwd_ref(q[None, a:e], k[None, a:e], v[None, a:e], do[None, a:e], 0.3, causal)
        np.testing.assert_allclose(O[a:e], o[0], atol=1e-13)
        np.testing.assert_allclose(L[:, a:e], l[0], atol=1e-13)
        for x, y in zip(G, g):
            np.testing.assert_allclose(x[a:e], y[0], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_block_diagonal_mask(causal):
    """Packed attention == one dense problem with a block-diagonal (causal) mask (torch fp64)."""
    r = rng(15)
    lens = [4, 11, 1, 6]
    H, d = 2, 4
    total = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, do = (r.standard_normal((total, H, d)) for _ in range(4))
    O, L = oracle.attn_varlen_fwd_ref(q, k, v, cu, 0.5, causal)
    dQ, dK, dV = oracle.attn_varlen_bwd_ref(q, k, v, do, cu, 0.5, causal)
    seg = np.repeat(np.arange(len(lens)), lens)
    allowed = seg[:, None] == seg[None, :]
    if causal:
        allowed &= np.arange(total)[None, :] <= np.arange(total)[:, None]
    mask = torch.tensor(allowed)
    tq, tk, tv = (torch.tensor(x).permute(1, 0, 2)[None].contiguous().requires_grad_(True) for x in (q, k, v))
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.5)
    to.backward(torch.tensor(do).permute(1, 0, 2)[None])
    np.testing.assert_allclose(O, to.detach()[0].permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dQ, tq.grad[0].permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad[0].permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad[0].permute(1, 0, 2).numpy(), atol=1e-12)


def test_heads_subset_matches_full():
    x = make_dense(2, 40, 3, 16, seed=3)
    a = {k: v.double().numpy() for k, v in x.items()}
    O, L = oracle.attn_fwd_ref(a["q"], a["k"], a["v"], 0.25, True)
    Os, Ls = oracle.attn_fwd_ref(a["q"], a["k"], a["v"], 0.25, True, heads=[(1, 2)])
    np.testing.assert_array_equal(Os[1, :, 2], O[1, :, 2])
    np.testing.assert_array_equal(Ls[1, 2], L[1, 2])
    assert np.isnan(Os[0, :, 0]).all()


# ------------------------------------------------------------- input recipe

def test_input_recipe_is_seeded_and_bf16():
    a = make_dense(1, 8, 2, 16, seed=0)
    b = make_dense(1, 8, 2, 16, seed=0)
    for k in a:
        assert a[k].dtype == torch.bfloat16 and a[k].shape == (1, 8, 2, 16)
        assert torch.equal(a[k], b[k])
    c = make_dense(1, 8, 2, 16, seed=0, qk_scale_factor=2.0)
    assert torch.equal(c["q"], a["q"] * 2) and torch.equal(c["k"], a["k"] * 2)
    assert torch.equal(c["v"], a["v"])


def test_varlen_lengths_recipe():
    w = WORKLOADS["varlen_total32768_h32_d128"]
    lens = varlen_lengths(w.varlen_total, w.varlen_lo, w.varlen_hi, 0)
    assert sum(lens) == 32768
    assert all(w.varlen_lo <= L <= w.varlen_hi for L in lens[:-1])
    assert 1 <= lens[-1] <= w.varlen_hi
    cu = cu_seqlens_of(lens)
    assert cu[0] == 0 and cu[-1] == 32768 and cu.dtype == torch.int32
