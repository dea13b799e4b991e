"""Pins of the decode oracle (oracle/decode.py), CPU only.

Each pin ties the decode definition to something other than itself: the
KV-cache identity with the dense causal oracle (itself pinned in
test_oracle.py), torch's float64 SDPA for rectangular non-causal problems,
closed forms, truncation by seqlens, fully masked rows, and scalar loops."""
import math

import numpy as np
import pytest
import torch

import oracle


def rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("nq,L", [(1, 37), (4, 50), (16, 16), (7, 130)])
def test_kv_cache_identity_with_dense_causal(nq, L):
    """Decoding the last nq tokens of a length-L sequence reproduces the last
    nq rows of the dense causal attention over the whole sequence."""
    r = rng(nq * 100 + L)
    B, H, d = 2, 3, 8
    q = r.standard_normal((B, L, H, d))
    k = r.standard_normal((B, L, H, d))
    v = r.standard_normal((B, L, H, d))
    s = 1 / math.sqrt(d)
    O_full, lse_full = oracle.attn_fwd_ref(q, k, v, s, True)
    O, lse = oracle.attn_decode_ref(q[:, L - nq:], k, v, None, s, True)
    assert np.allclose(O, O_full[:, L - nq:], atol=1e-12, rtol=0)
    assert np.allclose(lse, lse_full[:, :, L - nq:], atol=1e-12, rtol=0)


@pytest.mark.parametrize("nq,nk", [(1, 64), (3, 33), (16, 5)])
def test_noncausal_matches_torch_sdpa_float64(nq, nk):
    r = rng(nq + 7 * nk)
    B, H, d = 2, 2, 16
    q = r.standard_normal((B, nq, H, d))
    k = r.standard_normal((B, nk, H, d))
    v = r.standard_normal((B, nk, H, d))
    s = 0.37
    O, lse = oracle.attn_decode_ref(q, k, v, None, s, False)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)  # [B, H, N, d]
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=s)
    assert np.allclose(O, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12, rtol=0)
    S = torch.einsum("bhqd,bhkd->bhqk", t(q), t(k)) * s
    assert np.allclose(lse, torch.logsumexp(S, dim=-1).numpy(), atol=1e-12, rtol=0)


def test_seqlens_truncate_the_cache():
    r = rng(3)
    B, nq, nk, H, d = 3, 2, 40, 2, 8
    q = r.standard_normal((B, nq, H, d))
    k = r.standard_normal((B, nk, H, d))
    v = r.standard_normal((B, nk, H, d))
    lens = [40, 9, 23]
    O, lse = oracle.attn_decode_ref(q, k, v, lens, 0.3, True)
    for b, L in enumerate(lens):
        Ob, lb = oracle.attn_decode_ref(q[b:b + 1], k[b:b + 1, :L], v[b:b + 1, :L], None, 0.3, True)
        assert np.array_equal(O[b:b + 1], Ob) and np.array_equal(lse[b:b + 1], lb)
    # garbage past the valid length changes nothing
    k2, v2 = k.copy(), v.copy()
    k2[1, 9:] = 1e30
    v2[1, 9:] = np.nan
    O2, lse2 = oracle.attn_decode_ref(q, k2, v2, lens, 0.3, True)
    assert np.array_equal(O2, O) and np.array_equal(lse2, lse)


def test_fully_masked_rows_are_zero_with_minus_inf_lse():
    """Causal with L < nq: the first nq - L queries sit before the first key."""
    r = rng(4)
    nq, L, d = 5, 2, 4
    q = r.standard_normal((1, nq, 1, d))
    k = r.standard_normal((1, L, 1, d))
    v = r.standard_normal((1, L, 1, d))
    O, lse = oracle.attn_decode_ref(q, k, v, None, 0.5, True)
    assert np.all(O[0, :nq - L] == 0) and np.all(np.isneginf(lse[0, 0, :nq - L]))
    # query nq-L sits at position 0: sees key 0 only
    assert np.allclose(O[0, nq - L, 0], v[0, 0, 0]) and np.isclose(lse[0, 0, nq - L], 0.5 * q[0, nq - L, 0] @ k[0, 0, 0])
    assert np.all(np.isfinite(lse[0, 0, nq - L:]))


def test_single_query_causal_equals_noncausal():
    r = rng(5)
    q = r.standard_normal((2, 1, 3, 8))
    k = r.standard_normal((2, 21, 3, 8))
    v = r.standard_normal((2, 21, 3, 8))
    a = oracle.attn_decode_ref(q, k, v, [21, 6], 0.4, True)
    b = oracle.attn_decode_ref(q, k, v, [21, 6], 0.4, False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_identical_keys_closed_form():
    r = rng(6)
    L, d = 17, 8
    q = r.standard_normal((1, 1, 1, d))
    k = np.tile(r.standard_normal(d), (1, L, 1, 1)).reshape(1, L, 1, d)
    v = r.standard_normal((1, L, 1, d))
    O, lse = oracle.attn_decode_ref(q, k, v, None, 0.25, False)
    assert np.allclose(O[0, 0, 0], v[0, :, 0].mean(axis=0), atol=1e-13)
    assert np.isclose(lse[0, 0, 0], 0.25 * q[0, 0, 0] @ k[0, 0, 0] + math.log(L), atol=1e-13)


def _brute(q, k, v, L, scale, causal):
    nq, d = len(q), len(q[0])
    O = [[0.0] * d for _ in range(nq)]
    lse = [0.0] * nq
    for i in range(nq):
        last = (L - nq + i) if causal else (L - 1)
        if last < 0:
            lse[i] = -math.inf
            continue
        s = [scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in range(last + 1)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        tot = sum(e)
        for c in range(d):
            O[i][c] = sum(e[j] * v[j][c] for j in range(last + 1)) / tot
        lse[i] = m + math.log(tot)
    return O, lse


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_loops(causal):
    r = rng(7 + causal)
    nq, L, d = 3, 6, 4
    q = r.standard_normal((nq, d))
    k = r.standard_normal((L, d))
    v = r.standard_normal((L, d))
    O, lse = oracle.decode_head_fwd(q, k, v, 0.6, causal)
    Ob, lb = _brute(q.tolist(), k.tolist(), v.tolist(), L, 0.6, causal)
    assert np.allclose(O, np.array(Ob), atol=1e-13)
    assert np.allclose(lse, np.array(lb), atol=1e-13)
