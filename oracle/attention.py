"""Plain, slow, obviously correct fp64 CPU oracle for exact attention.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import or call this module.  The
product path (the CUDA library and its Python binding) never does, and this
module imports nothing from it: the two share no code.

What it computes, and where that is stated
------------------------------------------
All five pages describe one method: attention computed *exactly* -- the same
result as standard attention -- but without writing the N x N score matrix to
slow GPU memory ("FlashAttention: Fast and Memory-Efficient Exact Attention
with IO-Awareness", sections "En pocas palabras" and "Ideas clave";
"FlashAttention-2 (PT)", opening paragraph; "FlashAttention" (aiunderstanding),
section "Plongee profonde").  Because the method reaches the plain definition
exactly (up to rounding order), this oracle *is* the plain definition written
out, with the full S and P materialised, in float64:

    S = scale * Q K^T                      (N_q x N_k per batch entry and head)
    S_ij = -inf  where causal and j > i    (query i sees key j iff j <= i)
    P = row-softmax(S)
    O = P V
    LSE_i = ln sum_j exp(S_ij)             (natural log, over unmasked j)

The backward pass, for the scalar loss  l = sum(dO * O):

    dV = P^T dO
    dP = dO V^T
    dS_i = J_i dP_i,  J_i = diag(P_i) - P_i P_i^T      (softmax Jacobian, row i)
    dQ = scale * dS K
    dK = scale * dS^T Q

The pages give no equation for the scale, the mask or the logsumexp; they say
only that the result equals standard attention, that the backward pass
recomputes the attention blocks ("Recalcular en vez de guardar"), and that
sequence packing is supported ("Flash Attention", section "Con Sequence
Packing").  The readings taken: scale = 1/sqrt(d) (passed in), causal j <= i,
LSE in natural-log units; a packed batch is a list of independent sequences
given by prefix offsets ``cu_seqlens``; no attention crosses a sequence
boundary.

Inputs are whatever the caller passes (normally bf16 values widened to
float64, so the oracle and the GPU see identical numbers).  Layouts:
dense tensors are [B, N, H, d]; LSE is [B, H, N]; packed tensors are
[total, H, d] with LSE [H, total].
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "scores", "softmax_rows", "softmax_jacobian",
    "attn_head_fwd", "attn_head_bwd",
    "attn_fwd_ref", "attn_bwd_ref",
    "attn_varlen_fwd_ref", "attn_varlen_bwd_ref",
]

NEG_INF = -np.inf


def scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool) -> np.ndarray:
    """S = scale * q k^T with the causal mask as -inf (j > i).  q [Nq, d], k [Nk, d]."""
    S = scale * (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T)
    if causal:
        nq, nk = S.shape
        i = np.arange(nq)[:, None]
        j = np.arange(nk)[None, :]
        S = np.where(j > i, NEG_INF, S)
    return S


def softmax_rows(S: np.ndarray):
    """Row softmax of S and the row logsumexp (natural log).

    Every row must keep at least one finite entry (true for every causal or
    non-causal square problem: query i always sees key 0).
    """
    m = np.max(S, axis=-1, keepdims=True)
    E = np.exp(S - m)
    l = np.sum(E, axis=-1, keepdims=True)
    P = E / l
    lse = (m + np.log(l))[..., 0]
    return P, lse


def softmax_jacobian(p: np.ndarray) -> np.ndarray:
    """The textbook Jacobian d softmax / d s of one row: diag(p) - p p^T."""
    p = np.asarray(p, np.float64)
    return np.diag(p) - np.outer(p, p)


def attn_head_fwd(q, k, v, scale: float, causal: bool):
    """One (batch entry, head): returns O [Nq, d], LSE [Nq], P [Nq, Nk]."""
    S = scores(q, k, scale, causal)
    P, lse = softmax_rows(S)
    O = P @ np.asarray(v, np.float64)
    return O, lse, P


def attn_head_bwd(q, k, v, do, scale: float, causal: bool, explicit_jacobian: bool = False):
    """One (batch entry, head): gradients of sum(dO * O) w.r.t. q, k, v.

    With ``explicit_jacobian`` the N x N Jacobian of each row is built and
    applied (only sensible for tiny N); otherwise the same product is formed
    as P_i * dP_i - P_i (P_i . dP_i), which is that matrix times dP_i written
    out term by term.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    _, _, P = attn_head_fwd(q, k, v, scale, causal)
    dV = P.T @ do
    dP = do @ v.T
    if explicit_jacobian:
        dS = np.stack([softmax_jacobian(P[i]) @ dP[i] for i in range(P.shape[0])])
    else:
        dS = P * dP - P * np.sum(P * dP, axis=-1, keepdims=True)
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q)
    return dQ, dK, dV


def _as64(x):
    return np.asarray(x, np.float64)


def attn_fwd_ref(q, k, v, scale: float, causal: bool, heads=None):
    """Dense forward over [B, N, H, d] inputs.

    Returns O [B, N, H, d] and LSE [B, H, N] (float64).  ``heads`` optionally
    restricts the work to a list of (b, h) pairs; other entries are NaN.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, N, H, d = q.shape
    O = np.full(q.shape, np.nan)
    L = np.full((B, H, N), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        o, lse, _ = attn_head_fwd(q[b, :, h], k[b, :, h], v[b, :, h], scale, causal)
        O[b, :, h] = o
        L[b, h] = lse
    return O, L


def attn_bwd_ref(q, k, v, do, scale: float, causal: bool, heads=None):
    """Dense backward over [B, N, H, d]: returns dQ, dK, dV (float64)."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    B, N, H, d = q.shape
    dQ = np.full(q.shape, np.nan)
    dK = np.full(q.shape, np.nan)
    dV = np.full(q.shape, np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        gq, gk, gv = attn_head_bwd(q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale, causal)
        dQ[b, :, h] = gq
        dK[b, :, h] = gk
        dV[b, :, h] = gv
    return dQ, dK, dV


def _segments(cu_seqlens):
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    return [(cu[s], cu[s + 1]) for s in range(len(cu) - 1)]


def attn_varlen_fwd_ref(q, k, v, cu_seqlens, scale: float, causal: bool, seqs=None, heads=None):
    """Packed forward: q, k, v [total, H, d]; each sequence [cu[s], cu[s+1]) alone.

    Returns O [total, H, d] and LSE [H, total].  ``seqs`` / ``heads`` restrict
    the work (other entries NaN).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    total, H, d = q.shape
    O = np.full(q.shape, np.nan)
    L = np.full((H, total), np.nan)
    segs = _segments(cu_seqlens)
    for s in (seqs if seqs is not None else range(len(segs))):
        a, e = segs[s]
        if e <= a:
            continue
        for h in (heads if heads is not None else range(H)):
            o, lse, _ = attn_head_fwd(q[a:e, h], k[a:e, h], v[a:e, h], scale, causal)
            O[a:e, h] = o
            L[h, a:e] = lse
    return O, L


def attn_varlen_bwd_ref(q, k, v, do, cu_seqlens, scale: float, causal: bool, seqs=None, heads=None):
    """Packed backward: returns dQ, dK, dV [total, H, d]."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    total, H, d = q.shape
    dQ = np.full(q.shape, np.nan)
    dK = np.full(q.shape, np.nan)
    dV = np.full(q.shape, np.nan)
    segs = _segments(cu_seqlens)
    for s in (seqs if seqs is not None else range(len(segs))):
        a, e = segs[s]
        if e <= a:
            continue
        for h in (heads if heads is not None else range(H)):
            gq, gk, gv = attn_head_bwd(q[a:e, h], k[a:e, h], v[a:e, h], do[a:e, h], scale, causal)
            dQ[a:e, h] = gq
            dK[a:e, h] = gk
            dV[a:e, h] = gv
    return dQ, dK, dV
