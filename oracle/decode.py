"""fp64 CPU oracle for decode-shaped exact attention -- TEST INFRASTRUCTURE ONLY.

Only the tests and the bench's CPU baseline may import this module; it
imports nothing from the CUDA library or its binding.

The shape: a few new queries (N_q, often 1) attend to the keys and values
of a sequence already held in a cache of up to N_k rows, of which the first
L_b are valid for batch entry b.  The pages name this inference workload
only through the decoding systems they list next to FlashAttention
("FlashAttention-2 (PT)", section "Literatura": FlashDecoding++,
PagedAttention); the arithmetic is the plain attention definition of
"FlashAttention: Fast and Memory-Efficient Exact Attention with
IO-Awareness" (section "En pocas palabras": the result equals standard
attention), written out in float64 with the full score rows:

    S_ij = scale * q_i . k_j             j < L_b
    causal: query i is the token at position L_b - N_q + i of the sequence
            and sees key j iff j <= L_b - N_q + i
    O_i  = sum_j softmax(S_i)_j v_j,    LSE_i = ln sum_j exp(S_ij)

A query that sees no key (causal with L_b < N_q) has O_i = 0 and
LSE_i = -inf.  Layouts: q, o [B, N_q, H, d]; k, v caches [B, N_k, H, d];
LSE [B, H, N_q]; seqlens_k gives L_b (all N_k when omitted).
"""
from __future__ import annotations

import numpy as np

__all__ = ["decode_head_fwd", "attn_decode_ref"]


def decode_head_fwd(q, k, v, scale: float, causal: bool):
    """One (batch entry, head): q [N_q, d] against the L valid cache rows k, v
    [L, d].  Returns O [N_q, d] and LSE [N_q] (float64)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, L = q.shape[0], k.shape[0]
    S = scale * (q @ k.T)
    if causal:
        pos = (L - nq + np.arange(nq))[:, None]  # absolute position of each query
        S = np.where(np.arange(L)[None, :] > pos, -np.inf, S)
    O = np.zeros((nq, v.shape[1]))
    lse = np.full(nq, -np.inf)
    for i in range(nq):
        row = S[i]
        if not np.any(np.isfinite(row)):
            continue  # sees no key
        m = np.max(row)
        e = np.exp(row - m)
        s = np.sum(e)
        O[i] = (e / s) @ v
        lse[i] = m + np.log(s)
    return O, lse


def attn_decode_ref(q, k_cache, v_cache, seqlens_k, scale: float, causal: bool, heads=None):
    """Decode forward over q [B, N_q, H, d] and caches [B, N_k, H, d].

    Returns O [B, N_q, H, d] and LSE [B, H, N_q].  ``heads`` optionally
    restricts the work to (b, h) pairs (other entries NaN)."""
    q = np.asarray(q, np.float64)
    k_cache = np.asarray(k_cache, np.float64)
    v_cache = np.asarray(v_cache, np.float64)
    B, nq, H, d = q.shape
    nk = k_cache.shape[1]
    lens = [nk] * B if seqlens_k is None else [int(x) for x in np.asarray(seqlens_k).reshape(-1)]
    O = np.full(q.shape, np.nan)
    LSE = np.full((B, H, nq), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        L = lens[b]
        o, lse = decode_head_fwd(q[b, :, h], k_cache[b, :L, h], v_cache[b, :L, h], scale, causal)
        O[b, :, h] = o
        LSE[b, h] = lse
    return O, LSE
