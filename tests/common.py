"""Shared helpers for the parity tests: run the CUDA path, run the oracle on the
same seeded inputs, and compare with the tolerances of the specification:
O max-abs <= 2e-2, LSE max-abs <= 1e-3, dQ/dK/dV relative Frobenius <= 5e-2."""
import math

import numpy as np
import torch

O_ATOL = 2e-2
LSE_ATOL = 1e-3
GRAD_RTOL_FRO = 5e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


GRAD_ATOL_WHEN_ZERO = 1e-3


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    """Relative Frobenius error.  Where the exact gradient is identically zero
    (a single key: softmax of one entry has zero derivative) the ratio is
    undefined; there the error is the max-abs deviation scaled so that the
    same 5e-2 bar means max|a| <= 1e-3."""
    nb = float(np.linalg.norm(b))
    if nb == 0.0:
        return float(np.max(np.abs(a))) * (5e-2 / GRAD_ATOL_WHEN_ZERO) if a.size else 0.0
    return float(np.linalg.norm(a - b) / nb)


def max_abs(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def scale_of(d: int) -> float:
    return 1.0 / math.sqrt(d)


def cuda(x: dict) -> dict:
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


# ---------------------------------------------------------------- full-size parity
# The oracle handles one (batch entry, head) -- or one packed sequence and head
# -- at a time with full N x N matrices.  At full sizes every head is run,
# several at once: NumPy releases the GIL inside its array operations, so a
# thread pool spreads the heads over the host cores.

def oracle_workers(n_items: int, mem_per_item: float) -> int:
    """Threads for the oracle: bounded by the host cores and by host memory
    (each item materialises a few N x N float64 matrices)."""
    import os
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    try:
        avail = os.sysconf("SC_AVPHYS_PAGES") * os.sysconf("SC_PAGE_SIZE")
    except Exception:
        avail = 16 << 30
    by_mem = max(1, int(0.5 * avail // max(mem_per_item, 1.0)))
    return max(1, min(n_items, cores, by_mem, 16))


def oracle_per_head(slices, scale: float, causal: bool, grads: bool):
    """Run the oracle on every item of `slices`: a list of (key, q, k, v, do)
    with q, k, v, do as [L, d] float64 arrays of one head.  Returns
    {key: (O, LSE, dQ, dK, dV)} (gradients None without `grads`)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    def one(item):
        key, q, k, v, do = item
        o, lse, _ = oracle.attn_head_fwd(q, k, v, scale, causal)
        g = oracle.attn_head_bwd(q, k, v, do, scale, causal) if grads else (None, None, None)
        return key, (o, lse) + tuple(g)

    if not slices:
        return {}
    L = max(s[1].shape[0] for s in slices)
    workers = oracle_workers(len(slices), 8.0 * L * L * 8)
    with ThreadPoolExecutor(workers) as ex:
        return dict(ex.map(one, slices))


class Agg:
    """Accumulates errors over heads: O and LSE max-abs, and per gradient the
    relative Frobenius error of the whole tensor (sum of squared differences
    over sum of squared references) plus the worst single head."""

    def __init__(self):
        self.eo = 0.0
        self.el = 0.0
        self.num = [0.0, 0.0, 0.0]
        self.den = [0.0, 0.0, 0.0]
        self.worst_head = [0.0, 0.0, 0.0]

    def fwd(self, o, O, lse, LSE):
        self.eo = max(self.eo, max_abs(o, O))
        self.el = max(self.el, max_abs(lse, LSE))

    def bwd(self, got, ref):
        for i, (a, b) in enumerate(zip(got, ref)):
            self.num[i] += float(np.sum((a - b) ** 2))
            self.den[i] += float(np.sum(b ** 2))
            self.worst_head[i] = max(self.worst_head[i], rel_fro(a, b))

    def grads(self):
        return [math.sqrt(n / d) if d > 0 else math.sqrt(n) for n, d in zip(self.num, self.den)]


def nan_like(t):
    import torch
    return torch.full_like(t, float("nan"))
