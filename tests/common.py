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
