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


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def max_abs(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def scale_of(d: int) -> float:
    return 1.0 / math.sqrt(d)


def cuda(x: dict) -> dict:
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
