"""Seeded synthetic inputs for exact attention, shared by the tests and the bench.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic.  Both the CPU oracle's callers and the CUDA path's
callers take their inputs from here, so the two see bit-identical bf16 values.

Recipe (the pages print no workload data, so every input is i.i.d. N(0, 1)):

* one ``torch.Generator('cpu')`` seeded with ``seed``; fp32 ``randn`` drawn in
  the order Q, K, V, dO, each then rounded to bf16 (round-to-nearest-even);
* the "softmax range stress" workload multiplies Q and K by 2 after the cast
  (exact in bf16);
* packed variable-length workloads draw their lengths from a second generator
  with the same seed: ``randint(lo, hi + 1)`` until the running sum reaches the
  token total, and the last length is cut so that the lengths sum to the total
  exactly (it may come out shorter than ``lo``; that is kept as an edge case).

Shapes follow the pages' workloads: GPT-style training at 2k-16k context
("FlashAttention-2 (PT)", section "Desempenho e eficiencia"), sequence packing
("Flash Attention", section "Con Sequence Packing").
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Tuple, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_dense", "make_varlen", "varlen_lengths", "cu_seqlens_of",
           "DecodeWorkload", "DECODE_WORKLOADS", "make_decode", "quantize_e4m3", "make_fp8_dense"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    d: int
    causal: tuple          # modes exercised, e.g. (False,) or (False, True)
    backward: bool
    qk_scale_factor: float = 1.0
    varlen_total: int = 0  # >0: packed sequences of this many tokens (B is 1)
    varlen_lo: int = 0
    varlen_hi: int = 0


# The five workloads the path is specified on, by what they are.
WORKLOADS: Dict[str, Workload] = {
    "tiny_fwd_bwd_b1_h2_n128_d64": Workload("tiny_fwd_bwd_b1_h2_n128_d64", 1, 128, 2, 64, (False,), True),
    "fwd_b8_h16_n2048_d64": Workload("fwd_b8_h16_n2048_d64", 8, 2048, 16, 64, (False, True), False),
    "fwd_bwd_causal_b4_h16_n4096_d128_qk2x": Workload(
        "fwd_bwd_causal_b4_h16_n4096_d128_qk2x", 4, 4096, 16, 128, (True,), True, qk_scale_factor=2.0),
    "long_b1_h16_n16384_d128": Workload("long_b1_h16_n16384_d128", 1, 16384, 16, 128, (False, True), True),
    "varlen_total32768_h32_d128": Workload(
        "varlen_total32768_h32_d128", 1, 0, 32, 128, (True,), True,
        varlen_total=32768, varlen_lo=64, varlen_hi=4096),
}


def _draw(gen: torch.Generator, shape, count: int, qk_scale_factor: float):
    out = []
    for i in range(count):
        t = torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)
        if i < 2 and qk_scale_factor != 1.0:
            t = t * qk_scale_factor  # exact for a power of two in bf16
        out.append(t)
    return out


def make_dense(B: int, N: int, H: int, d: int, seed: int = 0, qk_scale_factor: float = 1.0,
               with_grad: bool = True) -> Dict[str, torch.Tensor]:
    """Q, K, V (and dO) as contiguous bf16 CPU tensors of shape [B, N, H, d]."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    names = ["q", "k", "v", "do"] if with_grad else ["q", "k", "v"]
    ts = _draw(gen, (B, N, H, d), len(names), qk_scale_factor)
    return dict(zip(names, ts))


def varlen_lengths(total: int, lo: int, hi: int, seed: int = 0) -> List[int]:
    """Sequence lengths drawn uniformly from [lo, hi], cut to sum to ``total``."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    lens: List[int] = []
    s = 0
    while s < total:
        L = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
        lens.append(L)
        s += L
    lens[-1] = total - (s - lens[-1])
    return lens


def cu_seqlens_of(lengths: List[int]) -> torch.Tensor:
    """Prefix offsets [0, L0, L0+L1, ...] as int32."""
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def make_varlen(lengths: List[int], H: int, d: int, seed: int = 0,
                with_grad: bool = True) -> Dict[str, torch.Tensor]:
    """Packed Q, K, V (and dO) [total, H, d] bf16 plus cu_seqlens (int32)."""
    total = int(sum(lengths))
    gen = torch.Generator(device="cpu").manual_seed(seed)
    names = ["q", "k", "v", "do"] if with_grad else ["q", "k", "v"]
    ts = _draw(gen, (total, H, d), len(names), 1.0)
    out = dict(zip(names, ts))
    out["cu_seqlens"] = cu_seqlens_of(lengths)
    out["lengths"] = list(int(x) for x in lengths)
    return out


def make_workload(w: Workload, seed: int = 0) -> Dict[str, torch.Tensor]:
    if w.varlen_total:
        lens = varlen_lengths(w.varlen_total, w.varlen_lo, w.varlen_hi, seed)
        return make_varlen(lens, w.H, w.d, seed, with_grad=w.backward)
    return make_dense(w.B, w.N, w.H, w.d, seed, w.qk_scale_factor, with_grad=True)


@dataclass(frozen=True)
class DecodeWorkload:
    """Decode-shaped inputs: Nq new queries per batch entry against a cache of
    Nk rows, of which seqlens are valid (all Nk when lo == hi == Nk)."""
    name: str
    B: int
    Nq: int
    Nk: int
    H: int
    d: int
    lo: int
    hi: int


# Serving-style decode: one new token per sequence against a 16k-token cache,
# with every cache full, and with lengths spread over [1024, 16384].
DECODE_WORKLOADS: Dict[str, DecodeWorkload] = {
    "decode_b16_h16_nk16384_d128_full": DecodeWorkload("decode_b16_h16_nk16384_d128_full", 16, 1, 16384, 16, 128,
                                                       16384, 16384),
    "decode_b16_h16_nk16384_d128_ragged": DecodeWorkload("decode_b16_h16_nk16384_d128_ragged", 16, 1, 16384, 16,
                                                         128, 1024, 16384),
}


def make_decode(B: int, Nq: int, Nk: int, H: int, d: int, lo: int, hi: int, seed: int = 0) -> Dict[str, torch.Tensor]:
    """q [B, Nq, H, d], k, v caches [B, Nk, H, d] (bf16, fp32 randn drawn in
    the order q, k, v from one generator), and seqlens int32 [B] drawn
    uniformly from [lo, hi] by a second generator seeded with ``seed``."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((B, Nq, H, d), generator=gen, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((B, Nk, H, d), generator=gen, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((B, Nk, H, d), generator=gen, dtype=torch.float32).to(torch.bfloat16)
    g2 = torch.Generator(device="cpu").manual_seed(seed)
    lens = torch.randint(lo, hi + 1, (B,), generator=g2, dtype=torch.int64).to(torch.int32)
    return {"q": q, "k": k, "v": v, "seqlens": lens}


def quantize_e4m3(x: torch.Tensor) -> Tuple[torch.Tensor, float]:
    """Per-tensor 8-bit input: scale = amax / 448 (the largest finite e4m3
    value) in fp32, and x / scale converted to torch.float8_e4m3fn (round to
    nearest even).  The attention is then taken of scale * result."""
    amax = float(x.float().abs().max())
    scale = amax / 448.0 if amax > 0 else 1.0
    return (x.float() / scale).to(torch.float8_e4m3fn), scale


def make_fp8_dense(B: int, N: int, H: int, d: int, seed: int = 0, qk_scale_factor: float = 1.0):
    """The dense recipe (make_dense, same draws) quantized per tensor to e4m3:
    returns {"q", "k", "v"} e4m3 tensors and {"q", "k", "v"} scales."""
    x = make_dense(B, N, H, d, seed=seed, qk_scale_factor=qk_scale_factor, with_grad=False)
    out, scales = {}, {}
    for n in ("q", "k", "v"):
        out[n], scales[n] = quantize_e4m3(x[n])
    return out, scales
