"""Autograd entry points over the C ABI, and packing helpers.

The step directly above the fused kernels that the pages show users calling:
a training loop switches its attention to FlashAttention ("Flash Attention"
(docs.monostate.ai), section "Parametros": use_flash_attention_2 /
attn_implementation) and packs variable-length sequences into one batch
(section "Con Sequence Packing").  ``attention`` and ``varlen_attention`` are
differentiable torch functions whose forward and backward are the library's
fa_fwd / fa_bwd (dense) and fa_varlen_fwd / fa_varlen_bwd (packed); ``pack``
and ``unpack`` build and split the packed layout.  No other attention
backend is consulted: these functions only call the CUDA library.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import bwd as _bwd
from . import fwd as _fwd
from . import varlen_bwd as _varlen_bwd
from . import varlen_fwd as _varlen_fwd

__all__ = ["attention", "varlen_attention", "pack", "unpack"]


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal: bool, scale: Optional[float], deterministic: bool):
        o, lse = _fwd(q, k, v, causal=causal, scale=scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale, ctx.deterministic = causal, scale, deterministic
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = _bwd(q, k, v, o, lse, do.contiguous(), causal=ctx.causal, scale=ctx.scale,
                          deterministic=ctx.deterministic)
        return dq, dk, dv, None, None, None


class _VarlenAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, cu_seqlens, max_seqlen: int, causal: bool, scale: Optional[float],
                deterministic: bool):
        o, lse = _varlen_fwd(q, k, v, cu_seqlens, max_seqlen, causal=causal, scale=scale)
        ctx.save_for_backward(q, k, v, o, lse, cu_seqlens)
        ctx.max_seqlen, ctx.causal, ctx.scale, ctx.deterministic = max_seqlen, causal, scale, deterministic
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, cu = ctx.saved_tensors
        dq, dk, dv = _varlen_bwd(q, k, v, o, lse, do.contiguous(), cu, ctx.max_seqlen, causal=ctx.causal,
                                 scale=ctx.scale, deterministic=ctx.deterministic)
        return dq, dk, dv, None, None, None, None, None


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
              scale: Optional[float] = None, deterministic: bool = False) -> torch.Tensor:
    """Exact attention over dense bf16 [B, N, H, d] tensors; differentiable in q, k, v.
    deterministic=True makes the gradients bitwise reproducible."""
    return _Attention.apply(q, k, v, bool(causal), scale, bool(deterministic))


def varlen_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                     max_seqlen: int, causal: bool = False, scale: Optional[float] = None,
                     deterministic: bool = False) -> torch.Tensor:
    """Exact attention over a packed batch ([total, H, d], cu_seqlens int32 on the device);
    every sequence attends only to itself.  Differentiable in q, k, v."""
    return _VarlenAttention.apply(q, k, v, cu_seqlens, int(max_seqlen), bool(causal), scale, bool(deterministic))


def pack(seqs: Sequence[torch.Tensor]) -> Tuple[torch.Tensor, torch.Tensor, int]:
    """Concatenate [L_s, H, d] tensors into one [total, H, d] tensor.

    Returns (packed, cu_seqlens int32 on the same device, max_seqlen).  Empty
    sequences are allowed and occupy no rows."""
    if len(seqs) == 0:
        raise ValueError("pack needs at least one sequence")
    shape = seqs[0].shape[1:]
    for s in seqs:
        if s.dim() != 3 or s.shape[1:] != shape:
            raise ValueError("every sequence must be [L, H, d] with the same H and d")
    lengths = [int(s.shape[0]) for s in seqs]
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    packed = torch.cat(list(seqs), dim=0).contiguous()
    return packed, torch.tensor(cu, dtype=torch.int32, device=packed.device), max(lengths)


def unpack(packed: torch.Tensor, cu_seqlens: torch.Tensor) -> List[torch.Tensor]:
    """Split a [total, ...] tensor back into its sequences (views)."""
    cu = [int(x) for x in cu_seqlens.tolist()]
    return [packed[cu[i]:cu[i + 1]] for i in range(len(cu) - 1)]
