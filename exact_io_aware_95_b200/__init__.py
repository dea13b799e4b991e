"""Python binding of the sm_100a exact-attention library (``libfa_b200.so``).

Argument marshalling only: every step of the forward and backward pass runs
in the library's CUDA kernels.  Torch provides device memory and the current
stream.  There is no CPU or library fallback: if the compiled library is
missing, importing any entry point raises.

Layouts (see include/fa.h): dense tensors bf16 [B, N, H, d], LSE fp32
[B, H, N]; packed tensors bf16 [total, H, d], LSE fp32 [H, total],
cu_seqlens int32 [nseq + 1] on the device.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

__all__ = ["FaError", "lib", "fwd", "bwd", "varlen_fwd", "varlen_bwd", "workspace_size", "check_device_error",
           "decode_fwd", "decode_workspace_size", "fwd_fp8", "fwd_fp8_workspace_size", "record_launch_events",
           "FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA", "FA_ERR_TIMEOUT", "FA_ERR_WORKSPACE",
           "EXPORTS", "LIB_PATH"]

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_WORKSPACE = range(6)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/fa.h
EXPORTS = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_varlen_fwd": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_workspace_size": (_S, [_I, _I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _I, _I, _I, _I, _F, _I, _P]),
    "fa_varlen_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_deterministic": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _I, _I, _I, _I, _F, _I, _P]),
    "fa_varlen_bwd_deterministic": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P, _I, _I, _I, _I, _I, _F, _I,
                                         _P]),
    "fa_decode_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "fa_fwd_fp8_workspace_size": (_S, [_I, _I, _I, _I]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _F, _F, _F, _P, _P, _P, _S, _I, _I, _I, _I, _F, _I, _P]),
    "fa_decode_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _S, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_record_launch_events": (_I, [ctypes.POINTER(ctypes.c_void_p), _I]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_get_device_error": (_I, [_P]),
}


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def lib(path: Optional[str] = None):
    """Load the compiled library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"CUDA library {p} is missing; build it with exact_io_aware_95_b200.build.build()")
    L = ctypes.CDLL(p)
    for name, (res, args) in EXPORTS.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    if path is None:
        _lib = L
    return L


def status_string(s: int) -> str:
    return lib().fa_status_string(int(s)).decode()


def _check(status: int, where: str):
    if status != FA_OK:
        raise FaError(status, where)


def _stream_ptr(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _on(t: torch.Tensor):
    """Make the tensors' device current for the call: the library launches on
    the calling thread's current device and stream."""
    return torch.cuda.device(t.device)


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need_shape(t, name: str, dtype, shape):
    """`t` must be a contiguous tensor of `dtype` and exactly `shape`:
    the kernels index every buffer from the sizes of q, so a smaller one
    would be read or written past its end."""
    _need(t, name, dtype, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _need_workspace(ws, need: int):
    if not isinstance(ws, torch.Tensor):
        raise TypeError("workspace must be a torch.Tensor")
    if not ws.is_contiguous():
        raise ValueError("workspace must be contiguous")
    if ws.numel() * ws.element_size() < need:
        raise FaError(FA_ERR_WORKSPACE, f"workspace of {ws.numel() * ws.element_size()} bytes < {need} needed")


def _same_device(*ts):
    """Every tensor on one CUDA device (checked after dtypes and shapes, right
    before the call)."""
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda:
            raise ValueError(f"all tensors must be on a CUDA device; got one on {t.device}")
        if t.device != dev:
            raise ValueError(f"all tensors must be on {dev}; got one on {t.device}")


def _scale(scale: Optional[float], d: int) -> float:
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def workspace_size(B: int, N: int, H: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_size(B, N, H, d))


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, scale: Optional[float] = None,
        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """O, LSE = attention(q, k, v) for dense [B, N, H, d] bf16 inputs."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 4)
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, N, H, d]")
    B, N, H, d = q.shape
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _need_shape(o, "out", torch.bfloat16, q.shape)
    _need_shape(l, "lse", torch.float32, (B, H, N))
    _same_device(q, k, v, o, l)
    with _on(q):
        st = lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), B, N, H, d,
                          _scale(scale, d), int(bool(causal)), _stream_ptr(q))
    _check(st, "fa_fwd")
    return o, l


def bwd(q, k, v, o, lse, do, causal: bool = False, scale: Optional[float] = None,
        workspace: Optional[torch.Tensor] = None, dq=None, dk=None, dv=None, deterministic: bool = False):
    """dQ, dK, dV for dense [B, N, H, d] inputs (o, lse from fwd).

    deterministic=True: bitwise reproducible gradients (fa_bwd_deterministic:
    dQ summed in a fixed order by a second pass instead of fp32 atomics)."""
    _need(q, "q", torch.bfloat16, 4)
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _need_shape(t, n, torch.bfloat16, q.shape)
    B, N, H, d = q.shape
    _need_shape(lse, "lse", torch.float32, (B, H, N))
    ws_need = workspace_size(B, N, H, d)
    ws = torch.empty(ws_need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need_shape(t, n, torch.bfloat16, q.shape)
    _need_workspace(ws, ws_need)
    _same_device(q, k, v, o, lse, do, ws, dq, dk, dv)
    with _on(q):
        fn = lib().fa_bwd_deterministic if deterministic else lib().fa_bwd
        st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                B, N, H, d, _scale(scale, d), int(bool(causal)), _stream_ptr(q))
    _check(st, "fa_bwd_deterministic" if deterministic else "fa_bwd")
    return dq, dk, dv


def varlen_fwd(q, k, v, cu_seqlens: torch.Tensor, max_seqlen: int, causal: bool = False,
               scale: Optional[float] = None, out=None, lse=None):
    """Packed forward: q, k, v [total, H, d]; returns O [total, H, d], LSE [H, total]."""
    _need(q, "q", torch.bfloat16, 3)
    for t, n in ((k, "k"), (v, "v")):
        _need_shape(t, n, torch.bfloat16, q.shape)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    total, H, d = q.shape
    nseq = cu_seqlens.numel() - 1
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((H, total), dtype=torch.float32, device=q.device) if lse is None else lse
    _need_shape(o, "out", torch.bfloat16, q.shape)
    _need_shape(l, "lse", torch.float32, (H, total))
    _same_device(q, k, v, o, l, cu_seqlens)
    with _on(q):
        st = lib().fa_varlen_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                                 cu_seqlens.data_ptr(), nseq, total, int(max_seqlen), H, d, _scale(scale, d),
                                 int(bool(causal)), _stream_ptr(q))
    _check(st, "fa_varlen_fwd")
    return o, l


def varlen_bwd(q, k, v, o, lse, do, cu_seqlens: torch.Tensor, max_seqlen: int, causal: bool = False,
               scale: Optional[float] = None, workspace=None, dq=None, dk=None, dv=None, deterministic: bool = False):
    """Packed backward; deterministic=True as for bwd (fa_varlen_bwd_deterministic)."""
    _need(q, "q", torch.bfloat16, 3)
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _need_shape(t, n, torch.bfloat16, q.shape)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    total, H, d = q.shape
    _need_shape(lse, "lse", torch.float32, (H, total))
    nseq = cu_seqlens.numel() - 1
    ws_need = workspace_size(1, total, H, d)
    ws = torch.empty(ws_need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need_shape(t, n, torch.bfloat16, q.shape)
    _need_workspace(ws, ws_need)
    _same_device(q, k, v, o, lse, do, cu_seqlens, ws, dq, dk, dv)
    with _on(q):
        fn = lib().fa_varlen_bwd_deterministic if deterministic else lib().fa_varlen_bwd
        st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                cu_seqlens.data_ptr(), nseq, total, int(max_seqlen), H, d, _scale(scale, d), int(bool(causal)),
                _stream_ptr(q))
    _check(st, "fa_varlen_bwd_deterministic" if deterministic else "fa_varlen_bwd")
    return dq, dk, dv


def fwd_fp8_workspace_size(B: int, N: int, H: int, d: int) -> int:
    return int(lib().fa_fwd_fp8_workspace_size(B, N, H, d))


def fwd_fp8(q, k, v, descale_q: float, descale_k: float, descale_v: float, causal: bool = False,
            scale: Optional[float] = None, out=None, lse=None, workspace=None):
    """Forward with e4m3 inputs [B, N, H, 128] (torch.float8_e4m3fn): attention of
    descale_q*q, descale_k*k, descale_v*v.  Returns O bf16 [B, N, H, 128], LSE [B, H, N]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.float8_e4m3fn, 4)
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, N, H, d]")
    B, N, H, d = q.shape
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    ws = workspace
    if ws is None:
        ws = torch.empty(max(fwd_fp8_workspace_size(B, N, H, d), 256), dtype=torch.uint8, device=q.device)
    _need_shape(o, "out", torch.bfloat16, q.shape)
    _need_shape(l, "lse", torch.float32, (B, H, N))
    _need_workspace(ws, fwd_fp8_workspace_size(B, N, H, d))
    _same_device(q, k, v, o, l, ws)
    with _on(q):
        st = lib().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(descale_q), float(descale_k),
                              float(descale_v), o.data_ptr(), l.data_ptr(), ws.data_ptr(),
                              ws.numel() * ws.element_size(), B, N, H, d, _scale(scale, d), int(bool(causal)),
                              _stream_ptr(q))
    _check(st, "fa_fwd_fp8")
    return o, l


def decode_workspace_size(B: int, Nq: int, Nk: int, H: int, d: int) -> int:
    return int(lib().fa_decode_workspace_size(B, Nq, Nk, H, d))


def decode_fwd(q, k_cache, v_cache, seqlens_k: Optional[torch.Tensor] = None, causal: bool = False,
               scale: Optional[float] = None, out=None, lse=None, workspace=None):
    """Decode-shaped forward: q [B, Nq, H, d] (Nq <= 16) against caches
    [B, Nk, H, d] with seqlens_k int32 [B] valid rows per entry (None: all).
    Returns O [B, Nq, H, d] bf16 and LSE [B, H, Nq] fp32."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    B, Nq, H, d = q.shape
    Nk = k_cache.shape[1]
    if k_cache.shape != (B, Nk, H, d) or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must be [B, Nk, H, d] matching q")
    if seqlens_k is not None:
        _need(seqlens_k, "seqlens_k", torch.int32, 1)
        if seqlens_k.numel() != B:
            raise ValueError("seqlens_k must have B entries")
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _need_shape(o, "out", torch.bfloat16, q.shape)
    _need_shape(l, "lse", torch.float32, (B, H, Nq))
    ws_need = decode_workspace_size(B, Nq, Nk, H, d)
    ws = workspace
    if ws is None and ws_need > 0:
        ws = torch.empty(ws_need, dtype=torch.uint8, device=q.device)
    if ws is not None:
        _need_workspace(ws, ws_need)
    ts = [q, k_cache, v_cache, o, l] + [t for t in (seqlens_k, ws) if t is not None]
    _same_device(*ts)
    with _on(q):
        st = lib().fa_decode_fwd(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), o.data_ptr(), l.data_ptr(),
                                 None if seqlens_k is None else seqlens_k.data_ptr(),
                                 None if ws is None else ws.data_ptr(),
                                 0 if ws is None else ws.numel() * ws.element_size(),
                                 B, Nq, Nk, H, d, _scale(scale, d), int(bool(causal)), _stream_ptr(q))
    _check(st, "fa_decode_fwd")
    return o, l


def record_launch_events(events):
    """Measurement hook: the next library call made by this thread records the
    given torch.cuda.Event objects on its stream, events[0] before its first
    kernel launch and events[i] after its i-th launch.  Each event must have
    been recorded once already (so that torch has created it)."""
    handles = [int(e.cuda_event) for e in events]
    if not all(handles):
        raise ValueError("record each event once before passing it (torch creates events lazily)")
    arr = (ctypes.c_void_p * len(handles))(*handles)
    _check(lib().fa_record_launch_events(arr, len(handles)), "fa_record_launch_events")


def check_device_error(stream: Optional[torch.cuda.Stream] = None):
    """Synchronise the stream and raise if a kernel gave up on a bounded wait."""
    s = (stream or torch.cuda.current_stream()).cuda_stream
    _check(lib().fa_get_device_error(s), "fa_get_device_error")


from .autograd import attention, varlen_attention, pack, unpack  # noqa: E402

__all__ += ["attention", "varlen_attention", "pack", "unpack"]
