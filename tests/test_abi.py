"""The C-ABI library loads without a GPU, exports every symbol include/fa.h
declares, and rejects bad arguments on the host (no compute call is made)."""
import ctypes
import os
import re

import pytest

import exact_io_aware_95_b200 as fa
from exact_io_aware_95_b200 import build as fabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    txt = open(os.path.join(ROOT, "include", "fa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def L():
    fabuild.build()
    return fa.lib()


def test_every_declared_symbol_is_exported(L):
    names = header_functions()
    assert "fa_fwd" in names and "fa_varlen_bwd" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(fa.EXPORTS), (names, sorted(fa.EXPORTS))


def test_status_strings(L):
    for s in range(6):
        assert len(fa.status_string(s)) > 0
    assert fa.status_string(99) == "unknown status"


def test_workspace_size(L):
    # fp32 dQ accumulator + fp32 D, each rounded up to 256 bytes
    assert fa.workspace_size(4, 4096, 16, 128) == 4 * 4096 * 16 * 128 * 4 + 4 * 4096 * 16 * 4
    assert fa.workspace_size(1, 3, 1, 64) == 768 + 256
    assert fa.workspace_size(1, 8, 1, 96) == 0
    assert fa.workspace_size(0, 8, 1, 64) == 0


def test_host_validation(L):
    P = 4096  # a 16-byte-aligned fake address; never dereferenced on these paths
    assert L.fa_fwd(None, P, P, P, P, 1, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd(P + 8, P, P, P, P, 1, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd(P, P, P, P, P, 0, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd(P, P, P, P, P, 1, 0, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd(P, P, P, P, P, 1, 8, 1, 64, 1.0, 2, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd(P, P, P, P, P, 1, 8, 1, 64, float("nan"), 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd(P, P, P, P, P, 1, 8, 1, 96, 1.0, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_varlen_fwd(P, P, P, P, P, None, 1, 8, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_varlen_fwd(P, P, P, P, P, P, 0, 8, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    ws = fa.workspace_size(1, 8, 1, 64)
    args = [P] * 10
    assert L.fa_bwd(*args, ws - 1, 1, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_WORKSPACE
    assert L.fa_bwd(*args[:9], P + 16, ws, 1, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG  # ws not 256-aligned
    assert L.fa_bwd(*args, ws, 1, 8, 1, 128, 1.0, 3, None) == fa.FA_ERR_INVALID_ARG
    # the deterministic entry points validate exactly as fa_bwd / fa_varlen_bwd
    assert L.fa_bwd_deterministic(*args, ws - 1, 1, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_WORKSPACE
    assert L.fa_bwd_deterministic(*args, ws, 1, 8, 1, 96, 1.0, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_bwd_deterministic(None, *args[1:], ws, 1, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_varlen_bwd_deterministic(*args, ws, None, 1, 8, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_varlen_bwd_deterministic(*args, ws, P + 2, 1, 8, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    # decode: q, k, v, o, lse, seqlens, workspace, ws_bytes, B, Nq, Nk, H, d, scale, causal, stream
    dws = fa.decode_workspace_size(1, 1, 16384, 1, 128)
    assert dws > 0 and fa.decode_workspace_size(64, 1, 300, 16, 128) > 0
    assert fa.decode_workspace_size(1, 1, 16384, 1, 128) == fa.decode_workspace_size(1, 1, 64, 1, 128)  # not Nk
    assert fa.decode_workspace_size(1, 17, 100, 1, 128) == 0 and fa.decode_workspace_size(1, 1, 100, 1, 96) == 0
    assert L.fa_decode_fwd(P, P, P, P, P, None, None, 0, 1, 17, 64, 1, 64, 1.0, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_decode_fwd(P, P, P, P, P, None, None, 0, 1, 1, 64, 1, 96, 1.0, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_decode_fwd(P, P, P, P, P, P + 2, None, 0, 1, 1, 64, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_decode_fwd(P, P, P, P, P, None, None, 0, 1, 1, 0, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_decode_fwd(None, P, P, P, P, None, None, 0, 1, 1, 64, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_decode_fwd(P, P, P, P, P, None, None, 0, 1, 1, 16384, 1, 128, 1.0, 0, None) == fa.FA_ERR_WORKSPACE
    assert L.fa_decode_fwd(P, P, P, P, P, None, P * 64, dws - 1, 1, 1, 16384, 1, 128, 1.0, 0, None) == \
        fa.FA_ERR_WORKSPACE
    assert L.fa_decode_fwd(P, P, P, P, P, None, P + 16, dws, 1, 1, 16384, 1, 128, 1.0, 0, None) == \
        fa.FA_ERR_INVALID_ARG  # workspace not 256-aligned
    assert L.fa_decode_fwd(P, P, P, P, P, None, None, 0, 65536, 1, 64, 1, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_decode_fwd(P, P, P, P, P, None, None, 0, 1, 1, 64, 65536, 64, 1.0, 0, None) == fa.FA_ERR_INVALID_ARG


@pytest.mark.skipif(os.path.exists("/dev/nvidia0"), reason="host without a GPU driver only")
def test_compute_call_without_gpu_reports_cuda_error(L):
    P = 4096
    assert L.fa_fwd(P, P, P, P, P, 1, 8, 1, 64, 1.0, 0, None) == fa.FA_ERR_CUDA


def test_launch_event_hook_validates_on_the_host(L):
    import ctypes
    assert L.fa_record_launch_events(None, 1) == fa.FA_ERR_INVALID_ARG
    arr = (ctypes.c_void_p * 2)(4096, 0)
    assert L.fa_record_launch_events(arr, 2) == fa.FA_ERR_INVALID_ARG   # null entry
    assert L.fa_record_launch_events(arr, 0) == fa.FA_ERR_INVALID_ARG
    assert L.fa_record_launch_events(arr, 9) == fa.FA_ERR_INVALID_ARG
