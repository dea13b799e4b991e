"""The C ABI used from plain C (tests/c_abi/fa_c_smoke.c): it compiles and
links against the library without a GPU, and on a GPU its output is
bitwise equal to the Python binding's on the same inputs (the forward pass
is deterministic)."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import exact_io_aware_95_b200 as fa
from exact_io_aware_95_b200 import build as fabuild

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CUDA = fabuild.cuda_home()


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    fabuild.build()
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    out = str(tmp_path_factory.mktemp("c_abi") / "fa_c_smoke")
    libdir = os.path.dirname(fabuild.LIB_PATH)
    cmd = [cc, "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-o", out, os.path.join(HERE, "c_abi", "fa_c_smoke.c"),
           "-I" + os.path.join(ROOT, "include"), "-I" + os.path.join(CUDA, "include"),
           "-L" + libdir, "-l:libfa_b200.so", "-Wl,-rpath," + libdir,
           "-L" + os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return out


def test_c_program_compiles_and_links(exe):
    assert os.path.exists(exe)


def _inputs(B, N, H, d):
    # the same integer pattern as the C program (exact in float32), rounded to
    # bf16 by torch (round to nearest even, as the C program does)
    n = B * N * H * d
    i = np.arange(n, dtype=np.int64)
    out = []
    for w in range(3):
        k = (i * 7919 + 104729 * w) % 2001
        x = (k - 1000).astype(np.float32) / np.float32(1024.0)
        out.append(torch.from_numpy(x).to(torch.bfloat16).reshape(B, N, H, d))
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("shape,causal", [((1, 128, 2, 64), 0), ((2, 300, 3, 128), 1)])
def test_c_program_matches_binding_bitwise(exe, shape, causal):
    B, N, H, d = shape
    r = subprocess.run([exe, str(B), str(N), str(H), str(d), str(causal)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    vals = r.stdout.split()
    n, nl = B * N * H * d, B * H * N
    o_c = np.array([int(x, 16) for x in vals[:n]], dtype=np.uint16)
    lse_c = np.array([int(x, 16) for x in vals[n:n + nl]], dtype=np.uint32)
    q, k, v = (t.cuda() for t in _inputs(B, N, H, d))
    scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))  # 1.0f / sqrtf(d), as in the C program
    o, lse = fa.fwd(q, k, v, causal=bool(causal), scale=scale)
    assert np.array_equal(o.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1), o_c)
    assert np.array_equal(lse.cpu().view(torch.int32).numpy().view(np.uint32).reshape(-1), lse_c)
