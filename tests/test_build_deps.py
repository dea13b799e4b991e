"""The in-tree build notices an edit to any file the library is compiled
from, so the GPU tests never run on a stale libfa_b200.so.  CPU only."""
import os
import shutil

import pytest

from exact_io_aware_95_b200 import build as fabuild


def test_every_kernel_source_is_a_dependency():
    csrc = os.path.join(fabuild.HERE, "csrc")
    deps = set(fabuild.deps())
    for f in os.listdir(csrc):
        if f.endswith((".cu", ".cuh", ".h")):
            assert os.path.join(csrc, f) in deps, f
    assert os.path.join(fabuild.ROOT, "include", "fa.h") in deps


@pytest.mark.parametrize("edited", ["fa_decode.cuh", "fa_bwd_dq.cuh", "fa_fwd_fp8.cuh", "fa_api.cu"])
def test_touching_one_source_makes_the_library_stale(tmp_path, monkeypatch, edited):
    # a copy of the sources with controlled modification times
    here = tmp_path / "pkg"
    shutil.copytree(os.path.join(fabuild.HERE, "csrc"), here / "csrc")
    shutil.copytree(os.path.join(fabuild.ROOT, "include"), tmp_path / "include")
    monkeypatch.setattr(fabuild, "HERE", str(here))
    monkeypatch.setattr(fabuild, "ROOT", str(tmp_path))
    out = tmp_path / "lib.so"
    out.write_bytes(b"")
    t0 = 1_000_000_000
    for f in fabuild.deps():
        os.utime(f, (t0, t0))
    os.utime(out, (t0 + 10, t0 + 10))
    assert fabuild.up_to_date(str(out))
    os.utime(here / "csrc" / edited, (t0 + 20, t0 + 20))
    assert not fabuild.up_to_date(str(out))


def test_cuda_home_holds_nvcc():
    assert os.path.exists(fabuild.nvcc())
    assert os.path.isdir(os.path.join(fabuild.cuda_home(), "include"))
