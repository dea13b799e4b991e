"""In-tree build of the CUDA library (sm_100a only).

``build()`` compiles ``csrc/fa_api.cu`` (which includes every kernel) into
``libfa_b200.so`` next to this file.  The CUDA runtime is linked statically
and the driver is reached through the runtime's entry-point query, so the
library loads on a machine without a GPU driver (its compute calls then
return FA_ERR_CUDA).
"""
from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libfa_b200.so")
SOURCES = [os.path.join(HERE, "csrc", "fa_api.cu")]
DEPS = [os.path.join(HERE, "csrc", f) for f in ("fa_api.cu", "fa_fwd.cuh", "fa_bwd.cuh", "sm100_ptx.cuh")] + [
    os.path.join(ROOT, "include", "fa.h")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB_PATH, defines=()) -> list:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"), "-o", out]
    cmd += ["-D" + d for d in defines]
    return cmd + SOURCES


def up_to_date(out: str = LIB_PATH) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, out: str = LIB_PATH, defines=()) -> str:
    if not force and not defines and up_to_date(out):
        return out
    cmd = command(out, defines)
    if verbose:
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose=True))
