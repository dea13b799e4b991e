"""In-tree build of the CUDA library (sm_100a only).

``build()`` compiles ``csrc/fa_api.cu`` (which includes every kernel) into
``libfa_b200.so`` next to this file.  The CUDA runtime is linked statically
and the driver is reached through the runtime's entry-point query, so the
library loads on a machine without a GPU driver (its compute calls then
return FA_ERR_CUDA).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libfa_b200.so")
SOURCES = [os.path.join(HERE, "csrc", "fa_api.cu")]


def deps() -> list:
    """Every file the library is compiled from: all sources under csrc/ and
    the public header (sorted, so hashes over the list are stable)."""
    files = glob.glob(os.path.join(HERE, "csrc", "*.cu")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh"))
    files += glob.glob(os.path.join(HERE, "csrc", "*.h")) + [os.path.join(ROOT, "include", "fa.h")]
    return sorted(set(files))


def cuda_home() -> str:
    """The CUDA toolkit root: $CUDA_HOME / $CUDA_PATH, else the directory above
    the bin/ that holds the nvcc on PATH."""
    for var in ("CUDA_HOME", "CUDA_PATH"):
        p = os.environ.get(var)
        if p and os.path.exists(os.path.join(p, "bin", "nvcc")):
            return p
    n = shutil.which("nvcc")
    if n:
        return os.path.dirname(os.path.dirname(os.path.realpath(n)))
    raise RuntimeError("nvcc not found (set CUDA_HOME or put nvcc on PATH)")


def nvcc() -> str:
    return os.path.join(cuda_home(), "bin", "nvcc")


def command(out: str = LIB_PATH, defines=(), sources=None) -> list:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"), "-o", out]
    cmd += ["-D" + d for d in defines]
    return cmd + list(sources or SOURCES)


def up_to_date(out: str = LIB_PATH, extra=()) -> bool:
    """The library at `out` is newer than every source (and `extra` file)."""
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in deps() + list(extra))


def build(force: bool = False, verbose: bool = False, out: str = LIB_PATH, defines=(), sources=None) -> str:
    """Compile the library (or, with `sources`, a variant built from other
    top-level files that include it) unless it is up to date.  A build with
    `defines` but no `sources` is always redone: its output carries no record
    of the defines."""
    if not force and (sources or not defines) and up_to_date(out, extra=sources or ()):
        return out
    cmd = command(out, defines, sources)
    if verbose:
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose=True))
