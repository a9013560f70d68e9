"""Build libexl3.so (sm_100a) in-tree with nvcc.

    python -m gemm_exl3_gemv_b200.build [--force]

The shared library lands next to this file; the ctypes binding loads it from
there.  nvcc cross-compiles, so no GPU is needed to build.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libexl3.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++20", "-lineinfo", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "exl3.h")]


# The debug-bounds variant: every product kernel checks the index of each
# access to the packed words, the workspace and the outputs, records a failed
# check in the workspace status word and skips the access (no trap).
LIB_DEBUG = os.path.join(HERE, "libexl3_debug.so")


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def _compile(lib: str, extra, verbose: bool):
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *ARCH, *FLAGS, *extra, "-shared", "-I", os.path.join(ROOT, "include"), "-o", tmp, *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Build libexl3.so (and, unless debug=False, libexl3_debug.so) if stale."""
    if force or stale(LIB):
        _compile(LIB, [], verbose)
    if debug and (force or stale(LIB_DEBUG)):
        _compile(LIB_DEBUG, ["-DEXL3_DEBUG_BOUNDS"], verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
