"""Builds libic_b200.so in-tree with nvcc for sm_100a (no JIT, no torch extension)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libic_b200.so")
# the same sources with -DIC_DEBUG_BOUNDS: device-side index checks (see ic.h)
LIB_DEBUG = os.path.join(PKG, "libic_b200_debug.so")
NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(ROOT, "include", "ic.h")])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          debug_bounds: bool = False) -> str:
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc()] + NVCC_FLAGS + (["-DIC_DEBUG_BOUNDS"] if debug_bounds else []) + (extra or []) + [
        "-I", os.path.join(ROOT, "include"), "-o", tmp, os.path.join(CSRC, "libic.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None,
          debug_bounds="--debug-bounds" in sys.argv)
