"""Compile libddtree.so (sm_100a) in-tree with nvcc.

Usage: ``python -m draft_tree_build_ddtree_b200.build_lib [--force]``.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libddtree.so")
LIB_DEBUG = os.path.join(PKG, "libddtree_debug.so")   # -DDDTREE_DEBUG: internal bounds checks into the status word

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(INCLUDE, "ddtree.h")])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build libddtree.so (or, with debug, libddtree_debug.so with -DDDTREE_DEBUG)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not stale(lib):
        return lib
    extra = ["-DDDTREE_DEBUG"] if debug else []
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-I" + INCLUDE, os.path.join(CSRC, "ddtree.cu"), "-o", lib + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
