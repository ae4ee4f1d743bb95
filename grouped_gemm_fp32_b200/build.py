"""Build ``libmoe.so`` (the C-ABI CUDA library) in-tree with nvcc for sm_100a, and
``libmoe_debug.so``, the same sources with MOE_DEBUG=1 (device-side checks of the
group table and tile coordinates that report MOE_ERR_BAD_ROUTING instead of
following a bad entry; loaded instead of libmoe.so when MOE_LIB_DEBUG=1).

    python -m grouped_gemm_fp32_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe.so")
LIB_DEBUG = os.path.join(HERE, "libmoe_debug.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        [os.path.join(INCLUDE, "moe.h"), os.path.abspath(__file__)]


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in deps())


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def _build_one(lib: str, extra, force: bool, verbose: bool):
    if not force and not stale(lib):
        return
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Both libraries (the debug one unless ``debug`` is False); returns libmoe.so's path."""
    _build_one(LIB, [], force, verbose)
    if debug:
        _build_one(LIB_DEBUG, ["-DMOE_DEBUG=1"], force, verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
