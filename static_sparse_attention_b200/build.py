"""Build libradattn.so in-tree: nvcc for sm_100a, static CUDA runtime.

    python static_sparse_attention_b200/build.py [--force] [--verbose] [--debug]

`--verbose` adds -Xptxas -v (registers, spills, shared memory per kernel).
`--debug` builds libradattn_debug.so instead: the same sources with
-DRA_DEBUG_BOUNDS, whose kernels check every global index and TMA coordinate
they derive from their inputs and record a failure in the device error word
(RA_ERR_DEVICE_BOUNDS) instead of making the access.  The binding loads it when
RA_LIBRARY_VARIANT=debug is set.
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
LIB = os.path.join(PKG, "libradattn.so")
LIB_DEBUG = os.path.join(PKG, "libradattn_debug.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-O3",
    "--cudart", "static",
    "-shared",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DRA_DEBUG_BOUNDS"] if debug else []), "-I", INCLUDE, "-I", CSRC, *sources(),
           "-o", tmp]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
