"""Builds libcsa.so in-tree with nvcc for sm_100a (no GPU needed to build),
and its debug twin libcsa_debug.so (compiled with CSA_DEBUG: the kernels
check the indices they compute before each global access and record a status
bit instead of accessing out of range; same entry points, same results).

CSA_NVTX=1 in the environment compiles in NVTX ranges named after the stages
(host side, around each stage's launches) for profiler timelines; it takes
effect on a forced rebuild (``python build.py --force``).
"""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")
LIB = os.path.join(PKG, "libcsa.so")
LIB_DEBUG = os.path.join(PKG, "libcsa_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC,-O2",
    "--expt-relaxed-constexpr",
]


def _sources():
    out = []
    for d in (CSRC, INCLUDE):
        for f in sorted(os.listdir(d)):
            if f.endswith((".cu", ".cuh", ".h")):
                out.append(os.path.join(d, f))
    return out


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def _compile(lib: str, defines, verbose: bool, extra) -> None:
    tmp = lib + ".tmp"
    nvtx = ["-DCSA_NVTX"] if os.environ.get("CSA_NVTX") == "1" else []
    cmd = [NVCC, *FLAGS, *nvtx, *defines, *extra, "-o", tmp, os.path.join(CSRC, "csa_lib.cu")]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile csrc/csa_lib.cu (which includes every kernel) into libcsa.so
    and libcsa_debug.so; returns the release library's path."""
    for lib, defines in ((LIB, []), (LIB_DEBUG, ["-DCSA_DEBUG"])):
        if force or needs_build(lib):
            _compile(lib, defines, verbose, extra)
    return LIB


if __name__ == "__main__":
    import sys
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
