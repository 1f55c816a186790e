"""Builds libcsa.so in-tree with nvcc for sm_100a (no GPU needed to build).

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


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile csrc/csa_lib.cu (which includes every kernel) into libcsa.so."""
    if not force and not needs_build():
        return LIB
    tmp = LIB + ".tmp"
    nvtx = ["-DCSA_NVTX"] if os.environ.get("CSA_NVTX") == "1" else []
    cmd = [NVCC, *FLAGS, *nvtx, *extra, "-o", tmp, os.path.join(CSRC, "csa_lib.cu")]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
