"""Build ``libqlinear.so`` (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libqlinear.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2", "-shared",
    # exact IEEE arithmetic: no fast-math, no flush-to-zero, no contraction
    # beyond what the kernels write explicitly
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(ROOT, "include", "qlinear.h")])


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    srcs = sources()
    stale = not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(s) for s in srcs)
    if force or stale:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose_ptxas else []), "-o", tmp,
               os.path.join(CSRC, "qlinear.cu")]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="-v" in sys.argv))
