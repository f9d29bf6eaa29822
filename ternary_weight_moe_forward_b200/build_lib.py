"""Build libmaple_moe.so (the CUDA library) in-tree for sm_100a.

    python -m ternary_weight_moe_forward_b200.build_lib
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmaple_moe.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
         "-Xcompiler", "-fPIC", "-shared", "-fmad=false", "-Xptxas", "-warn-spills"]


def sources():
    return [os.path.join(CSRC, "maple_moe.cu")]


def _deps():
    return glob.glob(os.path.join(CSRC, "*")) + [os.path.join(ROOT, "include", "maple_moe.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(d) <= t for d in _deps()):
            return LIB
    cmd = [NVCC, *FLAGS, "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp", *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
