"""Build the CPU oracle shared library (test infrastructure).

    python oracle/build.py        -> oracle/liboracle.so

Flags: -O2 -ffp-contract=off so that gcc never fuses a product into a sum
(fmaf() is written where a fused multiply-add is meant), no fast-math, and
-mfma only when the host CPU has FMA (fmaf is exact either way).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "maple_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def _host_has_fma() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("flags"):
                    return " fma " in (line + " ")
    except OSError:
        pass
    return False


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    if _host_has_fma():
        cmd.insert(3, "-mfma")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
