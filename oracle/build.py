"""Compile the fp64 CPU oracle (plain C, gcc) into ``oracle/libsdoracle.so``.

Test infrastructure: the library is only loaded by the tests, the smoke check and the
benchmark's CPU-baseline leg.  Flags keep the arithmetic plain: no fast-math, no FMA
contraction, so every sum is evaluated exactly as written.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sd_oracle.c")
HDR = os.path.join(HERE, "sd_oracle.h")
LIB = os.path.join(HERE, "libsdoracle.so")


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in (SRC, HDR, __file__))


def build(force: bool = False) -> str:
    if force or is_stale():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
