"""Build the float64 oracle as a shared library (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg load it.
Compiled without FMA contraction or fast-math so every operation in oracle.c
is one IEEE double operation in the order written.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
HDR = os.path.join(HERE, "oracle.h")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fno-finite-math-only", "-fPIC", "-shared", "-pthread",
          "-Wall", "-Wextra", "-Werror"]


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in (SRC, HDR, __file__))


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source if missing or out of date."""
    if force or is_stale():
        tmp = LIB + ".tmp"
        cmd = ["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
