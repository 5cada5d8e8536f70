"""Compile the CPU oracle (plain C) into ``oracle/liboracle.so``.

Test infrastructure: the oracle is built so the test suite, the smoke check and
the benchmark's CPU-baseline leg can call it.  Run as a script or call
``build_oracle()``; it rebuilds only when the source is newer than the library.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp8bw_oracle.c")
HDR = os.path.join(HERE, "fp8bw_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")

# IEEE binary32 arithmetic: no contraction into FMA, no fast-math, SSE on x86-64.
CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def build_oracle(force: bool = False) -> str:
    """Build the oracle shared library if missing or stale; return its path."""
    stale = force or not os.path.exists(LIB) or any(
        os.path.getmtime(p) > os.path.getmtime(LIB) for p in (SRC, HDR, __file__))
    if stale:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build_oracle(force="--force" in sys.argv))
