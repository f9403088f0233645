"""Compile the CPU oracle (oracle.c) into oracle/liboracle.so with gcc.

Test infrastructure only. Flags keep binary32 arithmetic exactly as written: SSE math (no x87
extended precision), no contraction of a*b+c into fused multiply-adds, no fast-math.
OpenMP parallelises the decode over (sequence, query head) pairs.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

FLAGS = [
    "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
    "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
    "-mfpmath=sse", "-msse2",
]


def build(force: bool = False) -> str:
    """Build liboracle.so if missing or older than its sources; return its path."""
    deps = [SRC, os.path.join(HERE, "oracle.h"), __file__]
    if not force and os.path.exists(LIB):
        lib_mtime = os.path.getmtime(LIB)
        if all(os.path.getmtime(p) <= lib_mtime for p in deps):
            return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *FLAGS, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
