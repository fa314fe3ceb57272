"""Compile the CPU oracle (test infrastructure) into oracle/libnvfp4_oracle.so.

Run as a script (``python oracle/build.py``) or through ``oracle.build()``.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nvfp4_oracle.c")
LIB_PATH = os.path.join(HERE, "libnvfp4_oracle.so")

# -fno-fast-math / -ffp-contract=off / SSE math: every float operation in the
# oracle is one IEEE binary32 operation (no FMA contraction, no x87 excess
# precision).
CFLAGS = [
    "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
    "-fno-fast-math", "-ffp-contract=off", "-msse2", "-mfpmath=sse",
]


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB_PATH) or (
        os.path.getmtime(LIB_PATH) < os.path.getmtime(SRC)
    ):
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
