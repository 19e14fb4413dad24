"""Build the oracle shared library (plain C, gcc, IEEE binary32 arithmetic).

Run ``python -m oracle.build`` or call ``build()``.  The flags matter for
parity: no FMA contraction, no fast-math, SSE arithmetic (no x87 excess
precision), so each float operation in the source is one IEEE operation.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nvfp4_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-msse2",
          "-mfpmath=sse", "-fno-finite-math-only", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
