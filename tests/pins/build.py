"""Compile the exhaustive pin harness together with the oracle source."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
LIB = os.path.join(HERE, "libpins.so")
SRCS = [os.path.join(HERE, "exhaustive.c"), os.path.join(HERE, "kernel_shortcuts.c"),
        os.path.join(ROOT, "oracle", "nvfp4_oracle.c")]


def build():
    newest = max(os.path.getmtime(s) for s in SRCS)
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-msse2",
                    "-mfpmath=sse", "-fPIC", "-shared", "-pthread", *SRCS, "-o", tmp, "-lm"],
                   check=True)
    os.replace(tmp, LIB)
    return LIB
