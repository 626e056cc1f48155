"""Compile the C oracle into oracle/liboracle.so with plain gcc.

The oracle is test infrastructure; building it is part of building the
checker, not of the product path.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "split12_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(src: str = SRC, out: str = LIB, extra=()) -> str:
    cmd = ["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-fno-fast-math", *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def ensure_built() -> str:
    if (not os.path.exists(LIB)) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        build()
    return LIB


if __name__ == "__main__":
    print(build(*sys.argv[1:2]))
