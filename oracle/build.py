"""Compile the CPU oracle (plain C) into oracle/libw8a8_oracle.so.

Test infrastructure only.  The flags keep every float operation a single IEEE
binary32 operation rounded to nearest even: no fast-math, no FMA contraction,
no flush-to-zero.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "w8a8_oracle.c")
LIB = os.path.join(HERE, "libw8a8_oracle.so")

CFLAGS = [
    "-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off",
    "-fno-unsafe-math-optimizations", "-frounding-math",
    "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
]


def needs_build() -> bool:
    return (not os.path.exists(LIB)) or os.path.getmtime(LIB) < os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
