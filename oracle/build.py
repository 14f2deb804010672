"""Compile the C oracle (cf_oracle.c) into oracle/libcf_oracle.so with gcc.

Test infrastructure: the flags keep the arithmetic plain IEEE binary32/64
(no FMA contraction, no fast-math) so that the oracle computes exactly the
rounding sequence its comments state.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cf_oracle.c")
LIB = os.path.join(HERE, "libcf_oracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-fno-finite-math-only", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
