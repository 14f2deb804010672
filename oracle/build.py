"""Compile the C oracle (cf_oracle.c) into oracle/libcf_oracle.so with gcc.

Test infrastructure: the flags keep the arithmetic plain IEEE binary32/64
(no FMA contraction, no fast-math) so that the oracle computes exactly the
rounding sequence its comments state.
"""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cf_oracle.c")
LIB = os.path.join(HERE, "libcf_oracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-fno-finite-math-only", "-Wall", "-Wextra"]


STAMP = LIB + ".sources"    # hash of the source and flags the library was built from


def _inputs_hash() -> str:
    # content, not file times: a copy of the tree may round the times
    h = hashlib.sha256(" ".join(CFLAGS).encode())
    with open(SRC, "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def build(force: bool = False) -> str:
    digest = _inputs_hash()
    if not force and os.path.exists(LIB) and os.path.exists(STAMP):
        with open(STAMP) as f:
            if f.read().strip() == digest:
                return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"])
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(digest + "\n")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
