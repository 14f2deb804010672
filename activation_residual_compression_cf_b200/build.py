"""Build libcf.so in-tree with nvcc for sm_100a (B200).

    python -m activation_residual_compression_cf_b200.build [--force] [--debug] [-v]

The library is the product: hand-written CUDA kernels plus the C ABI of
include/cf.h.  It links the CUDA runtime statically, so it depends only on
the driver (libcuda) at run time.  --debug builds libcf_debug.so instead:
the same kernels compiled with CF_DEBUG_BOUNDS, whose index checks record
an out-of-range access in a status word and skip it (include/cf_diag.h).
"""
from __future__ import annotations

import fcntl
import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libcf.so")
DEBUG_LIB = os.path.join(PKG, "libcf_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2",
         "--expt-relaxed-constexpr", "-Xcudafe", "--diag_suppress=177"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__])


def _flags(debug: bool):
    return FLAGS + (["-DCF_DEBUG_BOUNDS"] if debug else [])


def _lib(debug: bool) -> str:
    return DEBUG_LIB if debug else LIB


def _inputs_hash(debug: bool = False) -> str:
    """Content hash of every source, header and flag the library depends on.
    File times are not used: a copy of the tree to another machine may round
    them, and a source edited within the same second as the build would then
    look older than the library."""
    h = hashlib.sha256()
    h.update(" ".join([NVCC, *ARCH, *_flags(debug)]).encode())
    for p in sorted(_deps()):
        h.update(os.path.relpath(p, ROOT).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def up_to_date(debug: bool = False) -> bool:
    lib, stamp = _lib(debug), _lib(debug) + ".sources"
    if not (os.path.exists(lib) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == _inputs_hash(debug)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every source (in parallel) and link the library; nothing is
    done when the stamp shows it was built from the same inputs.  Processes
    that build at the same time (one per GPU of a multi-rank run) take turns
    on a lock file, and a process that finds the library current once it
    holds the lock does nothing."""
    lib = _lib(debug)
    if not force and up_to_date(debug):
        return lib
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    with open(os.path.join(ROOT, "_build", ".lock"), "w") as lk:
        fcntl.flock(lk, fcntl.LOCK_EX)
        try:
            if not force and up_to_date(debug):
                return lib
            return _compile(lib, verbose, debug)
        finally:
            fcntl.flock(lk, fcntl.LOCK_UN)


def _compile(lib: str, verbose: bool, debug: bool) -> str:
    digest = _inputs_hash(debug)
    objdir = os.path.join(ROOT, "_build", "debug" if debug else "release")
    os.makedirs(objdir, exist_ok=True)
    objs, procs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *_flags(debug), "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        procs.append((cmd, subprocess.Popen(cmd)))
        objs.append(obj)
    for cmd, p in procs:
        if p.wait() != 0:
            raise subprocess.CalledProcessError(p.returncode, cmd)
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp])
    os.replace(tmp, lib)
    with open(lib + ".sources", "w") as f:
        f.write(digest + "\n")
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
