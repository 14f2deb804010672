"""The bounds-checked debug build (libcf_debug.so, CF_DEBUG_BOUNDS): the same
kernels with an index check at their global and shared-memory accesses; a
failed check skips the access and records its file and line, nothing traps.
Compute-sanitizer is not available to these tests, so this build stands in
for its out-of-bounds checks.

  * The positive control: a kernel whose check declares half its buffer's
    extent records a failure in diag.cu and skips exactly the upper half;
    every write it makes stays inside the buffer whether or not the check
    works.
  * The ragged-shape parity tests (quantize and low-rank, the publishing and
    waiting kernels) run under the debug build in a child process and must
    pass with no failed check after any test (an autouse fixture in
    conftest.py reads the record after each one).
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_release_build_has_no_checks():
    from activation_residual_compression_cf_b200 import build, cf
    build.build()
    if os.environ.get("CF_LIBRARY") == "debug":
        pytest.skip("this process runs the debug build")
    assert cf.cf_debug_bounds_checked() is False
    assert cf.cf_debug_bounds_take() == 0


def test_debug_build_exports_the_same_symbols():
    import ctypes
    from activation_residual_compression_cf_b200 import build, cf
    lib = ctypes.CDLL(build.build(debug=True))
    for name in cf.EXPORTS + cf.DIAG_EXPORTS:
        assert hasattr(lib, name), name
    lib.cf_debug_bounds_checked.restype = ctypes.c_int32
    assert lib.cf_debug_bounds_checked() == 1


@pytest.mark.gpu
def test_debug_build_selftest_records_and_skips():
    env = dict(os.environ, CF_LIBRARY="debug")
    code = r"""
import torch
from activation_residual_compression_cf_b200 import build, cf
build.build(debug=True)
assert cf.cf_debug_bounds_checked()
assert cf.cf_debug_bounds_take() == 0
out = torch.full((512,), -1, dtype=torch.int32, device="cuda")
cf.cf_diag_bounds_selftest(out)
hit = cf.cf_debug_bounds_take()
assert hit >> 16 == cf.bounds_file_tag("diag.cu"), hit
assert out[:256].tolist() == list(range(256)) and out[256:].tolist() == [-1] * 256
assert cf.cf_debug_bounds_take() == 0          # cleared by the read
print("selftest ok")
"""
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert "selftest ok" in r.stdout


@pytest.mark.gpu
def test_ragged_parity_under_the_debug_build():
    env = dict(os.environ, CF_LIBRARY="debug")
    from activation_residual_compression_cf_b200 import build
    build.build(debug=True)
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_parity_quant.py", "tests/test_parity_lowrank.py",
           "tests/test_parity_publish.py",
           "-k", "ragged or tma_pipeline_bit_identical or publishing or waiting or batched_lowrank"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout
