"""The C-ABI library loads, exports every entry point include/cf.h declares,
and rejects bad arguments on the host without launching anything.  No GPU
needed: nothing here reaches a kernel launch."""
import ctypes
import os
import re

import pytest

from activation_residual_compression_cf_b200 import build, cf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header=None):
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h") and (header is None or fn == header):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(cf_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def L():
    build.build()
    return cf.lib()


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert declared, "no declarations found"
    for name in sorted(declared):
        assert hasattr(L, name), f"{name} declared in include/ but not exported"
    # the product header and the diagnostic header each match their list
    assert _declared("cf.h") == set(cf.EXPORTS)
    assert _declared("cf_diag.h") == set(cf.DIAG_EXPORTS)
    assert not set(cf.EXPORTS) & set(cf.DIAG_EXPORTS)
    assert declared == set(cf.EXPORTS) | set(cf.DIAG_EXPORTS)


def test_async_status_validates_before_any_cuda_call(L):
    h = ctypes.c_int32()
    assert L.cf_lowrank_status_async(256, 256, 0, None, None) == 0           # n == 0: nothing
    assert L.cf_lowrank_status_async(256, 256, -1, ctypes.byref(h), None) == 1
    assert L.cf_lowrank_status_async(None, 256, 1, ctypes.byref(h), None) == 1
    assert L.cf_lowrank_status_async(256, 256, 1, None, None) == 1
    assert L.cf_lowrank_status_async(256, 0, 1, ctypes.byref(h), None) == 1
    assert L.cf_lowrank_status_async(128, 256, 1, ctypes.byref(h), None) == 2  # workspace alignment
    assert L.cf_lowrank_status_async(256, 100, 1, ctypes.byref(h), None) == 2  # slice alignment


def test_abi_version_and_status_strings(L):
    assert cf.cf_abi_version() == 1
    for code, name in cf.STATUS_NAMES.items():
        assert cf.cf_status_string(code).startswith(name)


def test_sizing_queries(L):
    assert cf.cf_codes_words_per_row(cf.desc(10, 3072, 2)) == 192
    assert cf.cf_codes_words_per_row(cf.desc(10, 33, 1)) == 2
    assert cf.cf_codes_words_per_row(cf.desc(10, 64, 3)) == 0
    assert cf.cf_payload_bytes(cf.desc(1024, 3072, 1)) == 1024 * (384 + 4)
    assert cf.cf_payload_bytes(cf.desc(1024, 3072, 0, 32, 2)) == 1024 * 16 + 3072 * 16 + 256
    assert cf.cf_lowrank_factor_bytes(4096, 32) == 4096 * 16
    assert cf.cf_lowrank_factor_bytes(5, 3) == 10


@pytest.mark.parametrize("d,expect", [
    (dict(tokens=4, channels=64, bits=3), 3),          # unsupported bit width
    (dict(tokens=4, channels=64, bits=1, scale_kind=1), 3),
    (dict(tokens=-1, channels=64, bits=1), 1),
    (dict(tokens=4, channels=0, bits=1), 1),
    (dict(tokens=4, channels=64, bits=1, rank=2), 1),
    (dict(tokens=4, channels=16385, bits=1), 3),       # beyond the register-resident row
    (dict(tokens=4, channels=64, bits=1), 1),          # null pointers
])
def test_encode_rejects_bad_arguments_without_launch(L, d, expect):
    st = L.cf_encode(ctypes.byref(cf.desc(**d)), None, None, None, None, None, None)
    assert st == expect
    st = L.cf_decode(ctypes.byref(cf.desc(**d)), None, None, None, None)
    assert st == expect


def test_empty_problem_is_a_noop(L):
    assert L.cf_encode(ctypes.byref(cf.desc(0, 64, 1)), None, None, None, None, None, None) == 0
    assert L.cf_decode_batched(ctypes.byref(cf.desc(4, 64, 2)), 0, None, None, None) == 0
    assert L.cf_encode_batched(ctypes.byref(cf.desc(4, 64, 2)), -1, None, None, None) == 1


def test_misaligned_pointer_is_rejected_before_any_cuda_call(L):
    st = L.cf_encode(ctypes.byref(cf.desc(4, 64, 1)), 8, 16, 16, 16, 16, None)
    assert st == 2


def test_lowrank_descriptor_checks(L):
    ok = cf.desc(64, 48, 0, 8, 2)
    assert cf.cf_lowrank_workspace_bytes(ok) >= 0
    assert cf.cf_lowrank_workspace_bytes(cf.desc(64, 48, 0, 65, 2)) == 0
    assert cf.cf_lowrank_workspace_bytes(cf.desc(64, 48, 0, 8, 0)) == 0
    assert cf.cf_lowrank_workspace_bytes(cf.desc(4, 48, 0, 8, 2)) == 0   # rank > tokens


def test_launch_override_validation(L):
    assert L.cf_set_launch_override(2, 0, 0, 0) == 1
    assert L.cf_set_launch_override(0, 5, 128, 0) == 1
    assert L.cf_set_launch_override(0, 2, 100, 0) == 1
    assert L.cf_set_launch_override(0, 2, 0, 0) == 1
    assert L.cf_set_launch_override(0, 2, 128, 4) == 0
    assert L.cf_set_launch_override(0, 0, 0, 0) == 0


def test_pipeline_and_engine_knobs_validate(L):
    assert L.cf_set_quant_pipeline(2, 0, 0) == 1
    assert L.cf_set_quant_pipeline(0, 2, 0) == 1
    assert L.cf_set_quant_pipeline(0, 1, 1) == 1
    assert L.cf_set_quant_pipeline(0, 1, 9) == 1
    assert L.cf_set_quant_pipeline(0, 1, 4) == 0
    assert L.cf_set_quant_pipeline(0, 0, 0) == 0
    assert L.cf_set_quant_pipeline(0, 1, 0) == 0   # restore the default
    assert L.cf_set_lowrank_engine(2) == 1
    assert L.cf_set_lowrank_engine(0) == 0
    # the apply-event hook takes pairs: half a pair is rejected, all-null clears
    one = ctypes.c_void_p(1)
    assert L.cf_lowrank_set_apply_events(one, None, None, None) == 1
    assert L.cf_lowrank_set_apply_events(None, None, None, one) == 1
    assert L.cf_lowrank_set_apply_events(None, None, None, None) == 0


def test_bounded_wait_diagnostic_validates_before_any_cuda_call(L):
    assert L.cf_diag_bounded_wait(0, 16, None) == 1        # no polls
    assert L.cf_diag_bounded_wait(65537, 16, None) == 1    # above the cap
    assert L.cf_diag_bounded_wait(256, None, None) == 1    # null output
    assert L.cf_diag_bounded_wait(256, 18, None) == 2      # not 4-byte aligned


def test_binding_raises_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(cf, "_lib", None)
    monkeypatch.setattr(cf, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="not built"):
        cf.lib()


def test_publish_and_wait_validate_before_any_cuda_call(L):
    d = ctypes.byref(cf.desc(4, 64, 2))
    assert L.cf_encode_publish_batched(d, 1, None, 0, None, 0, None, None) == 1    # no destination
    assert L.cf_encode_publish_batched(d, 1, None, 9, None, 0, None, None) == 1    # above 8
    assert L.cf_encode_publish_batched(d, -1, None, 1, None, 0, None, None) == 1
    assert L.cf_encode_publish_batched(d, 0, None, 1, None, 0, None, None) == 0    # nothing to do
    assert L.cf_encode_publish_batched(ctypes.byref(cf.desc(4, 64, 3)), 1, None, 1, None, 0, None,
                                       None) == 3
    assert L.cf_decode_wait_batched(d, -1, None, 0, 0, None, None, None) == 1
    assert L.cf_decode_wait_batched(d, 0, None, 0, 65, None, None, None) == 1      # acks above 64
    assert L.cf_decode_wait_batched(d, 0, None, 0, 0, None, None, None) == 0
    assert L.cf_set_quant_unit(0, 6) == 1 and L.cf_set_quant_unit(2, 4) == 1
    assert L.cf_set_quant_unit(0, 4) == 0 and L.cf_set_quant_unit(0, 0) == 0
