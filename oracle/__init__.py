"""CPU oracle for CompactFusion-style residual compression.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and
bench.py's CPU-baseline leg may import this package; the product library
never does, and it shares no code with the CUDA path.

* Quantize mode (1/2-bit, per-token scales, error feedback): plain C in
  cf_oracle.c, called through ctypes on numpy arrays.
* Low-rank mode (subspace iteration, INT4 factors): numpy fp64 in
  lowrank.py.

Method source: "Accelerating Parallel Diffusion Model Serving with Residual
Compression" (atlas.scime.ai summary of CompactFusion), sections "Approach",
"Key results" and the "Measured effects" table.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build
from . import lowrank  # noqa: F401  (re-exported)

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        lib.orc_words_per_row.argtypes = [i64, i32]
        lib.orc_words_per_row.restype = i64
        lib.orc_state_init.argtypes = [i64, i64, vp, vp, vp]
        lib.orc_state_init.restype = None
        lib.orc_encode.argtypes = [i64, i64, i32, vp, vp, vp, vp, vp, vp]
        lib.orc_encode.restype = ctypes.c_int
        lib.orc_encode_delta.argtypes = [i64, i64, i32, vp, vp, vp, vp, vp, vp]
        lib.orc_encode_delta.restype = ctypes.c_int
        lib.orc_decode.argtypes = [i64, i64, i32, vp, vp, vp]
        lib.orc_decode.restype = ctypes.c_int
        lib.orc_decode_emit.argtypes = [i64, i64, i32, vp, vp, vp, vp]
        lib.orc_decode_emit.restype = ctypes.c_int
        lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.orc_f32_to_bf16.restype = ctypes.c_uint16
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(a, dtype, shape, name):
    if a.dtype != dtype or a.shape != tuple(shape) or not a.flags["C_CONTIGUOUS"]:
        raise ValueError(f"{name}: want contiguous {np.dtype(dtype)}{tuple(shape)}, "
                         f"got {a.dtype}{a.shape}")


def words_per_row(channels: int, bits: int) -> int:
    return int(_load().orc_words_per_row(channels, bits))


def state_init(x0_bits: np.ndarray):
    """Warmup step: returns (recon, err) = ((float)x0, 0)."""
    T, C = x0_bits.shape
    _check(x0_bits, np.uint16, (T, C), "x0")
    recon = np.empty((T, C), np.float32)
    err = np.empty((T, C), np.float32)
    _load().orc_state_init(T, C, _ptr(x0_bits), _ptr(recon), _ptr(err))
    return recon, err


def encode(x_bits: np.ndarray, recon_s: np.ndarray, bits: int):
    """One compressed sender step; ``recon_s`` is updated in place.
    Returns (codes uint32 [T, W], scales float32 [T], err float32 [T, C])."""
    T, C = x_bits.shape
    _check(x_bits, np.uint16, (T, C), "x")
    _check(recon_s, np.float32, (T, C), "recon_s")
    W = words_per_row(C, bits) if bits in (1, 2) else 0
    codes = np.empty((T, W), np.uint32)
    scales = np.empty((T,), np.float32)
    err = np.empty((T, C), np.float32)
    scratch = np.empty((max(C, 1),), np.float32)
    rc = _load().orc_encode(T, C, bits, _ptr(x_bits), _ptr(recon_s), _ptr(err),
                            _ptr(codes), _ptr(scales), _ptr(scratch))
    if rc != 0:
        raise ValueError(f"oracle encode: unsupported bits={bits}")
    return codes, scales, err


def encode_delta(x_bits: np.ndarray, xprev_bits: np.ndarray, err: np.ndarray, bits: int):
    """Delta-state sender step: v = ((float)x - (float)x_prev) + err, then
    as encode without the mirror; ``err`` is updated in place.
    Returns (codes uint32 [T, W], scales float32 [T])."""
    T, C = x_bits.shape
    _check(x_bits, np.uint16, (T, C), "x")
    _check(xprev_bits, np.uint16, (T, C), "x_prev")
    _check(err, np.float32, (T, C), "err")
    W = words_per_row(C, bits) if bits in (1, 2) else 0
    codes = np.empty((T, W), np.uint32)
    scales = np.empty((T,), np.float32)
    scratch = np.empty((max(C, 1),), np.float32)
    rc = _load().orc_encode_delta(T, C, bits, _ptr(x_bits), _ptr(xprev_bits), _ptr(err),
                                  _ptr(codes), _ptr(scales), _ptr(scratch))
    if rc != 0:
        raise ValueError(f"oracle encode: unsupported bits={bits}")
    return codes, scales


def decode(codes: np.ndarray, scales: np.ndarray, recon_r: np.ndarray, bits: int):
    """Receiver step; ``recon_r`` is updated in place."""
    T, C = recon_r.shape
    W = words_per_row(C, bits)
    _check(codes, np.uint32, (T, W), "codes")
    _check(scales, np.float32, (T,), "scales")
    _check(recon_r, np.float32, (T, C), "recon_r")
    rc = _load().orc_decode(T, C, bits, _ptr(codes), _ptr(scales), _ptr(recon_r))
    if rc != 0:
        raise ValueError(f"oracle decode: unsupported bits={bits}")


def decode_emit(codes: np.ndarray, scales: np.ndarray, recon_r: np.ndarray, bits: int):
    """Receiver step that also returns the bf16 reconstruction (uint16 bit
    patterns, round to nearest even); ``recon_r`` is updated in place."""
    T, C = recon_r.shape
    W = words_per_row(C, bits)
    _check(codes, np.uint32, (T, W), "codes")
    _check(scales, np.float32, (T,), "scales")
    _check(recon_r, np.float32, (T, C), "recon_r")
    out = np.empty((T, C), np.uint16)
    rc = _load().orc_decode_emit(T, C, bits, _ptr(codes), _ptr(scales), _ptr(recon_r), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle decode: unsupported bits={bits}")
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Element-wise fp32 -> bf16 (round to nearest even) through the C oracle."""
    f = _load().orc_f32_to_bf16
    flat = np.ascontiguousarray(a, np.float32).ravel()
    return np.array([f(float(v)) for v in flat], np.uint16).reshape(np.shape(a))


def quant_payload_bytes(tokens: int, channels: int, bits: int) -> int:
    """Bytes on the wire per buffer in quantize mode: packed codes plus one
    fp32 scale per token."""
    return tokens * words_per_row(channels, bits) * 4 + tokens * 4
