"""Thin ctypes binding of libcf.so (include/cf.h), same names as the C ABI.

Argument marshalling only: tensors become raw device pointers, the stream
defaults to torch's current stream, and a non-zero cf_status raises
CFError.  Every step of the compression runs in the library's CUDA kernels;
there is no Python or CPU fallback.  If libcf.so is missing, the first call
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# CF_LIBRARY=debug loads the bounds-checked debug build (libcf_debug.so)
LIB_PATH = os.path.join(_PKG, "libcf_debug.so" if os.environ.get("CF_LIBRARY") == "debug"
                        else "libcf.so")

CF_OK = 0
STATUS_NAMES = {0: "CF_OK", 1: "CF_ERR_INVALID_ARG", 2: "CF_ERR_ALIGNMENT",
                3: "CF_ERR_UNSUPPORTED", 4: "CF_ERR_WORKSPACE", 5: "CF_ERR_CUDA",
                6: "CF_ERR_NUMERIC", 7: "CF_ERR_TIMEOUT"}

# Every symbol include/cf.h declares (checked by the ABI test).
EXPORTS = ("cf_status_string", "cf_abi_version", "cf_codes_words_per_row",
           "cf_payload_bytes", "cf_state_init", "cf_encode", "cf_decode",
           "cf_encode_batched", "cf_decode_batched", "cf_lowrank_workspace_bytes",
           "cf_lowrank_factor_bytes", "cf_lowrank_encode", "cf_lowrank_decode",
           "cf_lowrank_status", "cf_lowrank_status_async", "cf_lowrank_encode_noalloc",
           "cf_decode_emit", "cf_decode_emit_batched", "cf_lowrank_encode_batched",
           "cf_lowrank_decode_batched", "cf_encode_delta", "cf_encode_delta_batched",
           "cf_encode_publish_batched", "cf_decode_wait_batched")
# Every symbol include/cf_diag.h declares: tuning knobs, measurement hooks
# and the bounded-wait self-test (process-wide state, not product calls).
DIAG_EXPORTS = ("cf_set_lowrank_engine", "cf_set_quant_pipeline", "cf_set_launch_override",
                "cf_set_quant_unit", "cf_set_lowrank_group", "cf_lowrank_set_apply_events",
                "cf_diag_bounded_wait", "cf_diag_stream_mix", "cf_diag_stream_mix_tma",
                "cf_debug_bounds_checked", "cf_debug_bounds_take", "cf_diag_bounds_selftest")


class CFError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().cf_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{where}: {msg}")


class cf_desc(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int64), ("channels", ctypes.c_int64),
                ("bits", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("iters", ctypes.c_int32), ("scale_kind", ctypes.c_int32)]


class cf_enc_buffer(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("recon_s", ctypes.c_void_p),
                ("err", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p)]


class cf_enc_delta_buffer(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("x_prev", ctypes.c_void_p),
                ("err", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p)]


class cf_dec_buffer(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("recon_r", ctypes.c_void_p)]


class cf_lowrank_buffer(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("recon_s", ctypes.c_void_p), ("err", ctypes.c_void_p),
                ("omega", ctypes.c_void_p), ("p_codes", ctypes.c_void_p),
                ("p_scales", ctypes.c_void_p), ("q_codes", ctypes.c_void_p),
                ("q_scales", ctypes.c_void_p)]


class cf_lowrank_dec_buffer(ctypes.Structure):
    _fields_ = [("p_codes", ctypes.c_void_p), ("p_scales", ctypes.c_void_p),
                ("q_codes", ctypes.c_void_p), ("q_scales", ctypes.c_void_p),
                ("recon_r", ctypes.c_void_p)]


class cf_dec_emit_buffer(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("recon_r", ctypes.c_void_p), ("out", ctypes.c_void_p)]


class cf_publish_dst(ctypes.Structure):
    _fields_ = [("payload", ctypes.c_void_p), ("ready", ctypes.c_void_p), ("ack", ctypes.c_void_p)]


class cf_enc_publish_buffer(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("recon_s", ctypes.c_void_p), ("err", ctypes.c_void_p),
                ("codes_offset", ctypes.c_int64), ("scales_offset", ctypes.c_int64)]


class cf_dec_wait_buffer(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("recon_r", ctypes.c_void_p), ("ready", ctypes.c_void_p)]


_lib = None


def lib():
    """Load libcf.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libcf.so not built ({LIB_PATH}); run "
                               "`python -m activation_residual_compression_cf_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        D = ctypes.POINTER(cf_desc)
        sig = {
            "cf_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "cf_abi_version": ([], i32),
            "cf_codes_words_per_row": ([D], i64),
            "cf_payload_bytes": ([D], i64),
            "cf_state_init": ([D, vp, vp, vp, vp], ctypes.c_int),
            "cf_encode": ([D, vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "cf_decode": ([D, vp, vp, vp, vp], ctypes.c_int),
            "cf_encode_batched": ([D, i32, vp, vp, vp], ctypes.c_int),
            "cf_encode_delta": ([D, vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "cf_encode_delta_batched": ([D, i32, vp, vp, vp], ctypes.c_int),
            "cf_decode_batched": ([D, i32, vp, vp, vp], ctypes.c_int),
            "cf_decode_emit": ([D, vp, vp, vp, vp, vp], ctypes.c_int),
            "cf_decode_emit_batched": ([D, i32, vp, vp, vp], ctypes.c_int),
            "cf_lowrank_workspace_bytes": ([D], i64),
            "cf_lowrank_factor_bytes": ([i64, i32], i64),
            "cf_lowrank_encode": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
            "cf_lowrank_decode": ([D, vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "cf_lowrank_status": ([vp, vp], ctypes.c_int),
            "cf_lowrank_status_async": ([vp, i64, i32, vp, vp], ctypes.c_int),
            "cf_lowrank_encode_batched": ([D, i32, vp, vp, sz, vp], ctypes.c_int),
            "cf_lowrank_decode_batched": ([D, i32, vp, vp, vp], ctypes.c_int),
            "cf_set_launch_override": ([i32, i32, i32, i32], ctypes.c_int),
            "cf_set_lowrank_engine": ([i32], ctypes.c_int),
            "cf_lowrank_set_apply_events": ([vp, vp, vp, vp], ctypes.c_int),
            "cf_diag_bounded_wait": ([i32, vp, vp], ctypes.c_int),
            "cf_set_quant_pipeline": ([i32, i32, i32], ctypes.c_int),
            "cf_set_quant_unit": ([i32, i32], ctypes.c_int),
            "cf_set_lowrank_group": ([i32], ctypes.c_int),
            "cf_diag_stream_mix": ([vp, vp, vp, i64, vp], ctypes.c_int),
            "cf_diag_stream_mix_tma": ([vp, vp, vp, i64, i64, i32, vp, vp], ctypes.c_int),
            "cf_debug_bounds_checked": ([], i32),
            "cf_debug_bounds_take": ([], i32),
            "cf_diag_bounds_selftest": ([vp, i32, vp], ctypes.c_int),
            "cf_encode_publish_batched": ([D, i32, vp, i32, vp, ctypes.c_uint64, vp, vp], ctypes.c_int),
            "cf_decode_wait_batched": ([D, i32, vp, ctypes.c_uint64, i32, vp, vp, vp], ctypes.c_int),
            "cf_lowrank_encode_noalloc": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes, f.restype = args, res
        _lib = L
    return _lib


def desc(tokens: int, channels: int, bits: int = 0, rank: int = 0, iters: int = 0,
         scale_kind: int = 0) -> cf_desc:
    return cf_desc(tokens, channels, bits, rank, iters, scale_kind)


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _chk(st: int, where: str):
    if st != CF_OK:
        raise CFError(st, where)


def cf_status_string(status: int) -> str:
    return lib().cf_status_string(status).decode()


def cf_abi_version() -> int:
    return lib().cf_abi_version()


def cf_codes_words_per_row(d: cf_desc) -> int:
    return lib().cf_codes_words_per_row(ctypes.byref(d))


def cf_payload_bytes(d: cf_desc) -> int:
    return lib().cf_payload_bytes(ctypes.byref(d))


def cf_state_init(d, x0, recon, err=None, stream=None):
    _chk(lib().cf_state_init(ctypes.byref(d), _p(x0), _p(recon), _p(err), _s(stream)),
         "cf_state_init")


def cf_encode(d, x, recon_s, err, codes, scales, stream=None):
    _chk(lib().cf_encode(ctypes.byref(d), _p(x), _p(recon_s), _p(err), _p(codes),
                         _p(scales), _s(stream)), "cf_encode")


def cf_encode_delta(d, x, x_prev, err, codes, scales, stream=None):
    _chk(lib().cf_encode_delta(ctypes.byref(d), _p(x), _p(x_prev), _p(err), _p(codes),
                               _p(scales), _s(stream)), "cf_encode_delta")


def cf_encode_delta_batched(d, n, bufs_dev, status_dev=None, stream=None):
    _chk(lib().cf_encode_delta_batched(ctypes.byref(d), n, _p(bufs_dev), _p(status_dev),
                                       _s(stream)), "cf_encode_delta_batched")


def cf_decode(d, codes, scales, recon_r, stream=None):
    _chk(lib().cf_decode(ctypes.byref(d), _p(codes), _p(scales), _p(recon_r), _s(stream)),
         "cf_decode")


def cf_decode_emit(d, codes, scales, recon_r, out, stream=None):
    _chk(lib().cf_decode_emit(ctypes.byref(d), _p(codes), _p(scales), _p(recon_r), _p(out),
                              _s(stream)), "cf_decode_emit")


def cf_decode_emit_batched(d, n, bufs_dev, status_dev=None, stream=None):
    _chk(lib().cf_decode_emit_batched(ctypes.byref(d), n, _p(bufs_dev), _p(status_dev),
                                      _s(stream)), "cf_decode_emit_batched")


def cf_encode_batched(d, n, bufs_dev, status_dev=None, stream=None):
    _chk(lib().cf_encode_batched(ctypes.byref(d), n, _p(bufs_dev), _p(status_dev), _s(stream)),
         "cf_encode_batched")


def cf_decode_batched(d, n, bufs_dev, status_dev=None, stream=None):
    _chk(lib().cf_decode_batched(ctypes.byref(d), n, _p(bufs_dev), _p(status_dev), _s(stream)),
         "cf_decode_batched")


def cf_lowrank_workspace_bytes(d) -> int:
    return lib().cf_lowrank_workspace_bytes(ctypes.byref(d))


def cf_lowrank_factor_bytes(rows: int, rank: int) -> int:
    return lib().cf_lowrank_factor_bytes(rows, rank)


def cf_lowrank_encode(d, x, recon_s, err, omega, p_codes, p_scales, q_codes, q_scales,
                      workspace, workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _chk(lib().cf_lowrank_encode(ctypes.byref(d), _p(x), _p(recon_s), _p(err), _p(omega),
                                 _p(p_codes), _p(p_scales), _p(q_codes), _p(q_scales),
                                 _p(workspace), nbytes, _s(stream)), "cf_lowrank_encode")


def cf_lowrank_encode_noalloc(d, x, recon_s, err, omega, p_codes, p_scales, q_codes, q_scales,
                              stream=None):
    """cf_lowrank_encode without a workspace, for callers that cannot allocate
    device memory: the library's fixed device scratch array is used instead
    (see include/cf.h for its size and sharing rules)."""
    _chk(lib().cf_lowrank_encode_noalloc(ctypes.byref(d), _p(x), _p(recon_s), _p(err),
                                         _p(omega), _p(p_codes), _p(p_scales), _p(q_codes),
                                         _p(q_scales), _s(stream)), "cf_lowrank_encode_noalloc")


def cf_lowrank_decode(d, p_codes, p_scales, q_codes, q_scales, recon_r, stream=None):
    _chk(lib().cf_lowrank_decode(ctypes.byref(d), _p(p_codes), _p(p_scales), _p(q_codes),
                                 _p(q_scales), _p(recon_r), _s(stream)), "cf_lowrank_decode")


def cf_lowrank_encode_batched(d, n, bufs_dev, workspace, workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _chk(lib().cf_lowrank_encode_batched(ctypes.byref(d), n, _p(bufs_dev), _p(workspace), nbytes,
                                         _s(stream)), "cf_lowrank_encode_batched")


def cf_lowrank_decode_batched(d, n, bufs_dev, status_dev=None, stream=None):
    _chk(lib().cf_lowrank_decode_batched(ctypes.byref(d), n, _p(bufs_dev), _p(status_dev),
                                         _s(stream)), "cf_lowrank_decode_batched")


def cf_lowrank_status(workspace, stream=None) -> int:
    """Synchronises the stream; returns (and clears) the workspace status."""
    return lib().cf_lowrank_status(_p(workspace), _s(stream))


def cf_lowrank_status_async(workspace, slice_bytes: int, n: int, host_status, stream=None):
    """Enqueues the copy of n status words (slice b at workspace + b *
    slice_bytes) into host_status (a pinned int32 tensor of >= n elements);
    returns without waiting."""
    if host_status.dtype != torch.int32 or host_status.device.type != "cpu" or host_status.numel() < n:
        raise ValueError("host_status must be a host int32 tensor with at least n elements")
    _chk(lib().cf_lowrank_status_async(_p(workspace), slice_bytes, n, _p(host_status), _s(stream)),
         "cf_lowrank_status_async")


def cf_encode_publish_batched(d, n, bufs_dev, ndst, dsts_dev, ack_target=0, status=None,
                              stream=None):
    _chk(lib().cf_encode_publish_batched(ctypes.byref(d), n, _p(bufs_dev), ndst, _p(dsts_dev),
                                         int(ack_target), _p(status), _s(stream)),
         "cf_encode_publish_batched")


def cf_decode_wait_batched(d, n, bufs_dev, ready_target, nack=0, acks_dev=None, status=None,
                           stream=None):
    _chk(lib().cf_decode_wait_batched(ctypes.byref(d), n, _p(bufs_dev), int(ready_target), nack,
                                      _p(acks_dev), _p(status), _s(stream)),
         "cf_decode_wait_batched")


def cf_debug_bounds_checked() -> bool:
    return lib().cf_debug_bounds_checked() == 1


def cf_debug_bounds_take() -> int:
    """First failed index check of the debug build since the last call, as
    (file tag << 16) | line, or 0; clears it (synchronises)."""
    return lib().cf_debug_bounds_take()


def cf_diag_bounds_selftest(out_dev, stream=None):
    _chk(lib().cf_diag_bounds_selftest(_p(out_dev), out_dev.numel(), _s(stream)),
         "cf_diag_bounds_selftest")


def bounds_file_tag(name: str) -> int:
    """The debug build's 15-bit tag of a source file's base name (FNV-1a)."""
    h = 2166136261
    for ch in os.path.basename(name).encode():
        h = ((h ^ ch) * 16777619) & 0xFFFFFFFF
    return (h ^ (h >> 15)) & 0x7FFF


def cf_diag_stream_mix(x, r, a, stream=None):
    """Streaming pass with the encode's byte mix over every element of x."""
    _chk(lib().cf_diag_stream_mix(_p(x), _p(r), _p(a), x.numel(), _s(stream)), "cf_diag_stream_mix")


def cf_diag_stream_mix_tma(x, r, a, rows, channels, status=None, stream=None, bulk=False):
    """The encode's byte mix through the encode's TMA row pipeline (rows x
    channels) and its store path (bulk=True: bulk stores from shared-memory
    output rows), without its per-row work."""
    _chk(lib().cf_diag_stream_mix_tma(_p(x), _p(r), _p(a), rows, channels, 1 if bulk else 0, _p(status),
                                      _s(stream)), "cf_diag_stream_mix_tma")


def cf_set_lowrank_group(buffers: int):
    _chk(lib().cf_set_lowrank_group(buffers), "cf_set_lowrank_group")


def cf_set_quant_unit(kernel: int, channels: int):
    _chk(lib().cf_set_quant_unit(kernel, channels), "cf_set_quant_unit")


def cf_set_lowrank_engine(engine: int):
    _chk(lib().cf_set_lowrank_engine(engine), "cf_set_lowrank_engine")


def _ev(e):
    """torch.cuda.Event (already recorded once, so that it exists) or None ->
    its cudaEvent_t handle."""
    return None if e is None else ctypes.c_void_p(e.cuda_event)


def cf_lowrank_set_apply_events(enc_start=None, enc_stop=None, dec_start=None, dec_stop=None):
    _chk(lib().cf_lowrank_set_apply_events(_ev(enc_start), _ev(enc_stop), _ev(dec_start),
                                           _ev(dec_stop)), "cf_lowrank_set_apply_events")


def cf_diag_bounded_wait(polls: int, out_dev, stream=None):
    _chk(lib().cf_diag_bounded_wait(polls, _p(out_dev), _s(stream)), "cf_diag_bounded_wait")


def cf_set_quant_pipeline(kernel: int, pipeline: int, stages: int = 0):
    _chk(lib().cf_set_quant_pipeline(kernel, pipeline, stages), "cf_set_quant_pipeline")


def cf_set_launch_override(kernel: int, groups_per_thread: int = 0, threads: int = 0,
                           blocks_per_sm: int = 0):
    _chk(lib().cf_set_launch_override(kernel, groups_per_thread, threads, blocks_per_sm),
         "cf_set_launch_override")


# ----------------------------------------------------------- small helpers
# Allocation helpers for callers that hold their buffers in torch tensors.
# They only size and place memory; the library itself never allocates.

def enc_buffer_array(sets, device) -> torch.Tensor:
    """Device array of cf_enc_buffer from [(x, recon_s, err, codes, scales), ...]."""
    arr = (cf_enc_buffer * len(sets))()
    for i, (x, r, e, c, s) in enumerate(sets):
        arr[i] = cf_enc_buffer(_p(x), _p(r), _p(e), _p(c), _p(s))
    host = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8)
    return host.to(device)


def enc_delta_buffer_array(sets, device) -> torch.Tensor:
    """Device array of cf_enc_delta_buffer from [(x, x_prev, err, codes, scales), ...]."""
    arr = (cf_enc_delta_buffer * len(sets))()
    for i, t in enumerate(sets):
        arr[i] = cf_enc_delta_buffer(*[_p(v) for v in t])
    return torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)


def dec_buffer_array(sets, device) -> torch.Tensor:
    """Device array of cf_dec_buffer from [(codes, scales, recon_r), ...]."""
    arr = (cf_dec_buffer * len(sets))()
    for i, (c, s, r) in enumerate(sets):
        arr[i] = cf_dec_buffer(_p(c), _p(s), _p(r))
    host = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8)
    return host.to(device)


def lowrank_buffer_array(sets, device) -> torch.Tensor:
    """Device array of cf_lowrank_buffer from
    [(x, recon_s, err, omega, p_codes, p_scales, q_codes, q_scales), ...]."""
    arr = (cf_lowrank_buffer * len(sets))()
    for i, t in enumerate(sets):
        arr[i] = cf_lowrank_buffer(*[_p(v) for v in t])
    return torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)


def lowrank_dec_buffer_array(sets, device) -> torch.Tensor:
    """Device array of cf_lowrank_dec_buffer from
    [(p_codes, p_scales, q_codes, q_scales, recon_r), ...]."""
    arr = (cf_lowrank_dec_buffer * len(sets))()
    for i, t in enumerate(sets):
        arr[i] = cf_lowrank_dec_buffer(*[_p(v) for v in t])
    return torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)


def publish_dst_array(dsts, device) -> torch.Tensor:
    """Device array of cf_publish_dst from [(payload, ready, ack or None), ...]."""
    arr = (cf_publish_dst * len(dsts))()
    for i, (pl, rd, ak) in enumerate(dsts):
        arr[i] = cf_publish_dst(_p(pl), _p(rd), _p(ak))
    return torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)


def enc_publish_buffer_array(sets, device) -> torch.Tensor:
    """Device array of cf_enc_publish_buffer from
    [(x, recon_s, err, codes_offset, scales_offset), ...]."""
    arr = (cf_enc_publish_buffer * len(sets))()
    for i, (x, r, e, co, so) in enumerate(sets):
        arr[i] = cf_enc_publish_buffer(_p(x), _p(r), _p(e), int(co), int(so))
    return torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)


def dec_wait_buffer_array(sets, device) -> torch.Tensor:
    """Device array of cf_dec_wait_buffer from [(codes, scales, recon_r, ready), ...]."""
    arr = (cf_dec_wait_buffer * len(sets))()
    for i, t in enumerate(sets):
        arr[i] = cf_dec_wait_buffer(*[_p(v) for v in t])
    return torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)


def pointer_array(ptrs, device) -> torch.Tensor:
    """Device array of raw pointers (uint64) from tensors or ints."""
    return torch.tensor([_p(t) for t in ptrs], dtype=torch.int64).to(device)


def dec_emit_buffer_array(sets, device) -> torch.Tensor:
    """Device array of cf_dec_emit_buffer from [(codes, scales, recon_r, out), ...]."""
    arr = (cf_dec_emit_buffer * len(sets))()
    for i, (c, s, r, o) in enumerate(sets):
        arr[i] = cf_dec_emit_buffer(_p(c), _p(s), _p(r), _p(o))
    host = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8)
    return host.to(device)


def bf16_as_u16(x: torch.Tensor) -> torch.Tensor:
    """View a bf16 tensor as its 16-bit patterns (no copy)."""
    return x.view(torch.int16)
