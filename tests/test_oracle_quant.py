"""Pins for the quantize-mode oracle (CPU only).

Each test checks the oracle against something other than its own formula:
invariants the method must satisfy (the error-feedback identity, a zero
residual leaving the reconstruction unchanged, sender/receiver agreement),
brute force (nearest reconstruction level), a library routine (math.fsum for
the mean-abs scale, np.unpackbits for the bit layout), perturbation
optimality of the scale, and hand-worked golden rows.

Method source: "Accelerating Parallel Diffusion Model Serving with Residual
Compression" -- "Approach" (residual against the previous reconstruction,
sender-side error feedback) and the "Measured effects" table (1-bit and 2-bit
variants, 1-step warmup).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from activation_residual_compression_cf_b200 import workloads as W
from conftest import GOLDEN


def _bits_from_f32(a):
    """bf16 bit patterns of float32 values that are exactly representable."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "values must be exact bf16"
    return (u >> 16).astype(np.uint16)


def _f32_from_bits(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def _ulp32(a):
    a = np.abs(np.asarray(a, np.float32))
    return np.spacing(a).astype(np.float64)


def _unpack_codes(codes, C, bits):
    """Independent unpack: numpy's little-endian bit order over the word bytes."""
    T = codes.shape[0]
    b = np.unpackbits(codes.view(np.uint8).reshape(T, -1), axis=1, bitorder="little")
    b = b[:, : C * bits].reshape(T, C, bits).astype(np.uint32)
    return sum(b[:, :, i] << i for i in range(bits))


def _traj(name, buffer=0, steps=None, **kw):
    wl = W.replace(W.WORKLOADS[name], **kw) if kw else W.WORKLOADS[name]
    xs = W.trajectory(wl, buffer, steps=steps, device="cpu")
    return wl, [W.bf16_bits(x) for x in xs]


def test_init_is_exact_and_error_is_zero():
    _, xs = _traj("tiny", steps=1)
    recon, err = oracle.state_init(xs[0])
    assert np.array_equal(recon, _f32_from_bits(xs[0]))
    assert not np.any(err)


@pytest.mark.parametrize("bits", [1, 2])
def test_golden_hand_row(bits):
    g = json.load(open(os.path.join(GOLDEN, "quant_hand_cases.json")))
    row = np.array(g["residual_row"], np.float32)[None, :]
    exp = g[f"bits{bits}"]
    recon = np.zeros_like(row)
    codes, scales, err = oracle.encode(_bits_from_f32(row), recon, bits)
    assert scales[0] == np.float32(exp["scale"])
    assert int(codes[0, 0]) == exp["packed_word0"]
    assert np.array_equal(_unpack_codes(codes, row.shape[1], bits)[0], exp["codes"])
    assert np.array_equal(recon[0], np.array(exp["deq"], np.float32))
    assert np.array_equal(err[0], np.array(exp["err"], np.float32))


@pytest.mark.parametrize("name", ["tiny", "flux_sp"])
def test_error_feedback_identity_and_mirror(name):
    """recon_s + err == x after every step, within the three fp32 roundings
    (residual, error, mirror update); the receiver's decode tracks the sender
    bit for bit."""
    kw = {} if name == "tiny" else dict(tokens=32, buffers=1)
    wl, xs = _traj(name, steps=6, **kw)
    recon_s, _ = oracle.state_init(xs[0])
    recon_r = recon_s.copy()
    for x in xs[1:]:
        xf = _f32_from_bits(x).astype(np.float64)
        v32 = (_f32_from_bits(x) - recon_s).astype(np.float32)
        codes, scales, err = oracle.encode(x, recon_s, wl.bits)
        bound = 0.5 * (_ulp32(v32) + _ulp32(err) + _ulp32(recon_s))
        gap = np.abs(recon_s.astype(np.float64) + err.astype(np.float64) - xf)
        assert np.all(gap <= bound * (1 + 1e-12) + 1e-300)
        oracle.decode(codes, scales, recon_r, wl.bits)
        assert np.array_equal(recon_r.view(np.uint32), recon_s.view(np.uint32))


@pytest.mark.parametrize("bits", [1, 2])
def test_zero_residual_leaves_reconstruction_unchanged(bits):
    _, xs = _traj("tiny", steps=1)
    recon, _ = oracle.state_init(xs[0])
    before = recon.copy()
    codes, scales, err = oracle.encode(xs[0], recon, bits)
    assert np.array_equal(recon.view(np.uint32), before.view(np.uint32))
    assert not np.any(scales) and not np.any(err)


def test_one_bit_code_is_sign_of_residual():
    """bit == [x >= recon], decided on the inputs in fp64 (exact), never on
    the oracle's fp32 residual: rounding cannot flip the sign of a
    difference of two finite floats."""
    wl, xs = _traj("tiny", steps=3)
    recon, _ = oracle.state_init(xs[0])
    for x in xs[1:]:
        sign = (_f32_from_bits(x).astype(np.float64) >= recon.astype(np.float64))
        codes, _, _ = oracle.encode(x, recon, 1)
        assert np.array_equal(_unpack_codes(codes, wl.channels, 1), sign.astype(np.uint32))


def test_one_bit_scale_is_mean_abs_and_l2_optimal():
    wl, xs = _traj("tiny", steps=2)
    recon, _ = oracle.state_init(xs[0])
    v = (_f32_from_bits(xs[1]) - recon).astype(np.float32)
    codes, scales, _ = oracle.encode(xs[1], recon, 1)
    C = wl.channels
    for t in range(wl.tokens):
        exact = np.float32(np.float32(math.fsum(abs(float(a)) for a in v[t])) / np.float32(C))
        assert abs(float(scales[t]) - float(exact)) <= float(np.spacing(exact))
        # first-order optimality of the scale for sign codes
        sgn = np.where(v[t] >= 0, 1.0, -1.0)
        e = lambda s: float(np.sum((v[t].astype(np.float64) - s * sgn) ** 2))
        s = float(scales[t])
        assert e(s) <= e(s * (1 + 1e-3)) and e(s) <= e(s * (1 - 1e-3))


def test_two_bit_is_nearest_level_brute_force():
    """Every 2-bit reconstruction is the nearest of the four levels
    {-3A/4, -A/4, A/4, 3A/4} (ties to the upper level), A = row absmax,
    and the layout matches numpy's little-endian bit order."""
    wl, xs = _traj("flux_sp", steps=2, tokens=16)
    recon, _ = oracle.state_init(xs[0])
    v = (_f32_from_bits(xs[1]) - recon).astype(np.float32)
    r0 = recon.copy()
    codes, scales, err = oracle.encode(xs[1], recon, 2)
    A = np.max(np.abs(v), axis=1)
    assert np.array_equal(scales, A)
    lv = np.array([-0.75, -0.25, 0.25, 0.75], np.float32)
    levels = (lv[None, :] * A[:, None]).astype(np.float32)              # [T,4]
    dist = np.abs(v[:, :, None].astype(np.float64) - levels[:, None, :])  # [T,C,4]
    best = np.min(dist, axis=2, keepdims=True)
    # highest index among the minimisers = tie to the upper level
    k = 3 - np.argmax((dist == best)[:, :, ::-1], axis=2)
    assert np.array_equal(_unpack_codes(codes, wl.channels, 2), k.astype(np.uint32))
    deq = levels[np.arange(k.shape[0])[:, None], k]
    assert np.array_equal(recon, (r0 + deq).astype(np.float32))
    assert np.all(np.abs(err) <= A[:, None] / 4 * (1 + 1e-6))


@pytest.mark.parametrize("C,bits", [(40, 1), (20, 2), (33, 1), (1, 2), (64, 2)])
def test_tail_padding_is_zero(C, bits):
    rng = np.random.default_rng(1)
    row = rng.standard_normal((3, C)).astype(np.float32)
    x = _bits_from_f32((row.view(np.uint32) & 0xFFFF0000).view(np.float32))
    recon = np.zeros((3, C), np.float32)
    codes, _, _ = oracle.encode(x, recon, bits)
    assert codes.shape[1] == (C * bits + 31) // 32
    b = np.unpackbits(codes.view(np.uint8).reshape(3, -1), axis=1, bitorder="little")
    assert not np.any(b[:, C * bits:])


def test_empty_rows():
    x = np.zeros((0, 64), np.uint16)
    recon = np.zeros((0, 64), np.float32)
    codes, scales, err = oracle.encode(x, recon, 1)
    assert codes.shape == (0, 2) and scales.shape == (0,)


def test_unsupported_bits_rejected():
    x = np.zeros((2, 32), np.uint16)
    with pytest.raises(ValueError):
        oracle.encode(x, np.zeros((2, 32), np.float32), 3)


def test_error_feedback_keeps_error_bounded():
    """Qualitative claim of the pages ("Approach", "Surprising findings"): with
    error feedback the reconstruction stays close to the true trajectory.
    Over all compressed steps of the tiny workload the error buffer norm
    stays within a small factor of the first step's, i.e. does not grow
    with the number of steps."""
    wl, xs = _traj("tiny")
    recon, _ = oracle.state_init(xs[0])
    norms = []
    for x in xs[1:]:
        _, _, err = oracle.encode(x, recon, wl.bits)
        norms.append(float(np.linalg.norm(err)))
    assert max(norms) <= 3.0 * norms[0]


def test_payload_ratio_closed_form():
    # 1-bit: 16 bits of bf16 -> 1 bit + 32 bits of scale per token
    assert oracle.quant_payload_bytes(1024, 3072, 1) == 1024 * (3072 // 8 + 4)
    r1 = 2 * 1024 * 3072 / oracle.quant_payload_bytes(1024, 3072, 1)
    assert abs(r1 - 16 / (1 + 32 / 3072)) < 1e-9


def test_bf16_rounding_matches_torch_and_ties_to_even():
    """The emitted bf16 reconstruction is round-to-nearest-even: checked
    against torch's CPU conversion (a library routine) on random values and on
    hand-picked ties."""
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(2000).astype(np.float32) * 10 ** rng.uniform(-30, 30, 2000).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, np.inf, -np.inf], np.float32)])
    ties = np.array([0x3f808000, 0x3f818000, 0xbf808000, 0x3f80c000], np.uint32).view(np.float32)
    vals = np.concatenate([vals, ties])
    ours = oracle.f32_to_bf16_bits(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # 1.00390625 = 0x3F808000 is a tie between 0x3F80 and 0x3F81: even -> 0x3F80
    assert ours[-4] == 0x3F80 and ours[-3] == 0x3F82 and ours[-2] == 0xBF80 and ours[-1] == 0x3F81
    nan = oracle.f32_to_bf16_bits(np.array([np.nan], np.float32))[0]
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x7F)


def test_decode_emit_is_decode_then_bf16():
    wl, xs = _traj("tiny", steps=2)
    recon_s, _ = oracle.state_init(xs[0])
    recon_r = recon_s.copy()
    codes, scales, _ = oracle.encode(xs[1], recon_s, 1)
    out = oracle.decode_emit(codes, scales, recon_r, 1)
    assert np.array_equal(recon_r, recon_s)
    ref = torch.from_numpy(recon_r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out, ref)


@pytest.mark.parametrize("name", ["tiny", "flux_sp"])
def test_delta_state_first_step_equals_standard_sender(name):
    """At the first compressed step after the warmup (err = 0, x_prev = x_0
    = recon_s) the delta-state residual ((x - x_prev) + 0) is the standard
    residual x - recon_s rounded once: codes, scales and err are identical."""
    kw = {} if name == "tiny" else dict(tokens=48, buffers=1)
    wl, xs = _traj(name, steps=2, **kw)
    recon_s, err0 = oracle.state_init(xs[0])
    c_std, s_std, e_std = oracle.encode(xs[1], recon_s, wl.bits)
    err = err0.copy()
    c_del, s_del = oracle.encode_delta(xs[1], xs[0], err, wl.bits)
    assert np.array_equal(c_std, c_del) and np.array_equal(s_std, s_del)
    assert np.array_equal(e_std.view(np.uint32), err.view(np.uint32))


@pytest.mark.parametrize("name", ["tiny", "flux_sp"])
def test_delta_state_ef_identity_drifts_only_by_its_roundings(name):
    """Delta-state bookkeeping: recon_r + err - x_t changes per step by
    exactly the four fp32 roundings of the step (x_t - x_prev, + err, the
    error, the receiver's add), so |recon_r + err - x_t| stays within their
    accumulated half-ulps (an exact accounting, element by element)."""
    kw = {} if name == "tiny" else dict(tokens=32, buffers=1)
    wl, xs = _traj(name, steps=8, **kw)
    recon_r, err = oracle.state_init(xs[0])
    bound = np.zeros(recon_r.shape, np.float64)
    for t in range(1, len(xs)):
        d1 = (_f32_from_bits(xs[t]) - _f32_from_bits(xs[t - 1])).astype(np.float32)
        v = (d1 + err).astype(np.float32)
        codes, scales = oracle.encode_delta(xs[t], xs[t - 1], err, wl.bits)
        oracle.decode(codes, scales, recon_r, wl.bits)
        bound += 0.5 * (_ulp32(d1) + _ulp32(v) + _ulp32(err) + _ulp32(recon_r))
        gap = np.abs(recon_r.astype(np.float64) + err.astype(np.float64)
                     - _f32_from_bits(xs[t]).astype(np.float64))
        assert np.all(gap <= bound * (1 + 1e-12) + 1e-300)
        assert np.all(np.abs(err) <= np.abs(v) + (scales[:, None] if wl.bits == 1 else 0.25 * scales[:, None]) + 1e-30)


@pytest.mark.parametrize("bits", [1, 2])
def test_delta_state_zero_residual(bits):
    """x_t == x_prev with err = 0 gives v = 0: zero scales, zero error, and a
    receiver that does not move."""
    _, xs = _traj("tiny", steps=1)
    _, err = oracle.state_init(xs[0])
    codes, scales = oracle.encode_delta(xs[0], xs[0], err, bits)
    assert not np.any(scales) and not np.any(err)
    recon_r, _ = oracle.state_init(xs[0])
    before = recon_r.copy()
    oracle.decode(codes, scales, recon_r, bits)
    assert np.array_equal(recon_r.view(np.uint32), before.view(np.uint32))
