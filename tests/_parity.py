"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerances (from the stated acceptance bar of the method's hot path):
  * packed codes bit-exact, except elements whose residual (as the oracle
    computes it) lies within 1e-5 * scale of a decision threshold, and at
    most 1e-5 of all elements may differ;
  * per-token scales within 1e-6 relative;
  * reconstructions and error buffers within 1e-5 relative, measured per
    token row against the row's largest |value| (elementwise relative error
    is meaningless at values near zero).
"""
import numpy as np
import torch

import oracle
from activation_residual_compression_cf_b200 import cf

CODE_BAND = 1e-5
CODE_FRAC = 1e-5
SCALE_RTOL = 1e-6
STATE_RTOL = 1e-5


def unpack(codes_u32: np.ndarray, C: int, bits: int) -> np.ndarray:
    T = codes_u32.shape[0]
    b = np.unpackbits(codes_u32.view(np.uint8).reshape(T, -1), axis=1, bitorder="little")
    b = b[:, : C * bits].reshape(T, C, bits).astype(np.uint8)
    return sum(b[:, :, i] << i for i in range(bits))


def thresholds(bits, scale):
    if bits == 1:
        return np.zeros((scale.shape[0], 1), np.float64)
    a = scale.astype(np.float64)[:, None]
    return np.concatenate([-0.5 * a, 0 * a, 0.5 * a], axis=1)


def compare_step(bits, v_oracle, ora, gpu, stats=None):
    """ora/gpu: dicts with codes (uint32 [T,W]), scales [T], err [T,C],
    recon_s [T,C] and optionally recon_r.  Raises AssertionError on a
    violation; returns the number of differing codes."""
    T, C = v_oracle.shape
    sc_o, sc_g = ora["scales"], gpu["scales"]
    assert np.all(np.abs(sc_g.astype(np.float64) - sc_o) <= SCALE_RTOL * np.abs(sc_o) + 1e-37), \
        f"scale mismatch: max rel {np.max(np.abs(sc_g - sc_o) / np.maximum(np.abs(sc_o), 1e-30))}"
    co, cg = unpack(ora["codes"], C, bits), unpack(gpu["codes"], C, bits)
    diff = co != cg
    nd = int(diff.sum())
    if nd:
        th = thresholds(bits, sc_o)
        near = np.min(np.abs(v_oracle.astype(np.float64)[:, :, None] - th[:, None, :]), axis=2)
        band = CODE_BAND * np.abs(sc_o.astype(np.float64))[:, None]
        assert np.all(near[diff] <= band[np.nonzero(diff)[0], 0]), "code differs away from a threshold"
        assert nd <= CODE_FRAC * T * C, f"{nd} codes differ (> {CODE_FRAC} of {T * C})"
    # padding bits beyond C*bits must be zero on the GPU too
    W = gpu["codes"].shape[1]
    if W * 32 > C * bits:
        pb = np.unpackbits(gpu["codes"].view(np.uint8).reshape(T, -1), axis=1, bitorder="little")
        assert not np.any(pb[:, C * bits:]), "non-zero padding bits"
    for key in ("recon_s", "err", "recon_r"):
        if key not in gpu:
            continue
        ref = ora["recon_s"] if key == "recon_r" else ora[key]
        o, g = ref.astype(np.float64), gpu[key].astype(np.float64)
        rowmax = np.max(np.abs(ref.astype(np.float64)), axis=1, keepdims=True) if C else 0
        assert np.all(np.abs(g - o) <= STATE_RTOL * rowmax + 1e-37), \
            f"{key} mismatch: max abs diff {np.max(np.abs(g - o))}"
    if stats is not None:
        stats["code_diffs"] = stats.get("code_diffs", 0) + nd
        stats["elems"] = stats.get("elems", 0) + T * C
        stats["recon_exact"] = stats.get("recon_exact", True) and np.array_equal(
            ora["recon_s"].view(np.uint32), gpu["recon_s"].view(np.uint32))
    return nd


def f32_of(bits_u16):
    return (bits_u16.astype(np.uint32) << 16).view(np.float32)


class GpuBuffer:
    """Device state for one buffer (sender + receiver) driven through the C ABI."""

    def __init__(self, T, C, bits, dev="cuda"):
        self.d = cf.desc(T, C, bits)
        self.T, self.C, self.bits = T, C, bits
        W = (C * bits + 31) // 32
        f32 = dict(dtype=torch.float32, device=dev)
        self.recon_s = torch.empty(T, C, **f32)
        self.recon_r = torch.empty(T, C, **f32)
        self.err = torch.empty(T, C, **f32)
        self.codes = torch.empty(T, W, dtype=torch.int32, device=dev)
        self.scales = torch.empty(T, **f32)

    def init(self, x0):
        cf.cf_state_init(self.d, x0.view(torch.int16), self.recon_s, self.err)
        cf.cf_state_init(self.d, x0.view(torch.int16), self.recon_r, None)

    def step(self, x):
        cf.cf_encode(self.d, x.view(torch.int16), self.recon_s, self.err, self.codes, self.scales)
        cf.cf_decode(self.d, self.codes, self.scales, self.recon_r)

    def host(self):
        torch.cuda.synchronize()
        return dict(codes=self.codes.cpu().numpy().view(np.uint32),
                    scales=self.scales.cpu().numpy(), err=self.err.cpu().numpy(),
                    recon_s=self.recon_s.cpu().numpy(), recon_r=self.recon_r.cpu().numpy())


def oracle_step(x_bits, recon_s, bits):
    """Runs the oracle on copies; returns (v, outputs dict) with recon_s updated."""
    v = (f32_of(x_bits) - recon_s).astype(np.float32)
    codes, scales, err = oracle.encode(x_bits, recon_s, bits)
    return v, dict(codes=codes, scales=scales, err=err, recon_s=recon_s.copy())


def compare_step_exact_first(bits, v_oracle, ora, gpu, stats=None):
    """compare_step, with a fast path: when codes, scales, err and recon_s
    are bit-identical (the usual case: the only non-exact step is the fp64
    order of the 1-bit sum), the bar is met without the elementwise work.
    Returns the number of differing codes."""
    same = all(np.array_equal(np.ascontiguousarray(gpu[k]).view(np.uint32),
                              np.ascontiguousarray(ora[k]).view(np.uint32))
               for k in ("codes", "scales", "err", "recon_s"))
    if same:
        if stats is not None:
            stats["elems"] = stats.get("elems", 0) + v_oracle.size
            stats["exact_steps"] = stats.get("exact_steps", 0) + 1
        return 0
    return compare_step(bits, v_oracle, ora, gpu, stats)
