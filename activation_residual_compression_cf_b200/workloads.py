"""Seeded synthetic workloads: the activation trajectories both the CUDA path
and the CPU oracle are fed.

This module generates inputs only.  It holds none of the compression
arithmetic, and it is the one piece of code the oracle side and the CUDA
side share (tests hand the same arrays to both).

The pages measure on FLUX.1-dev image generation with COCO Captions 2014
prompts and on CogVideoX-2b with VBench ("Experimental setup" of
"Accelerating Parallel Diffusion Model Serving with Residual Compression").
Neither the weights nor the datasets exist here, so a synthetic drift model
stands in for real activations with the shapes of those models' exchanged
K/V buffers:

  g_c          per-channel gain, lognormal(0, gain_sigma), drawn once per
               buffer (optionally 1% of channels x20 outliers)
  m_0 = xi * g                      xi ~ N(0, 1) elementwise
  m_t = m_{t-1} + drift * n_t * g   n_t ~ N(0, 1), or AR(1) over steps:
                                    n_t = rho n_{t-1} + sqrt(1 - rho^2) xi_t
  x_t = bf16_rne(m_t)

The low-rank workload instead drifts by a rank-16 signal plus noise:
  m_t = m_{t-1} + U_t W_t^T + noise * xi_t,
  U_t ~ N(0,1) [T,16],  W_t ~ N(0, signal_rms^2 / 16) [C,16]
and its subspace-iteration start Omega ~ N(0,1) [C, rank] is drawn per
(buffer, step) and passed to both sides as an input.

Every buffer has its own torch.Generator seeded from (seed, workload,
buffer), so any single buffer can be regenerated alone.  CPU and CUDA
generators give different streams: parity tests generate on one device and
copy the same tensor to the other side.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    tokens: int
    channels: int
    buffers: int
    steps: int               # including the uncompressed warmup step 0
    mode: str                # "quant" or "lowrank"
    bits: int = 0            # quant mode: 1 or 2
    rank: int = 0            # lowrank mode
    iters: int = 0           # lowrank mode: subspace iterations
    gain_sigma: float = 0.5
    drift: float = 0.05
    outlier_frac: float = 0.0
    outlier_gain: float = 1.0
    ar_rho: float = 0.0
    signal_rank: int = 0
    signal_rms: float = 0.0
    noise: float = 0.0
    note: str = ""

    @property
    def elems(self) -> int:
        return self.tokens * self.channels


# The five workloads: a tiny parity case, a FLUX-like 4-way sequence-parallel
# shard, a FLUX-like full sequence, a CogVideoX-like video latent and the
# low-rank mode on the full FLUX sequence.
WORKLOADS = {
    "tiny": Workload("tiny", 256, 64, 1, 8, "quant", bits=1, gain_sigma=0.5,
                     drift=0.05, note="1-bit mean-abs + EF"),
    "flux_sp": Workload("flux_sp", 1024, 3072, 114, 28, "quant", bits=2,
                        gain_sigma=0.5, drift=0.03, outlier_frac=0.01,
                        outlier_gain=20.0, note="2-bit absmax + EF, 1% x20 outlier channels"),
    "flux_full": Workload("flux_full", 4096, 3072, 114, 28, "quant", bits=1,
                          gain_sigma=0.7, drift=0.05, note="1-bit mean-abs + EF"),
    "cogvideox": Workload("cogvideox", 17550, 1920, 60, 50, "quant", bits=2,
                          gain_sigma=0.5, drift=0.02, ar_rho=0.9,
                          note="2-bit absmax + EF, AR(1) drift over steps; tokens = 13x45x30"),
    "lowrank": Workload("lowrank", 4096, 3072, 114, 28, "lowrank", rank=32,
                        iters=2, gain_sigma=0.7, drift=0.05, signal_rank=16,
                        signal_rms=0.1, noise=0.01,
                        note="rank 32, 2 iterations, INT4 factors + EF"),
}

_NAME_IDS = {n: i for i, n in enumerate(WORKLOADS)}


def replace(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some fields changed (e.g. fewer buffers)."""
    return dataclasses.replace(wl, **kw)


def _seed(seed: int, wl: Workload, buffer: int, salt: int = 0) -> int:
    # Simple deterministic mix; any injective-enough function will do.
    h = (seed * 1_000_003 + _NAME_IDS.get(wl.name, 97) * 10_007 + buffer) * 31 + salt
    return h % (2**63 - 1)


def _gen(device, s: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def channel_gain(wl: Workload, buffer: int, device="cpu", seed: int = 0) -> torch.Tensor:
    g = _gen(device, _seed(seed, wl, buffer, salt=1))
    gain = torch.exp(wl.gain_sigma * torch.randn(wl.channels, generator=g, device=device))
    if wl.outlier_frac > 0:
        n_out = int(round(wl.outlier_frac * wl.channels))
        idx = torch.randperm(wl.channels, generator=g, device=device)[:n_out]
        gain[idx] *= wl.outlier_gain
    return gain


class Trajectory:
    """The activation trajectory of one buffer: call ``next()`` for x_0,
    x_1, ... (bf16 [T, C]) on ``device``."""

    def __init__(self, wl: Workload, buffer: int, device="cpu", seed: int = 0):
        self.wl, self.buffer, self.device, self.seed = wl, buffer, device, seed
        self.gain = channel_gain(wl, buffer, device, seed)
        self.gen = _gen(device, _seed(seed, wl, buffer, salt=2))
        self.m = None
        self.ar = None
        self.t = 0

    def _randn(self, *shape):
        return torch.randn(*shape, generator=self.gen, device=self.device)

    def next(self) -> torch.Tensor:
        wl = self.wl
        T, C = wl.tokens, wl.channels
        if self.m is None:
            self.m = self._randn(T, C) * self.gain
        elif wl.mode == "lowrank":
            k = wl.signal_rank
            u = self._randn(T, k)
            w = self._randn(C, k) * (wl.signal_rms / math.sqrt(k))
            self.m += u @ w.T
            self.m += wl.noise * self._randn(T, C)
        else:
            xi = self._randn(T, C)
            if wl.ar_rho > 0:
                if self.ar is None:
                    self.ar = xi
                else:
                    self.ar.mul_(wl.ar_rho).add_(xi, alpha=math.sqrt(1 - wl.ar_rho**2))
                n = self.ar
            else:
                n = xi
            self.m += wl.drift * n * self.gain
        self.t += 1
        return self.m.to(torch.bfloat16)


def trajectory(wl: Workload, buffer: int, steps: int | None = None, device="cpu",
               seed: int = 0) -> torch.Tensor:
    """All steps of one buffer as one bf16 tensor [steps, T, C]."""
    steps = wl.steps if steps is None else steps
    tr = Trajectory(wl, buffer, device, seed)
    out = torch.empty((steps, wl.tokens, wl.channels), dtype=torch.bfloat16, device=device)
    for s in range(steps):
        out[s] = tr.next()
    return out


def omega(wl: Workload, buffer: int, step: int, device="cpu", seed: int = 0) -> torch.Tensor:
    """Gaussian start block for subspace iteration, fp32 [C, rank], drawn per
    (buffer, step) and handed to both implementations."""
    g = _gen(device, _seed(seed, wl, buffer, salt=1000 + step))
    return torch.randn(wl.channels, wl.rank, generator=g, device=device)


def bf16_bits(x: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy), for the oracle."""
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
