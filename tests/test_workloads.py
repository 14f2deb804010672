"""The seeded synthetic workloads: shapes, determinism and the stated drift
statistics (per-channel lognormal gain, 1% x20 outlier channels, drift
sigma, AR(1) correlation, rank-16 low-rank drift)."""
import math

import numpy as np
import torch

from activation_residual_compression_cf_b200 import workloads as W


def test_five_workloads_have_the_stated_shapes():
    w = W.WORKLOADS
    assert (w["tiny"].tokens, w["tiny"].channels, w["tiny"].buffers, w["tiny"].steps) == (256, 64, 1, 8)
    assert (w["flux_sp"].tokens, w["flux_sp"].channels, w["flux_sp"].buffers) == (1024, 3072, 114)
    assert (w["flux_full"].tokens, w["flux_full"].channels, w["flux_full"].bits) == (4096, 3072, 1)
    assert w["cogvideox"].tokens == 13 * 45 * 30 and w["cogvideox"].channels == 1920
    assert w["cogvideox"].steps == 50 and w["cogvideox"].buffers == 60
    assert (w["lowrank"].rank, w["lowrank"].iters, w["lowrank"].steps) == (32, 2, 28)


def test_deterministic_per_buffer():
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=8, channels=64)
    a = W.trajectory(wl, 3, steps=3)
    b = W.trajectory(wl, 3, steps=3)
    c = W.trajectory(wl, 4, steps=3)
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert a.dtype == torch.bfloat16 and a.shape == (3, 8, 64)


def test_outlier_channels_and_gain():
    wl = W.WORKLOADS["flux_sp"]
    g = W.channel_gain(wl, 0)
    ref = W.channel_gain(W.replace(wl, outlier_frac=0.0), 0)
    ratio = (g / ref)
    assert int(torch.isclose(ratio, torch.tensor(20.0)).sum()) == round(0.01 * wl.channels)
    lg = torch.log(ref)
    assert abs(float(lg.std()) - wl.gain_sigma) < 0.05


def test_drift_sigma_and_ar1():
    wl = W.replace(W.WORKLOADS["cogvideox"], tokens=512, channels=256)
    tr = W.Trajectory(wl, 0)
    xs = [tr.next().float() for _ in range(4)]
    g = tr.gain
    d1 = (xs[2] - xs[1]) / (wl.drift * g)
    d2 = (xs[3] - xs[2]) / (wl.drift * g)
    assert abs(float(d1.std()) - 1.0) < 0.1       # bf16 rounding adds a little
    rho = float((d1 * d2).mean() / (d1.std() * d2.std()))
    assert abs(rho - wl.ar_rho) < 0.1


def test_lowrank_drift_is_rank16_plus_noise():
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=256, channels=192)
    tr = W.Trajectory(wl, 0)
    tr.next()
    m0 = tr.m.clone()
    tr.next()
    d = (tr.m - m0).double().numpy()
    s = np.linalg.svd(d, compute_uv=False)
    noise_edge = wl.noise * (math.sqrt(256) + math.sqrt(192))
    assert s[15] > 5 * noise_edge and s[16] < 1.2 * noise_edge
    om = W.omega(wl, 0, 1)
    assert om.shape == (192, 32) and om.dtype == torch.float32
