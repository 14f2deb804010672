"""GPU parity of the quantize-mode kernels (cf_encode / cf_decode and the
batched forms) against the CPU oracle, through the C ABI.

Sizes: every workload shape, small enough for the oracle to finish in
seconds yet spanning many rows and a ragged tail of channel groups; the
scalar path (channels not a multiple of 8); the largest supported row; an
empty problem; and the full FLUX-like step (114 buffers in one batched
launch, as bench.py times it) checked on sampled buffers against the oracle
and on all buffers through properties that hold at any size.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W

from _parity import GpuBuffer, compare_step, oracle_step

pytestmark = pytest.mark.gpu


def _run_trajectory(wl, buffer, steps, stats=None):
    xs = W.trajectory(wl, buffer, steps=steps, device="cuda")
    xb = [W.bf16_bits(x) for x in xs]
    g = GpuBuffer(wl.tokens, wl.channels, wl.bits)
    g.init(xs[0].clone())
    recon_o, _ = oracle.state_init(xb[0])
    h = g.host()
    assert np.array_equal(h["recon_s"], recon_o) and not np.any(h["err"])
    for s in range(1, steps):
        g.step(xs[s].clone())          # a fresh allocation is 16-byte aligned
        v, ora = oracle_step(xb[s], recon_o, wl.bits)
        gh = g.host()
        compare_step(wl.bits, v, ora, gh, stats)
        # receiver tracks sender bit for bit on the GPU
        assert np.array_equal(gh["recon_r"].view(np.uint32), gh["recon_s"].view(np.uint32))
        # free-running: the oracle continues from its own state
    return stats


def test_tiny_full_trajectory():
    stats = _run_trajectory(W.WORKLOADS["tiny"], 0, 8, {})
    assert stats["code_diffs"] == 0


@pytest.mark.parametrize("name,tokens", [("flux_sp", 96), ("flux_full", 80), ("cogvideox", 70)])
def test_workload_shapes_trajectory(name, tokens):
    wl = W.replace(W.WORKLOADS[name], tokens=tokens)
    _run_trajectory(wl, 1, 5, {})


@pytest.mark.parametrize("T,C,bits", [
    (37, 3072, 1), (37, 3072, 2), (50, 1920, 1), (19, 200, 2), (64, 64, 2),
    (13, 33, 2), (9, 33, 1), (5, 1, 1), (6, 7, 2), (11, 1000, 1),   # scalar path: C % 8 != 0
    (3, 16384, 1), (3, 16384, 2),                                   # largest supported row
])
def test_shapes_and_ragged_tails(T, C, bits):
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, channels=C, bits=bits)
    _run_trajectory(wl, 0, 3, {})


def test_empty_tokens_is_noop():
    g = GpuBuffer(0, 64, 1)
    g.step(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()


def test_zero_residual_on_gpu():
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=16)
    x = W.trajectory(wl, 0, steps=1, device="cuda")[0]
    for bits in (1, 2):
        g = GpuBuffer(16, 3072, bits)
        g.init(x)
        before = g.host()["recon_s"].copy()
        g.step(x)
        h = g.host()
        assert np.array_equal(h["recon_s"], before) and np.array_equal(h["recon_r"], before)
        assert not np.any(h["scales"]) and not np.any(h["err"])


@pytest.mark.parametrize("bits", [1, 2])
def test_launch_shapes_agree_bitwise(bits):
    """Every launch shape the override allows gives the same bits."""
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=64, bits=bits)
    xs = W.trajectory(wl, 2, steps=2, device="cuda")
    ref = None
    try:
        for gpt, thr, bps in [(0, 0, 0), (3, 128, 0), (4, 96, 0), (2, 192, 2), (1, 384, 1), (4, 128, 0)]:
            cf.cf_set_launch_override(0, gpt, thr, bps)
            cf.cf_set_launch_override(1, gpt, thr, bps)
            g = GpuBuffer(64, 3072, bits)
            g.init(xs[0])
            g.step(xs[1])
            h = g.host()
            if ref is None:
                ref = h
            for k in ("codes", "scales", "err", "recon_s", "recon_r"):
                assert np.array_equal(h[k].view(np.uint8), ref[k].view(np.uint8)), (gpt, thr, k)
    finally:
        cf.cf_set_launch_override(0, 0, 0, 0)
        cf.cf_set_launch_override(1, 0, 0, 0)


@pytest.mark.parametrize("T,C,bits", [(64, 3072, 2), (64, 3072, 1), (33, 1920, 2), (17, 256, 1),
                                      (9, 64, 2), (5, 16384, 2), (40, 200, 2)])
@pytest.mark.parametrize("stages", [0, 2, 5])
def test_tma_pipeline_bit_identical(T, C, bits, stages):
    """The TMA row-staging pipeline computes the same bits as the
    register-resident one (and falls back to it where its alignment
    conditions fail, e.g. C = 200 at 2 bits for decode)."""
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, channels=C, bits=bits)
    xs = W.trajectory(wl, 4, steps=3, device="cuda")
    res = []
    try:
        for pipe in (0, 1):
            cf.cf_set_quant_pipeline(0, pipe, stages if pipe else 0)
            cf.cf_set_quant_pipeline(1, pipe, stages if pipe else 0)
            g = GpuBuffer(T, C, bits)
            g.init(xs[0].clone())
            g.step(xs[1].clone())
            g.step(xs[2].clone())
            res.append(g.host())
    finally:
        cf.cf_set_quant_pipeline(0, 1, 0)   # the library default
        cf.cf_set_quant_pipeline(1, 1, 0)
    for k in ("codes", "scales", "err", "recon_s", "recon_r"):
        assert np.array_equal(res[0][k].view(np.uint8), res[1][k].view(np.uint8)), k


def test_host_pointer_is_rejected():
    d = cf.desc(4, 64, 1)
    host = torch.zeros(4, 64)
    dev = torch.zeros(4, 64, device="cuda")
    with pytest.raises(cf.CFError) as ei:
        cf.cf_encode(d, host.view(torch.int16), dev, dev, dev, dev)
    assert ei.value.status == 1


def _batched_state(wl, n, dev="cuda"):
    T, C = wl.tokens, wl.channels
    Wd = (C * wl.bits + 31) // 32
    f32 = dict(dtype=torch.float32, device=dev)
    st = dict(recon_s=torch.empty(n, T, C, **f32), recon_r=torch.empty(n, T, C, **f32),
              err=torch.empty(n, T, C, **f32),
              codes=torch.empty(n, T, Wd, dtype=torch.int32, device=dev),
              scales=torch.empty(n, T, **f32))
    return st


def test_batched_bad_buffer_is_skipped_and_reported():
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=32, buffers=3)
    xs = torch.stack([W.trajectory(wl, b, steps=2, device="cuda") for b in range(3)], 1)  # [S,n,T,C]
    st = _batched_state(wl, 3)
    d = cf.desc(32, 3072, 2)
    for b in range(3):
        cf.cf_state_init(d, xs[0, b].view(torch.int16), st["recon_s"][b], st["err"][b])
    before = st["recon_s"].clone()
    x16 = xs[1].view(torch.int16)
    sets = [(x16[b], st["recon_s"][b], st["err"][b], st["codes"][b], st["scales"][b]) for b in range(3)]
    bad = list(sets[1])
    bad[1] = st["recon_s"][1].data_ptr() + 4           # misaligned recon
    bufs = cf.enc_buffer_array([sets[0], tuple(bad), sets[2]], "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cf.cf_encode_batched(d, 3, bufs, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 2
    assert torch.equal(st["recon_s"][1], before[1])     # skipped buffer untouched
    assert not torch.equal(st["recon_s"][0], before[0])
    bad[1] = 0                                           # null pointer
    bufs = cf.enc_buffer_array([tuple(bad)], "cuda")
    status.zero_()
    cf.cf_encode_batched(d, 1, bufs, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1


@pytest.mark.parametrize("pipe", [0, 1])
@pytest.mark.parametrize("name,steps,sample", [("flux_sp", 3, (0, 57, 113)),
                                               ("flux_full", 2, (0, 113)),
                                               ("cogvideox", 2, (0, 59))])
def test_full_size_batched_step(name, steps, sample, pipe):
    """The bench's launch: all buffers of a step in one batched encode and one
    batched decode.  Sampled buffers are checked against the oracle over all
    steps; every buffer is checked for the EF identity and for
    receiver == sender."""
    wl = W.WORKLOADS[name]
    n, T, C = wl.buffers, wl.tokens, wl.channels
    trs = [W.Trajectory(wl, b, device="cuda") for b in range(n)]
    st = _batched_state(wl, n)
    d = cf.desc(T, C, wl.bits)
    x = torch.stack([t.next() for t in trs])
    for b in range(n):
        cf.cf_state_init(d, x[b].view(torch.int16), st["recon_s"][b], st["err"][b])
        cf.cf_state_init(d, x[b].view(torch.int16), st["recon_r"][b], None)
    recon_o = {b: oracle.state_init(W.bf16_bits(x[b]))[0] for b in sample}
    x_buf = torch.empty_like(x)
    x16 = x_buf.view(torch.int16)
    enc = cf.enc_buffer_array([(x16[b], st["recon_s"][b], st["err"][b], st["codes"][b],
                                st["scales"][b]) for b in range(n)], "cuda")
    dec = cf.dec_buffer_array([(st["codes"][b], st["scales"][b], st["recon_r"][b])
                               for b in range(n)], "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cf.cf_set_quant_pipeline(0, pipe, 0)
    cf.cf_set_quant_pipeline(1, pipe, 0)
    try:
        _full_size_steps(wl, d, n, steps, sample, trs, st, x_buf, enc, dec, status, recon_o)
    finally:
        cf.cf_set_quant_pipeline(0, 1, 0)   # the library default
        cf.cf_set_quant_pipeline(1, 1, 0)


def _full_size_steps(wl, d, n, steps, sample, trs, st, x_buf, enc, dec, status, recon_o):
    for s in range(1, steps):
        for b in range(n):
            x_buf[b].copy_(trs[b].next())
        v = [x_buf[b].float() - st["recon_s"][b] for b in range(n)]   # one fp32 rounding
        cf.cf_encode_batched(d, n, enc, status)
        cf.cf_decode_batched(d, n, dec, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(st["recon_r"].view(torch.int32), st["recon_s"].view(torch.int32))
        # EF identity per buffer: recon_s + err == x within the three fp32
        # roundings (residual, error, mirror update)
        for b in range(n):
            rs, er, xb = st["recon_s"][b].double(), st["err"][b].double(), x_buf[b].double()
            vb = v[b].double().abs()
            gap = (rs + er - xb).abs()
            bound = (vb + er.abs() + rs.abs()) * 2.0**-24 * (1 + 1e-9) + 3 * 2.0**-149
            assert bool((gap <= bound).all()), b
            del rs, er, xb, vb, gap, bound
        del v
        for b in sample:
            xb = W.bf16_bits(x_buf[b])
            v, ora = oracle_step(xb, recon_o[b], wl.bits)
            gh = dict(codes=st["codes"][b].cpu().numpy().view(np.uint32),
                      scales=st["scales"][b].cpu().numpy(), err=st["err"][b].cpu().numpy(),
                      recon_s=st["recon_s"][b].cpu().numpy())
            compare_step(wl.bits, v, ora, gh)


@pytest.mark.parametrize("pipeline,bits", [(1, 2), (0, 1)])
def test_single_buffer_beyond_2_pow_31_elements(pipeline, bits):
    """One buffer of 700,000 x 3072 = 2.15e9 elements, past 2^31, so every
    element offset beyond row 699,050 needs 64-bit arithmetic (about 35 GB on
    the device).  Rows on both sides of that boundary, the first and last
    rows and random rows are checked against the oracle, which computes rows
    independently; the receiver must equal the sender everywhere."""
    T, C = 700_000, 3072
    assert T * C > 2 ** 31
    gen = torch.Generator(device="cuda").manual_seed(11)
    gain = torch.exp(0.5 * torch.randn(C, device="cuda", generator=gen))
    x0 = (torch.randn(T, C, device="cuda", generator=gen) * gain).to(torch.bfloat16)
    x1 = (x0.float() + 0.05 * gain * torch.randn(T, C, device="cuda", generator=gen)).to(torch.bfloat16)
    cf.cf_set_quant_pipeline(0, pipeline, 0)
    cf.cf_set_quant_pipeline(1, pipeline, 0)
    try:
        g = GpuBuffer(T, C, bits)
        g.init(x0)
        g.step(x1)
        torch.cuda.synchronize()
        assert torch.equal(g.recon_r, g.recon_s)
        edge = 2 ** 31 // C
        rng = np.random.default_rng(5)
        rows = np.unique(np.concatenate([[0, 1, T - 2, T - 1], np.arange(edge - 3, edge + 4),
                                         rng.integers(0, T, 16)]))
        idx = torch.from_numpy(rows).cuda()
        r0, _ = oracle.state_init(W.bf16_bits(x0[idx]))
        v, ora = oracle_step(W.bf16_bits(x1[idx]), r0, bits)
        gpu = dict(codes=g.codes[idx].cpu().numpy().view(np.uint32), scales=g.scales[idx].cpu().numpy(),
                   err=g.err[idx].cpu().numpy(), recon_s=g.recon_s[idx].cpu().numpy())
        compare_step(bits, v, ora, gpu)
    finally:
        cf.cf_set_quant_pipeline(0, 1, 0)
        cf.cf_set_quant_pipeline(1, 1, 0)


@pytest.mark.parametrize("C", [3072, 3068])
def test_rows_pipeline_bad_buffers_between_valid_ones(C):
    """Register-row pipeline (C = 3072 vector path, C = 3068 scalar path)
    with every other buffer of a batched call invalid (null pointer), on a
    grid of one CTA per SM, so each CTA meets valid and skipped rows in turn.
    The valid buffers must equal an all-valid run bit for bit and the oracle
    within the parity bar; a skipped row must not shift the scale slots that
    the next valid row shares with the previous one."""
    n, T = 24, 16
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, channels=C, buffers=n)
    xs = torch.stack([W.trajectory(wl, b, steps=2, device="cuda") for b in range(n)], 1)
    d = cf.desc(T, C, wl.bits)
    x16 = xs[1].view(torch.int16)
    runs = []
    try:
        cf.cf_set_quant_pipeline(0, 0, 0)
        G = (C + 7) // 8
        cf.cf_set_launch_override(0, 2, ((G + 1) // 2 + 31) // 32 * 32, 1)   # one CTA per SM
        for skip in (False, True):
            st = _batched_state(wl, n)
            for b in range(n):
                cf.cf_state_init(d, xs[0, b].view(torch.int16), st["recon_s"][b], st["err"][b])
            sets = [(x16[b], st["recon_s"][b], st["err"][b], st["codes"][b], st["scales"][b])
                    for b in range(n)]
            if skip:
                sets = [s if b % 2 == 0 else (0,) + s[1:] for b, s in enumerate(sets)]
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            cf.cf_encode_batched(d, n, cf.enc_buffer_array(sets, "cuda"), status)
            torch.cuda.synchronize()
            assert int(status.item()) == (1 if skip else 0)
            runs.append(st)
    finally:
        cf.cf_set_quant_pipeline(0, 1, 0)
        cf.cf_set_launch_override(0, 0, 0, 0)
    full, part = runs
    for b in range(0, n, 2):
        for k in ("codes", "scales", "err", "recon_s"):
            assert torch.equal(full[k][b].view(torch.int32), part[k][b].view(torch.int32)), (b, k)
        r0, _ = oracle.state_init(W.bf16_bits(xs[0, b]))
        v, ora = oracle_step(W.bf16_bits(xs[1, b]), r0, wl.bits)
        gh = dict(codes=part["codes"][b].cpu().numpy().view(np.uint32),
                  scales=part["scales"][b].cpu().numpy(), err=part["err"][b].cpu().numpy(),
                  recon_s=part["recon_s"][b].cpu().numpy())
        compare_step(wl.bits, v, ora, gh)


@pytest.mark.parametrize("C", [1920, 1024])
def test_bulk_encode_bad_buffers_between_valid_ones(C):
    """TMA encode with bulk stores (rows short enough for four CTAs per SM)
    on a grid of one CTA per SM, every other buffer of the batched call
    invalid: each CTA meets valid and skipped rows in turn, so a row's
    outputs wait in shared memory across skipped rows before their bulk
    store.  The valid buffers must equal an all-valid run bit for bit and
    the oracle within the parity bar; the skipped buffers stay untouched."""
    n, T = 24, 16
    wl = W.replace(W.WORKLOADS["cogvideox"], tokens=T, channels=C, buffers=n)
    xs = torch.stack([W.trajectory(wl, b, steps=2, device="cuda") for b in range(n)], 1)
    d = cf.desc(T, C, wl.bits)
    x16 = xs[1].view(torch.int16)
    runs = []
    G = C // 8
    try:
        cf.cf_set_launch_override(0, 4, ((G + 3) // 4 + 31) // 32 * 32, 1)   # one CTA per SM
        for skip in (False, True):
            st = _batched_state(wl, n)
            for b in range(n):
                cf.cf_state_init(d, xs[0, b].view(torch.int16), st["recon_s"][b], st["err"][b])
            before = st["recon_s"].clone()
            sets = [(x16[b], st["recon_s"][b], st["err"][b], st["codes"][b], st["scales"][b])
                    for b in range(n)]
            if skip:
                sets = [s if b % 2 == 0 else (0,) + s[1:] for b, s in enumerate(sets)]
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            cf.cf_encode_batched(d, n, cf.enc_buffer_array(sets, "cuda"), status)
            torch.cuda.synchronize()
            assert int(status.item()) == (1 if skip else 0)
            if skip:
                for b in range(1, n, 2):
                    assert torch.equal(st["recon_s"][b], before[b])
            runs.append(st)
    finally:
        cf.cf_set_launch_override(0, 0, 0, 0)
    full, part = runs
    for b in range(0, n, 2):
        for k in ("codes", "scales", "err", "recon_s"):
            assert torch.equal(full[k][b].view(torch.int32), part[k][b].view(torch.int32)), (b, k)
        r0, _ = oracle.state_init(W.bf16_bits(xs[0, b]))
        v, ora = oracle_step(W.bf16_bits(xs[1, b]), r0, wl.bits)
        gh = dict(codes=part["codes"][b].cpu().numpy().view(np.uint32),
                  scales=part["scales"][b].cpu().numpy(), err=part["err"][b].cpu().numpy(),
                  recon_s=part["recon_s"][b].cpu().numpy())
        compare_step(wl.bits, v, ora, gh)
