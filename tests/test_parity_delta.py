"""GPU parity of the delta-state sender (cf_encode_delta / _batched) against
the C oracle's orc_encode_delta, through the C ABI.

The sender keeps the previous activation and the error buffer; the receiver
is the ordinary decode.  Teacher-forced: every step both sides start from
the GPU's pre-step error buffer and receiver state.  Bar as for the standard
sender (codes bit-exact away from thresholds, scales 1e-6, state 1e-5 of the
row maximum); both TMA-staged and register pipelines, ragged shapes, and the
batched call against single calls bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W
from _parity import compare_step, f32_of

pytestmark = pytest.mark.gpu


class DeltaBuffer:
    def __init__(self, T, C, bits, dev="cuda"):
        self.d = cf.desc(T, C, bits)
        W_ = (C * bits + 31) // 32
        f32 = dict(dtype=torch.float32, device=dev)
        self.err = torch.empty(T, C, **f32)
        self.recon_r = torch.empty(T, C, **f32)
        self.codes = torch.empty(T, W_, dtype=torch.int32, device=dev)
        self.scales = torch.empty(T, **f32)

    def init(self, x0):
        cf.cf_state_init(self.d, x0.view(torch.int16), None, self.err)
        cf.cf_state_init(self.d, x0.view(torch.int16), self.recon_r, None)

    def step(self, x, x_prev):
        cf.cf_encode_delta(self.d, x.view(torch.int16), x_prev.view(torch.int16), self.err,
                           self.codes, self.scales)
        cf.cf_decode(self.d, self.codes, self.scales, self.recon_r)


def _run(xs, bits, pipeline):
    # fresh allocations: slices of one trajectory tensor are not 16-byte
    # aligned when T * C * 2 is not a multiple of 16
    xs = [x.clone() for x in xs]
    T, C = xs[0].shape
    cf.cf_set_quant_pipeline(0, pipeline, 0)
    try:
        g = DeltaBuffer(T, C, bits)
        g.init(xs[0])
        torch.cuda.synchronize()
        assert not torch.any(g.err)
        for t in range(1, len(xs)):
            err0 = g.err.cpu().numpy()
            rr0 = g.recon_r.cpu().numpy()
            g.step(xs[t], xs[t - 1])
            torch.cuda.synchronize()
            xb, pb = W.bf16_bits(xs[t]), W.bf16_bits(xs[t - 1])
            err_o = err0.copy()
            v = ((f32_of(xb) - f32_of(pb)).astype(np.float32) + err0).astype(np.float32)
            codes_o, scales_o = oracle.encode_delta(xb, pb, err_o, bits)
            rr_o = rr0.copy()
            oracle.decode(codes_o, scales_o, rr_o, bits)
            gpu = dict(codes=g.codes.cpu().numpy().view(np.uint32), scales=g.scales.cpu().numpy(),
                       err=g.err.cpu().numpy(), recon_r=g.recon_r.cpu().numpy())
            ora = dict(codes=codes_o, scales=scales_o, err=err_o, recon_s=rr_o)
            compare_step(bits, v, ora, gpu)
    finally:
        cf.cf_set_quant_pipeline(0, 1, 0)


@pytest.mark.parametrize("pipeline", [0, 1])
@pytest.mark.parametrize("name,kw", [("tiny", {}), ("flux_sp", dict(tokens=96)),
                                     ("flux_full", dict(tokens=64))])
def test_delta_trajectory(name, kw, pipeline):
    wl = W.replace(W.WORKLOADS[name], **kw)
    xs = W.trajectory(wl, 0, steps=5, device="cuda")
    _run(xs, wl.bits, pipeline)


@pytest.mark.parametrize("T,C,bits", [(37, 1003, 1), (21, 200, 2), (9, 16384, 1), (5, 16384, 2),
                                      (130, 8, 2)])
def test_delta_ragged_shapes(T, C, bits):
    """C % 8 != 0 (scalar register path), C = 16384 (too wide for the TMA
    ring: register path), tiny C."""
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, channels=C, bits=bits)
    xs = W.trajectory(wl, 1, steps=3, device="cuda")
    _run(xs, bits, 1)


@pytest.mark.parametrize("pipeline", [0, 1])
def test_delta_batched_equals_single_and_skips_bad_buffers(pipeline):
    T, C, bits, n = 200, 3072, 2, 5
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, buffers=n)
    xs = [W.trajectory(wl, b, steps=3, device="cuda") for b in range(n)]
    cf.cf_set_quant_pipeline(0, pipeline, 0)
    try:
        single = [DeltaBuffer(T, C, bits) for _ in range(n)]
        batch = [DeltaBuffer(T, C, bits) for _ in range(n)]
        for b in range(n):
            single[b].init(xs[b][0])
            batch[b].init(xs[b][0])
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for t in (1, 2):
            for b in range(n):
                single[b].step(xs[b][t], xs[b][t - 1])
            arr = cf.enc_delta_buffer_array(
                [(xs[b][t].view(torch.int16), xs[b][t - 1].view(torch.int16), batch[b].err,
                  batch[b].codes, batch[b].scales) for b in range(n)], "cuda")
            cf.cf_encode_delta_batched(batch[0].d, n, arr, status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            for b in range(n):
                for k in ("err", "codes", "scales"):
                    assert torch.equal(getattr(batch[b], k), getattr(single[b], k)), (t, b, k)
        # a buffer with a misaligned x_prev is skipped and reported
        before = batch[1].err.clone()
        arr = cf.enc_delta_buffer_array(
            [(xs[0][2].view(torch.int16), xs[0][1].view(torch.int16), batch[0].err,
              batch[0].codes, batch[0].scales),
             (xs[1][2].view(torch.int16), xs[1][1].data_ptr() + 2, batch[1].err,
              batch[1].codes, batch[1].scales)], "cuda")
        cf.cf_encode_delta_batched(batch[0].d, 2, arr, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 2
        assert torch.equal(batch[1].err, before)
    finally:
        cf.cf_set_quant_pipeline(0, 1, 0)


def test_delta_and_standard_senders_agree_on_the_first_step():
    """After the warmup, the first delta-state step equals the standard
    sender's bit for bit on the GPU too."""
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=128)
    xs = W.trajectory(wl, 0, steps=2, device="cuda")
    T, C, bits = wl.tokens, wl.channels, wl.bits
    g = DeltaBuffer(T, C, bits)
    g.init(xs[0])
    g.step(xs[1], xs[0])
    f32 = dict(dtype=torch.float32, device="cuda")
    recon_s, err = torch.empty(T, C, **f32), torch.empty(T, C, **f32)
    codes, scales = torch.empty_like(g.codes), torch.empty_like(g.scales)
    cf.cf_state_init(g.d, xs[0].view(torch.int16), recon_s, err)
    cf.cf_encode(g.d, xs[1].view(torch.int16), recon_s, err, codes, scales)
    torch.cuda.synchronize()
    assert torch.equal(codes, g.codes) and torch.equal(scales, g.scales) and torch.equal(err, g.err)
