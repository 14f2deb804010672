"""The publishing encode and the waiting decode (the exchange with the
payload transfer fused into the codec kernels), on one GPU: the
destinations are payload slots in this GPU's own memory, standing in for
the receivers' slots that peer access would map.

  * The publishing encode computes exactly what cf_encode_batched does:
    the codes and scales in every destination slot and the sender state
    equal the plain call's bit for bit, for both channel-unit widths and
    both bit widths, over two steps; each destination's ready counter grows
    by the rows published.
  * The waiting decode equals cf_decode_batched bit for bit once the
    counter has reached the target, and adds 1 to every ack counter.
  * Each bounded wait runs out when its counter never arrives (a counter
    that nothing advances): CF_ERR_TIMEOUT in the status word, nothing
    decoded or published, and the GPU takes the next launch.
  * Bad destinations are refused before any store.
Kernels that wait on each other never run concurrently here: a waiting
decode is always enqueued after the encode it waits for, on the same
stream, or waits for a counter that nothing advances.
"""
import time

import pytest
import torch

from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W
from activation_residual_compression_cf_b200.exchange import PayloadLayout

pytestmark = pytest.mark.gpu

SHAPES = [(96, 3072, 2, 5), (70, 1920, 2, 3), (64, 3072, 1, 4), (33, 1024, 1, 2), (40, 1920, 1, 3)]


def _setup(T, C, bits, n):
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, channels=C, bits=bits, buffers=n)
    xs = torch.stack([W.trajectory(wl, b, steps=3, device="cuda") for b in range(n)], 1)  # [S,n,T,C]
    f32 = dict(dtype=torch.float32, device="cuda")
    Wd = (C * bits + 31) // 32
    st = {k: torch.empty(n, T, C, **f32) for k in ("recon_s", "err", "recon_r")}
    st["codes"] = torch.empty(n, T, Wd, dtype=torch.int32, device="cuda")
    st["scales"] = torch.empty(n, T, **f32)
    d = cf.desc(T, C, bits)
    for b in range(n):
        cf.cf_state_init(d, xs[0, b].view(torch.int16), st["recon_s"][b], st["err"][b])
        cf.cf_state_init(d, xs[0, b].view(torch.int16), st["recon_r"][b], None)
    return xs, st, d


def _clone(st):
    return {k: v.clone() for k, v in st.items()}


def _bits_equal(a, b):
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.fixture(params=[4, 8], ids=["unit4", "unit8"])
def unit(request):
    cf.cf_set_quant_unit(0, request.param)
    cf.cf_set_quant_unit(1, request.param)
    yield request.param
    cf.cf_set_quant_unit(0, 0)
    cf.cf_set_quant_unit(1, 0)


@pytest.mark.parametrize("T,C,bits,n", SHAPES)
def test_publishing_encode_equals_plain_encode(T, C, bits, n, unit):
    xs, st, d = _setup(T, C, bits, n)
    L = PayloadLayout(T, C, bits, n)
    ref = _clone(st)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    slots = [torch.full((L.bytes_per_rank,), 0xCD, dtype=torch.uint8, device="cuda") for _ in range(2)]
    ready = torch.zeros(2, dtype=torch.int64, device="cuda")
    dsts = cf.publish_dst_array([(slots[k], ready[k:k + 1], None) for k in range(2)], "cuda")
    for step in (1, 2):
        x16 = xs[step].view(torch.int16)
        cf.cf_encode_batched(d, n, cf.enc_buffer_array(
            [(x16[b], ref["recon_s"][b], ref["err"][b], ref["codes"][b], ref["scales"][b])
             for b in range(n)], "cuda"), status)
        bufs = cf.enc_publish_buffer_array([(x16[b], st["recon_s"][b], st["err"][b], L.codes_offset(b),
                                             L.scales_offset(b)) for b in range(n)], "cuda")
        cf.cf_encode_publish_batched(d, n, bufs, 2, dsts, 0, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert ready.tolist() == [step * n * T] * 2
        for k in (0, 1):
            for b in range(n):
                assert torch.equal(L.codes(slots[k], b), ref["codes"][b]), (step, k, b)
                assert _bits_equal(L.scales(slots[k], b), ref["scales"][b]), (step, k, b)
        assert _bits_equal(st["recon_s"], ref["recon_s"]) and _bits_equal(st["err"], ref["err"])


@pytest.mark.parametrize("T,C,bits,n", SHAPES)
def test_waiting_decode_equals_plain_decode_and_acks(T, C, bits, n, unit):
    xs, st, d = _setup(T, C, bits, n)
    L = PayloadLayout(T, C, bits, n)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x16 = xs[1].view(torch.int16)
    cf.cf_encode_batched(d, n, cf.enc_buffer_array(
        [(x16[b], st["recon_s"][b], st["err"][b], st["codes"][b], st["scales"][b]) for b in range(n)],
        "cuda"), status)
    slot = torch.zeros(L.bytes_per_rank, dtype=torch.uint8, device="cuda")
    for b in range(n):
        L.codes(slot, b).copy_(st["codes"][b])
        L.scales(slot, b).copy_(st["scales"][b])
    ready = torch.full((1,), n * T, dtype=torch.int64, device="cuda")   # step 1 published
    recv = st["recon_r"].clone()
    cf.cf_decode_batched(d, n, cf.dec_buffer_array(
        [(st["codes"][b], st["scales"][b], st["recon_r"][b]) for b in range(n)], "cuda"), status)
    acks = torch.zeros(3, dtype=torch.int64, device="cuda")
    wbufs = cf.dec_wait_buffer_array([(L.codes(slot, b), L.scales(slot, b), recv[b], ready)
                                      for b in range(n)], "cuda")
    cf.cf_decode_wait_batched(d, n, wbufs, n * T, 3, cf.pointer_array([acks[k:k + 1] for k in range(3)],
                                                                      "cuda"), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert _bits_equal(recv, st["recon_r"])
    assert _bits_equal(recv, st["recon_s"])        # receiver == sender mirror
    assert acks.tolist() == [1, 1, 1]


def test_publish_then_wait_in_stream_order_over_steps():
    """Encode-publish and waiting decode alternate over four steps on one
    stream, with two slots used in turn and the ack target of each step
    (e - 2): the receiver tracks the sender bit for bit."""
    T, C, bits, n = 48, 1920, 2, 3
    wl = W.replace(W.WORKLOADS["cogvideox"], tokens=T, buffers=n)
    xs_all = torch.stack([W.trajectory(wl, b, steps=5, device="cuda") for b in range(n)], 1)
    f32 = dict(dtype=torch.float32, device="cuda")
    rs, er, rr = (torch.empty(n, T, C, **f32) for _ in range(3))
    d = cf.desc(T, C, bits)
    for b in range(n):
        cf.cf_state_init(d, xs_all[0, b].view(torch.int16), rs[b], er[b])
        cf.cf_state_init(d, xs_all[0, b].view(torch.int16), rr[b], None)
    L = PayloadLayout(T, C, bits, n)
    slots = [torch.zeros(L.bytes_per_rank, dtype=torch.uint8, device="cuda") for _ in range(2)]
    ready = torch.zeros(1, dtype=torch.int64, device="cuda")
    ack = torch.zeros(1, dtype=torch.int64, device="cuda")
    ackp = cf.pointer_array([ack], "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for e in range(1, 5):
        s = slots[e % 2]
        x16 = xs_all[e].view(torch.int16)
        dsts = cf.publish_dst_array([(s, ready, ack)], "cuda")
        bufs = cf.enc_publish_buffer_array([(x16[b], rs[b], er[b], L.codes_offset(b), L.scales_offset(b))
                                            for b in range(n)], "cuda")
        cf.cf_encode_publish_batched(d, n, bufs, 1, dsts, max(e - 2, 0), status)
        wb = cf.dec_wait_buffer_array([(L.codes(s, b), L.scales(s, b), rr[b], ready) for b in range(n)],
                                      "cuda")
        cf.cf_decode_wait_batched(d, n, wb, e * n * T, 1, ackp, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert ready.item() == 4 * n * T and ack.item() == 4
    assert _bits_equal(rr, rs)


def test_waiting_decode_times_out_when_nothing_is_published():
    T, C, bits, n = 64, 1920, 2, 2
    xs, st, d = _setup(T, C, bits, n)
    L = PayloadLayout(T, C, bits, n)
    slot = torch.zeros(L.bytes_per_rank, dtype=torch.uint8, device="cuda")
    ready = torch.zeros(1, dtype=torch.int64, device="cuda")       # nothing advances it
    before = st["recon_r"].clone()
    acks = torch.zeros(1, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    wb = cf.dec_wait_buffer_array([(L.codes(slot, b), L.scales(slot, b), st["recon_r"][b], ready)
                                   for b in range(n)], "cuda")
    t0 = time.time()
    cf.cf_decode_wait_batched(d, n, wb, 1, 1, cf.pointer_array([acks], "cuda"), status)
    torch.cuda.synchronize()
    waited = time.time() - t0
    assert int(status.item()) == 7                  # CF_ERR_TIMEOUT
    assert _bits_equal(st["recon_r"], before)       # nothing decoded
    assert acks.item() == 1                         # the ack is still sent
    assert waited < 30
    # the context takes the next launch
    status.zero_()
    ready.fill_(n * T)
    cf.cf_decode_wait_batched(d, n, wb, n * T, 0, None, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_publishing_encode_times_out_when_the_slot_is_never_acknowledged():
    T, C, bits, n = 64, 3072, 2, 2
    xs, st, d = _setup(T, C, bits, n)
    L = PayloadLayout(T, C, bits, n)
    slot = torch.full((L.bytes_per_rank,), 0x3C, dtype=torch.uint8, device="cuda")
    ready = torch.zeros(1, dtype=torch.int64, device="cuda")
    ack = torch.zeros(1, dtype=torch.int64, device="cuda")         # nothing advances it
    before = _clone(st)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x16 = xs[1].view(torch.int16)
    bufs = cf.enc_publish_buffer_array([(x16[b], st["recon_s"][b], st["err"][b], L.codes_offset(b),
                                         L.scales_offset(b)) for b in range(n)], "cuda")
    cf.cf_encode_publish_batched(d, n, bufs, 1, cf.publish_dst_array([(slot, ready, ack)], "cuda"), 1,
                                 status)
    torch.cuda.synchronize()
    assert int(status.item()) == 7
    assert bool((slot == 0x3C).all()) and ready.item() == 0
    assert _bits_equal(st["recon_s"], before["recon_s"]) and _bits_equal(st["err"], before["err"])


@pytest.mark.parametrize("which,expect", [("null_payload", 1), ("null_ready", 1),
                                          ("misaligned_payload", 2), ("misaligned_ready", 2)])
def test_bad_destination_is_refused_before_any_store(which, expect):
    T, C, bits, n = 32, 1920, 1, 2
    xs, st, d = _setup(T, C, bits, n)
    L = PayloadLayout(T, C, bits, n)
    slot = torch.full((L.bytes_per_rank + 64,), 0x11, dtype=torch.uint8, device="cuda")
    ready = torch.zeros(2, dtype=torch.int64, device="cuda")
    pl, rd = slot, ready
    if which == "null_payload":
        pl = 0
    elif which == "null_ready":
        rd = 0
    elif which == "misaligned_payload":
        pl = slot.data_ptr() + 8
    else:
        rd = ready.data_ptr() + 4
    before = _clone(st)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x16 = xs[1].view(torch.int16)
    bufs = cf.enc_publish_buffer_array([(x16[b], st["recon_s"][b], st["err"][b], L.codes_offset(b),
                                         L.scales_offset(b)) for b in range(n)], "cuda")
    cf.cf_encode_publish_batched(d, n, bufs, 1, cf.publish_dst_array([(pl, rd, None)], "cuda"), 0, status)
    torch.cuda.synchronize()
    assert int(status.item()) == expect
    assert bool((slot == 0x11).all()) and ready.tolist() == [0, 0]
    assert _bits_equal(st["recon_s"], before["recon_s"])


def test_publish_and_wait_refuse_shapes_off_the_tma_path():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dummy = torch.zeros(64, dtype=torch.int64, device="cuda")
    with pytest.raises(cf.CFError) as ei:      # C % 8 != 0
        cf.cf_encode_publish_batched(cf.desc(4, 36, 2), 1, dummy, 1, dummy, 0, status)
    assert ei.value.status == 3
    with pytest.raises(cf.CFError) as ei:      # ceil(C*bits/32) % 4 != 0 for the decode
        cf.cf_decode_wait_batched(cf.desc(4, 200, 2), 1, dummy, 1, 0, None, status)
    assert ei.value.status == 3
    with pytest.raises(cf.CFError) as ei:
        cf.cf_encode_publish_batched(cf.desc(4, 64, 2), 1, dummy, 9, dummy, 0, status)
    assert ei.value.status == 1
