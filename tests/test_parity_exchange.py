"""The sequence-parallel exchange (exchange.py) on one GPU through libcf's
kernels and a one-rank NCCL group, in loopback: the rank encodes its buffers
into the payload, all-gathers it and decodes its own payload.  Every
receiver state must equal the sender's mirror bit for bit, the payload's
codes and scales must equal the single-buffer calls on the same inputs, and
buffer 0 is checked step by step against the oracle (teacher-forced, the
quantize parity bar)."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W
from activation_residual_compression_cf_b200.exchange import (FusedShardExchange, LowrankShardExchange,
                                                                ShardExchange)
from _parity import compare_step, f32_of

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture(scope="module")
def nccl_group():
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("T,C,bits,B", [(1024, 3072, 2, 6), (100, 1003, 1, 3)])
def test_exchange_loopback_matches_single_calls_and_oracle(nccl_group, T, C, bits, B):
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, channels=C, bits=bits, buffers=B)
    trajs = [W.trajectory(wl, b, steps=4, device="cuda") for b in range(B)]
    ex = ShardExchange(T, C, bits, B, loopback=True)
    assert ex.world == 1 and ex.backend == "nccl"
    xs0 = [trajs[b][0].clone() for b in range(B)]
    ex.warmup(xs0)
    # the same buffers through the single-buffer calls
    d = cf.desc(T, C, bits)
    f32 = dict(dtype=torch.float32, device="cuda")
    ref = []
    for b in range(B):
        rs, e = torch.empty(T, C, **f32), torch.empty(T, C, **f32)
        cf.cf_state_init(d, xs0[b], rs, e)
        ref.append((rs, e, torch.empty(T, ex.layout.words_per_row, dtype=torch.int32, device="cuda"),
                    torch.empty(T, **f32)))
    for t in range(1, 4):
        xs = [trajs[b][t].clone() for b in range(B)]
        r0 = ex.recon_s[0].cpu().numpy()
        ex.step(xs)
        for b in range(B):
            rs, e, c, s = ref[b]
            cf.cf_encode(d, xs[b], rs, e, c, s)
        torch.cuda.synchronize()
        assert ex.codec.status_value() == 0
        for b in range(B):
            rs, e, c, s = ref[b]
            assert torch.equal(ex.layout.codes(ex.recv, b), c), (t, b)
            assert torch.equal(ex.layout.scales(ex.recv, b), s), (t, b)
            assert torch.equal(ex.recon_s[b], rs) and torch.equal(ex.err[b], e), (t, b)
            assert torch.equal(ex.recon_r[0][b], ex.recon_s[b]), (t, b)
        xb = W.bf16_bits(xs[0])
        v = (f32_of(xb) - r0).astype(np.float32)
        ro = r0.copy()
        co, so, eo = oracle.encode(xb, ro, bits)
        gpu = dict(codes=ex.layout.codes(ex.send, 0).cpu().numpy().view(np.uint32),
                   scales=ex.layout.scales(ex.send, 0).cpu().numpy(),
                   err=ex.err[0].cpu().numpy(), recon_s=ex.recon_s[0].cpu().numpy())
        compare_step(bits, v, dict(codes=co, scales=so, err=eo, recon_s=ro), gpu)


def test_exchange_emits_the_bf16_reconstruction(nccl_group):
    """With emit, the receivers' bf16 copy equals the warmup activation after
    the warmup and the bf16 rounding of the reconstruction after each step."""
    T, C, bits, B = 256, 3072, 2, 4
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, channels=C, bits=bits, buffers=B)
    trajs = [W.trajectory(wl, b, steps=3, device="cuda") for b in range(B)]
    ex = ShardExchange(T, C, bits, B, loopback=True, emit=True)
    xs0 = [trajs[b][0].clone() for b in range(B)]
    ex.warmup(xs0)
    torch.cuda.synchronize()
    for b in range(B):
        assert torch.equal(ex.out[0][b], xs0[b])
    for t in (1, 2):
        ex.step([trajs[b][t].clone() for b in range(B)])
        torch.cuda.synchronize()
        assert ex.codec.status_value() == 0
        for b in range(B):
            assert torch.equal(ex.recon_r[0][b], ex.recon_s[b])
            ref = ex.recon_r[0][b].to(torch.bfloat16)
            assert torch.equal(ex.out[0][b].view(torch.int16), ref.view(torch.int16)), (t, b)


def test_lowrank_exchange_loopback_matches_single_calls_and_oracle(nccl_group):
    """The low-rank exchange in loopback: the payload equals single-buffer
    cf_lowrank_encode calls on the same inputs bit for bit, the receivers
    mirror the senders, buffer 0's error is within 1 % of the oracle's, and
    a warm-started step (no start blocks) runs clean."""
    from oracle import lowrank as OL
    T, C, r, iters, B = 256, 192, 8, 2, 3
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r, iters=iters, buffers=B)
    trajs = [W.trajectory(wl, b, steps=4, device="cuda") for b in range(B)]
    ex = LowrankShardExchange(T, C, r, iters, B, loopback=True)
    ex.warmup([trajs[b][0].clone() for b in range(B)])
    d = cf.desc(T, C, 0, r, iters)
    ws = torch.empty(cf.cf_lowrank_workspace_bytes(d), dtype=torch.uint8, device="cuda")
    nb = (r + 1) // 2
    ref = [dict(rs=ex.recon_s[b].clone(), err=torch.empty_like(ex.err[b]),
                pc=torch.empty(T * nb, dtype=torch.uint8, device="cuda"), ps=torch.empty(r, device="cuda"),
                qc=torch.empty(C * nb, dtype=torch.uint8, device="cuda"), qs=torch.empty(r, device="cuda"))
           for b in range(B)]
    for t in (1, 2):
        xs = [trajs[b][t].clone() for b in range(B)]
        oms = [W.omega(wl, b, t, device="cuda") for b in range(B)]
        before0 = ex.recon_s[0].cpu().numpy()
        ex.step(xs, oms)
        for b in range(B):
            g = ref[b]
            cf.cf_lowrank_encode(d, xs[b], g["rs"], g["err"], oms[b], g["pc"], g["ps"], g["qc"], g["qs"], ws)
        torch.cuda.synchronize()
        assert ex.status() == [0] * B
        for b in range(B):
            pc, ps, qc, qs = ex.layout.parts(ex.recv, b)
            g = ref[b]
            assert torch.equal(pc.reshape(-1), g["pc"]) and torch.equal(qc.reshape(-1), g["qc"]), (t, b)
            assert torch.equal(ps, g["ps"]) and torch.equal(qs, g["qs"]), (t, b)
            assert torch.equal(ex.recon_s[b], g["rs"]) and torch.equal(ex.err[b], g["err"]), (t, b)
            assert torch.equal(ex.recon_r[0][b], ex.recon_s[b]), (t, b)
        out = OL.lowrank_encode(W.bf16_bits(xs[0]), before0.copy(), oms[0].cpu().numpy(), iters)
        v = out["V"].astype(np.float64)
        pc, ps, qc, qs = (a.cpu().numpy() for a in ex.layout.parts(ex.send, 0))
        e_gpu = np.linalg.norm(v - OL.reconstruct(pc, ps, qc, qs, r)) / np.linalg.norm(v)
        e_ora = np.linalg.norm(v - out["D"]) / np.linalg.norm(v)
        assert abs(e_gpu - e_ora) <= 0.01 * e_ora, (t, e_gpu, e_ora)
    # a checkpoint taken here resumes the warm start bit for bit
    resumed = LowrankShardExchange(T, C, r, iters, B, loopback=True)
    resumed.load_state_dict(ex.state_dict())
    x3 = [trajs[b][3].clone() for b in range(B)]
    ex.step(x3)                                           # warm start from the previous Q
    resumed.step(x3)
    torch.cuda.synchronize()
    assert ex.status() == [0] * B and resumed.status() == [0] * B
    for b in range(B):
        assert torch.equal(ex.recon_r[0][b], ex.recon_s[b])
        assert torch.equal(resumed.recon_s[b], ex.recon_s[b]) and torch.equal(resumed.err[b], ex.err[b])
        assert torch.equal(resumed.recon_r[0][b], ex.recon_r[0][b])


@pytest.mark.parametrize("T,C,bits,B", [(1024, 3072, 2, 6), (200, 1920, 1, 3), (96, 1920, 2, 2)])
def test_fused_exchange_loopback_equals_the_gather_exchange(nccl_group, T, C, bits, B):
    """The fused exchange (publishing encode into the slots, waiting decode,
    counters and acks) in loopback on one GPU: its slots hold exactly the
    gather exchange's payload, every state equals the gather exchange's bit
    for bit over five steps (both slots used twice, ack waits from step 3),
    buffer 0 meets the oracle's bar every step, and a checkpoint resumes on
    fresh slot memory bit for bit."""
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, channels=C, bits=bits, buffers=B)
    trajs = [W.trajectory(wl, b, steps=7, device="cuda") for b in range(B)]
    gx = ShardExchange(T, C, bits, B, loopback=True)
    fx = FusedShardExchange(T, C, bits, B, loopback=True)
    for ex in (gx, fx):
        ex.warmup([trajs[b][0].clone() for b in range(B)])
    for t in range(1, 6):
        xs = [trajs[b][t].clone() for b in range(B)]
        r0 = fx.recon_s[0].cpu().numpy()
        gx.step(xs)
        fx.step(xs)
        torch.cuda.synchronize()
        assert gx.codec.status_value() == 0 and fx.codec.status_value() == 0
        slot = fx.memory.recv[0][t % 2, 0]
        assert torch.equal(slot, gx.recv), t
        for b in range(B):
            for a, g in ((fx.recon_s[b], gx.recon_s[b]), (fx.err[b], gx.err[b]),
                         (fx.recon_r[0][b], gx.recon_r[0][b]), (fx.recon_r[0][b], fx.recon_s[b])):
                assert torch.equal(a.view(torch.int32), g.view(torch.int32)), (t, b)
        assert fx.memory.ready[0].item() == t * B * T and fx.memory.ack[0].item() == t
        xb = W.bf16_bits(xs[0])
        v = (f32_of(xb) - r0).astype(np.float32)
        ro = r0.copy()
        co, so, eo = oracle.encode(xb, ro, bits)
        gpu = dict(codes=fx.layout.codes(slot, 0).cpu().numpy().view(np.uint32),
                   scales=fx.layout.scales(slot, 0).cpu().numpy(),
                   err=fx.err[0].cpu().numpy(), recon_s=fx.recon_s[0].cpu().numpy())
        compare_step(bits, v, dict(codes=co, scales=so, err=eo, recon_s=ro), gpu)
    resumed = FusedShardExchange(T, C, bits, B, loopback=True)
    resumed.load_state_dict(fx.state_dict())
    x6 = [trajs[b][6].clone() for b in range(B)]
    fx.step(x6)
    resumed.step(x6)
    torch.cuda.synchronize()
    assert resumed.codec.status_value() == 0
    for b in range(B):
        assert torch.equal(resumed.recon_s[b], fx.recon_s[b]) and torch.equal(resumed.err[b], fx.err[b])
        assert torch.equal(resumed.recon_r[0][b], fx.recon_r[0][b])
