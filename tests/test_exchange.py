"""Host logic of the sequence-parallel exchange (exchange.py) on CPU ranks:
payload layout, the warmup's uncompressed all-gather, and the routing of
every peer's payload into that peer's receiver states.  The ranks run on the
gloo backend with the oracle standing in for libcf's kernels (the codec is
injected by the test); each rank regenerates every shard's trajectory from
the shared seeds and checks each receiver state bit for bit against the
oracle run directly on that peer's shard."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from activation_residual_compression_cf_b200.exchange import PayloadLayout


class OracleCodec:
    """The four codec methods of ShardExchange on CPU tensors, computed by
    the oracle in place through numpy views."""

    def __init__(self, bits):
        self.bits = bits

    def state_init(self, d, x, recon, err):
        import oracle
        from activation_residual_compression_cf_b200 import workloads as W
        r, e = oracle.state_init(W.bf16_bits(x))
        recon.copy_(torch.from_numpy(r))
        if err is not None:
            err.copy_(torch.from_numpy(e))

    def encode_batched(self, d, sets):
        import oracle
        from activation_residual_compression_cf_b200 import workloads as W
        for x, rs, e, c, s in sets:
            codes, scales, err = oracle.encode(W.bf16_bits(x), rs.numpy(), self.bits)
            c.numpy().view(np.uint32)[...] = codes
            s.numpy()[...] = scales
            e.numpy()[...] = err

    def decode_batched(self, d, sets):
        import oracle
        for c, s, rr in sets:
            oracle.decode(c.numpy().view(np.uint32).copy(), s.numpy().copy(), rr.numpy(), self.bits)

    def decode_emit_batched(self, d, sets):
        import oracle
        for c, s, rr, o in sets:
            out = oracle.decode_emit(c.numpy().view(np.uint32).copy(), s.numpy().copy(), rr.numpy(),
                                     self.bits)
            o.view(torch.int16).numpy().view(np.uint16)[...] = out


class OracleLowrankCodec(OracleCodec):
    """The low-rank codec methods on CPU tensors, computed by the numpy
    oracle in place through numpy views (cold start only)."""

    def __init__(self, rank, iters):
        super().__init__(0)
        self.rank, self.iters = rank, iters

    def lowrank_workspace_bytes(self, d):
        return 16

    def lowrank_status(self, workspace_slice):
        return 0

    def lowrank_encode_batched(self, d, sets, workspace):
        from oracle import lowrank as OL
        from activation_residual_compression_cf_b200 import workloads as W
        for x, rs, e, om, pc, ps, qc, qs in sets:
            out = OL.lowrank_encode(W.bf16_bits(x), rs.numpy(), om.numpy().astype(np.float64), self.iters)
            pc.numpy()[...] = out["p_codes"]
            ps.numpy()[...] = out["p_scales"]
            qc.numpy()[...] = out["q_codes"]
            qs.numpy()[...] = out["q_scales"]
            e.numpy()[...] = out["err"]

    def lowrank_decode_batched(self, d, sets):
        from oracle import lowrank as OL
        for pc, ps, qc, qs, rr in sets:
            OL.lowrank_decode(pc.numpy().copy(), ps.numpy().copy(), qc.numpy().copy(), qs.numpy().copy(),
                              rr.numpy(), self.rank)


@pytest.mark.parametrize("T,C,r,B", [(40, 72, 4, 2), (4096, 3072, 32, 114), (3, 5, 3, 1)])
def test_lowrank_payload_layout_is_aligned_and_disjoint(T, C, r, B):
    from activation_residual_compression_cf_b200.exchange import LowrankPayloadLayout
    L = LowrankPayloadLayout(T, C, r, B)
    nb = (r + 1) // 2
    spans = []
    p = torch.zeros(L.bytes_per_rank, dtype=torch.uint8)
    base = p.data_ptr()
    for b in range(B):
        parts = L.parts(p, b)
        assert [tuple(t.shape) for t in parts] == [(T, nb), (r,), (C, nb), (r,)]
        for t in parts:
            off = t.data_ptr() - base
            assert off % 16 == 0
            spans.append((off, off + t.numel() * t.element_size()))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:])) and spans[-1][1] <= L.bytes_per_rank
    # the payload is the page's factor bytes plus at most 60 bytes of padding per buffer
    assert L.stride - ((T + C) * nb + 8 * r) <= 60


@pytest.mark.parametrize("T,C,bits,B", [(48, 200, 1, 3), (1024, 3072, 2, 114), (7, 8, 2, 2),
                                        (3, 33, 1, 5)])
def test_payload_layout_is_aligned_and_disjoint(T, C, bits, B):
    L = PayloadLayout(T, C, bits, B)
    assert L.words_per_row == (C * bits + 31) // 32
    spans = []
    for b in range(B):
        for off, n in ((L.codes_offset(b), L.codes_bytes), (L.scales_offset(b), L.scales_bytes)):
            assert off % 16 == 0
            spans.append((off, off + n))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= L.bytes_per_rank
    # the padding costs at most 30 bytes per buffer over the packed payload
    assert L.bytes_per_rank - B * (L.codes_bytes + L.scales_bytes) <= 30 * B
    p = torch.zeros(L.bytes_per_rank, dtype=torch.uint8)
    assert L.codes(p, B - 1).shape == (T, L.words_per_row) and L.scales(p, 0).shape == (T,)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q, bits, loopback, emit=False):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    try:
        import torch.distributed as dist
        import oracle
        from activation_residual_compression_cf_b200 import workloads as W
        from activation_residual_compression_cf_b200.exchange import ShardExchange
        from test_exchange import OracleCodec
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=60))
        T, C, B, steps = 37, 203, 3, 4          # ragged: segments need padding
        wl = W.replace(W.WORKLOADS["flux_sp"], tokens=world * T, channels=C, bits=bits, buffers=B)
        trajs = [W.trajectory(wl, b, steps=steps) for b in range(B)]

        def shard(x, p):
            return x[p * T:(p + 1) * T].clone()

        ex = ShardExchange(T, C, bits, B, device="cpu", codec=OracleCodec(bits), loopback=loopback,
                           emit=emit)
        ex.warmup([shard(trajs[b][0], rank) for b in range(B)])
        for t in range(1, steps):
            ex.step([shard(trajs[b][t], rank) for b in range(B)])
        bad = []
        for p in range(world):
            for b in range(B):
                r, _ = oracle.state_init(W.bf16_bits(shard(trajs[b][0], p)))
                for t in range(1, steps):
                    oracle.encode(W.bf16_bits(shard(trajs[b][t], p)), r, bits)
                if p == rank and not np.array_equal(ex.recon_s[b].numpy(), r):
                    bad.append(("sender", p, b))
                if p in ex.peers and not np.array_equal(ex.recon_r[p][b].numpy(), r):
                    bad.append(("receiver", p, b))
                if emit and p in ex.peers and not torch.equal(ex.out[p][b], torch.from_numpy(r).to(torch.bfloat16)):
                    bad.append(("emitted bf16", p, b))
                if p not in ex.peers and ex.recon_r[p] is not None:
                    bad.append(("unexpected receiver", p))
        q.put((rank, "ok" if not bad else "bad", bad, len(ex.peers)))
        dist.destroy_process_group()
    except Exception as e:
        q.put((rank, "fail", repr(e), 0))


@pytest.mark.parametrize("bits,loopback,emit", [(1, False, False), (2, True, False), (2, False, True)])
def test_exchange_routes_every_peer_payload_world2(bits, loopback, emit):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q, bits, loopback, emit))
          for r in range(world)]
    for p in ps:
        p.start()
    out = sorted([q.get(timeout=180) for _ in range(world)], key=lambda t: t[0])
    for p in ps:
        p.join(timeout=60)
    for rank, status, info, npeers in out:
        assert status == "ok", (rank, info)
        assert npeers == (world if loopback else world - 1)


def test_exchange_rejects_bad_shapes():
    from activation_residual_compression_cf_b200.exchange import ShardExchange
    ex = ShardExchange(8, 64, 1, 2, device="cpu", codec=OracleCodec(1))
    with pytest.raises(ValueError):
        ex.step([torch.zeros(8, 64, dtype=torch.bfloat16)])
    with pytest.raises(ValueError):
        ex.step([torch.zeros(8, 64, dtype=torch.float32)] * 2)
    with pytest.raises(ValueError):
        ShardExchange(8, 64, 3, 2, device="cpu", codec=OracleCodec(1))


def _leaver(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    try:
        import torch.distributed as dist
        from activation_residual_compression_cf_b200 import workloads as W
        from activation_residual_compression_cf_b200.exchange import ShardExchange
        from test_exchange import OracleCodec
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=5))
        T, C, bits = 16, 64, 1
        wl = W.replace(W.WORKLOADS["tiny"], tokens=world * T, channels=C)
        xs = W.trajectory(wl, 0, steps=3)
        ex = ShardExchange(T, C, bits, 1, device="cpu", codec=OracleCodec(bits))
        ex.warmup([xs[0][rank * T:(rank + 1) * T].clone()])
        ex.step([xs[1][rank * T:(rank + 1) * T].clone()])
        if rank == 1:
            q.put((rank, "left"))
            q.close()
            q.join_thread()
            os._exit(0)                       # leaves between steps, nothing in flight
        try:
            ex.step([xs[2][rank * T:(rank + 1) * T].clone()])
            q.put((rank, "no error"))
        except Exception as e:                # the gather times out or the peer's socket closed
            q.put((rank, "error", type(e).__name__))
    except Exception as e:
        q.put((rank, "fail", repr(e)))


def test_a_rank_that_leaves_ends_the_survivors_next_step_with_an_error():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_leaver, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    out = sorted([q.get(timeout=180) for _ in range(world)], key=lambda t: t[0])
    for p in ps:
        p.join(timeout=60)
    assert out[1][1] == "left", out
    assert out[0][1] == "error", out


def _resumer(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    try:
        import torch.distributed as dist
        from activation_residual_compression_cf_b200 import workloads as W
        from activation_residual_compression_cf_b200.exchange import ShardExchange
        from test_exchange import OracleCodec
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=60))
        T, C, bits, B = 24, 96, 2, 2
        wl = W.replace(W.WORKLOADS["flux_sp"], tokens=world * T, channels=C, bits=bits, buffers=B)
        trajs = [W.trajectory(wl, b, steps=5) for b in range(B)]

        def xs(t):
            return [trajs[b][t][rank * T:(rank + 1) * T].clone() for b in range(B)]

        def make():
            return ShardExchange(T, C, bits, B, device="cpu", codec=OracleCodec(bits), emit=True)
        whole, first = make(), make()
        whole.warmup(xs(0))
        first.warmup(xs(0))
        for t in (1, 2):
            whole.step(xs(t))
            first.step(xs(t))
        sd = first.state_dict()
        del first
        resumed = make()
        resumed.load_state_dict(sd)
        for t in (3, 4):
            whole.step(xs(t))
            resumed.step(xs(t))
        same = all(torch.equal(a, b) for a, b in zip(whole.recon_s + whole.err, resumed.recon_s + resumed.err))
        for p in whole.peers:
            same &= all(torch.equal(a, b) for a, b in zip(whole.recon_r[p], resumed.recon_r[p]))
            same &= all(torch.equal(a, b) for a, b in zip(whole.out[p], resumed.out[p]))
        bad = make()
        sd["world"] = world + 1
        try:
            bad.load_state_dict(sd)
            rejected = False
        except ValueError:
            rejected = True
        q.put((rank, "ok" if same and rejected else "bad", same, rejected))
        dist.destroy_process_group()
    except Exception as e:
        q.put((rank, "fail", repr(e), None))


def test_exchange_resumes_bit_for_bit_from_a_state_dict_world2():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_resumer, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    out = sorted([q.get(timeout=180) for _ in range(world)], key=lambda t: t[0])
    for p in ps:
        p.join(timeout=60)
    for o in out:
        assert o[1] == "ok", o


def _lowrank_worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    try:
        import torch.distributed as dist
        from oracle import lowrank as OL
        from activation_residual_compression_cf_b200 import workloads as W
        from activation_residual_compression_cf_b200.exchange import LowrankShardExchange
        from test_exchange import OracleLowrankCodec
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=60))
        T, C, r, iters, B, steps = 40, 72, 4, 2, 2, 3
        wl = W.replace(W.WORKLOADS["lowrank"], tokens=world * T, channels=C, rank=r, iters=iters,
                       buffers=B)
        trajs = [W.trajectory(wl, b, steps=steps) for b in range(B)]
        oms = {(b, t): W.omega(wl, b, t) for b in range(B) for t in range(1, steps)}

        def shard(x, p):
            return x[p * T:(p + 1) * T].clone()

        ex = LowrankShardExchange(T, C, r, iters, B, device="cpu", codec=OracleLowrankCodec(r, iters))
        ex.warmup([shard(trajs[b][0], rank) for b in range(B)])
        for t in range(1, steps):
            ex.step([shard(trajs[b][t], rank) for b in range(B)], [oms[(b, t)] for b in range(B)])
        bad = []
        for p in range(world):
            for b in range(B):
                rec = W.bf16_bits(shard(trajs[b][0], p)).astype(np.uint32) << 16
                rec = rec.view(np.float32).copy()
                for t in range(1, steps):
                    OL.lowrank_encode(W.bf16_bits(shard(trajs[b][t], p)), rec,
                                      oms[(b, t)].numpy().astype(np.float64), iters)
                if p == rank and not np.array_equal(ex.recon_s[b].numpy(), rec):
                    bad.append(("sender", p, b))
                if p in ex.peers and not np.array_equal(ex.recon_r[p][b].numpy(), rec):
                    bad.append(("receiver", p, b))
        q.put((rank, "ok" if not bad else "bad", bad, ex.status()))
        dist.destroy_process_group()
    except Exception as e:
        q.put((rank, "fail", repr(e), None))


def test_lowrank_exchange_routes_every_peer_payload_world2():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_lowrank_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    out = sorted([q.get(timeout=180) for _ in range(world)], key=lambda t: t[0])
    for p in ps:
        p.join(timeout=60)
    for rank, status, info, st in out:
        assert status == "ok", (rank, info)
        assert st == [0, 0]


def test_lowrank_warm_start_before_any_encode_is_refused():
    """A warm start (no start block) needs the Q of an earlier encode of that
    buffer: on the first compressed step it raises at the call site instead
    of starting subspace iteration from an empty workspace.  After a step
    with start blocks it is accepted, and a checkpoint carries that state."""
    from activation_residual_compression_cf_b200 import workloads as W
    from activation_residual_compression_cf_b200.exchange import LowrankShardExchange
    T, C, r, iters, B = 24, 48, 4, 2, 2
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r, iters=iters, buffers=B)
    trajs = [W.trajectory(wl, b, steps=4) for b in range(B)]
    ex = LowrankShardExchange(T, C, r, iters, B, device="cpu", codec=OracleLowrankCodec(r, iters),
                              loopback=True)
    ex.warmup([trajs[b][0] for b in range(B)])
    with pytest.raises(ValueError, match="warm-start"):
        ex.step([trajs[b][1] for b in range(B)])
    with pytest.raises(ValueError, match=r"\[1\]"):
        ex.step([trajs[b][1] for b in range(B)], [W.omega(wl, 0, 1), None])
    ex.step([trajs[b][1] for b in range(B)], [W.omega(wl, b, 1) for b in range(B)])
    sd = ex.state_dict()
    fresh = LowrankShardExchange(T, C, r, iters, B, device="cpu", codec=OracleLowrankCodec(r, iters),
                                 loopback=True)
    with pytest.raises(ValueError):
        fresh.step([trajs[b][2] for b in range(B)])
    fresh.load_state_dict(sd)
    assert fresh.encoded == [True, True]


# ---------------------------------------------------------------- fused exchange

class OracleFusedCodec(OracleCodec):
    """The fused exchange's two calls on CPU tensors, computed by the oracle,
    with the counter protocol of the publishing encode and the waiting decode
    done by polling the shared counters (bounded by `timeout` seconds)."""

    def __init__(self, bits, timeout=30.0):
        super().__init__(bits)
        self.timeout = timeout

    def _wait(self, counter, target):
        import time
        t0 = time.time()
        while int(counter[0]) < target:
            if time.time() - t0 > self.timeout:
                raise TimeoutError(f"counter {int(counter[0])} < {target}")
            time.sleep(0.001)

    def encode_publish_batched(self, d, sets, dsts, ack_target):
        import oracle
        from activation_residual_compression_cf_b200 import workloads as W
        if ack_target:
            for _, _, ack in dsts:
                self._wait(ack, ack_target)
        for x, rs, e, co, so in sets:
            codes, scales, err = oracle.encode(W.bf16_bits(x), rs.numpy(), self.bits)
            e.numpy()[...] = err
            cb, sb = codes.view(np.uint8).reshape(-1), scales.view(np.uint8).reshape(-1)
            for payload, _, _ in dsts:
                payload[co:co + cb.size].copy_(torch.from_numpy(cb.copy()))
                payload[so:so + sb.size].copy_(torch.from_numpy(sb.copy()))
        for _, ready, _ in dsts:                 # after every store (one writer per counter)
            ready[0] += d.tokens * len(sets)

    def decode_wait_batched(self, d, sets, ready_target, acks):
        import oracle
        for c, s, rr, ready in sets:
            self._wait(ready, ready_target)
            oracle.decode(c.numpy().view(np.uint32).copy(), s.numpy().copy(), rr.numpy(), self.bits)
        for a in acks:
            a[0] += 1


def _file_slot_memory(layout, world, folder):
    """Every rank's slots and counters in files mapped shared by all the
    rank processes (stands in for peer-mapped GPU memory)."""
    from activation_residual_compression_cf_b200.exchange import SlotMemory
    mem = SlotMemory([], [], [])
    for r in range(world):
        recv = torch.from_file(os.path.join(folder, f"recv{r}"), shared=True,
                               size=2 * world * layout.bytes_per_rank, dtype=torch.uint8)
        mem.recv.append(recv.view(2, world, layout.bytes_per_rank))
        mem.ready.append(torch.from_file(os.path.join(folder, f"ready{r}"), shared=True, size=world,
                                         dtype=torch.int64))
        mem.ack.append(torch.from_file(os.path.join(folder, f"ack{r}"), shared=True, size=world,
                                       dtype=torch.int64))
    return mem


def _fused_worker(rank, world, port, folder, leave_after, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    try:
        import torch.distributed as dist
        import oracle
        from activation_residual_compression_cf_b200 import workloads as W
        from activation_residual_compression_cf_b200.exchange import FusedShardExchange, PayloadLayout
        from test_exchange import OracleFusedCodec, _file_slot_memory
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=60))
        T, C, bits, B, steps = 16, 64, 2, 2, 6
        wl = W.replace(W.WORKLOADS["flux_sp"], tokens=world * T, channels=C, bits=bits, buffers=B)
        trajs = [W.trajectory(wl, b, steps=steps) for b in range(B)]

        def shard(x, p):
            return x[p * T:(p + 1) * T].clone()

        mem = _file_slot_memory(PayloadLayout(T, C, bits, B), world, folder)
        codec = OracleFusedCodec(bits, timeout=3.0 if leave_after else 30.0)
        ex = FusedShardExchange(T, C, bits, B, device="cpu", codec=codec, memory=mem)
        ex.warmup([shard(trajs[b][0], rank) for b in range(B)])
        for t in range(1, steps):
            if leave_after and rank == 1 and t > leave_after:
                q.put((rank, "left"))
                q.close()
                q.join_thread()
                os._exit(0)                      # leaves between steps, nothing in flight
            try:
                ex.step([shard(trajs[b][t], rank) for b in range(B)])
            except TimeoutError as e:
                q.put((rank, "timeout", t, str(e)))
                return
        bad = []
        for p in ex.peers:
            for b in range(B):
                rec, _ = oracle.state_init(W.bf16_bits(shard(trajs[b][0], p)))
                for t in range(1, steps):
                    oracle.encode(W.bf16_bits(shard(trajs[b][t], p)), rec, bits)
                if not np.array_equal(ex.recon_r[p][b].numpy(), rec):
                    bad.append((p, b))
        dist.barrier()        # every rank's last decode (and its acks) is done
        counters = ([int(v) for v in mem.ready[rank]], [int(v) for v in mem.ack[rank]])
        q.put((rank, "ok" if not bad else "bad", bad, counters))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:
        q.put((rank, "fail", repr(e), None))


def _run_fused(tmp_path, world, leave_after):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_fused_worker, args=(r, world, port, str(tmp_path), leave_after, q))
          for r in range(world)]
    for p in ps:
        p.start()
    out = sorted([q.get(timeout=240) for _ in range(world)], key=lambda t: t[0])
    for p in ps:
        p.join(timeout=60)
    return out


def test_fused_exchange_routes_every_payload_through_the_slots_world2(tmp_path):
    """Two ranks exchange five compressed steps through each other's slots
    (shared memory standing in for peer-mapped GPU memory): every receiver
    state equals the oracle run on that peer's shard bit for bit, both slots
    are reused under the ack protocol, and the counters end at five steps."""
    out = _run_fused(tmp_path, 2, 0)
    for rank, status, info, counters in out:
        assert status == "ok", (rank, info)
        ready, ack = counters
        assert ready == [0 if p == rank else 5 * 2 * 16 for p in range(2)], (rank, ready)
        assert ack == [0 if p == rank else 5 for p in range(2)], (rank, ack)


def test_fused_exchange_a_rank_that_leaves_ends_the_survivors_next_step(tmp_path):
    out = _run_fused(tmp_path, 2, 1)
    assert out[1][1] == "left", out
    assert out[0][1] == "timeout" and out[0][2] == 2, out
