"""Sequence-parallel exchange of compressed activations between ranks.

In sequence-parallel serving every GPU computes the activations (K and V of
every layer) of its own token shard and needs every other shard's for
attention.  CompactFusion ("Accelerating Parallel Diffusion Model Serving
with Residual Compression", sections "Approach" and "Key results") sends,
instead of an activation, the compressed difference between it and the
reconstruction the receivers already hold; each receiver keeps one
reconstruction per (peer, buffer) and adds the decoded residual to it.  The
first step (the warmup) exchanges the activations uncompressed.

One compressed step on each rank is three device operations, all enqueued on
the current stream:

1. one batched encode of the rank's buffers, writing codes and scales
   straight into one contiguous payload (``PayloadLayout``);
2. one all-gather of the payloads over the process group (NCCL over NVLink
   on GPUs);
3. one batched decode of every peer's payload into that peer's receiver
   states.

``ShardExchange`` carries the quantize mode (1- or 2-bit codes and per-token
scales), ``LowrankShardExchange`` the low-rank mode (INT4 factors P and Q
and their column scales).  ``FusedShardExchange`` is the quantize mode with
the transfer fused into the kernels: the encode stores each row's payload
straight into every receiver's slot (peer memory) and advances counters
that the receivers' decode waits on, so no collective runs per step.

The arithmetic runs in libcf's kernels (``CudaCodec``); this module lays out
memory and orders the calls.  A caller may pass another codec object with
the same methods (the CPU tests drive the host logic that way).
"""
from __future__ import annotations

import collections
import dataclasses

import torch
import torch.distributed as dist

from . import cf


def _align16(n: int) -> int:
    return (n + 15) & ~15


def _seg(payload: torch.Tensor, off: int, nbytes: int) -> torch.Tensor:
    return payload[off:off + nbytes]


@dataclasses.dataclass(frozen=True)
class PayloadLayout:
    """Where each buffer's codes and scales sit in one rank's payload.

    Per buffer, in buffer order: the packed codes (uint32 [tokens, words]),
    then the per-token fp32 scales, each segment starting on a 16-byte
    boundary (the library's alignment rule), so the payload of a rank is one
    contiguous byte range and the all-gather is a single collective."""
    tokens: int
    channels: int
    bits: int
    buffers: int

    @property
    def words_per_row(self) -> int:
        return (self.channels * self.bits + 31) // 32

    @property
    def codes_bytes(self) -> int:
        return self.tokens * self.words_per_row * 4

    @property
    def scales_bytes(self) -> int:
        return self.tokens * 4

    @property
    def stride(self) -> int:
        return _align16(self.codes_bytes) + _align16(self.scales_bytes)

    @property
    def bytes_per_rank(self) -> int:
        return self.buffers * self.stride

    def codes_offset(self, b: int) -> int:
        return b * self.stride

    def scales_offset(self, b: int) -> int:
        return b * self.stride + _align16(self.codes_bytes)

    def codes(self, payload: torch.Tensor, b: int) -> torch.Tensor:
        """int32 [tokens, words] view of buffer b's codes in a payload."""
        o = self.codes_offset(b)
        return payload[o:o + self.codes_bytes].view(torch.int32).view(self.tokens, self.words_per_row)

    def scales(self, payload: torch.Tensor, b: int) -> torch.Tensor:
        """float32 [tokens] view of buffer b's scales in a payload."""
        o = self.scales_offset(b)
        return payload[o:o + self.scales_bytes].view(torch.float32)


@dataclasses.dataclass(frozen=True)
class LowrankPayloadLayout:
    """Where each buffer's low-rank payload sits in one rank's payload.

    Per buffer, in buffer order, each segment on a 16-byte boundary: the
    packed INT4 codes of P (uint8 [tokens, ceil(rank/2)]), P's column scales
    (fp32 [rank]), the packed codes of Q (uint8 [channels, ceil(rank/2)]),
    Q's column scales (fp32 [rank])."""
    tokens: int
    channels: int
    rank: int
    buffers: int

    @property
    def nibble_bytes(self) -> int:
        return (self.rank + 1) // 2

    def _sizes(self):
        nb = self.nibble_bytes
        return (self.tokens * nb, 4 * self.rank, self.channels * nb, 4 * self.rank)

    def _offsets(self):
        offs, o = [], 0
        for n in self._sizes():
            offs.append(o)
            o += _align16(n)
        return offs, o

    @property
    def stride(self) -> int:
        return self._offsets()[1]

    @property
    def bytes_per_rank(self) -> int:
        return self.buffers * self.stride

    def parts(self, payload: torch.Tensor, b: int):
        """(p_codes, p_scales, q_codes, q_scales) views of buffer b."""
        offs, _ = self._offsets()
        base = b * self.stride
        pc, ps, qc, qs = (_seg(payload, base + o, n) for o, n in zip(offs, self._sizes()))
        nb = self.nibble_bytes
        return (pc.view(self.tokens, nb), ps.view(torch.float32), qc.view(self.channels, nb),
                qs.view(torch.float32))


class CudaCodec:
    """The product path: libcf's batched kernels.  The device arrays of
    buffer pointers are kept for the last `cache` pointer sets, so inputs
    that cycle through a fixed set of tensors cost no host-to-device copy of
    pointers per step."""

    def __init__(self, device: torch.device, cache: int = 64):
        self.device = device
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self._cache = collections.OrderedDict()
        self._cache_size = cache

    def _array(self, kind, sets, make):
        key = (kind,) + tuple(0 if t is None else t if isinstance(t, int) else t.data_ptr()
                              for s in sets for t in s)
        arr = self._cache.get(key)
        if arr is None:
            arr = make(sets, self.device)
            self._cache[key] = arr
            if len(self._cache) > self._cache_size:
                self._cache.popitem(last=False)
        else:
            self._cache.move_to_end(key)
        return arr

    def state_init(self, d, x, recon, err):
        cf.cf_state_init(d, x, recon, err)

    def prepare_encode(self, d, sets):
        self._array("enc", sets, cf.enc_buffer_array)

    def encode_batched(self, d, sets):
        cf.cf_encode_batched(d, len(sets), self._array("enc", sets, cf.enc_buffer_array), self.status)

    def decode_batched(self, d, sets):
        if sets:
            cf.cf_decode_batched(d, len(sets), self._array("dec", sets, cf.dec_buffer_array), self.status)

    def decode_emit_batched(self, d, sets):
        if sets:
            cf.cf_decode_emit_batched(d, len(sets), self._array("emit", sets, cf.dec_emit_buffer_array),
                                      self.status)

    def lowrank_workspace_bytes(self, d) -> int:
        return cf.cf_lowrank_workspace_bytes(d)

    def lowrank_status(self, workspace_slice) -> int:
        return cf.cf_lowrank_status(workspace_slice)

    def lowrank_encode_batched(self, d, sets, workspace):
        cf.cf_lowrank_encode_batched(d, len(sets), self._array("lr_enc", sets, cf.lowrank_buffer_array),
                                     workspace)

    def lowrank_decode_batched(self, d, sets):
        if sets:
            cf.cf_lowrank_decode_batched(d, len(sets),
                                         self._array("lr_dec", sets, cf.lowrank_dec_buffer_array),
                                         self.status)

    def encode_publish_batched(self, d, sets, dsts, ack_target):
        arr = self._array("pub", sets, cf.enc_publish_buffer_array)
        dst = self._array("dst", dsts, cf.publish_dst_array)
        cf.cf_encode_publish_batched(d, len(sets), arr, len(dsts), dst, ack_target, self.status)

    def prepare_publish(self, enc, dsts, dec, acks):
        self._array("pub", enc, cf.enc_publish_buffer_array)
        self._array("dst", dsts, cf.publish_dst_array)
        if dec:
            self._array("wait", dec, cf.dec_wait_buffer_array)
        if acks:
            self._array("ack", [(a,) for a in acks], lambda v, dev: cf.pointer_array([t[0] for t in v], dev))

    def decode_wait_batched(self, d, sets, ready_target, acks):
        arr = self._array("wait", sets, cf.dec_wait_buffer_array) if sets else None
        ack = self._array("ack", [(a,) for a in acks], lambda v, dev: cf.pointer_array(
            [t[0] for t in v], dev)) if acks else None
        cf.cf_decode_wait_batched(d, len(sets), arr, ready_target, len(acks), ack, self.status)

    def status_value(self) -> int:
        """First error any batched call recorded (synchronises)."""
        return int(self.status.item())


class _Exchange:
    """What both modes share: the process group, this rank's sender state
    for its shard of `buffers` activations, a receiver state per peer, the
    payload buffers, the warmup and checkpoints."""

    def __init__(self, layout, d, tokens, channels, buffers, group, device, codec, loopback):
        if tokens < 1 or channels < 1 or buffers < 1:
            raise ValueError("tokens, channels and buffers must be positive")
        self.group = group
        if dist.is_available() and dist.is_initialized():
            self.world = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
            self.backend = dist.get_backend(group)
        else:
            self.world, self.rank, self.backend = 1, 0, None
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.device = torch.device(device)
        self.codec = codec if codec is not None else CudaCodec(self.device)
        self.layout, self.d = layout, d
        self.tokens, self.channels, self.buffers = tokens, channels, buffers
        n = layout.bytes_per_rank
        self.send = torch.zeros(n, dtype=torch.uint8, device=self.device)
        self.recv = torch.zeros(self.world * n, dtype=torch.uint8, device=self.device)
        f32 = dict(dtype=torch.float32, device=self.device)
        self.recon_s = [torch.empty(tokens, channels, **f32) for _ in range(buffers)]
        self.err = [torch.empty(tokens, channels, **f32) for _ in range(buffers)]
        self.peers = [p for p in range(self.world) if loopback or p != self.rank]
        self.recon_r = [[torch.empty(tokens, channels, **f32) for _ in range(buffers)]
                        if p in self.peers else None for p in range(self.world)]
        self.emit = False
        self.out = [None] * self.world

    def _payload(self, p: int) -> torch.Tensor:
        n = self.layout.bytes_per_rank
        return self.recv[p * n:(p + 1) * n]

    def _all_gather(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        if self.backend is None:
            out.copy_(inp)
        elif self.backend == "nccl":
            dist.all_gather_into_tensor(out, inp, group=self.group)
        else:
            dist.all_gather(list(out.chunk(self.world)), inp, group=self.group)

    def _check(self, xs):
        if len(xs) != self.buffers:
            raise ValueError(f"expected {self.buffers} activations, got {len(xs)}")
        for x in xs:
            if (x.dtype != torch.bfloat16 or tuple(x.shape) != (self.tokens, self.channels)
                    or not x.is_contiguous()):
                raise ValueError("each activation must be a contiguous bf16 [tokens, channels] tensor")
            if x.data_ptr() % 16:
                raise ValueError("each activation must start on a 16-byte boundary")

    def warmup(self, xs) -> None:
        """Step 0: exchange the activations uncompressed; every receiver
        state starts from the exact activation and the error buffers from 0."""
        self._check(xs)
        T, C, B = self.tokens, self.channels, self.buffers
        n = T * C * 2
        seg = _align16(n)            # every activation starts on a 16-byte boundary

        def at(buf, i):
            return buf[i * seg:i * seg + n].view(torch.bfloat16).view(T, C)

        local = torch.zeros(B * seg, dtype=torch.uint8, device=self.device)
        for b in range(B):
            at(local, b).copy_(xs[b])
        every = torch.empty(self.world * B * seg, dtype=torch.uint8, device=self.device)
        self._all_gather(every, local)
        for b in range(B):
            self.codec.state_init(self.d, xs[b], self.recon_s[b], self.err[b])
            for p in self.peers:
                self.codec.state_init(self.d, at(every, p * B + b), self.recon_r[p][b], None)
                if self.emit:
                    self.out[p][b].copy_(at(every, p * B + b))

    def state_dict(self) -> dict:
        """Everything a resumed exchange needs, as host copies, taken between
        steps: this rank's sender state (recon_s, err) and its receivers'
        reconstructions (and bf16 copies when emitting)."""
        host = lambda ts: [t.detach().cpu().clone() for t in ts]  # noqa: E731
        sd = {"layout": dataclasses.asdict(self.layout), "rank": self.rank, "world": self.world,
              "recon_s": host(self.recon_s), "err": host(self.err),
              "recon_r": {p: host(self.recon_r[p]) for p in self.peers}}
        if self.emit:
            sd["out"] = {p: host(self.out[p]) for p in self.peers}
        return sd

    def load_state_dict(self, sd: dict) -> None:
        """Restore a state_dict taken on the same rank of an exchange with
        the same layout, world size, peers and emit setting."""
        if (sd["layout"] != dataclasses.asdict(self.layout) or sd["rank"] != self.rank
                or sd["world"] != self.world or sorted(sd["recon_r"]) != self.peers
                or ("out" in sd) != self.emit):
            raise ValueError("state_dict was taken on a different exchange")
        for dst, src in ((self.recon_s, sd["recon_s"]), (self.err, sd["err"])):
            for d, s_ in zip(dst, src):
                d.copy_(s_)
        for p in self.peers:
            for d, s_ in zip(self.recon_r[p], sd["recon_r"][p]):
                d.copy_(s_)
            if self.emit:
                for d, s_ in zip(self.out[p], sd["out"][p]):
                    d.copy_(s_)

    def payload_bytes_per_step(self) -> int:
        """Bytes this rank sends per compressed step."""
        return self.layout.bytes_per_rank


class ShardExchange(_Exchange):
    """The quantize mode.  tokens, channels: this rank's shard of one buffer
    (every rank's shard has the same shape); bits: 1 or 2.  `loopback` also
    keeps a receiver for the rank's own shard and decodes its own payload,
    which on one GPU runs the whole path (its reconstruction must equal the
    sender's mirror bit for bit).  recon_r[p][b] is the reconstruction of
    peer p's buffer b (None for the rank's own shard unless `loopback`).
    With `emit`, the decode also writes out[p][b], the bf16 rounding of
    recon_r[p][b] that attention reads, in the same pass."""

    def __init__(self, tokens: int, channels: int, bits: int, buffers: int, *, group=None,
                 device=None, codec=None, loopback: bool = False, emit: bool = False):
        if bits not in (1, 2):
            raise ValueError(f"bits must be 1 or 2, got {bits}")
        super().__init__(PayloadLayout(tokens, channels, bits, buffers), cf.desc(tokens, channels, bits),
                         tokens, channels, buffers, group, device, codec, loopback)
        self.emit = emit
        self.out = [[torch.empty(tokens, channels, dtype=torch.bfloat16, device=self.device)
                     for _ in range(buffers)] if emit and p in self.peers else None
                    for p in range(self.world)]
        L = self.layout
        self._dec_sets = [(L.codes(self._payload(p), b), L.scales(self._payload(p), b), self.recon_r[p][b])
                          + ((self.out[p][b],) if emit else ())
                          for p in self.peers for b in range(buffers)]

    def _enc_sets(self, xs):
        if not hasattr(self, "_send_views"):   # built once: views cost host time every step
            L = self.layout
            self._send_views = [(L.codes(self.send, b), L.scales(self.send, b)) for b in range(L.buffers)]
        return [(xs[b], self.recon_s[b], self.err[b]) + self._send_views[b] for b in range(self.buffers)]

    def prepare(self, xs) -> None:
        """Optional: build the codec's per-call state (the device array of
        buffer pointers) for these input tensors ahead of their step."""
        self._check(xs)
        if hasattr(self.codec, "prepare_encode"):
            self.codec.prepare_encode(self.d, self._enc_sets(xs))

    def step(self, xs, events=None) -> None:
        """One compressed step: encode into the payload, all-gather, decode
        every peer's payload into its receiver states.  `events`, four CUDA
        events, are recorded on the current stream before the encode, after
        it, after the all-gather and after the decode."""
        self._check(xs)
        mark = (lambda i: events[i].record()) if events is not None else (lambda i: None)
        mark(0)
        self.codec.encode_batched(self.d, self._enc_sets(xs))
        mark(1)
        self._all_gather(self.recv, self.send)
        mark(2)
        if self.emit:
            self.codec.decode_emit_batched(self.d, self._dec_sets)
        else:
            self.codec.decode_batched(self.d, self._dec_sets)
        mark(3)


class LowrankShardExchange(_Exchange):
    """The low-rank mode: rank `rank` factors from `iters` subspace
    iterations, INT4-quantised.  Each step's encode takes one fp32 [C, rank]
    Gaussian start block per buffer (`omegas`), or None for the warm start
    from the previous step's Q (allowed only for a buffer that an earlier
    step encoded; otherwise step() raises ValueError).  The encode
    uses a device workspace of cf_lowrank_workspace_bytes per buffer;
    status() reads the numeric status of every buffer.  Otherwise as
    ShardExchange (no bf16 emission)."""

    def __init__(self, tokens: int, channels: int, rank: int, iters: int, buffers: int, *,
                 group=None, device=None, codec=None, loopback: bool = False):
        if rank < 1 or iters < 1:
            raise ValueError("rank and iters must be positive")
        super().__init__(LowrankPayloadLayout(tokens, channels, rank, buffers),
                         cf.desc(tokens, channels, 0, rank, iters),
                         tokens, channels, buffers, group, device, codec, loopback)
        self.ws_bytes = self.codec.lowrank_workspace_bytes(self.d)
        self.workspace = torch.zeros(buffers * self.ws_bytes, dtype=torch.uint8, device=self.device)
        # buffer b's workspace slice holds a Q to warm-start from only after
        # an encode of that buffer with a start block
        self.encoded = [False] * buffers
        L = self.layout
        self._dec_sets = [L.parts(self._payload(p), b) + (self.recon_r[p][b],)
                          for p in self.peers for b in range(buffers)]

    def step(self, xs, omegas=None) -> None:
        """One compressed step: encode into the payload, all-gather, decode
        every peer's payload into its receiver states."""
        self._check(xs)
        if omegas is None:
            omegas = [None] * self.buffers
        if len(omegas) != self.buffers:
            raise ValueError(f"expected {self.buffers} start blocks, got {len(omegas)}")
        cold = [b for b in range(self.buffers) if omegas[b] is None and not self.encoded[b]]
        if cold:
            raise ValueError(f"buffers {cold} have no earlier encode to warm-start from: "
                             "the first compressed step needs a start block for every buffer")
        for om in omegas:
            if om is not None and (om.dtype != torch.float32 or tuple(om.shape) != (self.channels, self.layout.rank)
                                   or not om.is_contiguous()):
                raise ValueError("each start block must be a contiguous fp32 [channels, rank] tensor")
        L = self.layout
        sets = [(xs[b], self.recon_s[b], self.err[b], omegas[b]) + L.parts(self.send, b)
                for b in range(self.buffers)]
        self.codec.lowrank_encode_batched(self.d, sets, self.workspace)
        self.encoded = [True] * self.buffers
        self._all_gather(self.recv, self.send)
        self.codec.lowrank_decode_batched(self.d, self._dec_sets)

    def state_dict(self) -> dict:
        """As for the quantize mode, plus the encode workspace: it holds each
        buffer's last Q, the warm start of the next step."""
        sd = super().state_dict()
        sd["workspace"] = self.workspace.detach().cpu().clone()
        sd["encoded"] = list(self.encoded)
        return sd

    def load_state_dict(self, sd: dict) -> None:
        if ("workspace" not in sd or sd["workspace"].numel() != self.workspace.numel()
                or len(sd.get("encoded", ())) != self.buffers):
            raise ValueError("state_dict was taken on a different exchange")
        super().load_state_dict(sd)
        self.workspace.copy_(sd["workspace"])
        self.encoded = list(sd["encoded"])

    def status(self) -> list:
        """Per-buffer numeric status of the last encodes (synchronises; the
        codec reads and clears each buffer's status word)."""
        return [self.codec.lowrank_status(self.workspace[b * self.ws_bytes:(b + 1) * self.ws_bytes])
                for b in range(self.buffers)]


# ---------------------------------------------------------------- fused exchange

@dataclasses.dataclass
class SlotMemory:
    """The memory the fused exchange writes through, as seen from one rank.

    For every rank r (all addressable from this rank: its own memory, and
    each peer's through peer access):
      recv[r]  uint8 [2, world, bytes_per_rank]: slot s of sender p's payload
               at receiver r is recv[r][s, p];
      ready[r] int64 [world]: rows sender p has published to receiver r;
      ack[r]   int64 [world]: steps receiver q has decoded from r's payloads.
    Counters only grow; a fresh SlotMemory starts them at zero."""
    recv: list
    ready: list
    ack: list


def local_slot_memory(layout, world: int, device) -> SlotMemory:
    """One process owning every rank's memory (one rank in loopback on one
    GPU, or a test that stands in for several ranks)."""
    return SlotMemory(
        recv=[torch.zeros(2, world, layout.bytes_per_rank, dtype=torch.uint8, device=device)
              for _ in range(world)],
        ready=[torch.zeros(world, dtype=torch.int64, device=device) for _ in range(world)],
        ack=[torch.zeros(world, dtype=torch.int64, device=device) for _ in range(world)])


def symmetric_slot_memory(layout, group, device) -> SlotMemory:
    """Every rank's slots and counters in one symmetric allocation per rank
    (torch symmetric memory), each peer's mapped for peer access.  The
    kernels only store to and atomically add into the peers' memory; no TMA
    load and no collective reads it."""
    import torch.distributed._symmetric_memory as symm_mem
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    nrecv = 2 * world * layout.bytes_per_rank
    total = nrecv + 16 * world                       # + ready[world] + ack[world], int64
    buf = symm_mem.empty(total, dtype=torch.uint8, device=device)
    buf.zero_()
    hdl = symm_mem.rendezvous(buf, group)
    dist.barrier(group)
    mem = SlotMemory([], [], [])
    for r in range(world):
        t = buf if r == rank else hdl.get_buffer(r, (total,), torch.uint8)
        mem.recv.append(t[:nrecv].view(2, world, layout.bytes_per_rank))
        mem.ready.append(t[nrecv:nrecv + 8 * world].view(torch.int64))
        mem.ack.append(t[nrecv + 8 * world:].view(torch.int64))
    mem._keep = (buf, hdl)  # the mapping lives as long as the exchange
    return mem


class FusedShardExchange(_Exchange):
    """The quantize-mode exchange with the transfer fused into the codec
    kernels: each step is one publishing encode, which stores every row's
    codes and scale straight into every receiver's slot for this rank and
    then advances the receivers' ready counters, and one waiting decode of
    every peer's slot, which reads a peer's rows once its counter shows them
    and then acknowledges the step to every sender.  Two slots per (receiver,
    sender) are used in turn; before it overwrites a slot the encode waits
    until the receiver has acknowledged the step that last used it.  No
    collective runs per step.  `memory` defaults to symmetric memory across
    the process group (one local allocation for a single rank)."""

    def __init__(self, tokens: int, channels: int, bits: int, buffers: int, *, group=None,
                 device=None, codec=None, loopback: bool = False, memory: SlotMemory = None):
        if bits not in (1, 2):
            raise ValueError(f"bits must be 1 or 2, got {bits}")
        super().__init__(PayloadLayout(tokens, channels, bits, buffers), cf.desc(tokens, channels, bits),
                         tokens, channels, buffers, group, device, codec, loopback)
        if not self.peers:
            raise ValueError("a single rank needs loopback=True: it has no other receiver")
        self.send = self.recv = None          # the slots replace the gather buffers
        if memory is None:
            memory = (local_slot_memory(self.layout, 1, self.device) if self.world == 1
                      else symmetric_slot_memory(self.layout, group, self.device))
        self.memory = memory
        self.epoch = 0          # compressed steps taken
        self.base = 0           # epoch at which this memory's counters were zero

    def _receivers(self):
        """Ranks whose slots this rank's payload goes to (the same set as the
        ranks it decodes: the exchange is symmetric)."""
        return self.peers

    def _sets(self, xs, s):
        """The encode's buffers, its destinations (slot s at every receiver)
        and the decode's buffers and ack counters for one step.  The views of
        a slot are built once and kept: a step would otherwise spend more
        host time making hundreds of tensor views than the GPU spends on its
        kernels."""
        me, L, m = self.rank, self.layout, self.memory
        cache = self.__dict__.setdefault("_slot_sets", {})
        if s not in cache:
            dsts = [(m.recv[r][s, me], m.ready[r][me:me + 1], m.ack[me][r:r + 1])
                    for r in self._receivers()]
            dec, acks = [], []
            for p in self.peers:
                slot = m.recv[me][s, p]
                dec += [(L.codes(slot, b), L.scales(slot, b), self.recon_r[p][b], m.ready[me][p:p + 1])
                        for b in range(self.buffers)]
                acks.append(m.ack[p][me:me + 1])
            cache[s] = (dsts, dec, acks)
        dsts, dec, acks = cache[s]
        enc = [(xs[b], self.recon_s[b], self.err[b], L.codes_offset(b), L.scales_offset(b))
               for b in range(self.buffers)]
        return enc, dsts, dec, acks

    def prepare(self, xs) -> None:
        """Optional: build the codec's device arrays of pointers for these
        input tensors (both slots) ahead of their steps."""
        self._check(xs)
        if hasattr(self.codec, "prepare_publish"):
            for s in (0, 1):
                enc, dsts, dec, acks = self._sets(xs, s)
                self.codec.prepare_publish(enc, dsts, dec, acks)

    def step(self, xs, events=None) -> None:
        """One compressed step: the publishing encode, then the waiting
        decode of every peer's slot.  `events`, four CUDA events, are
        recorded on the current stream before the encode, after it (twice:
        there is no collective in between) and after the decode."""
        self._check(xs)
        mark = (lambda i: events[i].record()) if events is not None else (lambda i: None)
        self.epoch += 1
        k = self.epoch - self.base           # steps on this memory's counters
        enc, dsts, dec, acks = self._sets(xs, self.epoch % 2)
        mark(0)
        self.codec.encode_publish_batched(self.d, enc, dsts, max(k - 2, 0))
        mark(1)
        mark(2)
        self.codec.decode_wait_batched(self.d, dec, k * self.buffers * self.tokens, acks)
        mark(3)

    def state_dict(self) -> dict:
        sd = super().state_dict()
        sd["epoch"] = self.epoch
        return sd

    def load_state_dict(self, sd: dict) -> None:
        """Restores the states into this exchange, whose slot memory must be
        fresh (counters at zero on every rank): the counters then count from
        the restored step on."""
        if "epoch" not in sd:
            raise ValueError("state_dict was taken on a different exchange")
        super().load_state_dict(sd)
        self.epoch = self.base = int(sd["epoch"])
