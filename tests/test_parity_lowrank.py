"""GPU parity of the low-rank mode (cf_lowrank_encode / cf_lowrank_decode)
against the fp64 CPU oracle, through the C ABI.

Bar: the relative Frobenius error ||V - D||_F / ||V||_F of the GPU payload is
within 1% of the oracle's on the same input (teacher-forced: both sides start
each step from the GPU's pre-step state).  Also checked at every step: the
error-feedback identity recon_s + err == x, receiver == sender bit for bit,
INT4 codes in [-7, 7] with the column maximum at +-7, and the payload ratio.
"""
import numpy as np
import pytest
import torch

from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W
from oracle import lowrank as L

pytestmark = pytest.mark.gpu

REL_FROB_TOL = 0.01


class GpuLowrank:
    def __init__(self, T, C, r, iters, dev="cuda"):
        self.d = cf.desc(T, C, 0, r, iters)
        self.T, self.C, self.r = T, C, r
        nb = (r + 1) // 2
        f32 = dict(dtype=torch.float32, device=dev)
        self.recon_s = torch.empty(T, C, **f32)
        self.recon_r = torch.empty(T, C, **f32)
        self.err = torch.empty(T, C, **f32)
        self.pc = torch.empty(T * nb + 16, dtype=torch.uint8, device=dev)
        self.qc = torch.empty(C * nb + 16, dtype=torch.uint8, device=dev)
        self.ps = torch.empty(r, **f32)
        self.qs = torch.empty(r, **f32)
        self.ws = torch.empty(cf.cf_lowrank_workspace_bytes(self.d), dtype=torch.uint8, device=dev)

    def init(self, x0):
        cf.cf_state_init(self.d, x0.view(torch.int16), self.recon_s, self.err)
        cf.cf_state_init(self.d, x0.view(torch.int16), self.recon_r, None)

    def step(self, x, omega):
        cf.cf_lowrank_encode(self.d, x.view(torch.int16), self.recon_s, self.err, omega,
                             self.pc, self.ps, self.qc, self.qs, self.ws)
        cf.cf_lowrank_decode(self.d, self.pc, self.ps, self.qc, self.qs, self.recon_r)

    def payload(self):
        nb = (self.r + 1) // 2
        return (self.pc[: self.T * nb].cpu().numpy().reshape(self.T, nb), self.ps.cpu().numpy(),
                self.qc[: self.C * nb].cpu().numpy().reshape(self.C, nb), self.qs.cpu().numpy())


def _rel_err(v, d):
    v64 = v.astype(np.float64)
    return np.linalg.norm(v64 - d.astype(np.float64)) / np.linalg.norm(v64)


def _check_codes(packed, scales, r):
    q = L.int4_unpack(packed, r)
    assert q.min() >= -7 and q.max() <= 7
    live = scales > 0
    assert np.all(np.abs(q[:, live]).max(axis=0) == 7)
    assert not np.any(q[:, ~live])


def _run(wl, steps, buffer=0, check_frob=True, warm=False):
    """Teacher-forced parity over a trajectory.  warm=True: from the second
    compressed step on, the GPU starts from the Q its previous encode left
    in the workspace (omega NULL) and the oracle from its own previous Q."""
    T, C, r, it = wl.tokens, wl.channels, wl.rank, wl.iters
    xs = W.trajectory(wl, buffer, steps=steps, device="cuda")
    g = GpuLowrank(T, C, r, it)
    g.init(xs[0].clone())
    errs = []
    q_prev = None
    for s in range(1, steps):
        x = xs[s].clone()
        om = W.omega(wl, buffer, s, device="cuda")
        om_ora = om.cpu().numpy()
        if warm and q_prev is not None:
            om, om_ora = None, q_prev
        recon_before = g.recon_s.cpu().numpy()
        g.step(x, om)
        torch.cuda.synchronize()
        assert cf.cf_lowrank_status(g.ws) in (0,)
        xb = W.bf16_bits(x)
        xf = L.bf16_bits_to_f32(xb)
        v = (xf - recon_before).astype(np.float32)
        rs, er, rr = g.recon_s.cpu().numpy(), g.err.cpu().numpy(), g.recon_r.cpu().numpy()
        # D as the GPU applied it, and the EF identity
        d_gpu = (rs.astype(np.float64) - recon_before)
        gap = np.abs(rs.astype(np.float64) + er - xf)
        assert gap.max() <= 4 * np.spacing(np.float32(np.abs(xf).max() + np.abs(v).max()))
        assert np.array_equal(rr.view(np.uint32), rs.view(np.uint32))
        pc, ps, qc, qs = g.payload()
        _check_codes(pc, ps, r)
        _check_codes(qc, qs, r)
        # the D the payload encodes (oracle reconstruction of the GPU payload)
        d_pay = L.reconstruct(pc, ps, qc, qs, r)
        tol = 4 * np.spacing(np.float32(np.abs(rs).max())) + 1e-5 * np.abs(d_pay).max()
        assert np.max(np.abs(d_pay - d_gpu)) <= tol
        # oracle on the same input
        ro = recon_before.copy()
        out = L.lowrank_encode(xb, ro, om_ora, it)
        q_prev = out["Q"]
        e_gpu, e_ora = _rel_err(v, d_pay), _rel_err(out["V"], out["D"])
        errs.append((e_gpu, e_ora))
        if check_frob:
            assert abs(e_gpu - e_ora) <= REL_FROB_TOL * e_ora, (s, e_gpu, e_ora)
    return errs


def test_small_lowrank_trajectory():
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=256, channels=192, rank=8)
    _run(wl, 4)


@pytest.mark.parametrize("T,C,r,iters", [(100, 200, 5, 1), (300, 136, 16, 3), (77, 64, 33, 2),
                                         (640, 512, 64, 2), (1000, 1000, 32, 2),
                                         (64, 8, 1, 1),        # rank 1, the narrowest rows
                                         (40, 64, 8, 16),      # the most iterations
                                         (33, 264, 32, 2),     # barely more tokens than the rank
                                         (17550, 1920, 32, 2)])  # 138 token tiles per Gram
def test_lowrank_ragged_shapes(T, C, r, iters):
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r, iters=iters)
    _run(wl, 3)


def test_lowrank_full_size_sampled():
    """The low-rank workload at full size (4096 x 3072, rank 32, 2
    iterations), one buffer, three compressed steps."""
    errs = _run(W.WORKLOADS["lowrank"], 4, buffer=7)
    assert all(e < 0.5 for e, _ in errs)


def test_lowrank_zero_residual_and_status():
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=128, channels=64, rank=4)
    x = W.trajectory(wl, 0, steps=1, device="cuda")[0].clone()
    g = GpuLowrank(128, 64, 4, 2)
    g.init(x)
    before = g.recon_s.clone()
    g.step(x, W.omega(wl, 0, 1, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(g.recon_s, before) and torch.equal(g.recon_r, before)
    assert not bool(g.err.any())
    assert cf.cf_lowrank_status(g.ws) == 6          # CF_ERR_NUMERIC: Y has no rank
    assert cf.cf_lowrank_status(g.ws) == 0          # cleared by the read


def test_lowrank_exact_rank_input():
    """A residual of rank 3 < r: Y has only 3 independent columns, the other
    Cholesky pivots are dead (status CF_ERR_NUMERIC, zero P columns), and the
    remaining error is the INT4 factor error, within 1% of the oracle's."""
    T, C, r = 256, 128, 8
    g = GpuLowrank(T, C, r, 2)
    gen = torch.Generator(device="cuda").manual_seed(5)
    x0 = torch.zeros(T, C, dtype=torch.bfloat16, device="cuda")
    g.init(x0)
    # small integers: u w^T is exact in bf16, so the input has rank exactly 3
    u = torch.randint(-3, 4, (T, 3), generator=gen, device="cuda").float()
    w = torch.randint(-3, 4, (C, 3), generator=gen, device="cuda").float()
    x = (u @ w.T).to(torch.bfloat16)
    assert torch.equal(x.float(), u @ w.T)
    om = torch.randn(C, r, generator=gen, device="cuda")
    g.step(x, om)
    torch.cuda.synchronize()
    assert cf.cf_lowrank_status(g.ws) == 6
    xb = W.bf16_bits(x)
    v = L.bf16_bits_to_f32(xb)
    d = g.recon_s.cpu().numpy()
    ro = np.zeros((T, C), np.float32)
    out = L.lowrank_encode(xb, ro, om.cpu().numpy(), 2)
    e_gpu, e_ora = _rel_err(v, d), _rel_err(out["V"], out["D"])
    assert abs(e_gpu - e_ora) <= REL_FROB_TOL * e_ora, (e_gpu, e_ora)
    pc, ps, qc, qs = g.payload()
    assert int((ps > 0).sum()) == 3 and int((qs > 0).sum()) == 3


@pytest.mark.parametrize("T,C,r", [(4096, 3072, 32), (300, 136, 16), (640, 512, 64), (77, 64, 33)])
def test_tensor_core_and_cuda_core_products_agree(T, C, r):
    """The tcgen05 products and the CUDA-core products read the same bf16
    operands and accumulate in fp32; the payloads they produce agree up to
    summation order, and both meet the oracle bar."""
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    xs = W.trajectory(wl, 3, steps=2, device="cuda")
    om = W.omega(wl, 3, 1, device="cuda")
    outs = []
    try:
        for engine in (1, 0):
            cf.cf_set_lowrank_engine(engine)
            g = GpuLowrank(T, C, r, 2)
            g.init(xs[0].clone())
            g.step(xs[1].clone(), om)
            torch.cuda.synchronize()
            assert cf.cf_lowrank_status(g.ws) == 0
            outs.append((g.payload(), g.recon_s.cpu().numpy()))
    finally:
        cf.cf_set_lowrank_engine(0)
    (p1, r1), (p0, r0) = outs
    # per-column scales of the weak (noise) directions may rotate with the
    # summation order; the leading columns and the product must agree
    assert np.allclose(p0[1][:8], p1[1][:8], rtol=1e-3)
    d0 = L.reconstruct(p0[0], p0[1], p0[2], p0[3], r)
    d1 = L.reconstruct(p1[0], p1[1], p1[2], p1[3], r)
    v = L.bf16_bits_to_f32(W.bf16_bits(xs[1])) - L.bf16_bits_to_f32(W.bf16_bits(xs[0]))
    e0, e1 = _rel_err(v, d0), _rel_err(v, d1)
    assert abs(e0 - e1) <= REL_FROB_TOL * e1, (e0, e1)
    assert np.linalg.norm(d0 - d1) <= 5e-2 * np.linalg.norm(d1)


def test_workspace_too_small_is_rejected():
    g = GpuLowrank(64, 64, 4, 1)
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    x = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    om = torch.zeros(64, 4, device="cuda")
    with pytest.raises(cf.CFError) as ei:
        cf.cf_lowrank_encode(g.d, x.view(torch.int16), g.recon_s, g.err, om, g.pc, g.ps, g.qc,
                             g.qs, small)
    assert ei.value.status == 4


# The larger batches give the apply kernel several token tiles per CTA (its
# persistent path), with ragged channel and token tails, at rank <= 32 and 64.
@pytest.mark.parametrize("T,C,r,n", [(4096, 3072, 32, 4), (300, 136, 16, 3), (77, 64, 33, 2),
                                     (1100, 264, 16, 64), (650, 520, 64, 32)])
def test_batched_lowrank_equals_single_calls(T, C, r, n):
    """One batched call over n buffers computes exactly what n single calls do
    (same kernels, fixed reduction orders), for the sender and the receiver;
    a buffer with a misaligned pointer is skipped and reported in its own
    workspace status word."""
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    d = cf.desc(T, C, 0, r, 2)
    wsb = cf.cf_lowrank_workspace_bytes(d)
    xs = [W.trajectory(wl, b, steps=2, device="cuda") for b in range(n)]
    oms = [W.omega(wl, b, 1, device="cuda") for b in range(n)]
    single = [GpuLowrank(T, C, r, 2) for _ in range(n)]
    batch = [GpuLowrank(T, C, r, 2) for _ in range(n)]
    for b in range(n):
        for g in (single[b], batch[b]):
            g.init(xs[b][0].clone())
    for b in range(n):
        single[b].step(xs[b][1].clone(), oms[b])
    xb = [xs[b][1].clone() for b in range(n)]
    ws = torch.empty(n * wsb, dtype=torch.uint8, device="cuda")
    enc = cf.lowrank_buffer_array([(xb[b].view(torch.int16), batch[b].recon_s, batch[b].err, oms[b],
                                    batch[b].pc, batch[b].ps, batch[b].qc, batch[b].qs)
                                   for b in range(n)], "cuda")
    dec = cf.lowrank_dec_buffer_array([(batch[b].pc, batch[b].ps, batch[b].qc, batch[b].qs,
                                        batch[b].recon_r) for b in range(n)], "cuda")
    cf.cf_lowrank_encode_batched(d, n, enc, ws)
    cf.cf_lowrank_decode_batched(d, n, dec)
    torch.cuda.synchronize()
    nb = (r + 1) // 2
    for b in range(n):
        assert cf.cf_lowrank_status(ws[b * wsb:]) == 0
        for k in ("recon_s", "recon_r", "err", "ps", "qs"):
            assert torch.equal(getattr(batch[b], k), getattr(single[b], k)), (b, k)
        # the code arrays carry 16 spare bytes past the payload; compare the payload
        assert torch.equal(batch[b].pc[:T * nb], single[b].pc[:T * nb]), b
        assert torch.equal(batch[b].qc[:C * nb], single[b].qc[:C * nb]), b
    # a misaligned recon pointer: that buffer is skipped, the others run
    bad = GpuLowrank(T, C, r, 2)
    bad.init(xs[0][0].clone())
    before = bad.recon_s.clone()
    rows = [(xb[0].view(torch.int16), bad.recon_s.data_ptr() + 4, bad.err, oms[0], bad.pc, bad.ps,
             bad.qc, bad.qs)]
    cf.cf_lowrank_encode_batched(d, 1, cf.lowrank_buffer_array(rows, "cuda"), ws)
    torch.cuda.synchronize()
    assert cf.cf_lowrank_status(ws) == 2
    assert torch.equal(bad.recon_s, before)


def test_apply_event_hook_times_the_apply_kernel_only():
    """Events handed to cf_lowrank_set_apply_events bracket the apply kernel
    of the next encode and decode: they are recorded (elapsed time > 0, less
    than the whole encode), results are unchanged, and clearing the hook
    stops the recording."""
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=1024, channels=3072)
    xs = W.trajectory(wl, 0, steps=2, device="cuda")
    om = W.omega(wl, 0, 1, device="cuda")
    plain, hooked = GpuLowrank(1024, 3072, 32, 2), GpuLowrank(1024, 3072, 32, 2)
    for g in (plain, hooked):
        g.init(xs[0].clone())
    plain.step(xs[1].clone(), om)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    try:
        cf.cf_lowrank_set_apply_events(ev[0], ev[1], ev[2], ev[3])
        ev[4].record()
        hooked.step(xs[1].clone(), om)
        ev[5].record()
    finally:
        cf.cf_lowrank_set_apply_events()
    torch.cuda.synchronize()
    for k in ("recon_s", "recon_r", "err"):
        assert torch.equal(getattr(plain, k), getattr(hooked, k)), k
    t_enc, t_dec, t_all = ev[0].elapsed_time(ev[1]), ev[2].elapsed_time(ev[3]), ev[4].elapsed_time(ev[5])
    assert 0 < t_enc < t_all and 0 < t_dec < t_all
    # the encode's apply ends before the decode's begins
    assert ev[1].elapsed_time(ev[2]) >= 0


@pytest.mark.parametrize("r", [32, 33])
def test_decode_with_unaligned_codes_matches_aligned(r):
    """Code arrays need only 1-byte alignment: a receiver given the same
    payload at an odd address (and so reading it byte by byte) adds exactly
    the same D as one reading it from an aligned copy."""
    T, C = 700, 264
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    xs = W.trajectory(wl, 0, steps=2, device="cuda")
    g = GpuLowrank(T, C, r, 2)
    g.init(xs[0].clone())
    g.step(xs[1].clone(), W.omega(wl, 0, 1, device="cuda"))
    nb = (r + 1) // 2
    odd_p = torch.zeros(T * nb + 32, dtype=torch.uint8, device="cuda")
    odd_q = torch.zeros(C * nb + 32, dtype=torch.uint8, device="cuda")
    odd_p[1:1 + T * nb] = g.pc[:T * nb]
    odd_q[3:3 + C * nb] = g.qc[:C * nb]
    ref = torch.zeros(T, C, dtype=torch.float32, device="cuda")
    got = torch.zeros(T, C, dtype=torch.float32, device="cuda")
    cf.cf_lowrank_decode(g.d, g.pc, g.ps, g.qc, g.qs, ref)
    cf.cf_lowrank_decode(g.d, odd_p.data_ptr() + 1, g.ps, odd_q.data_ptr() + 3, g.qs, got)
    torch.cuda.synchronize()
    assert torch.equal(ref, got)
    assert ref.abs().max() > 0


@pytest.mark.parametrize("r", [32, 64, 33])
def test_encode_into_unaligned_codes_matches_aligned(r):
    """The encode writes a row's INT4 codes as 16-byte vectors only where the
    row is 16-byte aligned (even rank 32 or 64) and byte by byte otherwise:
    code arrays at odd addresses receive exactly the bytes an aligned
    encode of the same input writes, and the states stay identical."""
    T, C = 700, 264
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    xs = W.trajectory(wl, 0, steps=2, device="cuda")
    om = W.omega(wl, 0, 1, device="cuda")
    a, b = GpuLowrank(T, C, r, 2), GpuLowrank(T, C, r, 2)
    a.init(xs[0].clone())
    b.init(xs[0].clone())
    nb = (r + 1) // 2
    odd_p = torch.zeros(T * nb + 32, dtype=torch.uint8, device="cuda")
    odd_q = torch.zeros(C * nb + 32, dtype=torch.uint8, device="cuda")
    a.step(xs[1].clone(), om)
    cf.cf_lowrank_encode(b.d, xs[1].clone().view(torch.int16), b.recon_s, b.err, om,
                         odd_p.data_ptr() + 1, b.ps, odd_q.data_ptr() + 5, b.qs, b.ws)
    torch.cuda.synchronize()
    assert cf.cf_lowrank_status(a.ws) == 0 and cf.cf_lowrank_status(b.ws) == 0
    assert torch.equal(odd_p[1:1 + T * nb], a.pc[:T * nb])
    assert torch.equal(odd_q[5:5 + C * nb], a.qc[:C * nb])
    assert not odd_p[0].item() and not odd_p[1 + T * nb:].any()      # nothing outside the rows
    assert not odd_q[:5].any() and not odd_q[5 + C * nb:].any()
    assert torch.equal(a.ps, b.ps) and torch.equal(a.qs, b.qs)
    assert torch.equal(a.recon_s, b.recon_s) and torch.equal(a.err, b.err)


def test_warm_start_trajectory():
    """omega NULL after the first compressed step: the iteration starts from
    the previous encode's Q (PowerSGD-style warm start); each step stays
    within the parity bar of the oracle started from its own previous Q."""
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=512, channels=384, iters=1)
    errs = _run(wl, steps=6, warm=True)
    assert len(errs) == 5


def test_warm_start_without_earlier_encode_is_refused():
    """A warm start on a workspace that never held this shape's Q skips the
    buffer (state untouched) and records CF_ERR_INVALID_ARG."""
    T, C, r = 256, 128, 8
    g = GpuLowrank(T, C, r, 2)
    g.ws.zero_()
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    xs = W.trajectory(wl, 0, steps=2, device="cuda")
    g.init(xs[0].clone())
    before = g.recon_s.clone()
    g.step(xs[1].clone(), None)
    torch.cuda.synchronize()
    assert cf.cf_lowrank_status(g.ws) == 1
    assert torch.equal(g.recon_s, before)
    # after one cold encode the same workspace accepts a warm start
    g.step(xs[1].clone(), W.omega(wl, 0, 1, device="cuda"))
    assert cf.cf_lowrank_status(g.ws) == 0
    g.step(xs[1].clone(), None)
    assert cf.cf_lowrank_status(g.ws) == 0
    # another rank on the same workspace does not match the tag
    d2 = cf.desc(T, C, 0, r - 1, 2)
    before = g.recon_s.clone()
    cf.cf_lowrank_encode(d2, xs[1].clone().view(torch.int16), g.recon_s, g.err, None, g.pc, g.ps,
                         g.qc, g.qs, g.ws)
    assert cf.cf_lowrank_status(g.ws) == 1
    assert torch.equal(g.recon_s, before)


def test_warm_start_batched_equals_single():
    """Warm-started batched encodes compute exactly what warm-started single
    encodes do, buffer by buffer."""
    T, C, r, n = 300, 136, 16, 3
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    d = cf.desc(T, C, 0, r, 1)
    wsb = cf.cf_lowrank_workspace_bytes(d)
    xs = [W.trajectory(wl, b, steps=3, device="cuda") for b in range(n)]
    single = [GpuLowrank(T, C, r, 1) for _ in range(n)]
    batch = [GpuLowrank(T, C, r, 1) for _ in range(n)]
    ws = torch.empty(n * wsb, dtype=torch.uint8, device="cuda")
    for b in range(n):
        for g in (single[b], batch[b]):
            g.init(xs[b][0].clone())
    for step in (1, 2):
        xb = [xs[b][step].clone() for b in range(n)]
        oms = [W.omega(wl, b, step, device="cuda") if step == 1 else None for b in range(n)]
        for b in range(n):
            single[b].step(xb[b], oms[b])
        enc = cf.lowrank_buffer_array([(xb[b].view(torch.int16), batch[b].recon_s, batch[b].err,
                                        oms[b], batch[b].pc, batch[b].ps, batch[b].qc, batch[b].qs)
                                       for b in range(n)], "cuda")
        cf.cf_lowrank_encode_batched(d, n, enc, ws)
        torch.cuda.synchronize()
        for b in range(n):
            assert cf.cf_lowrank_status(ws[b * wsb:]) == 0
            assert cf.cf_lowrank_status(single[b].ws) == 0
            for k in ("recon_s", "err", "ps", "qs"):
                assert torch.equal(getattr(batch[b], k), getattr(single[b], k)), (step, b, k)


def test_async_status_reads_every_slice_without_waiting():
    """cf_lowrank_status_async copies each buffer's status word of a batched
    encode into pinned host memory: a normal buffer (CF_OK), a zero residual
    (CF_ERR_NUMERIC), a misaligned pointer (CF_ERR_ALIGNMENT) and a warm
    start without an earlier encode (CF_ERR_INVALID_ARG), in one strided
    copy; the words agree with the blocking per-slice read."""
    T, C, r = 256, 192, 8
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    d = cf.desc(T, C, 0, r, 2)
    wsb = cf.cf_lowrank_workspace_bytes(d)
    n = 4
    xs = W.trajectory(wl, 0, steps=2, device="cuda")
    gs = [GpuLowrank(T, C, r, 2) for _ in range(n)]
    for g in gs:
        g.init(xs[0].clone())
    om = W.omega(wl, 0, 1, device="cuda")
    x1 = xs[1].clone().view(torch.int16)
    x0 = xs[0].clone().view(torch.int16)      # equals the state: zero residual
    rows = [(x1, gs[0].recon_s, gs[0].err, om, gs[0].pc, gs[0].ps, gs[0].qc, gs[0].qs),
            (x0, gs[1].recon_s, gs[1].err, om, gs[1].pc, gs[1].ps, gs[1].qc, gs[1].qs),
            (x1, gs[2].recon_s.data_ptr() + 4, gs[2].err, om, gs[2].pc, gs[2].ps, gs[2].qc, gs[2].qs),
            (x1, gs[3].recon_s, gs[3].err, None, gs[3].pc, gs[3].ps, gs[3].qc, gs[3].qs)]
    ws = torch.empty(n * wsb, dtype=torch.uint8, device="cuda")
    ws.fill_(0x11)   # no earlier encode on these slices: the warm tag is absent
    host = torch.full((n,), -1, dtype=torch.int32).pin_memory()
    cf.cf_lowrank_encode_batched(d, n, cf.lowrank_buffer_array(rows, "cuda"), ws)
    cf.cf_lowrank_status_async(ws, wsb, n, host)
    ev = torch.cuda.Event()
    ev.record()
    ev.synchronize()
    assert host.tolist() == [0, 6, 2, 1]
    assert [cf.cf_lowrank_status(ws[b * wsb:]) for b in range(n)] == [0, 6, 2, 1]
    # pageable host memory is refused: the copy would not be asynchronous
    with pytest.raises(cf.CFError) as ei:
        cf.cf_lowrank_status_async(ws, wsb, n, torch.zeros(n, dtype=torch.int32))
    assert ei.value.status == 1


@pytest.mark.parametrize("group", [1, 3])
def test_grouped_batched_encode_is_bit_identical(group):
    """A batched encode run g buffers at a time (cf_set_lowrank_group)
    computes exactly what the all-buffers launches do."""
    T, C, r, n = 640, 384, 16, 7
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    d = cf.desc(T, C, 0, r, 2)
    wsb = cf.cf_lowrank_workspace_bytes(d)
    xs = [W.trajectory(wl, b, steps=2, device="cuda") for b in range(n)]
    oms = [W.omega(wl, b, 1, device="cuda") for b in range(n)]
    outs = []
    try:
        for g in (0, group):
            cf.cf_set_lowrank_group(g)
            gs = [GpuLowrank(T, C, r, 2) for _ in range(n)]
            for b in range(n):
                gs[b].init(xs[b][0].clone())
            ws = torch.empty(n * wsb, dtype=torch.uint8, device="cuda")
            enc = cf.lowrank_buffer_array([(xs[b][1].view(torch.int16), gs[b].recon_s, gs[b].err, oms[b],
                                            gs[b].pc, gs[b].ps, gs[b].qc, gs[b].qs) for b in range(n)],
                                          "cuda")
            cf.cf_lowrank_encode_batched(d, n, enc, ws)
            torch.cuda.synchronize()
            assert [cf.cf_lowrank_status(ws[b * wsb:]) for b in range(n)] == [0] * n
            outs.append(gs)
    finally:
        cf.cf_set_lowrank_group(0)
    nb = (r + 1) // 2
    for a, b in zip(*outs):
        for k in ("recon_s", "err", "ps", "qs"):
            assert torch.equal(getattr(a, k), getattr(b, k)), k
        assert torch.equal(a.pc[:T * nb], b.pc[:T * nb]) and torch.equal(a.qc[:C * nb], b.qc[:C * nb])
