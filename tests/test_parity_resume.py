"""Checkpoint / resume: the codec's whole state is the sender's {recon_s,
err} (or {err} plus the caller's previous activation for the delta-state
sender) and the receiver's recon_r.  Copying it to the host mid-trajectory
and restoring it into fresh device buffers continues the trajectory bit for
bit, for the quantize and the low-rank (cold start) modes."""
import numpy as np
import pytest
import torch

from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _quant(T, C, bits, xs, split):
    d = cf.desc(T, C, bits)
    Wd = cf.cf_codes_words_per_row(d)
    f32 = dict(dtype=torch.float32, device="cuda")

    def fresh():
        return dict(rs=torch.empty(T, C, **f32), er=torch.empty(T, C, **f32),
                    rr=torch.empty(T, C, **f32))

    st = fresh()
    codes = torch.empty(T, Wd, dtype=torch.int32, device="cuda")
    sc = torch.empty(T, **f32)
    cf.cf_state_init(d, xs[0].view(torch.int16), st["rs"], st["er"])
    cf.cf_state_init(d, xs[0].view(torch.int16), st["rr"], None)
    for t in range(1, len(xs)):
        if t == split:
            saved = {k: v.cpu().numpy().copy() for k, v in st.items()}
            del st
            torch.cuda.empty_cache()
            st = fresh()
            for k in st:
                st[k].copy_(torch.from_numpy(saved[k]))
        cf.cf_encode(d, xs[t].view(torch.int16), st["rs"], st["er"], codes, sc)
        cf.cf_decode(d, codes, sc, st["rr"])
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in st.items()}


@pytest.mark.parametrize("bits", [1, 2])
def test_quantize_resume_is_bit_exact(bits):
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=128, bits=bits)
    xs = [x.clone() for x in W.trajectory(wl, 0, steps=7, device="cuda")]
    a = _quant(wl.tokens, wl.channels, bits, xs, split=None)
    b = _quant(wl.tokens, wl.channels, bits, xs, split=4)
    for k in a:
        assert np.array_equal(a[k].view(np.uint32), b[k].view(np.uint32)), k


def _lowrank(T, C, r, xs, oms, split):
    d = cf.desc(T, C, 0, r, 2)
    nb = (r + 1) // 2
    f32 = dict(dtype=torch.float32, device="cuda")

    def fresh():
        return dict(rs=torch.empty(T, C, **f32), er=torch.empty(T, C, **f32),
                    rr=torch.empty(T, C, **f32))

    st = fresh()
    pc = torch.empty(T * nb, dtype=torch.uint8, device="cuda")
    qc = torch.empty(C * nb, dtype=torch.uint8, device="cuda")
    ps, qs = torch.empty(r, **f32), torch.empty(r, **f32)
    ws = torch.empty(cf.cf_lowrank_workspace_bytes(d), dtype=torch.uint8, device="cuda")
    cf.cf_state_init(d, xs[0].view(torch.int16), st["rs"], st["er"])
    cf.cf_state_init(d, xs[0].view(torch.int16), st["rr"], None)
    for t in range(1, len(xs)):
        if t == split:
            saved = {k: v.cpu().numpy().copy() for k, v in st.items()}
            del st
            st = fresh()
            for k in st:
                st[k].copy_(torch.from_numpy(saved[k]))
            ws = torch.empty_like(ws)      # scratch: nothing in it carries over
        cf.cf_lowrank_encode(d, xs[t].view(torch.int16), st["rs"], st["er"], oms[t], pc, ps, qc,
                             qs, ws)
        cf.cf_lowrank_decode(d, pc, ps, qc, qs, st["rr"])
        assert cf.cf_lowrank_status(ws) == 0
    return {k: v.cpu().numpy() for k, v in st.items()}


def test_lowrank_resume_is_bit_exact():
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=384, channels=256, rank=16)
    xs = [x.clone() for x in W.trajectory(wl, 0, steps=5, device="cuda")]
    oms = [W.omega(wl, 0, s, device="cuda") for s in range(5)]
    a = _lowrank(wl.tokens, wl.channels, wl.rank, xs, oms, split=None)
    b = _lowrank(wl.tokens, wl.channels, wl.rank, xs, oms, split=3)
    for k in a:
        assert np.array_equal(a[k].view(np.uint32), b[k].view(np.uint32)), k
