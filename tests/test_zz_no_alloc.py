"""cf_lowrank_encode_noalloc: the low-rank sender for callers that cannot
allocate device memory (a plug-in inside a framework that owns all device
memory, or a serving loop that must not call cudaMalloc mid-step).  It uses
the library's fixed device scratch array instead of a caller workspace.

Checked through the C ABI against cf_lowrank_encode (caller workspace) on
the same inputs, on two calls in a row, within the low-rank parity
tolerances of the other tests.  This file is named to be collected last.
"""
import numpy as np
import pytest
import torch

from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W
from oracle import lowrank as L

pytestmark = pytest.mark.gpu

STATE_RTOL = 1e-5        # reconstructions / error buffers, per token row
REL_FROB_TOL = 0.01      # low-rank relative Frobenius error


def _state(T, C, r):
    nb = (r + 1) // 2
    f32 = dict(dtype=torch.float32, device="cuda")
    return dict(recon=torch.empty(T, C, **f32), err=torch.empty(T, C, **f32),
                pc=torch.empty(T * nb + 16, dtype=torch.uint8, device="cuda"),
                qc=torch.empty(C * nb + 16, dtype=torch.uint8, device="cuda"),
                ps=torch.empty(r, **f32), qs=torch.empty(r, **f32))


def _rows_close(a, b):
    rowmax = np.max(np.abs(b.astype(np.float64)), axis=1, keepdims=True)
    return np.all(np.abs(a.astype(np.float64) - b) <= STATE_RTOL * rowmax + 1e-37)


def test_noalloc_matches_workspace_entry_point_two_calls():
    wl = W.WORKLOADS["lowrank"]                 # 4096 x 3072, rank 32, 2 iterations
    T, C, r, it = wl.tokens, wl.channels, wl.rank, wl.iters
    d = cf.desc(T, C, 0, r, it)
    assert 0 < cf.cf_lowrank_workspace_bytes(d) <= (40 << 20)
    xs = W.trajectory(wl, 5, steps=3, device="cuda")
    a, b = _state(T, C, r), _state(T, C, r)
    ws = torch.empty(cf.cf_lowrank_workspace_bytes(d), dtype=torch.uint8, device="cuda")
    x0 = xs[0].clone().view(torch.int16)
    for s in (a, b):
        cf.cf_state_init(d, x0, s["recon"], s["err"])
    nb = (r + 1) // 2
    for step in (1, 2):
        x = xs[step].clone().view(torch.int16)
        om = W.omega(wl, 5, step, device="cuda")
        recon_before = a["recon"].cpu().numpy()
        cf.cf_lowrank_encode(d, x, a["recon"], a["err"], om, a["pc"], a["ps"], a["qc"], a["qs"], ws)
        cf.cf_lowrank_encode_noalloc(d, x, b["recon"], b["err"], om, b["pc"], b["ps"], b["qc"],
                                     b["qs"])
        torch.cuda.synchronize()
        ha = {k: v.cpu().numpy() for k, v in a.items()}
        hb = {k: v.cpu().numpy() for k, v in b.items()}
        assert _rows_close(hb["recon"], ha["recon"]) and _rows_close(hb["err"], ha["err"])
        da = L.reconstruct(ha["pc"][:T * nb].reshape(T, nb), ha["ps"],
                           ha["qc"][:C * nb].reshape(C, nb), ha["qs"], r)
        db = L.reconstruct(hb["pc"][:T * nb].reshape(T, nb), hb["ps"],
                           hb["qc"][:C * nb].reshape(C, nb), hb["qs"], r)
        v = (L.bf16_bits_to_f32(W.bf16_bits(xs[step])) - recon_before).astype(np.float64)
        ea = np.linalg.norm(v - da) / np.linalg.norm(v)
        eb = np.linalg.norm(v - db) / np.linalg.norm(v)
        assert abs(ea - eb) <= REL_FROB_TOL * ea, (step, ea, eb)


def test_noalloc_rejects_problems_beyond_the_scratch_array():
    d = cf.desc(8192, 4096, 0, 32, 2)           # needs ~85 MB of scratch
    assert cf.cf_lowrank_workspace_bytes(d) > (40 << 20)
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(cf.CFError) as ei:
        cf.cf_lowrank_encode_noalloc(d, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy)
    assert ei.value.status == 4                 # CF_ERR_WORKSPACE, nothing launched
