"""cf_lowrank_encode_noalloc: the low-rank sender for callers that cannot
allocate device memory (a plug-in inside a framework that owns all device
memory, or a serving loop that must not call cudaMalloc mid-step).  It uses
the library's fixed device scratch array instead of a caller workspace.

Both entry points run the same kernels, with fixed reduction orders, on the
same inputs, so their results must be identical bit for bit: codes, scales,
the sender's reconstruction and the error buffer.  The checks run two calls
in a row, and once after a larger problem has left its data in the shared
array, so stale contents from an earlier call would show.  This file is
named to be collected last.
"""
import pytest
import torch

from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W

pytestmark = pytest.mark.gpu

SCRATCH = 40 << 20


def _state(T, C, r):
    nb = (r + 1) // 2
    f32 = dict(dtype=torch.float32, device="cuda")
    return dict(recon=torch.empty(T, C, **f32), err=torch.empty(T, C, **f32),
                pc=torch.empty(T * nb + 16, dtype=torch.uint8, device="cuda"),
                qc=torch.empty(C * nb + 16, dtype=torch.uint8, device="cuda"),
                ps=torch.empty(r, **f32), qs=torch.empty(r, **f32))


def _compare_two_calls(wl, buffer, ws_fill):
    """Steps 1 and 2 of one buffer through both entry points; the caller
    workspace starts filled with `ws_fill` bytes."""
    T, C, r, it = wl.tokens, wl.channels, wl.rank, wl.iters
    d = cf.desc(T, C, 0, r, it)
    assert 0 < cf.cf_lowrank_workspace_bytes(d) <= SCRATCH
    xs = W.trajectory(wl, buffer, steps=3, device="cuda")
    a, b = _state(T, C, r), _state(T, C, r)
    # the payload buffers start different; both calls must overwrite them
    for k in ("pc", "qc", "ps", "qs"):
        a[k].zero_()
        b[k].fill_(0x5A if b[k].dtype == torch.uint8 else 3.0)
    ws = torch.full((cf.cf_lowrank_workspace_bytes(d),), ws_fill, dtype=torch.uint8, device="cuda")
    x0 = xs[0].clone().view(torch.int16)
    for s in (a, b):
        cf.cf_state_init(d, x0, s["recon"], s["err"])
    nb = (r + 1) // 2
    for step in (1, 2):
        x = xs[step].clone().view(torch.int16)
        om = W.omega(wl, buffer, step, device="cuda")
        cf.cf_lowrank_encode(d, x, a["recon"], a["err"], om, a["pc"], a["ps"], a["qc"], a["qs"], ws)
        cf.cf_lowrank_encode_noalloc(d, x, b["recon"], b["err"], om, b["pc"], b["ps"], b["qc"],
                                     b["qs"])
        torch.cuda.synchronize()
        assert cf.cf_lowrank_status(ws) == 0
        assert torch.equal(a["pc"][:T * nb], b["pc"][:T * nb]), step
        assert torch.equal(a["qc"][:C * nb], b["qc"][:C * nb]), step
        for k in ("ps", "qs", "recon", "err"):
            assert torch.equal(a[k].view(torch.int32), b[k].view(torch.int32)), (step, k)


def test_noalloc_equals_workspace_entry_point_two_calls():
    # the largest problem the scratch array holds: 4096 x 3072, rank 32, 2 iterations
    _compare_two_calls(W.WORKLOADS["lowrank"], 5, 0)


def test_noalloc_equals_workspace_entry_point_after_a_larger_call():
    big = W.WORKLOADS["lowrank"]
    T, C, r = big.tokens, big.channels, big.rank
    d = cf.desc(T, C, 0, r, big.iters)
    # a full-size call leaves its Gram partials, factors and residual copy in
    # the shared array ...
    xs = W.trajectory(big, 7, steps=2, device="cuda")
    s = _state(T, C, r)
    cf.cf_state_init(d, xs[0].view(torch.int16), s["recon"], s["err"])
    cf.cf_lowrank_encode_noalloc(d, xs[1].view(torch.int16), s["recon"], s["err"],
                                 W.omega(big, 7, 1, device="cuda"), s["pc"], s["ps"], s["qc"],
                                 s["qs"])
    torch.cuda.synchronize()
    del s, xs
    # ... then a smaller problem with another rank and a ragged token count
    # must still equal the workspace call (whose workspace starts as garbage)
    small = W.replace(big, tokens=1000, channels=1920, rank=24)
    _compare_two_calls(small, 3, 0xA7)


def test_noalloc_rejects_problems_beyond_the_scratch_array():
    d = cf.desc(8192, 4096, 0, 32, 2)           # needs ~85 MB of scratch
    assert cf.cf_lowrank_workspace_bytes(d) > SCRATCH
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(cf.CFError) as ei:
        cf.cf_lowrank_encode_noalloc(d, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy)
    assert ei.value.status == 4                 # CF_ERR_WORKSPACE, nothing launched
