"""The batched calls are capturable: no allocation, no synchronisation, no
host read of device state.  A CUDA graph of one whole step (encode then
decode of every buffer), replayed, gives exactly what the same calls made
eagerly give, for the quantize and the low-rank modes."""
import pytest
import torch

from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _quant_state(n, T, C, bits, xs):
    d = cf.desc(T, C, bits)
    Wd = cf.cf_codes_words_per_row(d)
    f32 = dict(dtype=torch.float32, device="cuda")
    st = dict(rs=torch.empty(n, T, C, **f32), rr=torch.empty(n, T, C, **f32),
              er=torch.empty(n, T, C, **f32),
              codes=torch.empty(n, T, Wd, dtype=torch.int32, device="cuda"),
              sc=torch.empty(n, T, **f32), x=torch.empty(n, T, C, dtype=torch.bfloat16, device="cuda"))
    for b in range(n):
        cf.cf_state_init(d, xs[b][0].view(torch.int16), st["rs"][b], st["er"][b])
        cf.cf_state_init(d, xs[b][0].view(torch.int16), st["rr"][b], None)
    x16 = st["x"].view(torch.int16)
    st["enc"] = cf.enc_buffer_array([(x16[b], st["rs"][b], st["er"][b], st["codes"][b], st["sc"][b])
                                     for b in range(n)], "cuda")
    st["dec"] = cf.dec_buffer_array([(st["codes"][b], st["sc"][b], st["rr"][b]) for b in range(n)],
                                    "cuda")
    return d, st


@pytest.mark.parametrize("pipe", [0, 1])
def test_quantize_step_graph_replay_equals_eager(pipe):
    n, T, C, bits, steps = 6, 256, 3072, 2, 4
    wl = W.replace(W.WORKLOADS["flux_sp"], tokens=T, buffers=n)
    xs = [W.trajectory(wl, b, steps=steps, device="cuda") for b in range(n)]
    cf.cf_set_quant_pipeline(0, pipe, 0)
    cf.cf_set_quant_pipeline(1, pipe, 0)
    try:
        d, eager = _quant_state(n, T, C, bits, xs)
        _, graph = _quant_state(n, T, C, bits, xs)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            # warm-up outside the capture (first-call set-up of the library)
            cf.cf_encode_batched(d, n, graph["enc"], status, s)
            s.synchronize()
        d, graph = _quant_state(n, T, C, bits, xs)
        with torch.cuda.graph(g, stream=s):
            cf.cf_encode_batched(d, n, graph["enc"], status, s)
            cf.cf_decode_batched(d, n, graph["dec"], status, s)
        for t in range(1, steps):
            for b in range(n):
                eager["x"][b].copy_(xs[b][t])
                graph["x"][b].copy_(xs[b][t])
            cf.cf_encode_batched(d, n, eager["enc"], status)
            cf.cf_decode_batched(d, n, eager["dec"], status)
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            for k in ("rs", "rr", "er", "codes", "sc"):
                assert torch.equal(eager[k], graph[k]), (t, k)
        assert int(status.item()) == 0
        del g
    finally:
        cf.cf_set_quant_pipeline(0, 1, 0)
        cf.cf_set_quant_pipeline(1, 1, 0)


def test_lowrank_step_graph_replay_equals_eager():
    n, T, C, r, steps = 3, 512, 768, 16, 3
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r, buffers=n)
    d = cf.desc(T, C, 0, r, 2)
    wsb = cf.cf_lowrank_workspace_bytes(d)
    xs = [W.trajectory(wl, b, steps=steps, device="cuda") for b in range(n)]
    oms = [W.omega(wl, b, 1, device="cuda") for b in range(n)]
    nb = (r + 1) // 2

    def state():
        f32 = dict(dtype=torch.float32, device="cuda")
        st = dict(rs=torch.empty(n, T, C, **f32), rr=torch.empty(n, T, C, **f32),
                  er=torch.empty(n, T, C, **f32),
                  pc=torch.empty(n, T * nb + 16, dtype=torch.uint8, device="cuda"),
                  qc=torch.empty(n, C * nb + 16, dtype=torch.uint8, device="cuda"),
                  ps=torch.empty(n, r, **f32), qs=torch.empty(n, r, **f32),
                  x=torch.empty(n, T, C, dtype=torch.bfloat16, device="cuda"),
                  ws=torch.empty(n * wsb, dtype=torch.uint8, device="cuda"))
        for b in range(n):
            cf.cf_state_init(d, xs[b][0].view(torch.int16), st["rs"][b], st["er"][b])
            cf.cf_state_init(d, xs[b][0].view(torch.int16), st["rr"][b], None)
        x16 = st["x"].view(torch.int16)
        st["enc"] = cf.lowrank_buffer_array([(x16[b], st["rs"][b], st["er"][b], oms[b], st["pc"][b],
                                              st["ps"][b], st["qc"][b], st["qs"][b])
                                             for b in range(n)], "cuda")
        st["dec"] = cf.lowrank_dec_buffer_array([(st["pc"][b], st["ps"][b], st["qc"][b], st["qs"][b],
                                                  st["rr"][b]) for b in range(n)], "cuda")
        return st

    eager, graph = state(), state()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        cf.cf_lowrank_decode_batched(d, n, graph["dec"], stream=s)   # first-call set-up
        s.synchronize()
    graph = state()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cf.cf_lowrank_encode_batched(d, n, graph["enc"], graph["ws"], stream=s)
        cf.cf_lowrank_decode_batched(d, n, graph["dec"], stream=s)
    for t in range(1, steps):
        for b in range(n):
            eager["x"][b].copy_(xs[b][t])
            graph["x"][b].copy_(xs[b][t])
        cf.cf_lowrank_encode_batched(d, n, eager["enc"], eager["ws"])
        cf.cf_lowrank_decode_batched(d, n, eager["dec"])
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        for k in ("rs", "rr", "er", "ps", "qs"):
            assert torch.equal(eager[k], graph[k]), (t, k)
        assert torch.equal(eager["pc"][:, :T * nb], graph["pc"][:, :T * nb])
        for b in range(n):
            assert cf.cf_lowrank_status(graph["ws"][b * wsb:]) == 0
    del g


def test_async_status_read_inside_a_captured_step():
    """cf_lowrank_status_async enqueues one strided device-to-host copy, so
    it captures with the batched encode: after each replay the pinned host
    words hold what the blocking per-slice read returns."""
    T, C, r, n = 256, 192, 8, 3
    wl = W.replace(W.WORKLOADS["lowrank"], tokens=T, channels=C, rank=r)
    d = cf.desc(T, C, 0, r, 2)
    wsb = cf.cf_lowrank_workspace_bytes(d)
    nb = (r + 1) // 2
    f32 = dict(dtype=torch.float32, device="cuda")
    xs = [W.trajectory(wl, b, steps=3, device="cuda") for b in range(n)]
    rs = torch.empty(n, T, C, **f32)
    er = torch.empty(n, T, C, **f32)
    x = torch.empty(n, T, C, dtype=torch.bfloat16, device="cuda")
    pc = torch.empty(n, T * nb + 16, dtype=torch.uint8, device="cuda")
    qc = torch.empty(n, C * nb + 16, dtype=torch.uint8, device="cuda")
    ps, qs = torch.empty(n, r, **f32), torch.empty(n, r, **f32)
    om = torch.stack([W.omega(wl, b, 1, device="cuda") for b in range(n)])
    for b in range(n):
        cf.cf_state_init(d, xs[b][0].view(torch.int16), rs[b], er[b])
    x16 = x.view(torch.int16)
    # buffer 1 gets a zero residual (CF_ERR_NUMERIC), the others real steps;
    # the capture warm-up below is step 1 of every buffer
    enc = cf.lowrank_buffer_array([(x16[b], rs[b], er[b], om[b], pc[b], ps[b], qc[b], qs[b])
                                   for b in range(n)], "cuda")
    ws = torch.empty(n * wsb, dtype=torch.uint8, device="cuda")
    host = torch.full((n,), -1, dtype=torch.int32).pin_memory()
    for b in range(n):
        x[b].copy_(xs[1][0] if b == 1 else xs[b][1])
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        cf.cf_lowrank_encode_batched(d, n, enc, ws, stream=s)    # first-call set-up outside capture
        s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cf.cf_lowrank_encode_batched(d, n, enc, ws, stream=s)
        cf.cf_lowrank_status_async(ws, wsb, n, host, stream=s)
    for t in (1, 2):
        # buffer 1 stays at its warmup activation: its state equals it
        # exactly, so its residual is zero at every step
        for b in range(n):
            x[b].copy_(xs[1][0] if b == 1 else xs[b][t])
        host.fill_(-1)
        g.replay()
        torch.cuda.synchronize()
        got = host.tolist()
        want = [cf.cf_lowrank_status(ws[b * wsb:]) for b in range(n)]
        assert got == want, (t, got, want)
        assert got[0] == 0 and got[2] == 0 and got[1] == 6, got
