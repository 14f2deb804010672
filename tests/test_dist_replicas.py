"""Multi-process (gloo, CPU) tests of the replica plumbing bench.py uses for
N > 1: barrier-bracketed timing, max/sum over ranks, whole-job rate, and a
rank that dies before a collective surfacing as an error on the survivor
(failure detected on the host; no GPU involved)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q, mode):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from activation_residual_compression_cf_b200 import replicas as R
    info = R.rank_info_from_env()
    try:
        R.init(info, backend="gloo", timeout_s=5.0 if mode == "die" else 60.0)
        if mode == "ok":
            with R.bracket():
                pass
            mx = R.reduce_scalar(rank + 1.5, "max")
            sm = R.reduce_scalar(rank + 1.5, "sum")
            rate = R.whole_job_rate(100.0, 1.0 + rank)   # slowest rank takes 1 + (world-1) s
            q.put((rank, mx, sm, rate))
            R.finish()
        else:
            if rank == 1:
                q.put((rank, "left"))
                q.close()
                q.join_thread()                             # flush before leaving
                os._exit(0)                                 # leaves between steps, no collective
            try:
                R.reduce_scalar(1.0, "sum")
                q.put((rank, "no error"))
            except Exception as e:                          # timeout / connection closed
                q.put((rank, "error", type(e).__name__))
    except Exception as e:
        q.put((rank, "fail", repr(e)))


def _run(world, mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q, mode)) for r in range(world)]
    for p in ps:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in ps:
        p.join(timeout=60)
    return sorted(out, key=lambda t: t[0])


def test_max_sum_and_whole_job_rate_world2():
    out = _run(2, "ok")
    for rank, mx, sm, rate in out:
        assert mx == 2.5 and sm == 4.0
        assert rate == pytest.approx(200.0 / 2.0)


def test_rank_that_leaves_is_detected_on_the_host():
    out = _run(2, "die")
    assert out[1][1] == "left"
    assert out[0][1] == "error", out[0]
