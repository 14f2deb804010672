"""Replica plumbing for multi-GPU runs of the codec (one process per GPU).

In the default multi-GPU run each rank compresses and decompresses its own
buffers, so N ranks are N independent replicas.  The only cross-rank
operations are host-side plumbing: a barrier around a timed region and a
max or sum of per-rank numbers.  torch.distributed provides them (NCCL on
GPUs, gloo on CPU).  The exchange of payloads between ranks is in
exchange.py.
"""
from __future__ import annotations

import contextlib
import dataclasses
import datetime
import os

import torch
import torch.distributed as dist


@dataclasses.dataclass(frozen=True)
class RankInfo:
    world: int
    rank: int
    local: int

    @property
    def distributed(self) -> bool:
        return self.world > 1


def rank_info_from_env() -> RankInfo:
    return RankInfo(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(info: RankInfo, backend: str | None = None, timeout_s: float = 120.0) -> None:
    """Join the process group (MASTER_ADDR/MASTER_PORT from the environment)
    with a short timeout, so a rank that never arrives ends the others'
    next collective with an error instead of a hang."""
    if not info.distributed or dist.is_initialized():
        return
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    dist.init_process_group(backend, rank=info.rank, world_size=info.world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _device():
    if dist.is_initialized() and dist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def reduce_scalar(x: float, op: str) -> float:
    """max or sum of a per-rank number over all ranks (identity when alone)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op={"max": dist.ReduceOp.MAX, "sum": dist.ReduceOp.SUM}[op])
    return float(t.item())


@contextlib.contextmanager
def bracket():
    """Barrier + device synchronisation on both sides of a timed region."""
    sync = torch.cuda.synchronize if torch.cuda.is_available() else (lambda: None)
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
    sync()
    yield
    sync()
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def whole_job_rate(units_per_rank: float, per_rank_seconds: float) -> float:
    """Aggregate throughput: every rank's units over the slowest rank's time."""
    total = reduce_scalar(units_per_rank, "sum")
    slowest = reduce_scalar(per_rank_seconds, "max")
    return total / slowest


def finish() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
