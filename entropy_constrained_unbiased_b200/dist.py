"""Multi-GPU plumbing for the benchmark: one process per GPU, no data-path
collective.

Every vector is an independent ECASQ problem (summary §1: one input vector X
per problem), so ranks never exchange solver data. The only collectives are on
the host path of the benchmark: a barrier around the timed region and one
all-reduce MAX of the measured device time (the job takes as long as its
slowest rank). Each rank draws its own vectors (weak scaling).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def world() -> tuple[int, int]:
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def setup(backend: str | None = None, timeout_s: float = 120.0) -> tuple[int, int]:
    """Join the process group when WORLD_SIZE > 1 (env:// rendezvous)."""
    rank, size = world()
    if size > 1 and not dist.is_initialized():
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, size


def _device():
    if dist.is_initialized() and dist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def barrier() -> None:
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float) -> float:
    """The largest value across ranks (the job's time is its slowest rank's)."""
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float) -> float:
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def teardown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
