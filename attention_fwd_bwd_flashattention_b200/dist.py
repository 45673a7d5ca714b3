"""Process-group plumbing for running the kernels data-parallel over GPUs.

One process per GPU (torchrun).  Every rank runs its own batch; the relative
tables are shared, so their gradients are summed across ranks with one
all-reduce (NCCL on GPUs, gloo on CPU in tests).  Timing is reduced with MAX.
"""
from __future__ import annotations

import datetime
import os
from typing import List

import torch
import torch.distributed as dist


def init_from_env(backend: str = "nccl", timeout_s: int = 120):
    """Initialise from RANK/WORLD_SIZE/LOCAL_RANK when WORLD_SIZE > 1.
    Returns (rank, world, local_rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return rank, world, local


def active() -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1


def barrier():
    if active():
        dist.barrier()


def max_over_ranks(x: float) -> float:
    if not active():
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_table_grads(drel: List[torch.Tensor]) -> None:
    """Sum the relative-table gradients over ranks (in place), one call per tensor
    in a fixed order so every rank issues the same collectives."""
    if not active():
        return
    for g in drel:
        dist.all_reduce(g, op=dist.ReduceOp.SUM)


def shutdown():
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
