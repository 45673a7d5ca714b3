"""Process-group plumbing for running the kernels data-parallel over GPUs.

One process per GPU (torchrun).  Every (batch, head) slice of the attention is
independent in both passes, so the work splits over ranks in two ways:

  * batch: every rank runs its own batch entries; the relative tables are shared by
    the batch, so their gradients are summed across ranks with one all-reduce per
    table (NCCL on GPUs, gloo on CPU in tests) -- data-parallel training;
  * heads: every rank runs a contiguous block of heads of the same batch with the
    matching rows of the (per-head) tables; nothing is exchanged -- the split for
    one long sequence (B = 1).

Timing is reduced with MAX.
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


def shard_range(n: int, rank: int, world: int):
    """Contiguous block [lo, hi) of n items for `rank` (sizes differ by at most one)."""
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def shard_inputs(inp: dict, mode: str, rank: int, world: int) -> dict:
    """This rank's part of a workload's inputs (dict q, k, v, do [B,H,L,d] and rel, the
    per-head tables [H,...]): batch entries (tables whole) or heads (tables' rows of
    those heads)."""
    if mode not in ("batch", "heads"):
        raise ValueError(mode)
    dim = 0 if mode == "batch" else 1
    lo, hi = shard_range(inp["q"].shape[dim], rank, world)
    out = {n: inp[n].narrow(dim, lo, hi - lo) for n in ("q", "k", "v", "do")}
    out["rel"] = list(inp["rel"]) if mode == "batch" else [r.narrow(0, lo, hi - lo) for r in inp["rel"]]
    return out


def gather_shards(t: torch.Tensor, dim: int) -> torch.Tensor:
    """Concatenate every rank's equally sized block of a tensor along `dim`, in rank
    order (all-gather)."""
    if not active():
        return t
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size())]
    dist.all_gather(parts, t.contiguous())
    return torch.cat(parts, dim=dim)


def shutdown():
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
