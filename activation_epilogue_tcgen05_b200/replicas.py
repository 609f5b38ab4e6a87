"""One process per GPU, independent replicas: host-side plumbing for N > 1.

The fused GEMM + epilogue has no exchange step: output tiles are independent,
so N GPUs run N independent problems (weak scaling) and no collective touches
the data path.  torch.distributed is used only for a barrier around the timed
region and for taking the slowest rank's time (max over ranks), as the
benchmark contract requires.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank():
    """(rank, world_size, local_rank) from the torchrun environment (defaults: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device_id=None) -> bool:
    """Join the process group when WORLD_SIZE > 1; returns whether one exists."""
    _, world, _ = env_rank()
    if world <= 1:
        return False
    if not dist.is_initialized():
        kw = {}
        if device_id is not None:
            kw["device_id"] = device_id
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return True


def barrier() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device="cpu") -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device="cpu") -> float:
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard(units: int, world: int, rank: int) -> range:
    """Contiguous near-equal share of `units` independent problems for `rank`."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(units, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def finalize() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
