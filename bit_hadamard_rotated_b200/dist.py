"""Multi-rank helpers for the benchmark: one process per GPU, torch.distributed
for the plumbing only.

The rotated linear shards without any exchange: every rank streams its own
weights (weak scaling: independent layers per rank), so the data path has no
collective.  The only cross-rank operations are the barrier around the timed
region and the max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_world() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (1 rank if absent)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0) -> bool:
    """Initialise the default process group when launched with more than one rank."""
    rank, _, world = env_world()
    if world <= 1 or dist.is_initialized():
        return dist.is_initialized()
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    kw = dict(backend=backend, rank=rank, world_size=world,
              timeout=datetime.timedelta(seconds=timeout_s))
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    dist.init_process_group(**kw)
    return True


def barrier(device=None) -> None:
    if dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Largest value across ranks (the job's time is its slowest rank's)."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard(n_units: int, rank: int, world: int) -> range:
    """Contiguous share of n_units for this rank (sizes differ by at most one)."""
    lo = (n_units * rank) // world
    hi = (n_units * (rank + 1)) // world
    return range(lo, hi)


def finish() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
