"""Rank logic of multi-GPU runs: one process per GPU, each running an independent replica of
the workload (documents and heads are independent units, so ranks share nothing on the data
path).  The only collectives are a barrier and the max of the per-rank device times."""
from __future__ import annotations

import os
from datetime import timedelta

import torch
import torch.distributed as dist


def env_rank():
    """(rank, world_size, local_rank) from the torchrun environment (defaults: single process)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init(world: int, backend: str = "nccl", device=None, timeout_s: float = 300.0):
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": timedelta(seconds=timeout_s)}
        if backend == "nccl" and device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)


def barrier(world: int):
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (every rank gets the result)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch of the same workload."""
    return base + rank


def throughput(units_per_rank: int, world: int, steps: int, max_elapsed_ms: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return units_per_rank * world * steps / (max_elapsed_ms / 1e3)


def shutdown(world: int):
    if world > 1 and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
