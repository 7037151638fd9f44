"""Data parallelism for the layer across the GPUs of one node.

Tokens are independent, so each rank holds the same weights and runs the
layer on its own batch: there is no collective on the data path. The only
cross-rank steps are the barriers around a timed region and the reduction of
its time to the maximum over ranks (the job's time is the slowest rank's).
"""
from __future__ import annotations

import os
from datetime import timedelta

import torch
import torch.distributed as dist


def env_ranks():
    """(world_size, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device=None) -> None:
    """Join the process group (rendezvous from MASTER_ADDR/MASTER_PORT)."""
    kw = {"timeout": timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def batch_seed(rank: int) -> int:
    """Seed of rank `rank`'s token batch (each rank draws a different batch)."""
    return 1000 + rank


def barrier() -> None:
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (the value itself on one rank)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens(tokens_per_rank: int, world: int, steps: int) -> int:
    """Tokens the whole job processes in `steps` steps (weak scaling)."""
    return tokens_per_rank * world * steps
