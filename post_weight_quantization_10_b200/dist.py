"""Multi-process plumbing for running independent layer solves on several GPUs.

Layers (and output-column blocks of a layer) are independent problems: every
rank solves its own units and nothing crosses ranks in the data path.  The
only collectives are the barrier around the timed region and the max over
ranks of the measured time.  Works with the nccl backend (one process per
GPU) and with gloo (CPU tests).
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def world() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def barrier(world_size: int) -> None:
    if world_size > 1:
        dist.barrier()


def max_over_ranks(value: float, world_size: int, device=None) -> float:
    """The largest `value` over all ranks (e.g. elapsed time)."""
    if world_size == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world_size: int, device=None) -> float:
    if world_size == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def my_units(n_units: int, rank: int, world_size: int) -> list[int]:
    """Round-robin share of `n_units` independent problems for this rank."""
    return list(range(rank, n_units, world_size))
