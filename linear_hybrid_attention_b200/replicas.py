"""Host-side logic for running the layer as independent replicas on several GPUs.

The hybrid layer has no exchange step on one sample: every head and every
query tile is independent.  Data parallelism therefore gives each rank its own
problem (its own synthetic batch element, seeded per rank) with no collective
on the data path; the only collectives are the timing barrier and the
max-over-ranks of the measured time.
"""
from __future__ import annotations

import os
from typing import Optional, Tuple

import torch
import torch.distributed as dist


def env_rank() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank r's batch element: distinct per rank, rank 0 keeps the base seed."""
    return base_seed + 7919 * rank


def max_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device: Optional[torch.device] = None) -> None:
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def job_throughput(tokens_per_rank_step: float, steps: int, seconds_per_rank: float,
                   device: Optional[torch.device] = None) -> Tuple[float, float]:
    """Whole-job tokens/s: tokens of all ranks / max-over-ranks time.  Returns (tokens/s, max s)."""
    t_max = max_over_ranks(seconds_per_rank, device)
    total = sum_over_ranks(tokens_per_rank_step * steps, device)
    return total / t_max, t_max
