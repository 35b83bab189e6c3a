"""Host-side logic for running the layer on several GPUs, one process per GPU.

The hybrid layer has no exchange step on one sample: every head and every
query tile is independent.  Two ways to use G GPUs follow from that:

  * replicas (what the bench runs under torchrun): each rank processes its own
    problem (its own synthetic batch element, seeded per rank) with no
    collective on the data path; the only collectives are the timing barrier
    and the max-over-ranks of the measured time (weak scaling);
  * a head partition of ONE sample: rank r runs the heads head_range(H, r, G)
    of every call (landmarks, selection, attention, linear state and fit are
    all per head), and the outputs are gathered only if the caller needs them
    in one place (gather_heads: one all-gather of H * N * d values; strong
    scaling of one layer).
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


def head_range(heads: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous, balanced block of heads [h0, h1) owned by `rank` (the first
    heads % world ranks hold one more head)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def gather_heads(local: torch.Tensor, heads: int) -> torch.Tensor:
    """All-gather the per-rank head blocks [h1 - h0, ...] of a head partition into
    the full [heads, ...] tensor on every rank.  Blocks are padded to the largest
    block so that one equal-size all-gather serves uneven partitions."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return local
    world, rank = dist.get_world_size(), dist.get_rank()
    h0, h1 = head_range(heads, rank, world)
    if local.shape[0] != h1 - h0:
        raise ValueError(f"rank {rank} holds {local.shape[0]} heads, its block is {h1 - h0}")
    width = -(-heads // world)
    pad = local.new_zeros((width,) + tuple(local.shape[1:]))
    pad[: h1 - h0] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([parts[r][: head_range(heads, r, world)[1] - head_range(heads, r, world)[0]]
                      for r in range(world)], dim=0)
