"""Data-parallel plumbing around the layer (one process per GPU).

kongchang, section 容量税 (capacity tax): under DDP every rank keeps its model
partition for the whole gradient-accumulation window and gradients are
synchronised once per optimizer step.  For this layer that means: each rank
runs route -> ... -> router grad on its own tokens with replicated expert
weights (no exchange inside a step), and the weight gradients are summed
across ranks once per optimizer step.

These helpers use ``torch.distributed`` only: the NCCL backend on GPUs, gloo
on CPU (tests).
"""

from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["rank_seed", "max_over_ranks", "allreduce_grads"]


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's own token batch (weak scaling: every rank draws its own tokens)."""
    return seed + rank


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (step times are reported as the slowest rank's)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_grads(grads, average: bool = False) -> None:
    """Sum (or average) weight gradients over ranks in place: the one exchange
    of data-parallel training, made once per optimizer step."""
    if not (dist.is_available() and dist.is_initialized()):
        return
    world = dist.get_world_size()
    for g in grads:
        dist.all_reduce(g, op=dist.ReduceOp.SUM)
        if average and world > 1:
            g.div_(world)
