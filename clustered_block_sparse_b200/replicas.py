"""Replica sharding for one-process-per-GPU runs.

Every stage of the path is independent per (batch, head) slice, so N ranks
run the whole path on disjoint slices and exchange nothing on the data path;
only the timing is combined (the slowest rank sets the step time)."""
from __future__ import annotations


def rank_heads(rank: int, heads_per_rank: int) -> list:
    """Global head indices owned by `rank` (weak scaling: a fixed count per rank)."""
    if rank < 0 or heads_per_rank < 1:
        raise ValueError("rank >= 0 and heads_per_rank >= 1 required")
    return list(range(rank * heads_per_rank, (rank + 1) * heads_per_rank))


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of `x` over the ranks of the default process group (x itself
    without one).  `device` places the reduction tensor (CUDA for NCCL, CPU
    for gloo)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_layer(ms_per_step_max: float, world: int) -> float:
    """Whole-job ms per layer: each of the `world` ranks runs one layer per
    step, and the step lasts as long as the slowest rank."""
    if world < 1:
        raise ValueError("world >= 1 required")
    return ms_per_step_max / world
