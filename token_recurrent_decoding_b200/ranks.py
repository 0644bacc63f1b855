"""One process per GPU: sequence sharding and device-time reduction.

Sequences are independent ("RLT Runs 96 Blocks Per Token With Recurrent State,
No Resets", "Three design principles and their caveats": ready updates from
independent sequences share one batched kernel), so N ranks split the
sequences of a job with no data-path collective. The only collective is the
max over ranks of each rank's device-timed region.
"""
from __future__ import annotations


def shard_range(n_global: int, rank: int, world: int):
    """Contiguous, balanced [start, stop) of the global sequences for `rank`."""
    if world < 1 or not 0 <= rank < world or n_global < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n_global, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """Max of a per-rank scalar over the process group (x itself without one)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, seconds_max: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return float(sum(units_per_rank)) / seconds_max
