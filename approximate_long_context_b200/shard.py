"""Data-parallel layout of the forward pass over ranks: host logic only, no device arithmetic.

The (batch, head) problems of the method ("HyperAttention: Long-context Attention in Near-Linear Time",
research-map summary, "Approach": every head is hashed, sorted and attended on its own) are independent,
so a job over G problems splits into contiguous ranges, one per rank, with no exchange of data. Each rank
passes its range's first global index as the `bh_offset` option. The sample draws of every problem are
then keyed by the global index, and the concatenation of the ranks' outputs equals one call over all G
problems. Timing is the only collective: the slowest rank's time is the job's time.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Shard:
    rank: int
    world: int
    offset: int   # global index of this rank's first problem
    count: int    # problems on this rank (>= 0)


def shard_problems(total: int, world: int, rank: int) -> Shard:
    """Contiguous split of `total` problems over `world` ranks. The first total % world ranks take one
    more problem. The ranges cover 0..total-1 once, in rank order."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError(f"bad shard request total={total} world={world} rank={rank}")
    base, extra = divmod(total, world)
    count = base + (1 if rank < extra else 0)
    offset = rank * base + min(rank, extra)
    return Shard(rank, world, offset, count)


def weak_shard(per_rank: int, world: int, rank: int) -> Shard:
    """Weak scaling: every rank takes `per_rank` problems of a job of world * per_rank problems."""
    return shard_problems(per_rank * world, world, rank)


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks of the default process group (the value itself without one).
    `device` is where the reduction tensor lives (a CUDA device for NCCL, None for CPU / gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
