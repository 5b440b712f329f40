"""Multi-GPU plumbing for the indexer: sequences are independent, so a batch
is split into contiguous per-rank shards with no data-path collective; the
only collectives are a barrier and the max-over-ranks reduction of timings.
Works with any torch.distributed backend (NCCL on GPUs, gloo on CPU)."""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(n_items: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous share [lo, hi) of n_items for `rank`; sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world or n_items < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n_items, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(values, device=None) -> list[float]:
    """Element-wise maximum of a list of floats over all ranks (identity when
    torch.distributed is not initialised)."""
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_total(per_rank_units: float) -> float:
    """Units processed by the whole job when every rank processes the same amount."""
    world = dist.get_world_size() if (dist.is_available() and dist.is_initialized()) else 1
    return per_rank_units * world
