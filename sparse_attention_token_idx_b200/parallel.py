"""Multi-GPU plumbing for the indexer.

* Batch sharding: sequences are independent, so a batch is split into
  contiguous per-rank shards with no data-path collective (only a barrier and
  the max-over-ranks reduction of timings).
* Split-T: one sequence's keys spread over the ranks; each rank selects its
  slice's top-k, one all-gather exchanges the (score, position) candidates and
  every rank merges them into the sequence's top-k.

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


# ----------------------------------------------------------------------------
# Split-T: one sequence's keys spread over the ranks.  Each rank holds the
# cache positions [lo, hi) of every sequence, scores the (replicated) queries
# against them, selects its slice's k best, and the ranks exchange those as
# (score, global position) pairs; the merge keeps the row's k best.  The result
# equals the top-k over the whole sequence (a key of the row's k best is among
# its own slice's k best), which the broadcast-and-compare of the reference
# forward only asserts across ranks.

_NEG_INF_BITS = -8388608   # 0xFF800000, the float32 bits of −inf, as int32


def key_slice(T_cap: int, rank: int, world: int, align: int = 128) -> tuple[int, int]:
    """Cache positions [lo, hi) that `rank` holds: contiguous slices of a
    multiple of `align` positions (the last may be shorter or empty)."""
    if world <= 0 or not 0 <= rank < world or T_cap < 0 or align <= 0:
        raise ValueError("bad slice request")
    per = -(-T_cap // world)
    per = -(-per // align) * align
    lo = min(rank * per, T_cap)
    return lo, min(lo + per, T_cap)


def slice_counts(lengths, lo: int, hi: int):
    """Keys of each sequence inside [lo, hi): clamp(length − lo, 0, hi − lo)
    (torch tensor or numpy array in, same kind out)."""
    if isinstance(lengths, torch.Tensor):
        return (lengths - lo).clamp(0, hi - lo).to(lengths.dtype)
    import numpy as np
    return np.clip(np.asarray(lengths) - lo, 0, hi - lo).astype(np.asarray(lengths).dtype)


def exchange_candidates(cand: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's candidate pairs [rows, kin, 2] → [world, rows, kin, 2] in
    rank order: one all-gather (k·8 bytes per row from each rank)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return cand.unsqueeze(0)
    world = dist.get_world_size(group)
    rows = cand.shape[0]
    out = torch.empty((world * rows,) + tuple(cand.shape[1:]), dtype=cand.dtype, device=cand.device)
    dist.all_gather_into_tensor(out, cand.contiguous(), group=group)   # rank g's rows at [g·rows, (g+1)·rows)
    return out.view((world,) + tuple(cand.shape))


def slice_candidates(q_fp8, w, k_cache, k_scale_cache, lengths, lo: int, hi: int, k: int, stream=None):
    """This rank's half of a split-T decode call: score the queries q_fp8
    [B, 1, 64, 128] / w [B, 1, 64] against the slice's cache (k_cache
    [B, hi − lo, 128], k_scale_cache [B, hi − lo] fp32 holding positions
    [lo, hi)), select the slice's k best and return them as candidate pairs
    int32 [B, k, 2] (score bits, global position; −1 empty).  lengths [B] int32
    are the whole sequences' lengths."""
    from . import binding as X
    B = q_fp8.shape[0]
    span = hi - lo
    if span <= 0:                        # this rank holds no positions: only empty candidates (−inf, −1)
        cand = torch.full((B, k, 2), -1, dtype=torch.int32, device=q_fp8.device)
        cand[..., 0] = _NEG_INF_BITS
        return cand
    counts = slice_counts(lengths, lo, hi)
    eff = counts.clamp(min=1)            # an empty slice is scored as one key and dropped by the gather
    scores = X.score_visible(q_fp8, w, k_cache, k_scale_cache, eff, False, span, stream=stream)
    idx_local = X.topk(scores, eff, False, k, span, stream=stream)
    return X.gather_scores(scores.reshape(B, span), idx_local.reshape(B, k), lo, counts=counts, stream=stream)


def split_t_decode(q_fp8, w, k_cache, k_scale_cache, lengths, lo: int, hi: int, k: int, group=None, stream=None):
    """One decode call with the keys split over the ranks (arguments as in
    slice_candidates).  Returns [B, k] int32 global positions, the same on every
    rank: slice candidates, one all-gather, the merge."""
    from . import binding as X
    cand = slice_candidates(q_fp8, w, k_cache, k_scale_cache, lengths, lo, hi, k, stream=stream)
    return X.merge_topk(exchange_candidates(cand, group), k, stream=stream)
