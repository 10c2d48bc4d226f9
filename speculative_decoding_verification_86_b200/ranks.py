"""Sharding verification across ranks (one process per GPU).

Requests are independent, so ranks split a batch with no collective on the data
path.  A request keeps its global index through `request_offset` (the Philox
counter's request word), so the draws -- and therefore the outputs -- of a
sharded batch are those of the same batch verified in one call.  The only
collective is the timing reduction: a step takes as long as its slowest rank.
"""
import torch
import torch.distributed as dist


def shard_bounds(total: int, world: int, rank: int):
    """Contiguous near-equal split of `total` requests: rank's [lo, hi)."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError("bad shard request: total=%d world=%d rank=%d" % (total, world, rank))
    return total * rank // world, total * (rank + 1) // world


def weak_offset(per_rank: int, rank: int) -> int:
    """request_offset of rank's batch when every rank verifies `per_rank`
    requests of one global batch (weak scaling)."""
    return per_rank * rank


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (a step time) over the process group; the value
    itself when no group is initialised or it has one rank."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
