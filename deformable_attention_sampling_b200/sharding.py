"""Batch sharding over GPUs, one process per GPU.

Every output of the operator reads only its own batch item's features and its
own offsets and masks (a DCN output pixel reads x[n]; an MSDA query reads
value[n]), so batch items are independent: a rank computes its contiguous
share of the batch and no data crosses GPUs.  Spatial splits are not offered:
learned offsets are unbounded, so a halo exchange would have no bounded width.

The only collective is host plumbing: the maximum of the ranks' device times.
"""


def shard_range(n_items, rank, world):
    """Contiguous, balanced share [start, start + count) of n_items for `rank`.

    The first n_items % world ranks get one extra item; shares are disjoint
    and cover range(n_items) in rank order.
    """
    if world < 1 or not 0 <= rank < world or n_items < 0:
        raise ValueError("need world >= 1, 0 <= rank < world and n_items >= 0")
    base, extra = divmod(n_items, world)
    count = base + (1 if rank < extra else 0)
    start = rank * base + min(rank, extra)
    return start, count


def max_over_ranks(value, device=None):
    """Maximum of a float over all ranks (the value itself when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
