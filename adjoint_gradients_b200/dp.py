"""Data-parallel helpers (one process per GPU, torch.distributed).

Samples are independent, so a global batch is split across ranks and the only
exchange is the gradient: every rank computes the gradient of the mean loss over
its own shard, and the ranks average them (the DistributedDataParallel training
the summaries mention, Gist-EN Technical Summary sec. 3).  With equal shards the
average equals the gradient of the mean loss over the global batch.
"""
from __future__ import annotations


def shard(global_batch: int, world: int, rank: int) -> slice:
    """Contiguous slice of the global batch owned by `rank` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def average_gradients(grad, group=None):
    """In-place mean of `grad` (a torch tensor) over the ranks of `group`."""
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        return grad
    world = dist.get_world_size(group)
    if world > 1:
        dist.all_reduce(grad, group=group)
        grad /= world
    return grad
