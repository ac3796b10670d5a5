"""Data-parallel training step over several GPUs (one process per GPU).

The anchors a, b, the phases phi, psi and the Gram weights D are parameters
shared by every rank; each rank applies the operator to its own batch of
vectors.  The loss is summed over the ranks' batches, so the gradient of a
shared parameter is the sum of the per-rank gradients (the operator is linear
in the vectors and the batch columns are independent): one all-reduce per
parameter gradient is the only exchange.  Vector gradients (gx) stay local.
"""
from __future__ import annotations

PARAM_GRADS = ("ga", "gb", "gphi", "gpsi", "gD")


def allreduce_param_grads(grads: dict, group=None, dist=None) -> dict:
    """Sum, in place, every shared-parameter gradient in `grads` over the group."""
    if dist is None:
        import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return grads
    for key in PARAM_GRADS:
        t = grads.get(key)
        if t is not None:
            dist.all_reduce(t, group=group)
    return grads


def shard_columns(B_total: int, rank: int, world: int) -> slice:
    """The batch columns rank owns when a global batch of B_total columns is split
    as evenly as possible (the first B_total % world ranks get one more)."""
    base, extra = divmod(B_total, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))
