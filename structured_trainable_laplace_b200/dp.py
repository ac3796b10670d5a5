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
    """Sum, in place, every shared-parameter gradient in `grads` over the group.

    The gradients present (in the fixed order of PARAM_GRADS, so that every rank
    lays them out alike) are packed into one flat buffer, reduced by a single
    all-reduce and unpacked: one collective per step instead of one per
    parameter, which matters because each of them is small (n + k floats) and
    latency-bound."""
    if dist is None:
        import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return grads
    import torch
    present = [grads[key] for key in PARAM_GRADS if grads.get(key) is not None]
    if not present:
        return grads
    if len(present) == 1:
        dist.all_reduce(present[0], group=group)
        return grads
    flat = torch.cat([t.reshape(-1) for t in present])
    dist.all_reduce(flat, group=group)
    off = 0
    for t in present:
        t.copy_(flat[off:off + t.numel()].view_as(t))
        off += t.numel()
    return grads


def shard_columns(B_total: int, rank: int, world: int) -> slice:
    """The batch columns rank owns when a global batch of B_total columns is split
    as evenly as possible (the first B_total % world ranks get one more)."""
    base, extra = divmod(B_total, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))
