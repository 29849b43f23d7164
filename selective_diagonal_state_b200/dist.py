"""Data-parallel plumbing of the scan (torch.distributed; NCCL on GPUs, gloo on CPU).

(batch, head) units of the scan are independent, so ranks take disjoint batch
rows and the forward needs no collective.  The only exchange of a
data-parallel training step is the sum over ranks of the per-head parameter
gradients (dA_log, dtheta, dD), a few KB: one all-reduce.
"""
from __future__ import annotations


def shard_batch(batch: int, world: int, rank: int) -> tuple:
    """Contiguous [start, stop) batch rows of `rank` (ragged when world does not divide batch)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_param_grads(tensors, group=None) -> None:
    """Sum the per-head parameter gradients over ranks, in place (None entries skipped)."""
    import torch.distributed as dist
    for t in tensors:
        if t is not None:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
