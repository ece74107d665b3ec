"""Data-parallel training of TT-compressed tables over several GPUs.

One process per GPU.  Every rank holds the same cores, runs the whole TT gather
(grouping, fused forward, fused backward) on its own shard of the bags, and the
ranks then exchange the one thing they share: the dense core gradients.  Because
the training loss is a sum over bags and every core gradient is linear in the
upstream gradient, the sum of the ranks' gradients is the gradient of the global
batch, so one all-reduce (sum) of the gradients followed by the same SGD step on
every rank keeps the cores identical everywhere.  The gradients of all tables and
cores live in one flat buffer so that the exchange is a single NCCL call.
"""
from __future__ import annotations

ALIGN_FLOATS = 4   # the library wants 16-byte aligned gradient buffers


def grad_layout(shapes):
    """Offsets (in floats) of each gradient inside one flat buffer, and its total size.

    shapes: list of core shapes; each offset is a multiple of ALIGN_FLOATS."""
    offsets, total = [], 0
    for shp in shapes:
        n = 1
        for x in shp:
            n *= int(x)
        offsets.append(total)
        total += (n + ALIGN_FLOATS - 1) // ALIGN_FLOATS * ALIGN_FLOATS
    return offsets, total


def allreduce_grads(emb, group=None):
    """Sums the core gradients of a TTEmbeddingBag over the ranks of `group` (in place).

    The handle must have been given its cores with ``flat_grads=True``; torch.distributed
    orders the NCCL call after the backward kernels on the current stream."""
    import torch.distributed as dist
    if emb.grad_flat is None:
        raise ValueError("allreduce_grads needs set_cores(..., flat_grads=True)")
    dist.all_reduce(emb.grad_flat, op=dist.ReduceOp.SUM, group=group)
