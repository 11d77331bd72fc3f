"""Data-parallel exchange for the GPT-2 step.

"Pré-treinar um LLM: dados, compute, leis de escala e custo" (parallelism
paragraph): data parallelism keeps a copy of the model on every GPU and
averages the gradients.  Each rank runs forward and backward on its own
micro-batch of equal size; since the loss is a mean over tokens, the mean of
the per-rank gradients is the gradient of the mean loss over the union of the
micro-batches, and every rank then applies the same AdamW step.

The exchange is one all-reduce (average) of the flat fp32 gradient buffer
between gpt2_backward and gpt2_adamw_step, NCCL over NVLink on GPUs (gloo in
the CPU tests).

With the optimizer state sharded (each rank owns the AdamW update of one
contiguous 1/world of the flat buffer, the ZeRO stage-1 scheme) the same step
is a reduce-scatter of the gradient (each rank receives the mean of its own
shard), the AdamW update of that shard only, and an all-gather of the updated
fp32 weights.  The bytes on the wire equal the all-reduce's (a reduce-scatter
plus an all-gather of the same buffer); the optimizer pass and its state are
cut by the world size.
"""
from __future__ import annotations


def average_gradients(grad, group=None):
    """In-place mean of the flat gradient buffer over all ranks of `group`."""
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return grad
    if dist.get_backend(group) == "nccl":
        dist.all_reduce(grad, op=dist.ReduceOp.AVG, group=group)
    else:  # gloo has no AVG
        dist.all_reduce(grad, op=dist.ReduceOp.SUM, group=group)
        grad.div_(dist.get_world_size(group))
    return grad


def shard_range(n: int, world: int, rank: int):
    """(offset, count) of rank's shard of an n-element flat buffer: equal
    contiguous shards, each a multiple of 4 elements (the update kernel works
    on float4 groups).  n must be a multiple of 4 * world."""
    if n % (4 * world):
        raise ValueError(f"{n} elements do not split into {world} shards of whole float4 groups")
    count = n // world
    return rank * count, count


def zero1_step(grad, master, local_update, refresh, group=None):
    """One sharded-optimizer step on the flat fp32 buffers of this rank.

    grad: this rank's micro-batch gradient (overwritten: its own shard ends up
    holding the mean over ranks).  local_update(offset, count) applies AdamW to
    master / m / v [offset, offset + count) from grad there (the library's
    gpt2_adamw_step_range on GPUs).  Afterwards master holds every rank's
    updated shard and refresh() is called to rebuild what derives from it (the
    bf16 shadow)."""
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        local_update(0, grad.numel())
        refresh()
        return
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    off, cnt = shard_range(grad.numel(), world, rank)
    shard = grad[off:off + cnt]
    if dist.get_backend(group) == "nccl":
        dist.reduce_scatter_tensor(shard, grad, op=dist.ReduceOp.AVG, group=group)
    else:  # gloo has no AVG
        dist.reduce_scatter_tensor(shard, grad, op=dist.ReduceOp.SUM, group=group)
        shard.div_(world)
    local_update(off, cnt)
    dist.all_gather_into_tensor(master, master[off:off + cnt].clone(), group=group)
    refresh()
