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


# ------------------------------------------------------ bucketed exchange ---
# The exchange per bucket instead of one buffer after the backward: the
# backward (gpt2_backward_bucketed) records one CUDA event per bucket as soon
# as the bucket's gradients are final, and each bucket's collective runs on a
# side stream after its event, overlapped with the rest of the backward.
# Buckets, indexed like the backward's events: 0 .. L-1 the decoder blocks,
# L the final LayerNorm, L + 1 the token and position embeddings (the tied
# wte gradient takes the embedding scatter last); the backward finishes them
# in the order L, L-1, ..., 0, L + 1.

def gradient_buckets(tensors, n_layer: int):
    """(offset, count) of each bucket of the flat parameter layout, from the
    (name, offset, rows, cols) tensor list of gpt2_tensors."""
    off = {name: o for name, o, r, c in tensors}
    end = max(o + r * c for name, o, r, c in tensors)
    lay = [off[f"h{l}.ln1_g"] for l in range(n_layer)] + [off["lnf_g"]]
    buckets = [(lay[l], lay[l + 1] - lay[l]) for l in range(n_layer)]
    buckets.append((off["lnf_g"], end - off["lnf_g"]))
    buckets.append((0, lay[0]))
    return buckets


def completion_order(n_layer: int):
    """Bucket indices in the order the backward finishes them."""
    return [n_layer] + list(range(n_layer - 1, -1, -1)) + [n_layer + 1]


def bucket_parts(buckets, world: int, rank: int):
    """With the optimizer state sharded: rank's part of every bucket, each an
    equal contiguous 1/world of its bucket (whole float4 groups)."""
    parts = []
    for off, cnt in buckets:
        if cnt % (4 * world):
            raise ValueError(f"bucket of {cnt} elements does not split into {world} parts of whole float4 groups")
        part = cnt // world
        parts.append((off + rank * part, part))
    return parts


class BucketedExchange:
    """Gradient averaging per bucket, overlapped with the backward.

    bucket_ready(grad, i): start bucket i's collective (on GPUs: on the side
    stream, after the event the backward records for it; gloo: at once).
    finish(): the caller's stream waits for every collective.
    zero1: each collective is a reduce-scatter that leaves in rank r's part
    of the bucket the mean of that part; optimizer_step then updates only the
    rank's parts and all-gathers the weights bucket by bucket."""

    def __init__(self, buckets, group=None, zero1=False, events=None, stream=None):
        import torch.distributed as dist
        self.buckets = list(buckets)
        self.group = group
        self.zero1 = zero1
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.events = events
        self.stream = stream
        self.parts = bucket_parts(self.buckets, self.world, self.rank) if zero1 else None

    def _collective(self, grad, i):
        import torch.distributed as dist
        off, cnt = self.buckets[i]
        view = grad[off:off + cnt]
        nccl = dist.get_backend(self.group) == "nccl"
        if not self.zero1:
            if nccl:
                dist.all_reduce(view, op=dist.ReduceOp.AVG, group=self.group)
            else:  # gloo has no AVG
                dist.all_reduce(view, op=dist.ReduceOp.SUM, group=self.group)
                view.div_(self.world)
            return
        poff, pcnt = self.parts[i]
        mine = grad[poff:poff + pcnt]
        if nccl:
            dist.reduce_scatter_tensor(mine, view, op=dist.ReduceOp.AVG, group=self.group)
        else:
            dist.reduce_scatter_tensor(mine, view, op=dist.ReduceOp.SUM, group=self.group)
            mine.div_(self.world)

    def bucket_ready(self, grad, i):
        import torch.distributed as dist
        if not dist.is_initialized() or self.world == 1:
            return
        if self.stream is None:
            self._collective(grad, i)
            return
        import torch
        self.stream.wait_event(self.events[i])
        with torch.cuda.stream(self.stream):
            self._collective(grad, i)

    def finish(self):
        if self.stream is not None:
            import torch
            torch.cuda.current_stream().wait_stream(self.stream)

    def optimizer_step(self, master, local_update, refresh):
        """After finish(): AdamW over the rank's parts of every bucket
        (local_update(offset, count)) and an all-gather of the updated fp32
        weights per bucket (zero1), or over the whole buffer."""
        import torch.distributed as dist
        if not self.zero1 or not dist.is_initialized() or self.world == 1:
            local_update(0, master.numel())
            refresh()
            return
        for poff, pcnt in self.parts:
            local_update(poff, pcnt)
        for (off, cnt), (poff, pcnt) in zip(self.buckets, self.parts):
            dist.all_gather_into_tensor(master[off:off + cnt], master[poff:poff + pcnt].clone(), group=self.group)
        refresh()
