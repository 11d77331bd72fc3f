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
