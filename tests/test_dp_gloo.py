"""The data-parallel exchange on two CPU ranks (gloo): each rank takes the
oracle gradient of its own micro-batch, the all-reduce average equals the
oracle gradient of the two micro-batches together, and the AdamW step that
follows is identical on both ranks."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import forward, backward, adamw_step, flatten, unflatten, param_shapes
from decoder_only_transformer_step_b200 import inputs
from decoder_only_transformer_step_b200.dp import average_gradients


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from oracle_fixtures import TINY, params_for
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    params = params_for(TINY, seed=90)
    tok, tgt = inputs.uniform_tokens(2 * world, 32, TINY.vocab, seed=91)
    mine = slice(2 * rank, 2 * rank + 2)
    _, cache = forward(params, TINY, tok[mine], tgt[mine])
    g = torch.from_numpy(flatten(backward(params, TINY, cache), TINY))
    average_gradients(g)
    zeros = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    p1, _, _ = adamw_step(params, unflatten(g.numpy(), TINY), zeros, zeros, 1, TINY)
    out[rank] = (g.numpy().copy(), flatten(p1, TINY))
    dist.destroy_process_group()


def test_two_rank_gradient_average():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from oracle_fixtures import TINY, params_for
    params = params_for(TINY, seed=90)
    tok, tgt = inputs.uniform_tokens(2 * world, 32, TINY.vocab, seed=91)
    _, cache = forward(params, TINY, tok, tgt)
    full = flatten(backward(params, TINY, cache), TINY)
    for r in range(world):
        np.testing.assert_allclose(out[r][0], full, rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(out[0][1], out[1][1])
