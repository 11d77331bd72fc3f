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


# ----------------------------------------- sharded optimizer state (ZeRO-1) ---

def _zero1_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from oracle_fixtures import TINY, params_for
    from decoder_only_transformer_step_b200.dp import zero1_step
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    params = params_for(TINY, seed=92)
    tok, tgt = inputs.uniform_tokens(2 * world, 32, TINY.vocab, seed=93)
    mine = slice(2 * rank, 2 * rank + 2)
    _, cache = forward(params, TINY, tok[mine], tgt[mine])
    g_local = flatten(backward(params, TINY, cache), TINY)
    master = torch.from_numpy(flatten(params, TINY))
    m = np.zeros(master.numel())
    v = np.zeros(master.numel())
    refreshed = []
    for step in (1, 2):
        grad = torch.from_numpy(g_local.copy())

        def local_update(off, cnt, step=step, grad=grad):
            # stand-in for the library's range update: the oracle's AdamW over
            # the whole buffer, of which only this rank's shard is kept
            P, Mo, Vo = adamw_step(unflatten(master.numpy(), TINY), unflatten(grad.numpy(), TINY),
                                   unflatten(m, TINY), unflatten(v, TINY), step, TINY)
            sl = slice(off, off + cnt)
            master[sl] = torch.from_numpy(flatten(P, TINY)[sl])
            m[sl] = flatten(Mo, TINY)[sl]
            v[sl] = flatten(Vo, TINY)[sl]

        zero1_step(grad, master, local_update, lambda: refreshed.append(step))
    out[rank] = (master.numpy().copy(), refreshed)
    dist.destroy_process_group()


def test_two_rank_sharded_adamw_equals_full_step():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_zero1_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from oracle_fixtures import TINY, params_for
    params = params_for(TINY, seed=92)
    tok, tgt = inputs.uniform_tokens(2 * world, 32, TINY.vocab, seed=93)
    _, cache = forward(params, TINY, tok, tgt)
    g = backward(params, TINY, cache)
    zeros = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    P, Mo, Vo = adamw_step(params, g, zeros, zeros, 1, TINY)
    P, _, _ = adamw_step(P, g, Mo, Vo, 2, TINY)
    want = flatten(P, TINY)
    for r in range(world):
        np.testing.assert_allclose(out[r][0], want, rtol=1e-12, atol=1e-15)
        assert list(out[r][1]) == [1, 2]


def test_shard_ranges_partition_the_buffer():
    from decoder_only_transformer_step_b200.dp import shard_range
    import pytest
    n = 124475904  # GPT-2 124M flat layout
    for world in (1, 2, 4, 8):
        rs = [shard_range(n, world, r) for r in range(world)]
        assert rs[0][0] == 0 and sum(c for _, c in rs) == n
        assert all(o % 4 == 0 and c % 4 == 0 for o, c in rs)
        assert all(rs[i][0] + rs[i][1] == rs[i + 1][0] for i in range(world - 1))
    with pytest.raises(ValueError):
        shard_range(4 * 3 * 5 + 4, 3, 0)


# ------------------------------------------------- bucketed exchange ---------

def _bucketed_worker(rank, world, port, out, zero1):
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from oracle_fixtures import TINY, params_for
    import decoder_only_transformer_step_b200 as gp
    from decoder_only_transformer_step_b200 import dp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    params = params_for(TINY, seed=96)
    tok, tgt = inputs.uniform_tokens(2 * world, 32, TINY.vocab, seed=97)
    mine = slice(2 * rank, 2 * rank + 2)
    _, cache = forward(params, TINY, tok[mine], tgt[mine])
    grad = torch.from_numpy(flatten(backward(params, TINY, cache), TINY))
    cfg = gp.make_config(TINY.n_layer, TINY.d_model, TINY.n_head, TINY.n_ctx, TINY.vocab, TINY.vocab, 4, 0)
    buckets = dp.gradient_buckets(gp.gpt2_tensors(cfg), TINY.n_layer)
    ex = dp.BucketedExchange(buckets, zero1=zero1)
    # buckets in the order the backward finishes them
    for b in dp.completion_order(TINY.n_layer):
        ex.bucket_ready(grad, b)
    ex.finish()
    master = torch.from_numpy(flatten(params, TINY))
    zeros = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    updated = []

    def local_update(off, cnt):
        # stand-in for the library's range update: the oracle's AdamW over the
        # whole buffer from this rank's gradient buffer, of which only the
        # range is kept (with zero1 only the rank's parts hold the mean)
        P, _, _ = adamw_step(unflatten(master.numpy(), TINY), unflatten(grad.numpy(), TINY), zeros, zeros, 1, TINY)
        sl = slice(off, off + cnt)
        master[sl] = torch.from_numpy(flatten(P, TINY)[sl])
        updated.append((off, cnt))

    ex.optimizer_step(master, local_update, lambda: None)
    out[rank] = (master.numpy().copy(), updated, buckets)
    dist.destroy_process_group()


import pytest  # noqa: E402


@pytest.mark.parametrize("zero1", [False, True])
def test_two_rank_bucketed_exchange_equals_the_union_step(zero1):
    """Per-bucket averaging (all-reduce, or reduce-scatter of equal bucket
    parts with the AdamW update of the rank's parts and a per-bucket
    all-gather) in the order the backward finishes the buckets: both ranks end
    with the oracle's AdamW step of the gradient of the two micro-batches
    together."""
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_bucketed_worker, args=(world, _free_port(), out, zero1), nprocs=world, join=True)
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from oracle_fixtures import TINY, params_for
    params = params_for(TINY, seed=96)
    tok, tgt = inputs.uniform_tokens(2 * world, 32, TINY.vocab, seed=97)
    _, cache = forward(params, TINY, tok, tgt)
    g = backward(params, TINY, cache)
    zeros = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    P, _, _ = adamw_step(params, g, zeros, zeros, 1, TINY)
    want = flatten(P, TINY)
    for r in range(world):
        np.testing.assert_allclose(out[r][0], want, rtol=1e-12, atol=1e-15)
    # the buckets tile the flat layout; with zero1 each rank updated exactly
    # its half of every bucket
    buckets = sorted(out[0][2])
    assert buckets[0][0] == 0 and all(buckets[i][0] + buckets[i][1] == buckets[i + 1][0]
                                      for i in range(len(buckets) - 1))
    assert buckets[-1][0] + buckets[-1][1] == want.size
    if zero1:
        for r in range(world):
            assert sorted(out[r][1]) == sorted((o + r * (c // 2), c // 2) for o, c in out[0][2])
