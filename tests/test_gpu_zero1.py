"""The range form of the AdamW step (one shard of the optimizer state): the
update of [offset, offset + count) pieces, applied over a partition of the
flat buffer, is bitwise the full step (master, m, v and the bf16 shadow), and
ranges outside the layout or not in float4 groups are rejected on the host."""
import numpy as np
import pytest
import torch

import decoder_only_transformer_step_b200 as gp
from decoder_only_transformer_step_b200.dp import shard_range

pytestmark = pytest.mark.gpu


def _state(model):
    return [t.clone() for t in (model.master, model.m, model.v, model.grad, model.shadow)]


def _restore(model, st):
    for t, s in zip((model.master, model.m, model.v, model.grad, model.shadow), st):
        t.copy_(s)


@pytest.mark.parametrize("mode", [0, 1])
def test_range_updates_partition_equals_full_step(mode):
    mc = gp.ModelConfig(2, 128, 2, 64, 1000, 1024, 2, mode)
    model = gp.GPT2(mc)
    model.init_params(seed=5)
    g = torch.Generator(device="cuda").manual_seed(6)
    model.grad.copy_(torch.randn(model.n_params, device="cuda", generator=g) * 1e-2)
    model.m.copy_(torch.randn(model.n_params, device="cuda", generator=g) * 1e-3)
    model.v.copy_(torch.rand(model.n_params, device="cuda", generator=g) * 1e-5)
    start = _state(model)
    model.adamw_step(3)
    want = [t.clone() for t in (model.master, model.m, model.v, model.shadow)]
    n = model.n_params
    for world in (2, 4):
        _restore(model, start)
        for r in range(world):
            off, cnt = shard_range(n, world, r)
            model.adamw_step_range(3, off, cnt)
        got = (model.master, model.m, model.v, model.shadow)
        for a, b in zip(got, want):
            assert torch.equal(a, b)
    # an uneven partition at float4 boundaries that cut through tensors
    _restore(model, start)
    cuts = [0, 4, 4100, 70000, n - 8, n]
    for a, b in zip(cuts[:-1], cuts[1:]):
        model.adamw_step_range(3, a, b - a)
    for x, y in zip((model.master, model.m, model.v, model.shadow), want):
        assert torch.equal(x, y)
    torch.cuda.synchronize()
    assert model.status() == 0


def test_range_arguments_are_checked():
    model = gp.GPT2(gp.ModelConfig(2, 64, 4, 64, 512, 512, 2, 1))
    n = model.n_params
    for off, cnt in [(2, 4), (0, 6), (n - 4, 8), (n + 4, 0)]:
        with pytest.raises(gp.Gpt2Error):
            model.adamw_step_range(1, off, cnt)
    model.adamw_step_range(1, n, 0)  # empty range at the end: nothing to do


@pytest.mark.parametrize("accumulate", [0, 1])
def test_bucketed_backward_equals_backward_and_orders_its_events(accumulate):
    """gpt2_backward_bucketed: the same gradients as gpt2_backward (each bias
    / LayerNorm reduction is the same fixed-order sum, only launched per
    bucket; the attention backward's fp32 dQ reductions arrive in no fixed
    order in either, hence a tolerance rather than bitwise equality), and each
    bucket's event recorded in the stated order (final LayerNorm, blocks
    L-1 .. 0, embeddings)."""
    from decoder_only_transformer_step_b200 import dp, inputs
    L = 3
    mc = gp.ModelConfig(L, 128, 2, 128, 1000, 1024, 2, 0)
    model = gp.GPT2(mc)
    model.init_params(seed=8)
    tok, tgt = inputs.uniform_tokens(2, 128, 1000, seed=9)
    tok, tgt = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    g0 = torch.randn(model.n_params, device="cuda") * 1e-3
    model.grad.copy_(g0)
    model.forward_loss(tok, tgt)
    model.backward(1.0, accumulate)
    want = model.grad.clone()
    model.grad.copy_(g0)
    events = [torch.cuda.Event(enable_timing=True) for _ in range(L + 2)]
    for ev in events:
        ev.record()
    start = torch.cuda.Event(enable_timing=True)
    model.forward_loss(tok, tgt)
    start.record()
    model.backward_bucketed(events, 1.0, accumulate)
    torch.cuda.synchronize()
    assert model.status() == 0
    diff = (model.grad - want).double()
    assert diff.norm().item() <= 1e-4 * want.double().norm().item()
    times = [start.elapsed_time(events[b]) for b in dp.completion_order(L)]
    assert all(t >= 0 for t in times)
    assert all(times[i] <= times[i + 1] for i in range(len(times) - 1)), times
    # the buckets tile the flat layout
    buckets = sorted(dp.gradient_buckets(gp.gpt2_tensors(mc.c()), L))
    assert buckets[0][0] == 0 and buckets[-1][0] + buckets[-1][1] == model.n_params
    assert all(buckets[i][0] + buckets[i][1] == buckets[i + 1][0] for i in range(len(buckets) - 1))
