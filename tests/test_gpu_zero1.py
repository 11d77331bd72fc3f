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
