"""The micro-step as a CUDA graph (gpt2_graph_capture / gpt2_graph_step): the
replayed graph computes what gpt2_forward_loss + gpt2_backward compute on the
same ids — bitwise in the repeatable bf16 mode (mode 2), so any difference
would be a captured pointer or argument that went stale — for new ids on
every replay, the launch counter counts the graph's kernels, and the calls
are checked on the host."""
import numpy as np
import pytest
import torch

import decoder_only_transformer_step_b200 as gp
from decoder_only_transformer_step_b200 import inputs

pytestmark = pytest.mark.gpu


def _ids(B, T, Vr, seed):
    tok, tgt = inputs.zipf_tokens(B, T, n_ids=Vr, seed=seed)
    return torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()


@pytest.mark.parametrize("accumulate", [0, 1])
def test_graph_step_equals_eager_step_bitwise(accumulate):
    B, T, Vr, V = 2, 256, 1000, 1024
    model = gp.GPT2(gp.ModelConfig(2, 256, 4, T, Vr, V, B, 2))
    model.init_params(seed=11)
    batches = [_ids(B, T, Vr, 40 + i) for i in range(3)]
    base = torch.randn(model.n_params, device="cuda", generator=torch.Generator(device="cuda").manual_seed(3))
    # eager reference for each batch
    want = []
    for tok, tgt in batches:
        model.grad.copy_(base)
        model.forward_loss(tok, tgt)
        model.backward(0.5, accumulate)
        torch.cuda.synchronize()
        want.append((model.loss.clone(), model.grad.clone()))
    model.graph_capture(B, grad_scale=0.5, accumulate=accumulate)
    for (tok, tgt), (loss, grad) in zip(batches, want):
        model.grad.copy_(base)
        model.loss.zero_()
        model.graph_step(tok, tgt)
        torch.cuda.synchronize()
        assert torch.equal(model.loss, loss)
        assert torch.equal(model.grad, grad)
    assert model.status() == 0
    # the step the graph leaves behind feeds the optimizer like an eager one
    model.adamw_step(1)
    torch.cuda.synchronize()
    assert model.status() == 0


def test_graph_launch_count_and_host_checks():
    B, T, Vr, V = 2, 128, 500, 512
    model = gp.GPT2(gp.ModelConfig(2, 128, 2, T, Vr, V, B, 0))
    model.init_params(seed=2)
    tok, tgt = _ids(B, T, Vr, 7)
    with pytest.raises(gp.Gpt2Error):  # no graph yet
        model.graph_step(tok, tgt)
    model.forward_loss(tok, tgt)
    model.backward()
    torch.cuda.synchronize()
    l0 = gp.gpt2_kernel_launches()
    model.forward_loss(tok, tgt)
    model.backward()
    eager = gp.gpt2_kernel_launches() - l0
    l1 = gp.gpt2_kernel_launches()
    model.graph_capture(B)
    assert gp.gpt2_kernel_launches() == l1  # capturing launches nothing
    model.graph_step(tok, tgt)
    model.graph_step(tok, tgt)
    torch.cuda.synchronize()
    assert gp.gpt2_kernel_launches() - l1 == 2 * eager
    # the legacy default stream (NULL) cannot be captured
    assert gp._lib().gpt2_graph_capture(model.ctx, B, 1.0, 0, None, None) == \
        gp.ERRORS_BY_NAME["GPT2_ERR_INVALID_ARG"]
    with pytest.raises(gp.Gpt2Error):
        model.graph_capture(B + 1)
    gp.gpt2_graph_release(model.ctx)
    with pytest.raises(gp.Gpt2Error):
        model.graph_step(tok, tgt)
    assert np.isfinite(float(model.loss.item()))
    assert model.status() == 0


def test_step_host_replays_the_graph_bitwise():
    """gpt2_step_host with a captured micro-step of the same shape (grad_scale
    1, accumulate 0) takes the graph: parameters and loss after the step are
    bitwise those of the step without a graph (mode 2), and the graph's
    kernels are counted."""
    B, T, Vr, V = 2, 256, 1000, 1024
    tok, tgt = inputs.zipf_tokens(B, T, n_ids=Vr, seed=91)
    th, gh = torch.from_numpy(tok).pin_memory(), torch.from_numpy(tgt).pin_memory()
    out = []
    for use_graph in (False, True):
        model = gp.GPT2(gp.ModelConfig(2, 256, 4, T, Vr, V, B, 2))
        model.init_params(seed=12)
        model.forward_loss(th.cuda(), gh.cuda())
        model.backward()
        torch.cuda.synchronize()
        model.grad.zero_()
        if use_graph:
            model.graph_capture(B)
        lh = torch.zeros(1).pin_memory()
        l0 = gp.gpt2_kernel_launches()
        model.step_host(th, gh, lh, 1)
        launched = gp.gpt2_kernel_launches() - l0
        assert model.status() == 0
        out.append((float(lh.item()), model.master.clone(), launched))
    assert out[0][0] == out[1][0]
    assert torch.equal(out[0][1], out[1][1])
    assert out[0][2] == out[1][2]
