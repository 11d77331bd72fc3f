"""Whole-step parity: the CUDA path through the C ABI against the fp64 oracle
on the same seeded inputs.  Tolerances: loss within 1e-2 relative in bf16
(1e-4 in the fp32 mode); every parameter gradient with cosine similarity
>= 0.999 and max|delta| / max|g_ref| <= 2e-2 (a per-element relative error is
meaningless where g_ref ~ 0); parameters after 10 AdamW steps within 1e-2
(relative L2 per tensor)."""
import numpy as np
import pytest
import torch

import decoder_only_transformer_step_b200 as gp
from decoder_only_transformer_step_b200 import inputs
import oracle
from oracle import Config, forward, backward, adamw_step, param_shapes
from oracle_fixtures import TINY, SMALL_124M_L2, params_for

pytestmark = pytest.mark.gpu


def make_model(oc: Config, vocab_real, batch, mode):
    mc = gp.ModelConfig(oc.n_layer, oc.d_model, oc.n_head, oc.n_ctx, vocab_real, oc.vocab, batch, mode)
    return gp.GPT2(mc)


def load_params(model, params, oc):
    flat32 = oracle.flatten(params, oc).astype(np.float32)
    model.master.copy_(torch.from_numpy(flat32))
    model.refresh_shadow()
    # the oracle sees exactly the fp32 values the GPU holds
    return oracle.unflatten(flat32.astype(np.float64), oc)


def gpu_grads(model, oc):
    g = model.grad.double().cpu().numpy()
    return oracle.unflatten(g, oc)


def compare_grads(g_gpu, g_ref, cos_min, rel_max):
    worst = []
    for n in g_ref:
        a, r = g_gpu[n].ravel(), g_ref[n].ravel()
        nr = np.linalg.norm(r)
        if nr == 0:
            assert np.abs(a).max() <= 1e-6, n
            continue
        cos = float(a @ r / (np.linalg.norm(a) * nr + 1e-300))
        rel = float(np.abs(a - r).max() / np.abs(r).max())
        worst.append((n, cos, rel))
        assert cos >= cos_min and rel <= rel_max, (n, cos, rel)
    return worst


def run_step(model, tok, tgt):
    tok_d = torch.from_numpy(tok).cuda()
    tgt_d = torch.from_numpy(tgt).cuda()
    loss = model.forward_loss(tok_d, tgt_d)
    model.backward(1.0, 0)
    torch.cuda.synchronize()
    assert model.status() == 0
    return float(loss.item())


@pytest.mark.parametrize("mode", [1, 0])
def test_tiny_loss_and_grads(mode):
    params = params_for(TINY, seed=21)
    tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=22)
    model = make_model(TINY, TINY.vocab, 4, mode)
    p32 = load_params(model, params, TINY)
    loss = run_step(model, tok, tgt)
    ref_loss, cache = forward(p32, TINY, tok, tgt)
    ref_g = backward(p32, TINY, cache)
    tol_loss = 1e-4 if mode == 1 else 1e-2
    assert abs(loss - ref_loss) <= tol_loss * abs(ref_loss), (loss, ref_loss)
    if mode == 1:
        compare_grads(gpu_grads(model, TINY), ref_g, 0.99999, 1e-3)
    else:
        compare_grads(gpu_grads(model, TINY), ref_g, 0.999, 2e-2)


def test_tiny_ten_adamw_steps():
    params = params_for(TINY, seed=31)
    model = make_model(TINY, TINY.vocab, 4, 0)
    p = load_params(model, params, TINY)
    m = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    v = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    for step in range(1, 11):
        tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=300 + step)
        loss = run_step(model, tok, tgt)
        model.adamw_step(step)
        ref_loss, cache = forward(p, TINY, tok, tgt)
        g = backward(p, TINY, cache)
        p, m, v = adamw_step(p, g, m, v, step, TINY)
        assert abs(loss - ref_loss) <= 1e-2 * abs(ref_loss)
    torch.cuda.synchronize()
    got = oracle.unflatten(model.master.double().cpu().numpy(), TINY)
    d = TINY.d_model
    for n in p:
        a, r = got[n], p[n]
        if n.endswith("b_qkv"):
            # The key-bias gradient is exactly zero in exact arithmetic (a shift
            # of every key leaves the softmax unchanged; pinned in the oracle
            # tests), so Adam's normalised step turns each side's rounding noise
            # into updates of either sign.  That block is held to Adam's
            # per-step bound instead: |m_hat| / sqrt(v_hat) <= 1/sqrt(1-beta2).
            kb = slice(d, 2 * d)
            assert np.abs(a[kb] - r[kb]).max() <= 2 * 10 * 6e-4 / np.sqrt(1 - 0.95)
            a = np.concatenate([a[:d], a[2 * d:]])
            r = np.concatenate([r[:d], r[2 * d:]])
        rel = np.linalg.norm(a - r) / np.linalg.norm(r)
        assert rel <= 1e-2, (n, rel)


HD64_L2 = Config(n_layer=2, d_model=256, n_head=4, n_ctx=256, vocab=1024)


def ten_step_param_errors(oc, batch, seed, mode=0):
    """Ten forward + backward + AdamW steps on the GPU and in the oracle from
    the same fp32 parameters, a new uniform batch each step; per tensor (the
    element-wise max|p_gpu - p_ref| / max|p_ref|, the relative L2 error, the
    fraction of elements beyond 1e-2 max|p_ref|, max|p_gpu - p_ref| / lr).
    The key-bias block of b_qkv is returned separately (its true gradient is
    exactly zero, so both sides' updates are Adam-normalised rounding noise)."""
    params = params_for(oc, seed=seed)
    model = make_model(oc, oc.vocab, batch, mode)
    p = load_params(model, params, oc)
    m = {n: np.zeros(s) for n, s in param_shapes(oc)}
    v = {n: np.zeros(s) for n, s in param_shapes(oc)}
    for step in range(1, 11):
        tok, tgt = inputs.uniform_tokens(batch, oc.n_ctx, oc.vocab, seed=seed * 100 + step)
        loss = run_step(model, tok, tgt)
        model.adamw_step(step)
        ref_loss, cache = forward(p, oc, tok, tgt)
        g = backward(p, oc, cache)
        p, m, v = adamw_step(p, g, m, v, step, oc)
        assert abs(loss - ref_loss) <= 1e-2 * abs(ref_loss), (step, loss, ref_loss)
    torch.cuda.synchronize()
    got = oracle.unflatten(model.master.double().cpu().numpy(), oc)
    d = oc.d_model
    errs, key_bias = {}, []
    for n in p:
        a, r = got[n], p[n]
        if n.endswith("b_qkv"):
            kb = slice(d, 2 * d)
            key_bias.append(float(np.abs(a[kb] - r[kb]).max()))
            a = np.concatenate([a[:d], a[2 * d:]])
            r = np.concatenate([r[:d], r[2 * d:]])
        dev = np.abs(a - r)
        errs[n] = (float(dev.max() / np.abs(r).max()), float(np.linalg.norm(a - r) / np.linalg.norm(r)),
                   float((dev > 1e-2 * np.abs(r).max()).mean()), float(dev.max() / 6e-4))
    return errs, key_bias


def test_ten_adamw_steps_tensor_core_path():
    """The production kernels: head_dim 64 takes the tcgen05 attention forward
    and backward, d = 256 the CTA-pair GEMM tiles, bf16 with the fused
    cross-entropy.  Parameters after 10 AdamW steps against the oracle's, per
    tensor:
    - relative L2 error <= 1e-2 (the stated 1e-2);
    - element-wise |dp| <= 1e-2 max |p_ref| for at least 99 % of the elements;
    - every element within 20 lr.
    Adam divides each coordinate's step by the root of its own squared-gradient
    average, so a coordinate whose gradient is below the bf16 path's rounding
    noise moves by about lr per step with a sign the noise picks, on either
    side, whatever the gradient's size: such coordinates (measured 0.1-0.8 %
    per tensor, at most 5 lr) can sit beyond 1e-2 of max |p| while the
    tensor's L2 error stays below 0.7 %.  The fp32 mode, whose gradients carry
    no such noise, is held to 1e-2 element-wise for every element
    (test_ten_adamw_steps_fp32_elementwise).  The key-bias block is held to
    Adam's per-step bound (its true gradient is exactly zero)."""
    errs, key_bias = ten_step_param_errors(HD64_L2, 4, seed=51)
    lr = 6e-4
    for n, (mx, l2, frac, mlr) in errs.items():
        assert l2 <= 1e-2 and frac <= 1e-2 and mlr <= 20, (n, mx, l2, frac, mlr)
    for kb in key_bias:
        assert kb <= 2 * 10 * lr / np.sqrt(1 - 0.95)


def test_ten_adamw_steps_fp32_elementwise():
    """The same ten steps in the fp32 mode (no bf16 rounding anywhere): every
    parameter element within 1e-2 of max |p_ref| of its tensor."""
    errs, key_bias = ten_step_param_errors(HD64_L2, 4, seed=52, mode=1)
    for n, (mx, l2, frac, mlr) in errs.items():
        assert mx <= 1e-2 and l2 <= 1e-2, (n, mx, l2)
    for kb in key_bias:
        assert kb <= 2 * 10 * 6e-4 / np.sqrt(1 - 0.95)


@pytest.mark.slow
def test_124m_shaped_two_layers():
    """d=768, 12 heads, T=1024, V=50304 (production tile paths, padded vocab),
    two layers, batch 1, Zipf ids."""
    oc = SMALL_124M_L2
    params = params_for(oc, seed=41)
    tok, tgt = inputs.zipf_tokens(1, 1024, seed=42)
    model = make_model(oc, 50257, 1, 0)
    p32 = load_params(model, params, oc)
    loss = run_step(model, tok, tgt)
    ref_loss, cache = forward(p32, oc, tok, tgt)
    ref_g = backward(p32, oc, cache)
    assert abs(loss - ref_loss) <= 1e-2 * abs(ref_loss), (loss, ref_loss)
    compare_grads(gpu_grads(model, oc), ref_g, 0.999, 2e-2)


def test_gradient_accumulation_and_scale():
    """Two micro-batches with grad_scale 1/2 and accumulate: the sum of the
    two scaled gradients (fp32 mode, tight)."""
    params = params_for(TINY, seed=51)
    model = make_model(TINY, TINY.vocab, 4, 1)
    p32 = load_params(model, params, TINY)
    ref = None
    for k in range(2):
        tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=500 + k)
        model.forward_loss(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda())
        model.backward(0.5, k)
        _, cache = forward(p32, TINY, tok, tgt)
        g = backward(p32, TINY, cache, grad_scale=0.5)
        ref = g if ref is None else {n: ref[n] + g[n] for n in g}
    torch.cuda.synchronize()
    compare_grads(gpu_grads(model, TINY), ref, 0.99999, 1e-3)


def test_init_params_statistics():
    model = gp.GPT2(gp.ModelConfig(4, 256, 4, 128, 1000, 1024, 1, 0))
    model.init_params(seed=7)
    torch.cuda.synchronize()
    L = 4
    for name, off, r, c in model.layout:
        t = model.master[off:off + r * c].double()
        short = name.split(".")[-1]
        if short in ("w_o", "w_mp"):
            assert abs(t.std().item() - 0.02 / np.sqrt(2 * L)) < 0.0005, name
        elif c > 1:
            assert abs(t.std().item() - 0.02) < 0.0005 and abs(t.mean().item()) < 5e-4, name
        elif short.endswith("_g"):
            assert torch.all(t == 1.0), name
        else:
            assert torch.all(t == 0.0), name
    assert torch.all(model.grad == 0) and torch.all(model.m == 0) and torch.all(model.v == 0)
    assert torch.equal(model.shadow, model.master.to(torch.bfloat16))
    # same seed -> identical; other seed -> different
    a = model.master.clone()
    model.init_params(seed=7)
    assert torch.equal(a, model.master)
    model.init_params(seed=8)
    assert not torch.equal(a, model.master)


def test_init_loss_near_log_vocab():
    model = gp.GPT2(gp.ModelConfig(2, 768, 12, 1024, 50257, 50304, 1, 0))
    model.init_params(seed=0)
    tok, tgt = inputs.zipf_tokens(1, 1024, seed=1000)
    loss = model.forward_loss(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()).item()
    assert abs(loss - (np.log(50304) + 0.5 * 0.02 ** 2 * 768)) < 0.15, loss


def test_device_errors_are_reported():
    model = make_model(TINY, 500, 4, 0)
    model.init_params(seed=1)
    tok, tgt = inputs.uniform_tokens(4, 64, 500, seed=60)
    tok[1, 5] = 505                       # >= vocab_real: clamped, flagged
    model.forward_loss(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda())
    assert model.status() == -5
    assert model.status() == 0            # reading clears it
    model.master[3] = float("nan")
    model.refresh_shadow()
    tok[1, 5] = 3
    model.forward_loss(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda())
    assert model.status() == -6
    with pytest.raises(gp.Gpt2Error):
        gp.GPT2(gp.ModelConfig(2, 64, 4, 64, 512, 512, 4, 0)).backward()


def test_fp32_mode_is_deterministic():
    params = params_for(TINY, seed=71)
    tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=72)
    outs = []
    for _ in range(2):
        model = make_model(TINY, TINY.vocab, 4, 1)
        load_params(model, params, TINY)
        run_step(model, tok, tgt)
        outs.append(model.grad.clone())
    assert torch.equal(outs[0], outs[1])


def test_step_host_matches_device_path():
    params = params_for(TINY, seed=81)
    tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=82)
    a = make_model(TINY, TINY.vocab, 4, 1)
    b = make_model(TINY, TINY.vocab, 4, 1)
    load_params(a, params, TINY)
    load_params(b, params, TINY)
    loss_a = run_step(a, tok, tgt)
    a.adamw_step(1)
    th = torch.from_numpy(tok).pin_memory()
    gh = torch.from_numpy(tgt).pin_memory()
    lh = torch.zeros(1).pin_memory()
    b.step_host(th, gh, lh, 1)
    assert abs(lh.item() - loss_a) <= 1e-6 * abs(loss_a)
    torch.cuda.synchronize()
    assert (a.master - b.master).abs().max().item() <= 1e-6


def test_grad_norm_matches_torch_and_repeats():
    """gpt2_grad_norm against a plain PyTorch fp64 norm of the same buffer,
    against the oracle's norm of its own gradients, and bitwise repeatable."""
    params = params_for(TINY, seed=41)
    tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=42)
    model = make_model(TINY, TINY.vocab, 4, 0)
    p32 = load_params(model, params, TINY)
    run_step(model, tok, tgt)
    n1 = model.grad_norm()
    n2 = model.grad_norm()
    torch.cuda.synchronize()
    ref = torch.linalg.vector_norm(model.grad.double()).item()
    assert abs(n1.item() - ref) <= 1e-5 * ref, (n1.item(), ref)
    assert torch.equal(n1, n2)
    _, cache = forward(p32, TINY, tok, tgt)
    _, total = oracle.gpt2_oracle.clip_grad_norm(backward(p32, TINY, cache), 1.0)
    assert abs(n1.item() - total) <= 1e-2 * total, (n1.item(), total)


def test_tiny_clipped_adamw_steps():
    """Five steps with global-norm clipping active (max_norm below every
    step's gradient norm): parameters against the oracle's clipped AdamW."""
    params = params_for(TINY, seed=51)
    model = make_model(TINY, TINY.vocab, 4, 0)
    p = load_params(model, params, TINY)
    m = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    v = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    max_norm = None
    for step in range(1, 6):
        tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=500 + step)
        run_step(model, tok, tgt)
        ref_loss, cache = forward(p, TINY, tok, tgt)
        g = backward(p, TINY, cache)
        if max_norm is None:
            max_norm = 0.3 * oracle.gpt2_oracle.clip_grad_norm(g, 1.0)[1]
        assert oracle.gpt2_oracle.clip_grad_norm(g, max_norm)[1] > max_norm  # clipping is active
        model.adamw_step(step, max_norm=max_norm)
        p, m, v = adamw_step(p, g, m, v, step, TINY, max_norm=max_norm)
    torch.cuda.synchronize()
    assert model.status() == 0
    got = oracle.unflatten(model.master.double().cpu().numpy(), TINY)
    d = TINY.d_model
    for n in p:
        a, r = got[n], p[n]
        if n.endswith("b_qkv"):
            # zero true gradient for the key bias: Adam's per-step bound (see
            # test_tiny_ten_adamw_steps)
            kb = slice(d, 2 * d)
            assert np.abs(a[kb] - r[kb]).max() <= 2 * 5 * 6e-4 / np.sqrt(1 - 0.95)
            a = np.concatenate([a[:d], a[2 * d:]])
            r = np.concatenate([r[:d], r[2 * d:]])
        rel = np.linalg.norm(a - r) / np.linalg.norm(r)
        assert rel <= 1e-2, (n, rel)


@pytest.mark.parametrize("mode", [1, 0])
def test_tiny_masked_loss_and_grads(mode):
    """Targets of -1 take no part (instruction-tuning loss): loss and every
    gradient against the oracle, with about a third of the positions masked,
    including one fully masked sequence."""
    params = params_for(TINY, seed=61)
    tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=62)
    rng = np.random.default_rng(63)
    tgt = tgt.copy()
    tgt[rng.random(tgt.shape) < 0.3] = -1
    tgt[2, :] = -1
    model = make_model(TINY, TINY.vocab, 4, mode)
    p32 = load_params(model, params, TINY)
    loss = run_step(model, tok, tgt)
    ref_loss, cache = forward(p32, TINY, tok, tgt)
    ref_g = backward(p32, TINY, cache)
    tol_loss = 1e-4 if mode == 1 else 1e-2
    assert abs(loss - ref_loss) <= tol_loss * abs(ref_loss), (loss, ref_loss)
    if mode == 1:
        compare_grads(gpu_grads(model, TINY), ref_g, 0.99999, 1e-3)
    else:
        compare_grads(gpu_grads(model, TINY), ref_g, 0.999, 2e-2)


def test_target_minus_one_is_masked_other_negatives_flagged():
    model = make_model(TINY, 500, 4, 0)
    model.init_params(seed=2)
    tok, tgt = inputs.uniform_tokens(4, 64, 500, seed=64)
    tgt[0, :10] = -1                      # masked: no error
    model.forward_loss(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda())
    assert model.status() == 0
    tgt[0, 3] = -2                        # neither an id nor the mask value
    model.forward_loss(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda())
    assert model.status() == -5
    assert model.status() == 0


def test_full_size_step_gradients_through_masked_targets():
    # the step in the bench's launch configuration (GPT-2 124M, 16 x 1024
    # tokens, 12 layers, bf16): with targets only at positions < n_b of row b
    # (-1 elsewhere) the loss and every gradient depend on the rows' first
    # n_b tokens alone (causality), which the oracle computes in full
    from oracle_fixtures import GPT2_124M
    B, T = 16, 1024
    model = make_model(GPT2_124M, 50257, B, 0)
    model.init_params(seed=5)
    p32 = oracle.unflatten(model.master.double().cpu().numpy(), GPT2_124M)
    tok, tgt = inputs.zipf_tokens(B, T, n_ids=50257, seed=1001)
    nb = (np.arange(B) * 7 + 9) % 40 + 8
    tgt = tgt.copy()
    for b in range(B):
        tgt[b, nb[b]:] = -1
    loss = run_step(model, tok, tgt)
    n = int(nb.max())
    ref_loss, cache = forward(p32, GPT2_124M, tok[:, :n], tgt[:, :n])
    ref_g = backward(p32, GPT2_124M, cache)
    assert abs(loss - ref_loss) <= 1e-2 * abs(ref_loss), (loss, ref_loss)
    compare_grads(gpu_grads(model, GPT2_124M), ref_g, 0.999, 2e-2)


@pytest.mark.parametrize("d,H,T", [(1024, 16, 256), (1600, 25, 256), (768, 12, 4096)],
                         ids=["350m-shaped", "1.5b-shaped", "t4096-shaped"])
def test_other_config_shapes_one_layer(d, H, T):
    """The widths and the context of the other configurations (GPT-2 medium
    d 1024 / 16 heads, XL d 1600 / 25 heads, long context T 4096): one layer,
    vocabulary 50304, bf16, Zipf ids; loss and every gradient against the
    oracle.  d 1024 and 1600 take the two-kernel LayerNorm backward and (1600)
    ragged GEMM tiles; T 4096 fills the attention backward's 32 query-block
    slots."""
    oc = Config(n_layer=1, d_model=d, n_head=H, n_ctx=T, vocab=50304)
    params = params_for(oc, seed=43)
    B = 1
    tok, tgt = inputs.zipf_tokens(B, T, seed=44)
    model = make_model(oc, 50257, B, 0)
    p32 = load_params(model, params, oc)
    loss = run_step(model, tok, tgt)
    ref_loss, cache = forward(p32, oc, tok, tgt)
    ref_g = backward(p32, oc, cache)
    assert abs(loss - ref_loss) <= 1e-2 * abs(ref_loss), (loss, ref_loss)
    compare_grads(gpu_grads(model, oc), ref_g, 0.999, 2e-2)


def test_deterministic_mode_repeats_bitwise_and_matches_oracle():
    """Mode 2 (bf16, attention dQ summed in key-block order): the same step
    twice gives bitwise the same loss and gradients, and they match the
    oracle within the bf16 tolerances."""
    oc = HD64_L2
    params = params_for(oc, seed=61)
    tok, tgt = inputs.uniform_tokens(4, oc.n_ctx, oc.vocab, seed=62)
    model = make_model(oc, oc.vocab, 4, 2)
    p32 = load_params(model, params, oc)
    losses, grads = [], []
    for _ in range(2):
        losses.append(run_step(model, tok, tgt))
        grads.append(model.grad.clone())
    assert losses[0] == losses[1]
    assert torch.equal(grads[0], grads[1])
    ref_loss, cache = forward(p32, oc, tok, tgt)
    assert abs(losses[0] - ref_loss) <= 1e-2 * abs(ref_loss)
    compare_grads(gpu_grads(model, oc), backward(p32, oc, cache), 0.999, 2e-2)


@pytest.mark.slow
def test_deterministic_mode_full_size_step_repeats_bitwise():
    """The bench's workload (GPT-2 124M, 16 x 1024 Zipf tokens) in mode 2:
    two identical steps give bitwise the same loss and every gradient."""
    mc = gp.ModelConfig(12, 768, 12, 1024, 50257, 50304, 16, 2)
    model = gp.GPT2(mc)
    model.init_params(seed=0)
    tok, tgt = inputs.zipf_tokens(16, 1024, seed=63)
    tok_d, tgt_d = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    out = []
    for _ in range(2):
        loss = model.forward_loss(tok_d, tgt_d)
        model.backward(1.0, 0)
        torch.cuda.synchronize()
        assert model.status() == 0
        out.append((float(loss.item()), model.grad.clone()))
    assert out[0][0] == out[1][0]
    assert torch.equal(out[0][1], out[1][1])


@pytest.mark.slow
def test_full_size_gradient_scale_equivariance_bitwise():
    """The page's 32-fold accumulation scales each micro-batch's gradients by
    grad_scale = 1/32.  In mode 2 every reduction is fixed-order and the
    embedding scatter's fixed-point unit is relative to grad_scale, so at the
    bench's full size (124M, 16 x 1024 Zipf tokens) the gradient at
    grad_scale 1/32 is bitwise 1/32 of the gradient at grad_scale 1 — the
    scale costs no precision anywhere (the grad_scale-1 gradient is itself
    checked against the oracle at this size by the prefix-masked test)."""
    mc = gp.ModelConfig(12, 768, 12, 1024, 50257, 50304, 16, 2)
    model = gp.GPT2(mc)
    model.init_params(seed=0)
    tok, tgt = inputs.zipf_tokens(16, 1024, seed=64)
    tok_d, tgt_d = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    grads = []
    for scale in (1.0, 1.0 / 32):
        model.forward_loss(tok_d, tgt_d)
        model.backward(scale, 0)
        torch.cuda.synchronize()
        assert model.status() == 0
        grads.append(model.grad.clone())
    g1, g32 = grads
    assert torch.equal(g32 * 32, g1)
    # the embedding rows of ids that occur, where the fixed point acts
    wte = g1[: 50304 * 768].view(50304, 768)
    assert torch.count_nonzero(wte[:1000]) > 0
