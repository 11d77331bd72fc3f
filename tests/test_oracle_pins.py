"""Pins the oracle to closed forms, invariants, library routines and the numbers
the pages print (tests/golden/pages_numbers.json)."""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle
from oracle import (Config, forward, backward, adamw_step, param_shapes, param_count,
                    MatmulCounter, flatten, unflatten)
from oracle import gpt2_oracle as G
from oracle import flops as FL
from decoder_only_transformer_step_b200 import inputs
from oracle_fixtures import TINY, SMALL_124M_L2, GPT2_124M, params_for

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))


def gold(key):
    return GOLD[key]["value"]


# ----------------------------------------------------- building blocks ---

def test_layernorm_constant_row_gives_shift():
    x = np.full((3, 16), 2.5)
    g = np.linspace(0.5, 2.0, 16)
    b = np.linspace(-1.0, 1.0, 16)
    y, _ = G.layernorm_fwd(x, g, b)
    np.testing.assert_array_equal(y, np.broadcast_to(b, y.shape))


def test_layernorm_standardises():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 64)) * 3.0 + 1.0
    y, _ = G.layernorm_fwd(x, np.ones(64), np.zeros(64))
    np.testing.assert_allclose(y.mean(axis=-1), 0.0, atol=1e-12)
    var = x.var(axis=-1)
    np.testing.assert_allclose(y.var(axis=-1), var / (var + G.LN_EPS), rtol=1e-12)


def test_cross_entropy_zero_logits_is_log_vocab():
    V = 50304
    z = np.zeros((2, 3, V))
    tgt = np.array([[0, 5, V - 1], [7, 50256, 1]])
    loss, lse = G.cross_entropy_fwd(z, tgt)
    np.testing.assert_allclose(loss, math.log(V), rtol=1e-15)


def test_cross_entropy_matches_scipy_logsumexp():
    rng = np.random.default_rng(1)
    z = rng.standard_normal((4, 7, 300)) * 5.0
    tgt = rng.integers(0, 300, size=(4, 7))
    loss, lse = G.cross_entropy_fwd(z, tgt)
    ref = scipy.special.logsumexp(z, axis=-1) - np.take_along_axis(z, tgt[..., None], -1)[..., 0]
    np.testing.assert_allclose(loss, ref, rtol=1e-13)


def test_gelu_tanh_form():
    u = np.linspace(-6, 6, 1001)
    exact = 0.5 * u * (1.0 + scipy.special.erf(u / math.sqrt(2.0)))
    assert np.abs(G.gelu_fwd(u) - exact).max() < 1e-3      # tanh form ~ erf form
    assert G.gelu_fwd(np.array([0.0]))[0] == 0.0
    assert G.gelu_bwd(np.array([1.0]), np.array([0.0]))[0] == 0.5
    np.testing.assert_allclose(G.gelu_fwd(np.array([20.0])), [20.0])


def test_attention_single_token_returns_value():
    rng = np.random.default_rng(2)
    q, k, v = (rng.standard_normal((2, 3, 1, 16)) for _ in range(3))
    o, p = G.attention_fwd(q, k, v, None)
    np.testing.assert_array_equal(p, np.ones_like(p))
    np.testing.assert_allclose(o, v, rtol=1e-15)


def test_attention_equal_keys_gives_causal_running_mean():
    """All keys equal -> every allowed score of a query is the same, so the
    output at position i is the mean of v_0..v_i."""
    rng = np.random.default_rng(3)
    B, H, T, hd = 2, 2, 9, 8
    q = rng.standard_normal((B, H, T, hd))
    k = np.broadcast_to(rng.standard_normal((B, H, 1, hd)), (B, H, T, hd)).copy()
    v = rng.standard_normal((B, H, T, hd))
    o, _ = G.attention_fwd(q, k, v, None)
    ref = np.cumsum(v, axis=2) / np.arange(1, T + 1)[None, None, :, None]
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------- the model ---

def test_causality_bit_exact():
    """Perturbing the token at position t0+k (k >= 1) leaves the logits at
    positions <= t0 bit-identical."""
    params = params_for(TINY, seed=11)
    tok, tgt = inputs.uniform_tokens(2, 32, TINY.vocab, seed=12)
    _, c0 = forward(params, TINY, tok, tgt)
    t0 = 13
    for k in (1, 5, 18):
        tok2 = tok.copy()
        tok2[:, t0 + k] = (tok2[:, t0 + k] + 123) % TINY.vocab
        _, c1 = forward(params, TINY, tok2, tgt)
        np.testing.assert_array_equal(c1["z"][:, :t0 + 1], c0["z"][:, :t0 + 1])
        assert np.abs(c1["z"][:, t0 + k] - c0["z"][:, t0 + k]).max() > 0


def test_tied_embedding_decomposition():
    """With a separate head copy equal to wte, the tied wte gradient equals the
    untied head gradient plus the untied embedding gradient, exactly."""
    params = params_for(TINY, seed=13)
    tok, tgt = inputs.uniform_tokens(2, 16, TINY.vocab, seed=14)
    _, ct = forward(params, TINY, tok, tgt)
    gt = backward(params, TINY, ct)
    _, cu = forward(params, TINY, tok, tgt, head=params["wte"].copy())
    gu = backward(params, TINY, cu)
    np.testing.assert_allclose(gt["wte"], gu["head"] + gu["wte"], rtol=0, atol=1e-17)
    assert np.abs(gu["head"]).max() > 0 and np.abs(gu["wte"]).max() > 0


def _expected_init_lse(cfg):
    # LN_f output has squared norm ~ d at gain 1, shift 0; logits of (nearly)
    # independent N(0, 0.02^2) rows then have variance 0.02^2 d, and the mean of
    # LSE over V such logits is ln V + var / 2.
    return math.log(cfg.vocab) + 0.5 * 0.02 ** 2 * cfg.d_model


def test_init_loss_tiny():
    lses, losses = [], []
    for seed in range(3):
        params = params_for(TINY, seed=seed, kind="init")
        tok, tgt = inputs.uniform_tokens(4, 64, TINY.vocab, seed=50 + seed)
        loss, cache = forward(params, TINY, tok, tgt)
        lses.append(cache["lse"].mean())
        losses.append(loss)
    assert abs(np.mean(lses) - _expected_init_lse(TINY)) < 0.01, lses
    assert abs(np.mean(losses) - _expected_init_lse(TINY)) < 0.02, losses


@pytest.mark.slow
def test_init_loss_124m_shaped():
    """Mean LSE at init against the closed form; the loss itself also carries
    the mean target logit, which fluctuates with the seed because Zipf targets
    concentrate on a few ids, so it gets the page's number with a wider band."""
    params = params_for(SMALL_124M_L2, seed=0, kind="init")
    tok, tgt = inputs.zipf_tokens(1, 1024, seed=1000)
    loss, cache = forward(params, SMALL_124M_L2, tok, tgt)
    assert abs(cache["lse"].mean() - _expected_init_lse(SMALL_124M_L2)) < 0.01
    # the page: initial loss 10.95 with ln(50304) ~ 10.83
    assert abs(math.log(gold("vocab_padded")) - gold("ln_vocab_padded")) < 0.005
    assert abs(loss - gold("init_loss_step0")) < 0.15, loss


def test_adamw_step_one_closed_form():
    """At t = 1, m_hat = g and v_hat = g^2, so
    p1 = p0 (1 - lr wd) - lr g / (|g| + eps) on decayed tensors (no decay factor
    on the others)."""
    params = params_for(TINY, seed=15)
    rng = np.random.default_rng(16)
    g = {n: rng.standard_normal(s) * 1e-3 for n, s in param_shapes(TINY)}
    z = {n: np.zeros(s) for n, s in param_shapes(TINY)}
    lr, wd, eps = 6e-4, 0.1, 1e-8
    p1, m1, v1 = adamw_step(params, g, z, z, 1, TINY, lr=lr, beta1=0.9, beta2=0.95, eps=eps,
                            weight_decay=wd)
    for n, s in param_shapes(TINY):
        decay = (1.0 - lr * wd) if len(s) == 2 else 1.0
        ref = params[n] * decay - lr * g[n] / (np.abs(g[n]) + eps)
        np.testing.assert_allclose(p1[n], ref, rtol=1e-12, atol=1e-16)
        np.testing.assert_allclose(m1[n], 0.1 * g[n], rtol=1e-15)
        np.testing.assert_allclose(v1[n], 0.05 * g[n] ** 2, rtol=1e-14)


def test_flatten_roundtrip_and_count():
    params = params_for(TINY, seed=17)
    flat = flatten(params, TINY)
    assert flat.size == param_count(TINY) == FL.n_params_total(2, 64, 512, 64)
    back = unflatten(flat, TINY)
    for n in params:
        np.testing.assert_array_equal(back[n], params[n])


# ------------------------------------------------------- compute model ---

def test_flop_ratio_is_three():
    """Matmul FLOPs of forward+backward over forward = 3.000 exactly (the
    page's FlopCounterMode measurement)."""
    params = params_for(TINY, seed=18)
    tok, tgt = inputs.uniform_tokens(2, 48, TINY.vocab, seed=19)
    ctr = MatmulCounter()
    _, cache = forward(params, TINY, tok, tgt, counter=ctr)
    backward(params, TINY, cache, counter=ctr)
    assert (ctr.fwd + ctr.bwd) / ctr.fwd == gold("fwd_bwd_over_fwd_matmul_flops")
    # and the count equals the shape formula 6 N_matmul + 12 L T d per token
    per_tok = FL.flops_per_token_matmul_only(TINY.n_layer, TINY.d_model, TINY.vocab, 48)
    assert ctr.fwd + ctr.bwd == per_tok * tok.size


@pytest.mark.parametrize("d,L,H,key", [(768, 12, 12, "measured_over_6ND_d768_T1024"),
                                       (1600, 48, 25, "measured_over_6ND_d1600_T1024")])
def test_measured_over_6nd_matches_page(d, L, H, key):
    T, V = 1024, gold("vocab_padded")
    measured = FL.flops_per_token_matmul_only(L, d, V, T)
    ratio = measured / (6 * FL.n_params_total(L, d, V, T))
    assert abs(ratio - gold(key)) < 0.001, ratio
    lo, hi = gold("measured_over_6ND_band")
    assert lo <= ratio <= hi


def test_parameter_counts():
    assert FL.n_params_total(12, 768, 50304, 1024) == 124_475_904 == param_count(GPT2_124M)
    assert FL.n_params_total(48, 1600, 50304, 1024) == 1_557_686_400


def test_memory_model_sixteen_bytes_per_param():
    n = FL.n_params_total(12, 768, 50304, 1024)
    # weight, gradient, m, v in fp32
    assert 4 * 4 == gold("bytes_per_param_fp32_adamw")
    assert abs(16 * n / 1e9 - 1.99) < 0.01
    assert abs(16 * FL.n_params_total(48, 1600, 50304, 1024) / 1e9 - 24.9) < 0.05
    # logits: one vocabulary-sized fp32 vector per token
    assert gold("logit_bytes_per_vocab_entry_per_token") * 50304 * 16 * 1024 / 1e9 == pytest.approx(3.30, abs=0.01)


def test_zipf_inputs():
    tok, tgt = inputs.zipf_tokens(16, 1024, seed=1000)
    assert tok.dtype == np.int32 and tok.shape == (16, 1024)
    np.testing.assert_array_equal(tok[:, 1:], tgt[:, :-1])
    assert tok.min() >= 0 and tok.max() < gold("vocab_real")
    p0 = inputs.zipf_cdf(50257)[0]
    assert abs(p0 - 0.139) < 0.001
    assert abs((tok == 0).mean() - p0) < 0.01


# ------------------------------------ optimizer-side steps around the path ---

def test_clip_grad_norm_matches_torch():
    """The oracle's global-norm clip against torch.nn.utils.clip_grad_norm_
    (a library routine) on the same tensors, clipping and not clipping."""
    import torch
    rng = np.random.default_rng(3)
    grads = {"a": rng.standard_normal((7, 5)), "b": rng.standard_normal(11), "c": rng.standard_normal((2, 3, 4))}
    for max_norm in (0.5, 1e6):
        ts = [torch.from_numpy(g.copy()) for g in grads.values()]
        for t in ts:
            t.grad = t.clone()
        total_t = torch.nn.utils.clip_grad_norm_(ts, max_norm)
        clipped, total = G.clip_grad_norm(grads, max_norm)
        assert abs(total - float(total_t)) <= 1e-12 * total
        for t, (n, g) in zip(ts, clipped.items()):
            np.testing.assert_allclose(g, t.grad.numpy(), rtol=1e-14, atol=0)


def test_clipped_adamw_equals_adamw_on_scaled_grads():
    """Clipping only rescales the gradients: AdamW with max_norm equals AdamW
    on gradients multiplied by max_norm / (norm + 1e-6) by hand."""
    cfg = TINY
    params = params_for(cfg, 5)
    rng = np.random.default_rng(6)
    grads = {n: rng.standard_normal(s) for n, s in param_shapes(cfg)}
    zeros = {n: np.zeros(s) for n, s in param_shapes(cfg)}
    norm = math.sqrt(sum(float(np.sum(g * g)) for g in grads.values()))
    coef = 0.25 / (norm + 1e-6)
    assert coef < 1.0
    P1, M1, V1 = adamw_step(params, grads, zeros, zeros, 1, cfg, max_norm=0.25)
    P2, M2, V2 = adamw_step(params, {n: g * coef for n, g in grads.items()}, zeros, zeros, 1, cfg)
    for n, _ in param_shapes(cfg):
        np.testing.assert_allclose(M1[n], M2[n], rtol=1e-15, atol=0)
        np.testing.assert_allclose(P1[n], P2[n], rtol=1e-15, atol=0)


def test_lr_schedule_closed_forms():
    from decoder_only_transformer_step_b200.schedule import lr_at, steps_for_budget
    max_lr, min_lr = 6e-4, 6e-5
    # the page's step: 16 x 1024 tokens with 32-fold accumulation
    assert steps_for_budget(16 * 1024 * 32 * 1000, 16, 1024, 32) == 1000
    total, warm = 1000, 100
    assert lr_at(0, max_lr, total, warm, min_lr) == pytest.approx(max_lr / warm)
    assert lr_at(warm - 1, max_lr, total, warm, min_lr) == pytest.approx(max_lr)
    assert lr_at(warm, max_lr, total, warm, min_lr) == pytest.approx(max_lr)        # cos 0
    mid = warm + (total - warm) // 2
    assert lr_at(mid, max_lr, total, warm, min_lr) == pytest.approx((max_lr + min_lr) / 2)  # cos(pi/2)
    assert lr_at(total, max_lr, total, warm, min_lr) == min_lr
    # plain cosine (no warm-up) decays to zero at the budget and is monotone
    lrs = [lr_at(s, max_lr, total) for s in range(total + 1)]
    assert lrs[0] == pytest.approx(max_lr) and lrs[-1] == 0.0
    assert all(a >= b for a, b in zip(lrs, lrs[1:]))
    with pytest.raises(ValueError):
        lr_at(0, max_lr, 10, 10)


def test_masked_cross_entropy_matches_torch():
    """Targets equal to IGNORE (-1) take no part: loss and dloss/dz against
    torch.nn.functional.cross_entropy(ignore_index=-1) and its autograd."""
    import torch
    rng = np.random.default_rng(8)
    z = rng.standard_normal((2, 5, 13)) * 2.0
    t = rng.integers(0, 13, size=(2, 5))
    t[0, 1] = t[1, 3] = t[1, 4] = G.IGNORE
    loss_pos, lse = G.cross_entropy_fwd(z, t)
    assert (loss_pos[t == G.IGNORE] == 0).all()
    zt = torch.from_numpy(z.reshape(-1, 13)).requires_grad_(True)
    ref = torch.nn.functional.cross_entropy(zt, torch.from_numpy(t.reshape(-1)), ignore_index=-1)
    ref.backward()
    n_valid = int((t != G.IGNORE).sum())
    assert abs(loss_pos.sum() / n_valid - ref.item()) <= 1e-13
    # the oracle's dz (as backward forms it) against autograd
    dz = np.exp(z - lse[..., None])
    valid = t != G.IGNORE
    safe = np.where(valid, t, 0)
    np.put_along_axis(dz, safe[..., None], np.take_along_axis(dz, safe[..., None], axis=-1) - 1.0, axis=-1)
    dz *= np.where(valid, 1.0 / n_valid, 0.0)[..., None]
    np.testing.assert_allclose(dz.reshape(-1, 13), zt.grad.numpy(), rtol=1e-12, atol=1e-15)


def test_masked_forward_backward_reduces_to_subset():
    """Masking positions equals dropping them from the mean: with only the
    first sequence's targets kept, loss and gradients equal the unmasked
    model run on that sequence alone (the other sequence still shares
    nothing with it: attention is per sequence)."""
    cfg = TINY
    params = params_for(cfg, 9)
    tok, tgt = inputs.uniform_tokens(2, cfg.n_ctx, cfg.vocab, seed=10)
    masked = tgt.copy()
    masked[1, :] = G.IGNORE
    loss_m, cache_m = forward(params, cfg, tok, masked)
    g_m = backward(params, cfg, cache_m)
    loss_1, cache_1 = forward(params, cfg, tok[:1], tgt[:1])
    g_1 = backward(params, cfg, cache_1)
    assert abs(loss_m - loss_1) <= 1e-12 * abs(loss_1)
    for n in g_1:
        np.testing.assert_allclose(g_m[n], g_1[n], rtol=1e-9, atol=1e-14)
