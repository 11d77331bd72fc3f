"""Pins the oracle against an independent PyTorch (CPU, fp64) model assembled
from library routines -- F.embedding, F.layer_norm, F.linear,
F.scaled_dot_product_attention(is_causal=True), F.gelu(approximate="tanh"),
F.cross_entropy -- differentiated by autograd, and against torch.optim.AdamW.
A dropped term, a wrong sign, a transposed operand or a wrong index in the
oracle's forward, backward or optimiser makes one of these fail."""
import numpy as np
import torch
import torch.nn.functional as F

from oracle import forward, backward, adamw_step, param_shapes, decay_mask
from decoder_only_transformer_step_b200 import inputs
from oracle_fixtures import TINY, params_for


def witness_loss(tp, cfg, tok, tgt):
    B, T = tok.shape
    d, H = cfg.d_model, cfg.n_head
    x = F.embedding(tok, tp["wte"]) + tp["wpe"][:T]
    for l in range(cfg.n_layer):
        P = lambda t: tp[f"h{l}.{t}"]  # noqa: E731
        h = F.layer_norm(x, (d,), P("ln1_g"), P("ln1_b"), eps=1e-5)
        q, k, v = F.linear(h, P("w_qkv"), P("b_qkv")).split(d, dim=-1)
        q, k, v = (t.view(B, T, H, d // H).transpose(1, 2) for t in (q, k, v))
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
        x = x + F.linear(o.transpose(1, 2).reshape(B, T, d), P("w_o"), P("b_o"))
        h = F.layer_norm(x, (d,), P("ln2_g"), P("ln2_b"), eps=1e-5)
        x = x + F.linear(F.gelu(F.linear(h, P("w_fc"), P("b_fc")), approximate="tanh"),
                         P("w_mp"), P("b_mp"))
    z = F.linear(F.layer_norm(x, (d,), tp["lnf_g"], tp["lnf_b"], eps=1e-5), tp["wte"])
    return F.cross_entropy(z.reshape(-1, cfg.vocab), tgt.reshape(-1))


def _torch_params(params):
    return {n: torch.tensor(a, dtype=torch.float64, requires_grad=True) for n, a in params.items()}


def test_loss_and_grads_match_autograd_witness():
    params = params_for(TINY, seed=3)
    tok, tgt = inputs.uniform_tokens(3, 40, TINY.vocab, seed=4)
    loss, cache = forward(params, TINY, tok, tgt)
    grads = backward(params, TINY, cache)
    tp = _torch_params(params)
    wl = witness_loss(tp, TINY, torch.tensor(tok, dtype=torch.long), torch.tensor(tgt, dtype=torch.long))
    wl.backward()
    assert abs(loss - wl.item()) <= 1e-12 * abs(loss)
    for n, _ in param_shapes(TINY):
        ref = tp[n].grad.numpy()
        err = np.abs(grads[n] - ref).max()
        assert err <= 1e-10 * (np.abs(ref).max() + 1e-30), (n, err)


def test_adamw_matches_torch_optim():
    """Ten AdamW steps with decay on the 2-D tensors only, against
    torch.optim.AdamW with two parameter groups."""
    params = params_for(TINY, seed=5)
    hp = dict(lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)
    names = [n for n, _ in param_shapes(TINY)]
    dm = decay_mask(TINY)
    tp = {n: torch.tensor(params[n], dtype=torch.float64, requires_grad=True) for n in names}
    opt = torch.optim.AdamW(
        [{"params": [tp[n] for n in names if dm[n]], "weight_decay": hp["weight_decay"]},
         {"params": [tp[n] for n in names if not dm[n]], "weight_decay": 0.0}],
        lr=hp["lr"], betas=(hp["beta1"], hp["beta2"]), eps=hp["eps"], foreach=False)
    m = {n: np.zeros_like(params[n]) for n in names}
    v = {n: np.zeros_like(params[n]) for n in names}
    rng = np.random.default_rng(6)
    p = params
    for step in range(1, 11):
        g = {n: rng.standard_normal(params[n].shape) * 10.0 ** rng.integers(-6, 0) for n in names}
        for n in names:
            tp[n].grad = torch.tensor(g[n])
        opt.step()
        p, m, v = adamw_step(p, g, m, v, step, TINY, **hp)
    for n in names:
        np.testing.assert_allclose(p[n], tp[n].detach().numpy(), rtol=1e-12, atol=1e-15)


def test_train_steps_match_witness():
    """Three full steps (forward, backward, AdamW) against the witness model
    trained by torch.optim.AdamW on the same tokens."""
    params = params_for(TINY, seed=8)
    names = [n for n, _ in param_shapes(TINY)]
    dm = decay_mask(TINY)
    tp = _torch_params(params)
    opt = torch.optim.AdamW(
        [{"params": [tp[n] for n in names if dm[n]], "weight_decay": 0.1},
         {"params": [tp[n] for n in names if not dm[n]], "weight_decay": 0.0}],
        lr=6e-4, betas=(0.9, 0.95), eps=1e-8, foreach=False)
    m = {n: np.zeros_like(params[n]) for n in names}
    v = {n: np.zeros_like(params[n]) for n in names}
    p = params
    for step in range(1, 4):
        tok, tgt = inputs.uniform_tokens(2, 32, TINY.vocab, seed=100 + step)
        loss, cache = forward(p, TINY, tok, tgt)
        g = backward(p, TINY, cache)
        p, m, v = adamw_step(p, g, m, v, step, TINY)
        opt.zero_grad()
        wl = witness_loss(tp, TINY, torch.tensor(tok, dtype=torch.long), torch.tensor(tgt, dtype=torch.long))
        wl.backward()
        opt.step()
        assert abs(loss - wl.item()) <= 1e-11 * abs(loss)
    for n in names:
        np.testing.assert_allclose(p[n], tp[n].detach().numpy(), rtol=1e-9, atol=1e-12)
