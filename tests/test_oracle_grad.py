"""Pins the oracle's hand-written backward to its forward by central finite
differences in fp64 (the backward must be the exact derivative of the forward),
plus exact invariances of the gradient."""
import zlib

import numpy as np
import pytest

from oracle import forward, backward, param_shapes
from decoder_only_transformer_step_b200 import inputs
from oracle_fixtures import TINY, params_for

H = 1e-5


def _loss(params, tok, tgt):
    return forward(params, TINY, tok, tgt)[0]


@pytest.fixture(scope="module")
def setup():
    params = params_for(TINY, seed=1)
    tok, tgt = inputs.uniform_tokens(2, 16, TINY.vocab, seed=2)
    loss, cache = forward(params, TINY, tok, tgt)
    grads = backward(params, TINY, cache)
    return params, tok, tgt, grads


def _shifted(params, name, delta):
    p = dict(params)
    p[name] = params[name] + delta
    return p


@pytest.mark.parametrize("name", [n for n, _ in param_shapes(TINY)])
def test_directional_derivative(setup, name):
    """(L(p + h u) - L(p - h u)) / 2h = <grad, u> for random directions u that
    move one tensor; relative to |grad|*|u| the error must be below 1e-6."""
    params, tok, tgt, grads = setup
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    g = grads[name]
    for _ in range(3):
        u = rng.standard_normal(g.shape)
        fd = (_loss(_shifted(params, name, H * u), tok, tgt)
              - _loss(_shifted(params, name, -H * u), tok, tgt)) / (2 * H)
        an = float((g * u).sum())
        scale = np.linalg.norm(g) * np.linalg.norm(u) + 1e-12
        assert abs(fd - an) <= 1e-6 * scale + 1e-11, (name, fd, an, scale)


@pytest.mark.parametrize("name", [n for n, _ in param_shapes(TINY)])
def test_coordinates(setup, name):
    """Single-coordinate central differences at random entries."""
    params, tok, tgt, grads = setup
    rng = np.random.default_rng(7 + zlib.crc32(name.encode()))
    g = grads[name]
    gmax = np.abs(g).max() + 1e-12
    for _ in range(4):
        idx = tuple(int(rng.integers(0, s)) for s in g.shape)
        e = np.zeros(g.shape)
        e[idx] = 1.0
        fd = (_loss(_shifted(params, name, H * e), tok, tgt)
              - _loss(_shifted(params, name, -H * e), tok, tgt)) / (2 * H)
        assert abs(fd - g[idx]) <= 1e-6 * gmax + 1e-11, (name, idx, fd, g[idx])


def test_tied_wte_rows(setup):
    """wte rows of an input token, a target-only id and an id that never occurs
    (a padded-vocabulary row is one): the tied gradient is right in each case."""
    params, tok, tgt, grads = setup
    used_in = set(tok.reshape(-1).tolist())
    used_tg = set(tgt.reshape(-1).tolist())
    in_only = next(iter(used_in - used_tg))
    tg_only = next(iter(used_tg - used_in))
    unused = next(i for i in range(TINY.vocab - 1, -1, -1) if i not in used_in | used_tg)
    g = grads["wte"]
    gmax = np.abs(g).max()
    for row in (in_only, tg_only, unused):
        for col in (0, 17, TINY.d_model - 1):
            e = np.zeros(g.shape)
            e[row, col] = 1.0
            fd = (_loss(_shifted(params, "wte", H * e), tok, tgt)
                  - _loss(_shifted(params, "wte", -H * e), tok, tgt)) / (2 * H)
            assert abs(fd - g[row, col]) <= 1e-6 * gmax + 1e-11
        assert np.abs(g[row]).max() > 0.0


def test_key_bias_gradient_vanishes(setup):
    """Adding the same vector to every key shifts all scores of a query by one
    constant, which the softmax ignores, so the key-bias gradient is zero."""
    params, tok, tgt, grads = setup
    d = TINY.d_model
    for l in range(TINY.n_layer):
        gb = grads[f"h{l}.b_qkv"]
        assert np.abs(gb[d:2 * d]).max() <= 1e-12 * np.abs(gb).max() + 1e-18
        assert np.abs(gb[:d]).max() > 0 and np.abs(gb[2 * d:]).max() > 0


def test_grad_scale_is_linear(setup):
    params, tok, tgt, grads = setup
    _, cache = forward(params, TINY, tok, tgt)
    g2 = backward(params, TINY, cache, grad_scale=0.25)
    for n in grads:
        np.testing.assert_allclose(g2[n], 0.25 * grads[n], rtol=1e-13, atol=1e-18)
