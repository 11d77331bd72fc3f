"""Pins the oracle's incremental decoder (key/value cache) to the full forward.

The next-token logits after positions 0..p are, by definition, the forward's
logits at position p; the cache only avoids recomputing positions < p.  These
tests check that identity at every position, for rows at different positions
in the same step, and that the cache holds exactly the forward's K and V.  A
wrong cache index, a missing self-attention to the new token, an off-by-one
position embedding or a transposed head layout each break one of them.
"""
import numpy as np

from oracle import forward, kv_cache_empty, decode_step, prefill, greedy_next
from oracle import gpt2_oracle as G
from oracle_fixtures import TINY, params_for
from decoder_only_transformer_step_b200 import inputs


def _forward_logits(params, cfg, tokens):
    tgt = np.full(tokens.shape, G.IGNORE)
    _, cache = forward(params, cfg, tokens, tgt)
    return cache


def test_decode_matches_forward_at_every_position():
    p = params_for(TINY, seed=3)
    B, T = 3, 20
    tok, _ = inputs.uniform_tokens(B, T, 500, seed=11)
    full = _forward_logits(p, TINY, tok)["z"]                       # [B, T, V]
    cache = kv_cache_empty(TINY, B, 32)
    for t in range(T):
        z = decode_step(p, TINY, cache, tok[:, t], np.full(B, t))
        np.testing.assert_allclose(z, full[:, t], rtol=1e-10, atol=1e-12)


def test_rows_at_different_positions_in_one_step():
    p = params_for(TINY, seed=4)
    tok, _ = inputs.uniform_tokens(2, 12, 500, seed=12)
    full = _forward_logits(p, TINY, tok)["z"]
    cache = kv_cache_empty(TINY, 2, 16)
    # row 0 runs 5 positions ahead of row 1
    for t in range(5):
        decode_step(p, TINY, [dict(k=c["k"][:1], v=c["v"][:1]) for c in cache], tok[:1, t], np.array([t]))
    for t in range(7):
        z = decode_step(p, TINY, cache, np.array([tok[0, t + 5], tok[1, t]]), np.array([t + 5, t]))
        np.testing.assert_allclose(z[0], full[0, t + 5], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(z[1], full[1, t], rtol=1e-10, atol=1e-12)


def test_prefill_cache_holds_forward_k_v_and_last_logits():
    p = params_for(TINY, seed=5)
    tok, _ = inputs.uniform_tokens(3, 16, 500, seed=13)
    plen = np.array([16, 9, 1])
    fw = _forward_logits(p, TINY, tok)
    cache = kv_cache_empty(TINY, 3, 24)
    z = prefill(p, TINY, cache, tok, plen)
    for b in range(3):
        n = plen[b]
        np.testing.assert_allclose(z[b], fw["z"][b, n - 1], rtol=1e-10, atol=1e-12)
        for l in range(TINY.n_layer):
            np.testing.assert_allclose(cache[l]["k"][b, :, :n], fw["layers"][l]["k"][b, :, :n], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(cache[l]["v"][b, :, :n], fw["layers"][l]["v"][b, :, :n], rtol=1e-12, atol=1e-14)
            assert not cache[l]["k"][b, :, n:].any() and not cache[l]["v"][b, :, n:].any()


def test_position_zero_attends_to_itself_only():
    # one key: softmax weight 1, attention output = v of the new token, so the
    # logits equal a one-token forward whatever the rest of the cache holds
    p = params_for(TINY, seed=6)
    tok = np.array([[7], [301]])
    cache = kv_cache_empty(TINY, 2, 8)
    for c in cache:
        c["k"][:] = 5.0
        c["v"][:] = -3.0
    z = decode_step(p, TINY, cache, tok[:, 0], np.array([0, 0]))
    np.testing.assert_allclose(z, _forward_logits(p, TINY, tok)["z"][:, 0], rtol=1e-10, atol=1e-12)


def test_greedy_ties_padding_and_nan():
    z = np.zeros((4, 16))
    z[0, [3, 9]] = 2.0          # tie: lowest id
    z[1, 14] = 9.0              # padded id (vocab_real 12): not eligible
    z[1, 5] = 1.0
    z[2, :] = -np.inf
    z[2, 11] = -1e30
    z[3, 2] = np.nan            # NaN wins, first one
    z[3, 7] = np.nan
    z[3, 1] = 4.0
    np.testing.assert_array_equal(greedy_next(z, 12), [3, 5, 11, 2])
