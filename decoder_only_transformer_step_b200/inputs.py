"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module draws random numbers and nothing else: it holds none of the
model's arithmetic, so both the CUDA path and the CPU oracle may take their
inputs from it.

Token ids stand in for the FineWeb-Edu shards the GPT-2 run trained on ("Criei
GPT-2 do zero com uma RTX 4090", section "Preparação dos dados"), which are not
available offline.  Natural-language token frequencies are heavy-tailed, so
ids are drawn from a Zipf law P(id = k) proportional to (k+1)^-s over the
50257 real ids (rank = id, no permutation), by inverse-CDF sampling in fp64.
Each row is a stream of T+1 draws: tokens = stream[0:T], targets =
stream[1:T+1] (the label at position t is the token at t+1).
"""
from __future__ import annotations

import numpy as np


def zipf_cdf(n_ids: int, s: float = 1.1) -> np.ndarray:
    w = np.arange(1, n_ids + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def zipf_tokens(batch: int, T: int, n_ids: int = 50257, s: float = 1.1, seed: int = 0):
    """(tokens, targets) int32 [batch, T] from Zipf(s) streams of length T+1."""
    rng = np.random.default_rng(seed)
    u = rng.random((batch, T + 1))
    ids = np.searchsorted(zipf_cdf(n_ids, s), u, side="right")
    ids = np.minimum(ids, n_ids - 1).astype(np.int32)
    return np.ascontiguousarray(ids[:, :T]), np.ascontiguousarray(ids[:, 1:])


def uniform_tokens(batch: int, T: int, n_ids: int, seed: int = 0):
    """(tokens, targets) int32 [batch, T] from uniform streams of length T+1."""
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, n_ids, size=(batch, T + 1), dtype=np.int64).astype(np.int32)
    return np.ascontiguousarray(ids[:, :T]), np.ascontiguousarray(ids[:, 1:])


def normal_tensors(shapes, mean_std, seed: int = 0) -> dict:
    """Independent N(mean, std^2) fp64 arrays for each (name, shape).

    ``mean_std(name, shape)`` returns the (mean, std) pair for that tensor.
    """
    rng = np.random.default_rng(seed)
    out = {}
    for name, shape in shapes:
        mu, sd = mean_std(name, shape)
        out[name] = mu + sd * rng.standard_normal(shape)
    return out
