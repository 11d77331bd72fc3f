"""Compute accounting for the bench (host logic, no model arithmetic).

"Pré-treinar um LLM: dados, compute, leis de escala e custo", compute section:
training costs 6 FLOPs per parameter per token (forward 2, backward 4), with
N counting every parameter including the embedding matrices; the Kaplan
Eq. (2.2) paragraph adds the attention-score term that 6N leaves out, counted
the way a matmul counter sees it (q k^T and P v unmasked, 4 T d per layer per
token forward, three times that for forward + backward).  MFU divides the
resulting FLOP rate by the GPU's dense bf16 peak.
"""
from __future__ import annotations


def param_count(n_layer: int, d: int, vocab: int, n_ctx: int) -> int:
    embeddings = (vocab + n_ctx) * d
    per_block = (4 * d * d + 4 * d) + (8 * d * d + 5 * d) + 4 * d   # attn, mlp, two LayerNorms
    return embeddings + n_layer * per_block + 2 * d


def train_flops_per_token(n_layer: int, d: int, vocab: int, n_ctx: int, T: int) -> int:
    """6 N + 12 L T d: the MFU numerator."""
    return 6 * param_count(n_layer, d, vocab, n_ctx) + 12 * n_layer * T * d


def matmul_flops_per_token(n_layer: int, d: int, vocab: int, T: int) -> int:
    """6 N_matmul + 12 L T d with N_matmul the parameters that enter a matmul
    (the twelve d^2 per block and the tied head; not wpe, biases or LayerNorm
    gains): what a FLOP counter sees, with the attention products unmasked."""
    return 6 * (n_layer * 12 * d * d + vocab * d) + 12 * n_layer * T * d


def executed_matmul_flops_per_token(n_layer: int, d: int, vocab: int, T: int) -> float:
    """FLOPs the kernels actually execute per token: every weight matmul three
    times (forward, input gradient, weight gradient) and the attention products
    with the causal half skipped (forward 2 products, backward 4 plus the
    recomputed scores = 5 products of 2 T d / 2 each per layer)."""
    weights = 6 * (n_layer * 12 * d * d + vocab * d)
    attn = n_layer * (2 + 5) * 2 * T * d / 2
    return weights + attn


def mfu(tokens_per_s: float, flops_per_token: float, peak_flops: float) -> float:
    return tokens_per_s * flops_per_token / peak_flops
