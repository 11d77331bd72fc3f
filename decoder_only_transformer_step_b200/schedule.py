"""Learning-rate schedule for the training loop around the step (host side).

"Pré-treinar um LLM" (Chinchilla section): the cosine schedule must match the
token budget, decaying to its floor exactly when the planned tokens have been
seen.  `lr_at` is that schedule with an optional linear warm-up (the pages give
none; warmup_steps = 0 reproduces the plain cosine).

    step < warmup:            max_lr * (step + 1) / warmup
    warmup <= step < total:   min_lr + (max_lr - min_lr) * (1 + cos(pi * (step - warmup) / (total - warmup))) / 2
    step >= total:            min_lr

`total_steps` is the optimizer-step count the token budget allows:
budget_tokens / (micro_batch * seq_len * accumulation).
"""
from __future__ import annotations

import math


def steps_for_budget(budget_tokens: int, micro_batch: int, seq_len: int, accumulation: int = 1) -> int:
    """Optimizer steps that consume `budget_tokens` (rounded down, at least 1)."""
    per_step = micro_batch * seq_len * accumulation
    return max(1, budget_tokens // per_step)


def lr_at(step: int, max_lr: float, total_steps: int, warmup_steps: int = 0, min_lr: float = 0.0) -> float:
    """Learning rate of optimizer step `step` (0-based)."""
    if total_steps <= 0:
        raise ValueError("total_steps must be positive")
    if warmup_steps < 0 or warmup_steps >= total_steps:
        raise ValueError("need 0 <= warmup_steps < total_steps")
    if step < warmup_steps:
        return max_lr * (step + 1) / warmup_steps
    if step >= total_steps:
        return min_lr
    frac = (step - warmup_steps) / (total_steps - warmup_steps)
    return min_lr + (max_lr - min_lr) * 0.5 * (1.0 + math.cos(math.pi * frac))
