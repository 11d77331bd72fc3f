"""Shared helpers for the tests: configs and seeded parameter sets.

The standard deviations used here are test inputs, not model arithmetic.
"""
import math

from oracle import Config, param_shapes
from decoder_only_transformer_step_b200 import inputs

TINY = Config(n_layer=2, d_model=64, n_head=4, n_ctx=64, vocab=512)
SMALL_124M_L2 = Config(n_layer=2, d_model=768, n_head=12, n_ctx=1024, vocab=50304)
GPT2_124M = Config(n_layer=12, d_model=768, n_head=12, n_ctx=1024, vocab=50304)


def gpt2_init_std(cfg):
    """GPT-2 initialisation: N(0, 0.02) weights, residual projections scaled by
    1/sqrt(2L), zero biases, LayerNorm gain 1 and shift 0."""
    def f(name, shape):
        t = name.split(".")[-1]
        if t in ("w_o", "w_mp"):
            return 0.0, 0.02 / math.sqrt(2 * cfg.n_layer)
        if t.startswith("ln") and t.endswith("_g") or name == "lnf_g":
            return 1.0, 0.0
        if len(shape) == 1:
            return 0.0, 0.0
        return 0.0, 0.02
    return f


def perturbed_std(cfg):
    """Like the GPT-2 init but with non-trivial gains, shifts and biases so that
    every gradient path carries signal."""
    base = gpt2_init_std(cfg)

    def f(name, shape):
        t = name.split(".")[-1]
        if t.endswith("_g"):
            return 1.0, 0.1
        if len(shape) == 1:
            return 0.0, 0.02
        return base(name, shape)
    return f


def params_for(cfg, seed=0, kind="perturbed"):
    fn = perturbed_std(cfg) if kind == "perturbed" else gpt2_init_std(cfg)
    return inputs.normal_tensors(param_shapes(cfg), fn, seed=seed)
