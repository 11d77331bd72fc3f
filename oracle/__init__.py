"""CPU oracle for the GPT-2 pretraining step (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it and shares no code with it.
"""
from .gpt2_oracle import (  # noqa: F401
    Config, param_shapes, param_count, flatten, unflatten, decay_mask,
    forward, backward, adamw_step, train_step, MatmulCounter,
    kv_cache_empty, decode_step, prefill, greedy_next,
)
from .flops import (  # noqa: F401
    n_params_total, n_params_matmul, flops_per_token, flops_per_token_matmul_only,
)
