"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/gpt2.h declares, and its host-side logic (parameter layout,
workspace sizing, argument validation) agrees with the specification the
oracle implements independently."""
import ctypes
import os
import re

import pytest

import decoder_only_transformer_step_b200 as gp
from decoder_only_transformer_step_b200 import build_lib
import oracle
from oracle import flops as FL
from oracle_fixtures import TINY, GPT2_124M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()


def header_functions():
    src = open(os.path.join(ROOT, "include", "gpt2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt2_\w+)\s*\(", src)))


def test_exports_every_declared_symbol():
    lib = ctypes.CDLL(gp.LIB_PATH)
    declared = header_functions()
    assert len(declared) >= 17
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(gp.EXPORTS) == declared


def _cfg(oc, max_batch=4, vocab_real=None, mode=0):
    return gp.make_config(oc.n_layer, oc.d_model, oc.n_head, oc.n_ctx,
                          vocab_real or oc.vocab, oc.vocab, max_batch, mode)


@pytest.mark.parametrize("oc", [TINY, GPT2_124M])
def test_layout_matches_oracle_spec(oc):
    cfg = _cfg(oc)
    assert gp.gpt2_param_count(cfg) == oracle.param_count(oc)
    lib_tensors = gp.gpt2_tensors(cfg)
    off = 0
    shapes = oracle.param_shapes(oc)
    assert len(lib_tensors) == len(shapes)
    for (name, o, r, c), (oname, oshape) in zip(lib_tensors, shapes):
        assert name == oname
        assert o == off
        assert (r, c) == (oshape + (1,) if len(oshape) == 1 else oshape)
        off += r * c
        assert o % 8 == 0  # every tensor starts 16-byte aligned in the bf16 shadow


def test_param_counts_of_named_configs():
    for mc, n in [(gp.GPT2_124M, 124_475_904), (gp.GPT2_1558M, 1_557_686_400)]:
        assert gp.gpt2_param_count(mc.c()) == n
        assert n == FL.n_params_total(mc.n_layer, mc.d_model, mc.vocab_padded, mc.n_ctx)


def test_workspace_fits_b200():
    for mc in (gp.GPT2_124M, gp.GPT2_350M, gp.GPT2_1558M, gp.GPT2_124M_T4096):
        ws = gp.gpt2_workspace_bytes(mc.c(), mc.max_batch)
        n = gp.gpt2_param_count(mc.c())
        total = ws + n * (4 * 4 + 2)
        assert 0 < total < 170e9, (mc, total / 1e9)
    assert gp.gpt2_workspace_bytes(gp.GPT2_124M.c(), 2) < gp.gpt2_workspace_bytes(gp.GPT2_124M.c(), 16)


def test_invalid_configs_are_rejected_on_host():
    bad = gp.make_config(2, 64, 3, 64, 512, 512, 4, 0)      # d % heads
    assert gp.gpt2_param_count(bad) == 0
    assert gp.gpt2_workspace_bytes(bad, 4) == 0
    lib = gp._lib()
    ctx = ctypes.c_void_p()
    bufs = gp.gpt2_buffers()
    cfg = gp.make_config(2, 64, 4, 64, 512, 512, 4, 0)
    # NULL buffers
    assert lib.gpt2_create(ctypes.byref(cfg), ctypes.byref(bufs), ctypes.byref(ctx)) == -1
    # d not a multiple of 64 / head_dim unsupported / vocab not a multiple of 128
    for c in (gp.make_config(2, 96, 4, 64, 512, 512, 4, 0), gp.make_config(2, 128, 4, 64, 512, 512, 4, 0),
              gp.make_config(2, 64, 4, 64, 500, 500, 4, 0)):
        fake = gp.gpt2_buffers(16, 16, 16, 16, 16, 16, 1 << 40)
        assert lib.gpt2_create(ctypes.byref(c), ctypes.byref(fake), ctypes.byref(ctx)) == -2
    # misaligned pointer
    fake = gp.gpt2_buffers(16, 16, 24, 16, 16, 16, 1 << 40)
    assert lib.gpt2_create(ctypes.byref(cfg), ctypes.byref(fake), ctypes.byref(ctx)) == -1
    # workspace too small
    fake = gp.gpt2_buffers(16, 16, 16, 16, 16, 16, 1024)
    assert lib.gpt2_create(ctypes.byref(cfg), ctypes.byref(fake), ctypes.byref(ctx)) == -8
    assert lib.gpt2_backward(None, ctypes.c_float(1.0), 0, None) == -1
    assert lib.gpt2_strerror(-5) == b"token or target id out of range"


def test_kv_cache_bytes_layout():
    # K and V planes [batch][H][max_len][hd] of every layer (bf16 in mode 0,
    # fp32 in mode 1, each padded to 256 bytes) plus four fp32 row buffers
    c = gp.GPT2_124M.c()
    planes = 2 * 12 * 8 * 12 * 1024 * 64 * 2
    scratch = 3 * 8 * 768 * 4 + 8 * 3072 * 4
    assert gp.gpt2_kv_cache_bytes(c, 8, 1024) == planes + scratch
    c1 = gp.GPT2_TINY.c()
    assert gp.gpt2_kv_cache_bytes(c1, 1, 5) == 2 * 2 * (4 * 5 * 16 * 4) + 3 * 64 * 4 + 256 * 4
    for b, n in [(0, 8), (17, 8), (4, 0), (4, 1025)]:
        assert gp.gpt2_kv_cache_bytes(c, b, n) == 0


def test_null_context_calls_are_rejected_on_host():
    # every entry point validates its context and pointers before touching the
    # device, so these return GPT2_ERR_INVALID_ARG without a GPU
    L = gp._lib()
    bad = gp.ERRORS_BY_NAME["GPT2_ERR_INVALID_ARG"]
    assert L.gpt2_forward_loss(None, None, None, 1, None, None) == bad
    assert L.gpt2_backward(None, 1.0, 0, None) == bad
    assert L.gpt2_adamw_step(None, 6e-4, 0.9, 0.95, 1e-8, 0.1, 1, None) == bad
    assert L.gpt2_adamw_step_clip(None, 6e-4, 0.9, 0.95, 1e-8, 0.1, 1, 1.0, None) == bad
    assert L.gpt2_adamw_step_range(None, 6e-4, 0.9, 0.95, 1e-8, 0.1, 1, 0, 4, None) == bad
    assert L.gpt2_grad_norm(None, None, None) == bad
    assert L.gpt2_zero_grad(None, None) == bad
    assert L.gpt2_get_status(None, None) == bad
    assert L.gpt2_prefill(None, None, 0, 1, 1, None, None, None, None) == bad
    assert L.gpt2_decode_step(None, None, 0, 1, 1, None, None, None, None) == bad
    assert L.gpt2_greedy_next(None, None, 1, None, None, None) == bad


def test_noalloc_attention_backward_validates_shape_before_scratch_size():
    # a head size below 1 is an invalid argument and an unsupported head size
    # an unsupported shape, as for the scratch-taking call, even where the
    # problem would also exceed the built-in scratch; all decided on the host
    # before any CUDA call (dummy, never-dereferenced pointers)
    L = gp._lib()
    p = ctypes.c_void_p(256)
    inv = gp.ERRORS_BY_NAME["GPT2_ERR_INVALID_ARG"]
    uns = gp.ERRORS_BY_NAME["GPT2_ERR_UNSUPPORTED_SHAPE"]
    assert L.gpt2_op_attention_bwd_bf16_noalloc(p, p, p, p, p, 64, 1024, 12, -1, None) == inv
    assert L.gpt2_op_attention_bwd_bf16_noalloc(p, p, p, p, p, 64, 1024, 12, 0, None) == inv
    assert L.gpt2_op_attention_bwd_bf16_noalloc(p, p, p, p, p, 64, 1024, 12, 32, None) == uns
    assert L.gpt2_op_attention_bwd_bf16_noalloc(p, p, p, p, p, 1, 64, 2, 128, None) == uns
    assert L.gpt2_op_attention_bwd_bf16_noalloc(None, p, p, p, p, 1, 64, 2, 64, None) == inv
    # a supported shape just past the 4 Mi-float array
    assert L.gpt2_op_attention_bwd_bf16_noalloc(p, p, p, p, p, 1, 4096, 16, 64, None) == \
        gp.ERRORS_BY_NAME["GPT2_ERR_TOO_LARGE"]


def test_lm_head_cross_entropy_ops_validate_on_host():
    # scratch sizing and shape rules of the fused LM-head cross-entropy ops,
    # decided on the host before any CUDA call
    L = gp._lib()
    assert gp.gpt2_op_lm_head_ce_scratch_bytes(1024, 1000) == 0           # V not a multiple of 128
    n = gp.gpt2_op_lm_head_ce_scratch_bytes(1024, 1024)
    # status words, the bf16 [M, V] exponentials / dz, two [V/128, M] fp32 part arrays, the [M] target logits
    assert n >= 1024 * 1024 * 2 + 2 * 8 * 1024 * 4 + 1024 * 4
    p = ctypes.c_void_p(4096)
    uns = gp.ERRORS_BY_NAME["GPT2_ERR_UNSUPPORTED_SHAPE"]
    assert L.gpt2_op_lm_head_ce_fwd_bf16(p, p, p, 64, 1000, 64, 1000, p, p, p, 1 << 30, None) == uns
    assert L.gpt2_op_lm_head_ce_fwd_bf16(p, p, p, 64, 1024, 96, 1000, p, p, p, 1 << 30, None) == uns
    assert L.gpt2_op_lm_head_ce_fwd_bf16(p, p, p, 64, 1024, 64, 1000, p, p, p, 16, None) == \
        gp.ERRORS_BY_NAME["GPT2_ERR_WORKSPACE"]
    assert L.gpt2_op_lm_head_ce_bwd_bf16(None, p, 64, 1024, 64, 1.0, p, p, 0, p, 1 << 30, None) == \
        gp.ERRORS_BY_NAME["GPT2_ERR_INVALID_ARG"]


def test_status_gemm_validates_on_host():
    # the status-word GEMM rejects a missing or misaligned status pointer
    # before any CUDA call
    L = gp._lib()
    p = ctypes.c_void_p(4096)
    inv = gp.ERRORS_BY_NAME["GPT2_ERR_INVALID_ARG"]
    assert L.gpt2_op_gemm_bf16_status(p, 0, 64, p, 0, 64, p, 0, 64, 64, 64, 64, 1.0, 0.0, None, 0, 0, 0, None,
                                      None) == inv
    assert L.gpt2_op_gemm_bf16_status(p, 0, 64, p, 0, 64, p, 0, 64, 64, 64, 64, 1.0, 0.0, None, 0, 0, 0,
                                      ctypes.c_void_p(4098), None) == inv


def test_linear_op_validates_on_host():
    # argument and shape rules of the fused linear-layer op, decided on the
    # host before any CUDA call
    L = gp._lib()
    p = ctypes.c_void_p(4096)
    inv = gp.ERRORS_BY_NAME["GPT2_ERR_INVALID_ARG"]
    uns = gp.ERRORS_BY_NAME["GPT2_ERR_UNSUPPORTED_SHAPE"]
    assert L.gpt2_op_linear_bf16(p, p, p, None, p, None, 64, 64, 64, 3, None) == inv    # act out of range
    assert L.gpt2_op_linear_bf16(p, p, p, None, p, None, 64, 64, 64, 1, None) == inv    # act 1 needs resid
    assert L.gpt2_op_linear_bf16(p, p, p, None, p, None, 64, 64, 64, 2, None) == inv    # act 2 needs out2
    assert L.gpt2_op_linear_bf16(p, p, p, None, ctypes.c_void_p(4104), None, 64, 64, 64, 0, None) == inv
    assert L.gpt2_op_linear_bf16(p, p, None, None, p, None, 64, 64, 64, 0, None) == inv
    assert L.gpt2_op_linear_bf16(p, p, p, None, p, None, 64, 64, 96, 0, None) == uns    # K % 64
    assert L.gpt2_op_linear_bf16(p, p, p, None, p, None, 64, 60, 64, 0, None) == uns    # N % 8
    assert L.gpt2_op_linear_bf16(p, p, p, None, p, None, 0, 64, 64, 0, None) == 0       # empty: nothing to do
