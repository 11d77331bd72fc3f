"""Python binding of libgpt2.so: one GPT-2 pretraining step on one B200.

Argument marshalling only.  Every step of the path runs in the library's
CUDA kernels; PyTorch provides device memory and streams.  The library is
loaded on first use; a RuntimeError is raised if it has not been built (``python -m decoder_only_transformer_step_b200.build_lib``):
there is no CPU fallback.

Functions named like the C entry points take torch tensors (device memory)
and ints/floats; ``GPT2`` bundles the buffers a context needs.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgpt2.so")

GPT2_OK = 0
ERRORS = {
    -1: "GPT2_ERR_INVALID_ARG", -2: "GPT2_ERR_UNSUPPORTED_SHAPE", -3: "GPT2_ERR_CUDA",
    -4: "GPT2_ERR_BAD_STATE", -5: "GPT2_ERR_TOKEN_RANGE", -6: "GPT2_ERR_NONFINITE",
    -7: "GPT2_ERR_TIMEOUT", -8: "GPT2_ERR_WORKSPACE", -9: "GPT2_ERR_TOO_LARGE",
    -10: "GPT2_ERR_POSITION_RANGE",
}
ERRORS_BY_NAME = {v: k for k, v in ERRORS.items()}


class Gpt2Error(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {ERRORS.get(code, code)} ({_lib().gpt2_strerror(code).decode()})")
        self.code = code


class gpt2_config(ctypes.Structure):
    _fields_ = [("n_layer", ctypes.c_int), ("d_model", ctypes.c_int), ("n_head", ctypes.c_int),
                ("n_ctx", ctypes.c_int), ("vocab_real", ctypes.c_int), ("vocab_padded", ctypes.c_int),
                ("max_batch", ctypes.c_int), ("mode", ctypes.c_int)]


class gpt2_buffers(ctypes.Structure):
    _fields_ = [("master", ctypes.c_void_p), ("shadow", ctypes.c_void_p), ("grad", ctypes.c_void_p),
                ("m", ctypes.c_void_p), ("v", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


EXPORTS = [
    "gpt2_param_count", "gpt2_workspace_bytes", "gpt2_tensor_info", "gpt2_create", "gpt2_destroy",
    "gpt2_init_params", "gpt2_refresh_shadow", "gpt2_forward_loss", "gpt2_backward",
    "gpt2_adamw_step", "gpt2_adamw_step_clip", "gpt2_adamw_step_range", "gpt2_grad_norm", "gpt2_zero_grad", "gpt2_get_status", "gpt2_step_host", "gpt2_strerror",
    "gpt2_kernel_launches",
    "gpt2_kv_cache_bytes", "gpt2_prefill", "gpt2_decode_step", "gpt2_greedy_next",
    "gpt2_op_gemm_bf16", "gpt2_op_attention_fwd_bf16", "gpt2_op_attention_bwd_bf16",
    "gpt2_op_attention_bwd_bf16_noalloc",
    "gpt2_op_layernorm_fwd_bf16", "gpt2_op_layernorm_bwd_scratch_floats", "gpt2_op_layernorm_bwd_bf16",
    "gpt2_op_colsum_scratch_floats", "gpt2_op_colsum_bf16",
    "gpt2_op_lm_head_ce_scratch_bytes", "gpt2_op_lm_head_ce_fwd_bf16", "gpt2_op_lm_head_ce_bwd_bf16",
    "gpt2_set_wait_timeout_ns", "gpt2_op_gemm_bf16_status", "gpt2_backward_bucketed",
    "gpt2_op_linear_bf16", "gpt2_graph_capture", "gpt2_graph_step", "gpt2_graph_release",
]

_LIB = None


def _lib():
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m decoder_only_transformer_step_b200.build_lib`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, S, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
    cfgp = ctypes.POINTER(gpt2_config)
    sig = {
        "gpt2_param_count": (S, [cfgp]),
        "gpt2_workspace_bytes": (S, [cfgp, I]),
        "gpt2_tensor_info": (I, [cfgp, I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(S),
                                 ctypes.POINTER(S), ctypes.POINTER(S)]),
        "gpt2_create": (I, [cfgp, ctypes.POINTER(gpt2_buffers), ctypes.POINTER(P)]),
        "gpt2_destroy": (I, [P]),
        "gpt2_init_params": (I, [P, U64, P]),
        "gpt2_refresh_shadow": (I, [P, P]),
        "gpt2_forward_loss": (I, [P, P, P, I, P, P]),
        "gpt2_backward": (I, [P, F, I, P]),
        "gpt2_adamw_step": (I, [P, F, F, F, F, F, I, P]),
        "gpt2_adamw_step_clip": (I, [P, F, F, F, F, F, I, F, P]),
        "gpt2_adamw_step_range": (I, [P, F, F, F, F, F, I, S, S, P]),
        "gpt2_grad_norm": (I, [P, P, P]),
        "gpt2_zero_grad": (I, [P, P]),
        "gpt2_get_status": (I, [P, P]),
        "gpt2_step_host": (I, [P, P, P, I, P, F, F, F, F, F, I, P]),
        "gpt2_strerror": (ctypes.c_char_p, [I]),
        "gpt2_kernel_launches": (ctypes.c_uint64, []),
        "gpt2_kv_cache_bytes": (S, [cfgp, I, I]),
        "gpt2_prefill": (I, [P, P, S, I, I, P, P, P, P]),
        "gpt2_decode_step": (I, [P, P, S, I, I, P, P, P, P]),
        "gpt2_greedy_next": (I, [P, P, I, P, P, P]),
        "gpt2_op_gemm_bf16": (I, [P, I, I, P, I, I, P, I, I, I, I, I, F, F, P, S, I, I, P]),
        "gpt2_op_attention_fwd_bf16": (I, [P, P, P, I, I, I, I, P]),
        "gpt2_op_attention_bwd_bf16": (I, [P, P, P, P, P, P, I, I, I, I, P]),
        "gpt2_op_attention_bwd_bf16_noalloc": (I, [P, P, P, P, P, I, I, I, I, P]),
        "gpt2_op_layernorm_fwd_bf16": (I, [P, P, P, P, P, P, I, I, P]),
        "gpt2_op_layernorm_bwd_scratch_floats": (S, [I, I]),
        "gpt2_op_layernorm_bwd_bf16": (I, [P, P, P, P, P, P, I, P, P, S, I, I, P]),
        "gpt2_op_colsum_scratch_floats": (S, [I, I]),
        "gpt2_op_colsum_bf16": (I, [P, I, I, P, P, S, P]),
        "gpt2_op_lm_head_ce_scratch_bytes": (S, [I, I]),
        "gpt2_op_lm_head_ce_fwd_bf16": (I, [P, P, P, I, I, I, I, P, P, P, S, P]),
        "gpt2_op_lm_head_ce_bwd_bf16": (I, [P, P, I, I, I, F, P, P, I, P, S, P]),
        "gpt2_set_wait_timeout_ns": (I, [U64]),
        "gpt2_backward_bucketed": (I, [P, F, I, P, I, P]),
        "gpt2_op_gemm_bf16_status": (I, [P, I, I, P, I, I, P, I, I, I, I, I, F, F, P, S, I, I, P, P]),
        "gpt2_op_linear_bf16": (I, [P, P, P, P, P, P, I, I, I, I, P]),
        "gpt2_graph_capture": (I, [P, I, F, I, P, P]),
        "gpt2_graph_step": (I, [P, P, P, P]),
        "gpt2_graph_release": (I, [P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = L
    return L


def _check(rc: int, where: str):
    if rc != GPT2_OK:
        raise Gpt2Error(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# --------------------------------------------------------------- C names ---

def make_config(n_layer, d_model, n_head, n_ctx, vocab_real, vocab_padded, max_batch, mode=0):
    return gpt2_config(n_layer, d_model, n_head, n_ctx, vocab_real, vocab_padded, max_batch, mode)


def gpt2_param_count(cfg: gpt2_config) -> int:
    return int(_lib().gpt2_param_count(ctypes.byref(cfg)))


def gpt2_workspace_bytes(cfg: gpt2_config, batch: int) -> int:
    return int(_lib().gpt2_workspace_bytes(ctypes.byref(cfg), batch))


def gpt2_tensor_info(cfg: gpt2_config, index: int):
    """(name, offset, rows, cols) or None past the last tensor."""
    name = ctypes.c_char_p()
    off, r, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    rc = _lib().gpt2_tensor_info(ctypes.byref(cfg), index, ctypes.byref(name), ctypes.byref(off),
                                 ctypes.byref(r), ctypes.byref(c))
    if rc != GPT2_OK:
        return None
    return name.value.decode(), off.value, r.value, c.value


def gpt2_tensors(cfg: gpt2_config):
    out, i = [], 0
    while True:
        t = gpt2_tensor_info(cfg, i)
        if t is None:
            return out
        out.append(t)
        i += 1


def gpt2_create(cfg, master, shadow, grad, m, v, workspace):
    bufs = gpt2_buffers(master.data_ptr(), shadow.data_ptr() if shadow is not None else None,
                        grad.data_ptr(), m.data_ptr(), v.data_ptr(), workspace.data_ptr(),
                        workspace.numel() * workspace.element_size())
    ctx = ctypes.c_void_p()
    _check(_lib().gpt2_create(ctypes.byref(cfg), ctypes.byref(bufs), ctypes.byref(ctx)), "gpt2_create")
    return ctx


def gpt2_destroy(ctx):
    _check(_lib().gpt2_destroy(ctx), "gpt2_destroy")


def gpt2_init_params(ctx, seed: int, stream=None):
    _check(_lib().gpt2_init_params(ctx, seed, _stream(stream)), "gpt2_init_params")


def gpt2_refresh_shadow(ctx, stream=None):
    _check(_lib().gpt2_refresh_shadow(ctx, _stream(stream)), "gpt2_refresh_shadow")


def gpt2_forward_loss(ctx, tokens, targets, batch: int, loss_dev, stream=None):
    _check(_lib().gpt2_forward_loss(ctx, _ptr(tokens), _ptr(targets), batch, _ptr(loss_dev),
                                    _stream(stream)), "gpt2_forward_loss")


def gpt2_backward(ctx, grad_scale: float = 1.0, accumulate: int = 0, stream=None):
    _check(_lib().gpt2_backward(ctx, grad_scale, accumulate, _stream(stream)), "gpt2_backward")


def gpt2_backward_bucketed(ctx, grad_scale, accumulate, events, stream=None):
    """events: torch.cuda.Event objects (already created, e.g. recorded once),
    n_layer + 2 of them."""
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(_lib().gpt2_backward_bucketed(ctx, grad_scale, accumulate, arr, len(events), _stream(stream)),
           "gpt2_backward_bucketed")


def gpt2_graph_capture(ctx, batch, grad_scale, accumulate, loss_dev, stream):
    """Records forward + loss + backward into the context's graph; `stream` is
    a torch.cuda.Stream the caller created (not the default stream)."""
    _check(_lib().gpt2_graph_capture(ctx, batch, grad_scale, accumulate, _ptr(loss_dev), _stream(stream)),
           "gpt2_graph_capture")


def gpt2_graph_step(ctx, tokens, targets, stream=None):
    _check(_lib().gpt2_graph_step(ctx, _ptr(tokens), _ptr(targets), _stream(stream)), "gpt2_graph_step")


def gpt2_graph_release(ctx):
    _check(_lib().gpt2_graph_release(ctx), "gpt2_graph_release")


def gpt2_adamw_step(ctx, lr, beta1, beta2, eps, weight_decay, step, stream=None):
    _check(_lib().gpt2_adamw_step(ctx, lr, beta1, beta2, eps, weight_decay, step, _stream(stream)),
           "gpt2_adamw_step")


def gpt2_adamw_step_clip(ctx, lr, beta1, beta2, eps, weight_decay, step, max_norm, stream=None):
    _check(_lib().gpt2_adamw_step_clip(ctx, lr, beta1, beta2, eps, weight_decay, step, max_norm,
                                       _stream(stream)), "gpt2_adamw_step_clip")


def gpt2_adamw_step_range(ctx, lr, beta1, beta2, eps, weight_decay, step, offset, count, stream=None):
    _check(_lib().gpt2_adamw_step_range(ctx, lr, beta1, beta2, eps, weight_decay, step, offset, count,
                                        _stream(stream)), "gpt2_adamw_step_range")


def gpt2_grad_norm(ctx, norm_dev=None, stream=None):
    _check(_lib().gpt2_grad_norm(ctx, _ptr(norm_dev), _stream(stream)), "gpt2_grad_norm")


def gpt2_zero_grad(ctx, stream=None):
    _check(_lib().gpt2_zero_grad(ctx, _stream(stream)), "gpt2_zero_grad")


def gpt2_get_status(ctx, stream=None) -> int:
    return int(_lib().gpt2_get_status(ctx, _stream(stream)))


def gpt2_step_host(ctx, tokens_host, targets_host, batch, loss_host, lr, beta1, beta2, eps,
                   weight_decay, step, stream=None):
    """tokens_host/targets_host/loss_host: CPU (ideally pinned) torch tensors."""
    _check(_lib().gpt2_step_host(ctx, _ptr(tokens_host), _ptr(targets_host), batch, _ptr(loss_host),
                                 lr, beta1, beta2, eps, weight_decay, step, _stream(stream)),
           "gpt2_step_host")


def gpt2_kernel_launches() -> int:
    return int(_lib().gpt2_kernel_launches())


def gpt2_kv_cache_bytes(cfg: gpt2_config, batch: int, max_len: int) -> int:
    return int(_lib().gpt2_kv_cache_bytes(ctypes.byref(cfg), batch, max_len))


def _nbytes(t):
    return t.numel() * t.element_size()


def gpt2_prefill(ctx, cache, batch, max_len, tokens, prompt_len, logits, stream=None):
    """cache: a device tensor of at least gpt2_kv_cache_bytes(cfg, batch, max_len) bytes."""
    _check(_lib().gpt2_prefill(ctx, _ptr(cache), _nbytes(cache), batch, max_len, _ptr(tokens), _ptr(prompt_len),
                               _ptr(logits), _stream(stream)), "gpt2_prefill")


def gpt2_decode_step(ctx, cache, batch, max_len, tokens, pos, logits, stream=None):
    """cache: a device tensor of at least gpt2_kv_cache_bytes(cfg, batch, max_len) bytes."""
    _check(_lib().gpt2_decode_step(ctx, _ptr(cache), _nbytes(cache), batch, max_len, _ptr(tokens), _ptr(pos),
                                   _ptr(logits), _stream(stream)), "gpt2_decode_step")


def gpt2_greedy_next(ctx, logits, batch, next_tokens, pos=None, stream=None):
    _check(_lib().gpt2_greedy_next(ctx, _ptr(logits), batch, _ptr(next_tokens), _ptr(pos), _stream(stream)),
           "gpt2_greedy_next")


def gpt2_op_gemm_bf16(A, a_mn_major, lda, B, b_mn_major, ldb, C, c_fp32, ldc, M, N, K,
                      alpha=1.0, beta=0.0, workspace=None, bn=0, splits=0, stream=None):
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().gpt2_op_gemm_bf16(_ptr(A), a_mn_major, lda, _ptr(B), b_mn_major, ldb, _ptr(C), c_fp32,
                                    ldc, M, N, K, alpha, beta, _ptr(workspace), wsb, bn, splits,
                                    _stream(stream)), "gpt2_op_gemm_bf16")


def gpt2_op_attention_fwd_bf16(qkv, o, lse, B, T, H, hd, stream=None):
    _check(_lib().gpt2_op_attention_fwd_bf16(_ptr(qkv), _ptr(o), _ptr(lse), B, T, H, hd,
                                             _stream(stream)), "gpt2_op_attention_fwd_bf16")


def gpt2_op_attention_bwd_bf16(qkv, o, lse, dout, dqkv, scratch, B, T, H, hd, stream=None):
    _check(_lib().gpt2_op_attention_bwd_bf16(_ptr(qkv), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dqkv),
                                             _ptr(scratch), B, T, H, hd, _stream(stream)),
           "gpt2_op_attention_bwd_bf16")


def gpt2_op_attention_bwd_bf16_noalloc(qkv, o, lse, dout, dqkv, B, T, H, hd, stream=None):
    """Allocation-free attention backward: scratch lives in the library (see
    include/gpt2.h); for callers that cannot allocate device memory."""
    _check(_lib().gpt2_op_attention_bwd_bf16_noalloc(_ptr(qkv), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dqkv),
                                                     B, T, H, hd, _stream(stream)),
           "gpt2_op_attention_bwd_bf16_noalloc")


def gpt2_op_layernorm_fwd_bf16(x, gamma, beta, y, mean, rstd, M, d, stream=None):
    _check(_lib().gpt2_op_layernorm_fwd_bf16(_ptr(x), _ptr(gamma), _ptr(beta), _ptr(y), _ptr(mean), _ptr(rstd),
                                             M, d, _stream(stream)), "gpt2_op_layernorm_fwd_bf16")


def gpt2_op_linear_bf16(x, w, bias, resid, out, out2, M, N, K, act, stream=None):
    """act 0: out = x w^T + bias; 1: + resid; 2: out = GELU(u), out2 = GELU'(u)."""
    _check(_lib().gpt2_op_linear_bf16(_ptr(x), _ptr(w), _ptr(bias), _ptr(resid), _ptr(out), _ptr(out2), M, N, K,
                                      act, _stream(stream)), "gpt2_op_linear_bf16")


def gpt2_op_layernorm_bwd_scratch_floats(M, d) -> int:
    return int(_lib().gpt2_op_layernorm_bwd_scratch_floats(M, d))


def gpt2_op_layernorm_bwd_bf16(dy, x, mean, rstd, gamma, dx, accumulate, dgamma_dbeta, scratch, M, d, stream=None):
    _check(_lib().gpt2_op_layernorm_bwd_bf16(_ptr(dy), _ptr(x), _ptr(mean), _ptr(rstd), _ptr(gamma), _ptr(dx),
                                             accumulate, _ptr(dgamma_dbeta), _ptr(scratch), scratch.numel(), M, d,
                                             _stream(stream)), "gpt2_op_layernorm_bwd_bf16")


def gpt2_op_colsum_scratch_floats(M, N) -> int:
    return int(_lib().gpt2_op_colsum_scratch_floats(M, N))


def gpt2_op_colsum_bf16(x, M, N, out, scratch, stream=None):
    _check(_lib().gpt2_op_colsum_bf16(_ptr(x), M, N, _ptr(out), _ptr(scratch), scratch.numel(), _stream(stream)),
           "gpt2_op_colsum_bf16")


def gpt2_op_lm_head_ce_scratch_bytes(M, V) -> int:
    return int(_lib().gpt2_op_lm_head_ce_scratch_bytes(M, V))


def gpt2_op_lm_head_ce_fwd_bf16(x, w, targets, M, V, d, vocab_real, loss, loss_rows, scratch, stream=None):
    _check(_lib().gpt2_op_lm_head_ce_fwd_bf16(_ptr(x), _ptr(w), _ptr(targets), M, V, d, vocab_real, _ptr(loss),
                                              _ptr(loss_rows), _ptr(scratch), scratch.numel() * scratch.element_size(),
                                              _stream(stream)), "gpt2_op_lm_head_ce_fwd_bf16")


def gpt2_op_lm_head_ce_bwd_bf16(x, w, M, V, d, grad_scale, dx, dw, accumulate, scratch, stream=None):
    _check(_lib().gpt2_op_lm_head_ce_bwd_bf16(_ptr(x), _ptr(w), M, V, d, grad_scale, _ptr(dx), _ptr(dw), accumulate,
                                              _ptr(scratch), scratch.numel() * scratch.element_size(),
                                              _stream(stream)), "gpt2_op_lm_head_ce_bwd_bf16")


def gpt2_set_wait_timeout_ns(ns: int):
    _check(_lib().gpt2_set_wait_timeout_ns(ns), "gpt2_set_wait_timeout_ns")


def gpt2_op_gemm_bf16_status(A, a_mn, lda, B, b_mn, ldb, C, c_fp32, ldc, M, N, K, alpha=1.0, beta=0.0,
                             workspace=None, bn=0, splits=0, status=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().gpt2_op_gemm_bf16_status(_ptr(A), a_mn, lda, _ptr(B), b_mn, ldb, _ptr(C), c_fp32, ldc, M, N, K,
                                           alpha, beta, _ptr(workspace), ws_bytes, bn, splits, _ptr(status),
                                           _stream(stream)), "gpt2_op_gemm_bf16_status")


# ------------------------------------------------------------ convenience ---

@dataclass(frozen=True)
class ModelConfig:
    n_layer: int
    d_model: int
    n_head: int
    n_ctx: int
    vocab_real: int
    vocab_padded: int
    max_batch: int
    mode: int = 0  # 0 bf16 tensor cores, 1 fp32 correctness mode, 2 bf16 bitwise repeatable

    def c(self) -> gpt2_config:
        return make_config(self.n_layer, self.d_model, self.n_head, self.n_ctx, self.vocab_real,
                           self.vocab_padded, self.max_batch, self.mode)


GPT2_124M = ModelConfig(12, 768, 12, 1024, 50257, 50304, 16)
GPT2_350M = ModelConfig(24, 1024, 16, 1024, 50257, 50304, 16)
GPT2_1558M = ModelConfig(48, 1600, 25, 1024, 50257, 50304, 8)
GPT2_124M_T4096 = ModelConfig(12, 768, 12, 4096, 50257, 50304, 4)
GPT2_TINY = ModelConfig(2, 64, 4, 64, 512, 512, 4, mode=1)


class GPT2:
    """A context plus the torch-owned device buffers it runs on."""

    def __init__(self, mc: ModelConfig, device="cuda"):
        import torch
        self.mc = mc
        self.cfg = mc.c()
        n = gpt2_param_count(self.cfg)
        if n == 0:
            raise ValueError(f"invalid config {mc}")
        self.n_params = n
        f32 = dict(dtype=torch.float32, device=device)
        self.master = torch.zeros(n, **f32)
        self.grad = torch.zeros(n, **f32)
        self.m = torch.zeros(n, **f32)
        self.v = torch.zeros(n, **f32)
        self.shadow = torch.zeros(n, dtype=torch.bfloat16, device=device)
        wsb = gpt2_workspace_bytes(self.cfg, mc.max_batch)
        self.workspace = torch.empty(wsb, dtype=torch.uint8, device=device)
        self.loss = torch.zeros(1, **f32)
        self.ctx = gpt2_create(self.cfg, self.master, self.shadow, self.grad, self.m, self.v, self.workspace)
        self.layout = gpt2_tensors(self.cfg)

    def close(self):
        if self.ctx is not None:
            gpt2_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def view(self, flat, name):
        """View of one named tensor inside a flat buffer (master, grad, m, v)."""
        for nm, off, r, c in self.layout:
            if nm == name:
                t = flat[off:off + r * c]
                return t.view(r, c) if c > 1 else t
        raise KeyError(name)

    def init_params(self, seed=0):
        gpt2_init_params(self.ctx, seed)

    def refresh_shadow(self):
        gpt2_refresh_shadow(self.ctx)

    def forward_loss(self, tokens, targets):
        gpt2_forward_loss(self.ctx, tokens, targets, tokens.shape[0], self.loss)
        return self.loss

    def backward(self, grad_scale=1.0, accumulate=0):
        gpt2_backward(self.ctx, grad_scale, accumulate)

    def graph_capture(self, batch, grad_scale=1.0, accumulate=0, stream=None):
        """Record forward + loss + backward of one micro-batch into the
        context's CUDA graph (after at least one eager step).  The capture runs
        on a side stream of its own unless one is given."""
        import torch
        s = stream if stream is not None else torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        gpt2_graph_capture(self.ctx, batch, grad_scale, accumulate, self.loss, s)
        torch.cuda.current_stream().wait_stream(s)

    def graph_step(self, tokens, targets):
        """One captured micro-step on the current stream: the ids are copied in,
        then the graph runs (as forward_loss + backward)."""
        gpt2_graph_step(self.ctx, tokens, targets)

    def backward_bucketed(self, events, grad_scale=1.0, accumulate=0):
        """The backward recording events[i] when bucket i's gradients are
        final (see gpt2_backward_bucketed; n_layer + 2 events)."""
        gpt2_backward_bucketed(self.ctx, grad_scale, accumulate, events)

    def adamw_step(self, step, lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, max_norm=0.0):
        """AdamW over the flat buffer; max_norm > 0 clips the gradient to that
        global norm first (on the device)."""
        if max_norm > 0.0:
            gpt2_adamw_step_clip(self.ctx, lr, beta1, beta2, eps, weight_decay, step, max_norm)
        else:
            gpt2_adamw_step(self.ctx, lr, beta1, beta2, eps, weight_decay, step)

    def adamw_step_range(self, step, offset, count, lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1):
        """AdamW on elements [offset, offset + count) only (one shard of the
        optimizer state)."""
        gpt2_adamw_step_range(self.ctx, lr, beta1, beta2, eps, weight_decay, step, offset, count)

    def grad_norm(self):
        """Global L2 norm of the gradient buffer as a device fp32 scalar tensor."""
        import torch
        out = torch.empty(1, dtype=torch.float32, device=self.grad.device)
        gpt2_grad_norm(self.ctx, out)
        return out

    def zero_grad(self):
        gpt2_zero_grad(self.ctx)

    def status(self) -> int:
        return gpt2_get_status(self.ctx)

    def step_host(self, tokens_host, targets_host, loss_host, step, lr=6e-4, beta1=0.9, beta2=0.95,
                  eps=1e-8, weight_decay=0.1):
        gpt2_step_host(self.ctx, tokens_host, targets_host, tokens_host.shape[0], loss_host, lr, beta1,
                       beta2, eps, weight_decay, step)


class KVCache:
    """Key/value cache of one GPT2 context for ``batch`` sequences of up to
    ``max_len`` positions, with the device-side token, position and logits
    buffers a decode loop runs on (so the loop can be captured in a CUDA
    graph)."""

    def __init__(self, model: "GPT2", batch: int, max_len: int):
        import torch
        nbytes = gpt2_kv_cache_bytes(model.cfg, batch, max_len)
        if nbytes == 0:
            raise ValueError(f"invalid cache size batch={batch} max_len={max_len}")
        dev = model.master.device
        self.model, self.batch, self.max_len = model, batch, max_len
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.tokens = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.pos = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.logits = torch.zeros(batch, model.cfg.vocab_padded, dtype=torch.float32, device=dev)

    def prefill(self, tokens, prompt_len):
        """tokens: int32 [batch, n_ctx] (device); prompt_len: int32 [batch]
        (device).  Leaves the logits after each prompt in self.logits, the
        greedy next id in self.tokens and self.pos = prompt_len."""
        gpt2_prefill(self.model.ctx, self.buf, self.batch, self.max_len, tokens, prompt_len, self.logits)
        self.pos.copy_(prompt_len)
        gpt2_greedy_next(self.model.ctx, self.logits, self.batch, self.tokens)
        return self.logits

    def step(self, tokens=None, pos=None):
        """One decode step on self.tokens / self.pos (or the given device
        tensors); returns the logits [batch, vocab_padded]."""
        gpt2_decode_step(self.model.ctx, self.buf, self.batch, self.max_len,
                         self.tokens if tokens is None else tokens, self.pos if pos is None else pos, self.logits)
        return self.logits

    def greedy_advance(self):
        """self.tokens = greedy choice from self.logits; self.pos += 1."""
        gpt2_greedy_next(self.model.ctx, self.logits, self.batch, self.tokens, self.pos)
