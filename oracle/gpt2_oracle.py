"""Plain, slow fp64 CPU oracle of one GPT-2 pretraining step.

TEST INFRASTRUCTURE.  This module is the reference that the CUDA path is
checked against.  Only tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it; it shares no code with the CUDA library.

What it computes, and where it comes from (web pages, cited by title and
section):

* "Pré-treinar um LLM: dados, compute, leis de escala e custo" (neuralialabs),
  opening section: the objective is next-token prediction -- the label for
  position t is the token at t+1 -- the loss is cross-entropy and the
  optimiser is AdamW.
* same page, compute section (the 6ND derivation): every weight matrix is used
  once per token in the forward (2 FLOPs per parameter) and the backward
  computes two matmul-sized gradients per layer, one with respect to the
  layer input and one with respect to its weights (4N).  ``backward`` below
  has exactly that shape: each forward matmul has one input-gradient and one
  weight-gradient matmul of the same size.
* same page, memory section: fp32 weights, gradients and the two AdamW
  moments m and v (16 bytes per parameter).
* "Criei GPT-2 do zero com uma RTX 4090" (yasue.org), section "Configuração do
  treinamento": GPT-2 small (12 layers, 768 dims), vocabulary rounded up from
  50257 to 50304 (a multiple of 128); section "Resultado": the softmax at
  initialisation is close to uniform over all 50304 ids (ln 50304 = 10.83), so
  the padded ids take part in the softmax.

The block structure (pre-LayerNorm, learned positions, causal multi-head
attention, GELU MLP, LM head tied to the token embedding) is the GPT-2 model
the pages train.  Where the pages are silent this oracle takes the plainest
GPT-2 reading: tanh-form GELU, LayerNorm eps 1e-5 with biased variance,
biases on every linear layer except the tied head, no dropout, softmax scale
1/sqrt(head_dim), loss averaged over all B*T positions (over those with a
target when some targets are -1, the masked loss below), weight decay on 2-D
tensors only, AdamW with bias correction and eps 1e-8, no gradient clipping
(an optional global-norm clip is provided for the training loop around the
step; it is off unless asked for).  The end of the module holds the
incremental decoder with a key/value cache (decode step, prefill, greedy
choice), pinned to the full forward.

Pins (tests/test_oracle_*.py): central finite differences in fp64 for every
parameter tensor, an independent PyTorch autograd witness built from library
routines (F.layer_norm, scaled_dot_product_attention, F.gelu(tanh),
F.cross_entropy, torch.optim.AdamW), causal invariance, the tied-embedding
decomposition, closed forms (initial loss, uniform-key attention, constant-row
LayerNorm, zero-logit cross-entropy, AdamW step 1) and the FLOP identities of
the compute section.  Every function here is pinned; none is "parity
unpinned".

Flat parameter layout (shared *specification*, implemented independently on
each side): wte[V,d], wpe[n_ctx,d], then per layer ln1_g[d], ln1_b[d],
w_qkv[3d,d], b_qkv[3d], w_o[d,d], b_o[d], ln2_g[d], ln2_b[d], w_fc[4d,d],
b_fc[4d], w_mp[d,4d], b_mp[d], and finally lnf_g[d], lnf_b[d].  Weights are
[out, in] row-major; q|k|v are consecutive d-column blocks of the QKV output
and head h owns columns [h*hd, (h+1)*hd) of each block.
"""
from __future__ import annotations

from dataclasses import dataclass
import math

import numpy as np

LN_EPS = 1e-5
GELU_C = math.sqrt(2.0 / math.pi)
GELU_A = 0.044715


@dataclass(frozen=True)
class Config:
    n_layer: int
    d_model: int
    n_head: int
    n_ctx: int
    vocab: int  # padded vocabulary: the softmax runs over all of it

    @property
    def head_dim(self) -> int:
        return self.d_model // self.n_head


# ---------------------------------------------------------------- layout ---

_LAYER_TENSORS = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
                  "ln2_g", "ln2_b", "w_fc", "b_fc", "w_mp", "b_mp")


def param_shapes(cfg: Config):
    """Ordered (name, shape) list of the flat parameter layout."""
    d, V = cfg.d_model, cfg.vocab
    out = [("wte", (V, d)), ("wpe", (cfg.n_ctx, d))]
    per = {"ln1_g": (d,), "ln1_b": (d,), "w_qkv": (3 * d, d), "b_qkv": (3 * d,),
           "w_o": (d, d), "b_o": (d,), "ln2_g": (d,), "ln2_b": (d,),
           "w_fc": (4 * d, d), "b_fc": (4 * d,), "w_mp": (d, 4 * d), "b_mp": (d,)}
    for l in range(cfg.n_layer):
        for t in _LAYER_TENSORS:
            out.append((f"h{l}.{t}", per[t]))
    out += [("lnf_g", (d,)), ("lnf_b", (d,))]
    return out


def param_count(cfg: Config) -> int:
    return sum(int(np.prod(s)) for _, s in param_shapes(cfg))


def flatten(params: dict, cfg: Config) -> np.ndarray:
    return np.concatenate([np.asarray(params[n], dtype=np.float64).reshape(-1)
                           for n, _ in param_shapes(cfg)])


def unflatten(flat: np.ndarray, cfg: Config) -> dict:
    out, off = {}, 0
    for n, s in param_shapes(cfg):
        k = int(np.prod(s))
        out[n] = np.array(flat[off:off + k], dtype=np.float64).reshape(s)
        off += k
    assert off == flat.size
    return out


def decay_mask(cfg: Config) -> dict:
    """True for tensors that get decoupled weight decay (the 2-D ones)."""
    return {n: len(s) == 2 for n, s in param_shapes(cfg)}


# ------------------------------------------------------------- counting ---

class MatmulCounter:
    """Counts 2*m*n*k for every matmul the oracle performs, split by phase."""

    def __init__(self):
        self.fwd = 0
        self.bwd = 0
        self.phase = "fwd"

    def add(self, flops: int):
        if self.phase == "fwd":
            self.fwd += flops
        else:
            self.bwd += flops


def _mm(a, b, counter):
    """Matrix product (numpy) that reports its FLOPs: a[..., m, k] @ b[..., k, n]."""
    out = np.matmul(a, b)
    if counter is not None:
        batch = int(np.prod(out.shape[:-2])) if out.ndim > 2 else 1
        counter.add(2 * batch * a.shape[-2] * a.shape[-1] * b.shape[-1])
    return out


# --------------------------------------------------------- building blocks ---

def layernorm_fwd(x, g, b):
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)   # biased variance
    rstd = 1.0 / np.sqrt(var + LN_EPS)
    xhat = (x - mu) * rstd
    return xhat * g + b, (xhat, rstd)


def layernorm_bwd(dy, g, saved):
    xhat, rstd = saved
    dg = (dy * xhat).reshape(-1, xhat.shape[-1]).sum(axis=0)
    db = dy.reshape(-1, dy.shape[-1]).sum(axis=0)
    dxhat = dy * g
    dx = rstd * (dxhat - dxhat.mean(axis=-1, keepdims=True)
                 - xhat * (dxhat * xhat).mean(axis=-1, keepdims=True))
    return dx, dg, db


def gelu_fwd(u):
    return 0.5 * u * (1.0 + np.tanh(GELU_C * (u + GELU_A * u ** 3)))


def gelu_bwd(du_out, u):
    t = np.tanh(GELU_C * (u + GELU_A * u ** 3))
    dgelu = 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * GELU_C * (1.0 + 3.0 * GELU_A * u * u)
    return du_out * dgelu


def linear_fwd(x, w, b, counter):
    """y = x W^T (+ b); x [..., in], w [out, in]."""
    y = _mm(x, w.T, counter)
    return y if b is None else y + b


def linear_bwd(dy, x, w, counter):
    """The two gradients of one linear layer: w.r.t. its input and its weight."""
    dx = _mm(dy, w, counter)
    d2 = dy.reshape(-1, dy.shape[-1])
    x2 = x.reshape(-1, x.shape[-1])
    dw = _mm(d2.T, x2, counter)
    return dx, dw, d2.sum(axis=0)


def _split_heads(t, H):
    B, T, d = t.shape
    return t.reshape(B, T, H, d // H).transpose(0, 2, 1, 3)   # [B, H, T, hd]


def _merge_heads(t):
    B, H, T, hd = t.shape
    return t.transpose(0, 2, 1, 3).reshape(B, T, H * hd)


def attention_fwd(q, k, v, counter):
    """Causal softmax(q k^T / sqrt(hd)) v per (batch, head); inputs [B,H,T,hd]."""
    T, hd = q.shape[-2], q.shape[-1]
    s = _mm(q, np.swapaxes(k, -1, -2), counter) / math.sqrt(hd)
    future = np.triu(np.ones((T, T), dtype=bool), k=1)          # key j > query i
    s = np.where(future, -np.inf, s)
    s_max = s.max(axis=-1, keepdims=True)
    e = np.exp(s - s_max)
    p = e / e.sum(axis=-1, keepdims=True)
    o = _mm(p, v, counter)
    return o, p


def attention_bwd(do, q, k, v, p, counter):
    hd = q.shape[-1]
    dv = _mm(np.swapaxes(p, -1, -2), do, counter)
    dp = _mm(do, np.swapaxes(v, -1, -2), counter)
    dsum = (dp * p).sum(axis=-1, keepdims=True)                 # = rowsum(do * o)
    ds = p * (dp - dsum) / math.sqrt(hd)
    dq = _mm(ds, k, counter)
    dk = _mm(np.swapaxes(ds, -1, -2), q, counter)
    return dq, dk, dv


IGNORE = -1  # target id of a position that takes no part in the loss


def cross_entropy_fwd(z, targets):
    """Per-position loss LSE(z) - z[target] with an explicit max-shifted LSE;
    positions whose target is IGNORE get loss 0.  That is the masked loss of
    instruction tuning: "Criei GPT-2 do zero com uma RTX 4090", section "Usei
    SFT para fazê-lo conversar", trains only the assistant's answer and its
    end marker while the question is only read."""
    zmax = z.max(axis=-1, keepdims=True)
    lse = zmax[..., 0] + np.log(np.exp(z - zmax).sum(axis=-1))
    valid = targets != IGNORE
    z_t = np.take_along_axis(z, np.where(valid, targets, 0)[..., None], axis=-1)[..., 0]
    return np.where(valid, lse - z_t, 0.0), lse


# ------------------------------------------------------------- the model ---

def forward(params: dict, cfg: Config, tokens, targets, counter=None, head=None):
    """Mean next-token cross-entropy over the positions that have a target
    (all B*T of them unless some targets are IGNORE), plus a cache.

    ``head`` (optional) replaces the tied LM-head matrix by a separate copy;
    it exists only for the tied-embedding decomposition test.
    """
    tokens = np.asarray(tokens)
    targets = np.asarray(targets)
    B, T = tokens.shape
    assert T <= cfg.n_ctx
    H = cfg.n_head
    if counter is not None:
        counter.phase = "fwd"
    x = params["wte"][tokens] + params["wpe"][:T][None, :, :]
    layers = []
    for l in range(cfg.n_layer):
        P = lambda t: params[f"h{l}.{t}"]  # noqa: E731
        c = {"x_in": x}
        y1, c["ln1"] = layernorm_fwd(x, P("ln1_g"), P("ln1_b"))
        qkv = linear_fwd(y1, P("w_qkv"), P("b_qkv"), counter)
        d = cfg.d_model
        q, k, v = (_split_heads(qkv[..., i * d:(i + 1) * d], H) for i in range(3))
        o, prob = attention_fwd(q, k, v, counter)
        a = _merge_heads(o)
        x = x + linear_fwd(a, P("w_o"), P("b_o"), counter)
        c.update(y1=y1, q=q, k=k, v=v, p=prob, a=a, x_mid=x)
        y2, c["ln2"] = layernorm_fwd(x, P("ln2_g"), P("ln2_b"))
        u = linear_fwd(y2, P("w_fc"), P("b_fc"), counter)
        g = gelu_fwd(u)
        x = x + linear_fwd(g, P("w_mp"), P("b_mp"), counter)
        c.update(y2=y2, u=u, g=g)
        layers.append(c)
    yf, lnf = layernorm_fwd(x, params["lnf_g"], params["lnf_b"])
    w_head = params["wte"] if head is None else head
    z = linear_fwd(yf, w_head, None, counter)
    loss_pos, lse = cross_entropy_fwd(z, targets)
    # mean over the positions that have a target (all of them unless masked)
    n_valid = max(1, int(np.sum(targets != IGNORE)))
    loss = float(loss_pos.sum() / n_valid)
    cache = dict(tokens=tokens, targets=targets, layers=layers, yf=yf, lnf=lnf,
                 z=z, lse=lse, loss_pos=loss_pos, head=head)
    return loss, cache


def backward(params: dict, cfg: Config, cache: dict, grad_scale: float = 1.0, counter=None):
    """Gradient of grad_scale * loss with respect to every parameter.

    Returns a dict with the same keys as ``params`` (plus ``head`` when the
    untied variant was used in ``forward``).
    """
    if counter is not None:
        counter.phase = "bwd"
    tokens, targets = cache["tokens"], cache["targets"]
    B, T = tokens.shape
    M = B * T
    H = cfg.n_head
    grads = {n: np.zeros(s) for n, s in param_shapes(cfg)}

    # d loss / d z = (softmax(z) - onehot(target)) / n_valid on positions with
    # a target, 0 on masked ones (n_valid = M without masking)
    z = cache["z"]
    valid = targets != IGNORE
    n_valid = max(1, int(np.sum(valid)))
    safe_t = np.where(valid, targets, 0)
    dz = np.exp(z - cache["lse"][..., None])
    np.put_along_axis(dz, safe_t[..., None], np.take_along_axis(dz, safe_t[..., None], axis=-1) - 1.0, axis=-1)
    dz *= np.where(valid, grad_scale / n_valid, 0.0)[..., None]
    w_head = params["wte"] if cache["head"] is None else cache["head"]
    dyf, dw_head, _ = linear_bwd(dz, cache["yf"], w_head, counter)
    if cache["head"] is None:
        grads["wte"] += dw_head
    else:
        grads["head"] = dw_head
    dx, grads["lnf_g"], grads["lnf_b"] = layernorm_bwd(dyf, params["lnf_g"], cache["lnf"])

    for l in reversed(range(cfg.n_layer)):
        P = lambda t: params[f"h{l}.{t}"]  # noqa: E731
        G = f"h{l}."
        c = cache["layers"][l]
        # x_out = x_mid + gelu(ln2(x_mid) W_fc^T + b_fc) W_mp^T + b_mp
        dg, grads[G + "w_mp"], grads[G + "b_mp"] = linear_bwd(dx, c["g"], P("w_mp"), counter)
        du = gelu_bwd(dg, c["u"])
        dy2, grads[G + "w_fc"], grads[G + "b_fc"] = linear_bwd(du, c["y2"], P("w_fc"), counter)
        dln, grads[G + "ln2_g"], grads[G + "ln2_b"] = layernorm_bwd(dy2, P("ln2_g"), c["ln2"])
        dx = dx + dln
        # x_mid = x_in + attn(ln1(x_in)) W_o^T + b_o
        da, grads[G + "w_o"], grads[G + "b_o"] = linear_bwd(dx, c["a"], P("w_o"), counter)
        dq, dk, dv = attention_bwd(_split_heads(da, H), c["q"], c["k"], c["v"], c["p"], counter)
        dqkv = np.concatenate([_merge_heads(dq), _merge_heads(dk), _merge_heads(dv)], axis=-1)
        dy1, grads[G + "w_qkv"], grads[G + "b_qkv"] = linear_bwd(dqkv, c["y1"], P("w_qkv"), counter)
        dln, grads[G + "ln1_g"], grads[G + "ln1_b"] = layernorm_bwd(dy1, P("ln1_g"), c["ln1"])
        dx = dx + dln

    # x_0 = wte[token] + wpe[position]: scatter-add into the (tied) wte rows
    np.add.at(grads["wte"], tokens.reshape(-1), dx.reshape(M, -1))
    grads["wpe"][:T] += dx.sum(axis=0)
    return grads


def clip_grad_norm(grads: dict, max_norm: float):
    """Global-norm gradient clipping.  The pages do not use it; this is the
    common form: total = sqrt(sum over every tensor of sum g^2), and when
    max_norm / (total + 1e-6) < 1 every gradient is multiplied by that ratio.
    Returns (clipped grads, total)."""
    total = float(np.sqrt(sum(float(np.sum(np.square(g, dtype=np.float64))) for g in grads.values())))
    coef = max_norm / (total + 1e-6)
    if coef >= 1.0:
        return {n: g.copy() for n, g in grads.items()}, total
    return {n: g * coef for n, g in grads.items()}, total


def adamw_step(params: dict, grads: dict, m: dict, v: dict, step: int, cfg: Config,
               lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, max_norm=0.0):
    """Decoupled-weight-decay Adam (AdamW), step counter starting at 1.

    p <- p * (1 - lr*wd)             (2-D tensors only)
    m <- b1 m + (1-b1) g ;  v <- b2 v + (1-b2) g^2
    p <- p - lr * m_hat / (sqrt(v_hat) + eps),  m_hat = m/(1-b1^t), v_hat = v/(1-b2^t)
    With max_norm > 0 the gradients are first clipped to that global norm
    (clip_grad_norm).  Returns new (params, m, v) dicts; the inputs are left
    untouched.
    """
    if max_norm > 0.0:
        grads, _ = clip_grad_norm(grads, max_norm)
    decay = decay_mask(cfg)
    bc1 = 1.0 - beta1 ** step
    bc2 = 1.0 - beta2 ** step
    P, Mo, Vo = {}, {}, {}
    for n, _ in param_shapes(cfg):
        g = grads[n]
        p = params[n] * (1.0 - lr * weight_decay) if decay[n] else params[n].copy()
        mn = beta1 * m[n] + (1.0 - beta1) * g
        vn = beta2 * v[n] + (1.0 - beta2) * g * g
        p = p - lr * (mn / bc1) / (np.sqrt(vn / bc2) + eps)
        P[n], Mo[n], Vo[n] = p, mn, vn
    return P, Mo, Vo


def train_step(params, m, v, step, cfg, tokens, targets, **hp):
    """One forward + backward + AdamW step; returns (loss, grads, params, m, v)."""
    loss, cache = forward(params, cfg, tokens, targets)
    grads = backward(params, cfg, cache)
    P, Mo, Vo = adamw_step(params, grads, m, v, step, cfg, **hp)
    return loss, grads, P, Mo, Vo


# ------------------------------------------------ incremental decoding ---
#
# "Criei GPT-2 do zero com uma RTX 4090", sections "Vendo o modelo ficar mais
# inteligente aos poucos" and "Conversando de verdade com ele": the trained
# model continues a prompt one token at a time.  The distribution of the next
# token after positions 0..p is the forward's output at position p, and by
# causality that output depends on the keys and values of positions 0..p only.
# A decoder therefore keeps every layer's K and V of the positions seen so far
# (the key/value cache) and, per new token, computes one query row against
# them.  The pages fix no sampling rule; greedy (the most probable id) is the
# plainest.

def kv_cache_empty(cfg: Config, batch: int, max_len: int) -> list:
    """Per layer {"k", "v"}: [batch, H, max_len, hd] zeros."""
    shape = (batch, cfg.n_head, max_len, cfg.head_dim)
    return [dict(k=np.zeros(shape), v=np.zeros(shape)) for _ in range(cfg.n_layer)]


def decode_step(params: dict, cfg: Config, cache: list, tokens, pos):
    """Row b feeds token ``tokens[b]`` at position ``pos[b]``: its K and V are
    written into the cache at that position, its query attends to positions
    0..pos[b] of the row's cache, and the logits of the next token
    ([batch, vocab]) are returned."""
    tokens = np.asarray(tokens)
    pos = np.asarray(pos)
    B = tokens.shape[0]
    H, hd, d = cfg.n_head, cfg.head_dim, cfg.d_model
    x = params["wte"][tokens] + params["wpe"][pos]                      # [B, d]
    for l in range(cfg.n_layer):
        P = lambda t: params[f"h{l}.{t}"]  # noqa: E731
        y1, _ = layernorm_fwd(x, P("ln1_g"), P("ln1_b"))
        qkv = linear_fwd(y1, P("w_qkv"), P("b_qkv"), None)               # [B, 3d]
        q, k, v = (qkv[:, i * d:(i + 1) * d].reshape(B, H, hd) for i in range(3))
        a = np.zeros((B, H, hd))
        for b in range(B):
            p = int(pos[b])
            cache[l]["k"][b, :, p, :] = k[b]
            cache[l]["v"][b, :, p, :] = v[b]
            keys = cache[l]["k"][b, :, :p + 1, :]                         # [H, p+1, hd]
            vals = cache[l]["v"][b, :, :p + 1, :]
            s = np.einsum("hd,hjd->hj", q[b], keys) / math.sqrt(hd)
            e = np.exp(s - s.max(axis=-1, keepdims=True))
            prob = e / e.sum(axis=-1, keepdims=True)
            a[b] = np.einsum("hj,hjd->hd", prob, vals)
        x = x + linear_fwd(a.reshape(B, d), P("w_o"), P("b_o"), None)
        y2, _ = layernorm_fwd(x, P("ln2_g"), P("ln2_b"))
        x = x + linear_fwd(gelu_fwd(linear_fwd(y2, P("w_fc"), P("b_fc"), None)), P("w_mp"), P("b_mp"), None)
    yf, _ = layernorm_fwd(x, params["lnf_g"], params["lnf_b"])
    return linear_fwd(yf, params["wte"], None, None)


def prefill(params: dict, cfg: Config, cache: list, tokens, prompt_len):
    """Feeds row b's prompt ``tokens[b, :prompt_len[b]]`` through the cache one
    position at a time; returns each row's logits after its last prompt token
    ([batch, vocab])."""
    tokens = np.asarray(tokens)
    B = tokens.shape[0]
    out = np.zeros((B, cfg.vocab))
    for b in range(B):
        row = [dict(k=c["k"][b:b + 1], v=c["v"][b:b + 1]) for c in cache]  # views: writes land in cache
        for p in range(int(prompt_len[b])):
            out[b] = decode_step(params, cfg, row, tokens[b, p:p + 1], np.array([p]))[0]
    return out


def greedy_next(logits, vocab_real: int):
    """Most probable real id per row (padded ids never chosen); the lowest id
    among equal maxima, and the first NaN if a row holds one."""
    return np.argmax(np.asarray(logits)[:, :vocab_real], axis=-1).astype(np.int32)
