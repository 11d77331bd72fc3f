"""Kernel-level GPU tests through the C ABI: the tcgen05 GEMM in every operand
majorness, tile width and split, with ragged M/N tails; the causal attention
forward/backward against the oracle's attention on the same bf16 inputs."""
import math

import numpy as np
import pytest
import torch

import decoder_only_transformer_step_b200 as gp
from oracle import gpt2_oracle as G

pytestmark = pytest.mark.gpu


def bf16_rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("bn", [128, 256, 512])
@pytest.mark.parametrize("c_fp32", [0, 1])
def test_gemm_layouts(a_mn, b_mn, bn, c_fp32):
    """bn 128 / 256: single-CTA 128 x bn tiles; 512: the CTA-pair 256 x 256 tile."""
    M, N, K = 300, 520, 192
    lda = 304 if a_mn else K
    A_log = bf16_rand((M, K), 1)                       # logical A(m, k)
    B_log = bf16_rand((N, K), 2)                       # logical B(n, k)
    if a_mn:
        A_st = torch.zeros((K, lda), dtype=torch.bfloat16)
        A_st[:, :M] = A_log.t()
    else:
        A_st = A_log.contiguous()
    B_st = B_log.t().contiguous() if b_mn else B_log.contiguous()
    ldb = N if b_mn else K
    ref = A_log.double() @ B_log.double().t()
    alpha = 0.75
    dev = "cuda"
    # fp32 output accumulates onto existing values (beta = 1, the gradient
    # accumulation path); bf16 output overwrites
    C0 = torch.randn((M, N), generator=torch.Generator().manual_seed(9)) if c_fp32 else torch.zeros((M, N))
    C = C0.to(torch.float32 if c_fp32 else torch.bfloat16).to(dev)
    gp.gpt2_op_gemm_bf16(A_st.to(dev), a_mn, lda, B_st.to(dev), b_mn, ldb, C, c_fp32, N, M, N, K,
                         alpha=alpha, beta=1.0 if c_fp32 else 0.0, bn=bn, splits=1)
    torch.cuda.synchronize()
    out = C.double().cpu()
    expect = alpha * ref + (C0.double() if c_fp32 else 0.0)
    err = (out - expect).abs().max().item()
    scale = (alpha * ref).abs().max().item()
    assert err <= (1e-5 if c_fp32 else 8e-3) * scale, (err, scale)


@pytest.mark.parametrize("bn", [128, 512])
@pytest.mark.parametrize("splits", [2, 3, 5])
def test_gemm_split_k_accumulate(splits, bn):
    """Weight-gradient shape: MN-major operands, fp32 out, split along K with
    the deterministic partial-sum reduction, beta = 1 accumulation."""
    M, N, K = 200, 136, 640
    A_log = bf16_rand((M, K), 3)
    B_log = bf16_rand((N, K), 4)
    A_st = torch.zeros((K, 200), dtype=torch.bfloat16)
    A_st[:, :M] = A_log.t()
    B_st = B_log.t().contiguous()
    C0 = torch.randn((M, N), generator=torch.Generator().manual_seed(5))
    C = C0.clone().cuda()
    ws = torch.empty(splits * M * N * 4, dtype=torch.uint8, device="cuda")
    gp.gpt2_op_gemm_bf16(A_st.cuda(), 1, 200, B_st.cuda(), 1, N, C, 1, N, M, N, K, alpha=0.5, beta=1.0,
                         workspace=ws, bn=bn, splits=splits)
    ref = C0.double() + 0.5 * (A_log.double() @ B_log.double().t())
    err = (C.double().cpu() - ref).abs().max().item()
    assert err <= 1e-5 * ref.abs().max().item()
    # deterministic: the same call twice gives bitwise-identical output
    C2 = C0.clone().cuda()
    gp.gpt2_op_gemm_bf16(A_st.cuda(), 1, 200, B_st.cuda(), 1, N, C2, 1, N, M, N, K, alpha=0.5, beta=1.0,
                         workspace=ws, bn=bn, splits=splits)
    assert torch.equal(C, C2)


@pytest.mark.parametrize("M,N", [(100, 136), (257, 600), (384, 256)])
@pytest.mark.parametrize("a_mn", [0, 1])
def test_gemm_pair_ragged(M, N, a_mn):
    """CTA-pair tiles whose second CTA holds no valid row (M = 100), a single
    valid row (M = 257), or whose B half lies past N (N = 136, 600)."""
    K = 128
    A_log = bf16_rand((M, K), 11)
    B_log = bf16_rand((N, K), 12)
    lda = (M + 7) // 8 * 8 + 8 if a_mn else K
    if a_mn:
        A_st = torch.zeros((K, lda), dtype=torch.bfloat16)
        A_st[:, :M] = A_log.t()
    else:
        A_st = A_log.contiguous()
    C = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    gp.gpt2_op_gemm_bf16(A_st.cuda(), a_mn, lda, B_log.cuda(), 0, K, C, 0, N, M, N, K, bn=512, splits=1)
    ref = A_log.double() @ B_log.double().t()
    err = (C.double().cpu() - ref).abs().max().item()
    assert err <= 8e-3 * ref.abs().max().item(), err


def test_gemm_large_k_many_tiles():
    """More output tiles than SMs (the persistent scheduler wraps) and a long
    K loop (ring buffer phases wrap many times)."""
    M, N, K = 2048, 4608, 1024
    A = bf16_rand((M, K), 6)
    B = bf16_rand((N, K), 7)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    gp.gpt2_op_gemm_bf16(A.cuda(), 0, K, B.cuda(), 0, K, C, 1, N, M, N, K)
    ref = A.cuda().float() @ B.cuda().float().t()
    assert (C - ref).abs().max().item() <= 1e-4 * ref.abs().max().item()


def _attn_inputs(B, T, H, hd, seed):
    d = H * hd
    qkv = bf16_rand((B * T, 3 * d), seed, scale=1.0)
    return qkv


def _split(qkv, B, T, H, hd):
    d = H * hd
    x = qkv.double().numpy().reshape(B, T, 3, H, hd)
    return [x[:, :, i].transpose(0, 2, 1, 3) for i in range(3)]   # [B, H, T, hd]


@pytest.mark.parametrize("hd,T", [(64, 200), (64, 1024), (16, 64), (16, 77)])
def test_attention_forward(hd, T):
    B, H = 2, 3
    d = H * hd
    qkv = _attn_inputs(B, T, H, hd, 10 + T)
    o = torch.empty((B * T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    gp.gpt2_op_attention_fwd_bf16(qkv.cuda(), o, lse, B, T, H, hd)
    q, k, v = _split(qkv, B, T, H, hd)
    o_ref, p = G.attention_fwd(q, k, v, None)
    s = np.einsum("bhid,bhjd->bhij", q, k) / math.sqrt(hd)
    s = np.where(np.triu(np.ones((T, T), bool), 1), -np.inf, s)
    lse_ref = np.log(np.exp(s - s.max(-1, keepdims=True)).sum(-1)) + s.max(-1)
    o_gpu = o.double().cpu().numpy().reshape(B, T, H, hd).transpose(0, 2, 1, 3)
    assert np.abs(o_gpu - o_ref).max() <= 0.02 * np.abs(o_ref).max()
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() <= 2e-2


@pytest.mark.parametrize("B,H,T", [(4, 12, 512), (8, 12, 300)])
def test_attention_forward_many_items(B, H, T):
    """More (query block, batch, head) work items than SMs: the persistent
    forward carries its K/V ring and buffer phases across items."""
    hd = 64
    d = H * hd
    qkv = _attn_inputs(B, T, H, hd, 40 + T)
    o = torch.empty((B * T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    gp.gpt2_op_attention_fwd_bf16(qkv.cuda(), o, lse, B, T, H, hd)
    q, k, v = _split(qkv, B, T, H, hd)
    o_ref, p = G.attention_fwd(q, k, v, None)
    s = np.einsum("bhid,bhjd->bhij", q, k) / math.sqrt(hd)
    s = np.where(np.triu(np.ones((T, T), bool), 1), -np.inf, s)
    lse_ref = np.log(np.exp(s - s.max(-1, keepdims=True)).sum(-1)) + s.max(-1)
    o_gpu = o.double().cpu().numpy().reshape(B, T, H, hd).transpose(0, 2, 1, 3)
    assert np.abs(o_gpu - o_ref).max() <= 0.02 * np.abs(o_ref).max()
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() <= 2e-2


@pytest.mark.parametrize("B,H,T", [(4, 12, 512), (8, 12, 300)])
def test_attention_backward_many_items(B, H, T):
    """More (key block, batch, head) work items than SMs: the persistent
    backward carries its ring phases and dQ buffers across items."""
    hd = 64
    d = H * hd
    qkv = _attn_inputs(B, T, H, hd, 50 + T)
    dout = bf16_rand((B * T, d), 60 + T)
    o = torch.empty((B * T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    gp.gpt2_op_attention_fwd_bf16(qkv.cuda(), o, lse, B, T, H, hd)
    dqkv = torch.empty((B * T, 3 * d), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(B * T * d + B * H * T, dtype=torch.float32, device="cuda")
    gp.gpt2_op_attention_bwd_bf16(qkv.cuda(), o, lse, dout.cuda(), dqkv, scratch, B, T, H, hd)
    q, k, v = _split(qkv, B, T, H, hd)
    _, p = G.attention_fwd(q, k, v, None)
    do = dout.double().numpy().reshape(B, T, H, hd).transpose(0, 2, 1, 3)
    dq, dk, dv = G.attention_bwd(do, q, k, v, p, None)
    got = _split(dqkv.cpu(), B, T, H, hd)
    for name, g, r in zip("qkv", got, (dq, dk, dv)):
        cos = (g * r).sum() / (np.linalg.norm(g) * np.linalg.norm(r))
        rel = np.abs(g - r).max() / np.abs(r).max()
        assert cos >= 0.999 and rel <= 2e-2, (name, cos, rel)


@pytest.mark.parametrize("hd,T", [(64, 200), (64, 1024), (16, 64), (16, 77)])
def test_attention_backward(hd, T):
    B, H = 2, 3
    d = H * hd
    qkv = _attn_inputs(B, T, H, hd, 20 + T)
    dout = bf16_rand((B * T, d), 30 + T)
    o = torch.empty((B * T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    gp.gpt2_op_attention_fwd_bf16(qkv.cuda(), o, lse, B, T, H, hd)
    dqkv = torch.empty((B * T, 3 * d), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(B * T * d + B * H * T, dtype=torch.float32, device="cuda")
    gp.gpt2_op_attention_bwd_bf16(qkv.cuda(), o, lse, dout.cuda(), dqkv, scratch, B, T, H, hd)
    q, k, v = _split(qkv, B, T, H, hd)
    _, p = G.attention_fwd(q, k, v, None)
    do = dout.double().numpy().reshape(B, T, H, hd).transpose(0, 2, 1, 3)
    dq, dk, dv = G.attention_bwd(do, q, k, v, p, None)
    got = _split(dqkv.cpu(), B, T, H, hd)
    for name, g, r in zip("qkv", got, (dq, dk, dv)):
        cos = (g * r).sum() / (np.linalg.norm(g) * np.linalg.norm(r))
        rel = np.abs(g - r).max() / np.abs(r).max()
        assert cos >= 0.999 and rel <= 2e-2, (name, cos, rel)


@pytest.mark.parametrize("M,d", [(1000, 768), (77, 1600), (4096, 1024)])
def test_layernorm_ops_against_oracle(M, d):
    """The LayerNorm forward and backward kernels alone, on ragged row counts
    and the three model widths, against the oracle's LayerNorm on the same
    bf16 inputs: y and dx element-wise within 1e-2 of their largest entry,
    mean / rstd and the fp32 gamma / beta gradients within 1e-4."""
    x = bf16_rand((M, d), 70 + M, scale=2.0) + 0.5
    gamma = bf16_rand((d,), 71, scale=0.1) + 1.0
    beta = bf16_rand((d,), 72, scale=0.1)
    dy = bf16_rand((M, d), 73 + M)
    y = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    mean = torch.empty(M, device="cuda")
    rstd = torch.empty(M, device="cuda")
    gp.gpt2_op_layernorm_fwd_bf16(x.cuda(), gamma.cuda(), beta.cuda(), y, mean, rstd, M, d)
    X, Gm, Bt, DY = (t.double().numpy() for t in (x, gamma, beta, dy))
    y_ref, saved = G.layernorm_fwd(X, Gm, Bt)
    assert np.abs(y.double().cpu().numpy() - y_ref).max() <= 1e-2 * np.abs(y_ref).max()
    assert np.abs(mean.double().cpu().numpy() - X.mean(-1)).max() <= 1e-4 * np.abs(X).max()
    assert np.abs(rstd.double().cpu().numpy() / saved[1][:, 0] - 1).max() <= 1e-4
    dx_ref, dg_ref, db_ref = G.layernorm_bwd(DY, Gm, saved)
    scratch = torch.empty(gp.gpt2_op_layernorm_bwd_scratch_floats(M, d), device="cuda")
    dgb = torch.empty(2 * d, device="cuda")
    prev = bf16_rand((M, d), 74 + M)
    for accumulate in (0, 1):
        dx = prev.cuda().clone()
        gp.gpt2_op_layernorm_bwd_bf16(dy.cuda(), x.cuda(), mean, rstd, gamma.cuda(), dx, accumulate, dgb, scratch,
                                      M, d)
        want = dx_ref + (prev.double().numpy() if accumulate else 0.0)
        assert np.abs(dx.double().cpu().numpy() - want).max() <= 1e-2 * np.abs(want).max(), accumulate
        got = dgb.double().cpu().numpy()
        assert np.abs(got[:d] - dg_ref).max() <= 1e-4 * np.abs(dg_ref).max()
        assert np.abs(got[d:] - db_ref).max() <= 1e-4 * np.abs(db_ref).max()


@pytest.mark.parametrize("M,N", [(16384, 3072), (1000, 2304), (77, 64)])
def test_colsum_op_exact_sums(M, N):
    """Bias gradients: the column sums of a bf16 matrix against the exact
    (fp64) sums of the same values; fp32 accumulation keeps the error far
    below 1e-5 of the sum of magnitudes."""
    x = bf16_rand((M, N), 80 + M)
    out = torch.empty(N, device="cuda")
    scratch = torch.empty(gp.gpt2_op_colsum_scratch_floats(M, N), device="cuda")
    gp.gpt2_op_colsum_bf16(x.cuda(), M, N, out, scratch)
    X = x.double().numpy()
    assert np.abs(out.double().cpu().numpy() - X.sum(0)).max() <= 1e-5 * np.abs(X).sum(0).max()


@pytest.mark.parametrize("M,V,d,vocab_real", [(960, 1408, 128, 1400), (1024, 50304, 768, 50257)])
def test_lm_head_cross_entropy_ops_against_oracle(M, V, d, vocab_real):
    """The tied LM head with the fused softmax cross-entropy, alone: the
    forward's per-row losses and mean against the oracle's cross-entropy of
    z = x w^T (fp64, same bf16 x and w), and the backward's dx and dw against
    the chain rule of that loss, (softmax - onehot) / n_valid; every tenth
    target masked (-1).  The rows are not a multiple of the 256-row tile and
    the first vocabulary is not a multiple of the 256-column tile."""
    g = torch.Generator().manual_seed(90 + M)
    x = bf16_rand((M, d), 91 + M)
    w = bf16_rand((V, d), 92 + V, scale=0.1)
    tgt = torch.randint(0, vocab_real, (M,), generator=g, dtype=torch.int32)
    tgt[::10] = -1
    scratch = torch.empty(gp.gpt2_op_lm_head_ce_scratch_bytes(M, V), dtype=torch.uint8, device="cuda")
    loss = torch.empty(1, device="cuda")
    rows = torch.empty(M, device="cuda")
    xd, wd, td = x.cuda(), w.cuda(), tgt.cuda()
    gp.gpt2_op_lm_head_ce_fwd_bf16(xd, wd, td, M, V, d, vocab_real, loss, rows, scratch)
    dx = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    dw = torch.full((V, d), float("nan"), device="cuda")
    gp.gpt2_op_lm_head_ce_bwd_bf16(xd, wd, M, V, d, 0.5, dx, dw, 0, scratch)
    torch.cuda.synchronize()
    assert int(scratch[:4].view(torch.int32).item()) == 0
    X, W, Y = x.double().numpy(), w.double().numpy(), tgt.numpy().astype(np.int64)
    z = X @ W.T
    ref_rows, _ = G.cross_entropy_fwd(z, Y)
    valid = Y != G.IGNORE
    n_valid = int(valid.sum())
    ref_loss = ref_rows.sum() / n_valid
    assert abs(loss.item() - ref_loss) <= 1e-4 * abs(ref_loss), (loss.item(), ref_loss)
    assert np.abs(rows.double().cpu().numpy() - ref_rows).max() <= 1e-3 * np.abs(ref_rows).max()
    p = np.exp(z - z.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    p[np.arange(M)[valid], Y[valid]] -= 1.0
    dz = np.where(valid[:, None], p, 0.0) * (0.5 / n_valid)
    for name, got, ref in (("dx", dx, dz @ W), ("dw", dw, dz.T @ X)):
        a = got.double().cpu().numpy().ravel()
        r = ref.ravel()
        cos = float(a @ r / (np.linalg.norm(a) * np.linalg.norm(r)))
        rel = float(np.abs(a - r).max() / np.abs(r).max())
        assert cos >= 0.999 and rel <= 2e-2, (name, cos, rel)


@pytest.mark.parametrize("act", [0, 1, 2])
@pytest.mark.parametrize("M,N,K", [(300, 520, 192), (2048, 3072, 768)])
def test_linear_op_fused_epilogues_against_oracle(act, M, N, K):
    """One linear layer with the epilogue the forward fuses into its GEMM
    (bias; bias + residual; bias + GELU with the saved GELU') against the
    oracle's linear layer and GELU on the same bf16 inputs.  Ragged M and N
    against the 256 x 256 tile in the small case; the MLP fc shape of GPT-2
    small in the large one.  Each output is rounded once to bf16 from an fp32
    accumulator: element-wise within 2^-7 of the value plus 4e-3 absolute
    (the tanh of the GELU is the hardware approximation)."""
    x = bf16_rand((M, K), 90 + M)
    w = bf16_rand((N, K), 91 + N, scale=2.0 / math.sqrt(K))
    bias = bf16_rand((N,), 92, scale=0.5)
    resid = bf16_rand((M, N), 93 + M)
    X, W, Bv, R = (t.double().numpy() for t in (x, w, bias, resid))
    u = G.linear_fwd(X, W, Bv, None)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    out2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda") if act == 2 else None
    gp.gpt2_op_linear_bf16(x.cuda(), w.cuda(), bias.cuda(), resid.cuda() if act == 1 else None, out, out2,
                           M, N, K, act)
    torch.cuda.synchronize()
    if act == 0:
        wants = [(out, u)]
    elif act == 1:
        wants = [(out, u + R)]
    else:
        wants = [(out, G.gelu_fwd(u)), (out2, G.gelu_bwd(np.ones_like(u), u))]
    for got, want in wants:
        err = np.abs(got.double().cpu().numpy() - want)
        assert (err <= np.abs(want) / 128 + 4e-3).all(), (act, err.max())
