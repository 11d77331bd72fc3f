"""Incremental decoding (key/value cache) through the C ABI against the fp64
oracle on the same seeded inputs: prefill of ragged prompts, then decode steps
with seeded (teacher-forced) tokens, rows at different positions.  Tolerance:
max |z - z_ref| / max |z_ref| per step <= 1e-4 in the fp32 mode and <= 2e-2 in
bf16 (bf16 weights and cache, fp32 accumulation).  The greedy choice is an
integer decided in fp32 on both sides and must match exactly."""
import numpy as np
import pytest
import torch

import decoder_only_transformer_step_b200 as gp
from decoder_only_transformer_step_b200 import inputs
import oracle
from oracle import Config, forward, kv_cache_empty, decode_step, prefill, greedy_next
from oracle import gpt2_oracle as G
from oracle_fixtures import TINY, params_for

pytestmark = pytest.mark.gpu

HD64 = Config(n_layer=2, d_model=128, n_head=2, n_ctx=128, vocab=1024)


def make_model(oc: Config, vocab_real, batch, mode):
    mc = gp.ModelConfig(oc.n_layer, oc.d_model, oc.n_head, oc.n_ctx, vocab_real, oc.vocab, batch, mode)
    return gp.GPT2(mc)


def load_params(model, params, oc):
    flat32 = oracle.flatten(params, oc).astype(np.float32)
    model.master.copy_(torch.from_numpy(flat32))
    model.refresh_shadow()
    return oracle.unflatten(flat32.astype(np.float64), oc)


def rel_err(z, ref):
    return float(np.abs(z - ref).max() / np.abs(ref).max())


def i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("oc", [TINY, HD64], ids=["hd16", "hd64"])
@pytest.mark.parametrize("mode", [1, 0])
@pytest.mark.parametrize("batch", [3, 7, 16])
def test_prefill_and_decode_match_oracle(oc, mode, batch):
    vocab_real = oc.vocab - 12
    params = params_for(oc, seed=41)
    model = make_model(oc, vocab_real, batch, mode)
    p32 = load_params(model, params, oc)
    max_len = oc.n_ctx - 8
    rng = np.random.default_rng(42)
    plen = rng.integers(1, 20, size=batch).astype(np.int32)
    plen[0] = 1
    tok, _ = inputs.uniform_tokens(batch, oc.n_ctx, vocab_real, seed=43)
    cache = gp.KVCache(model, batch, max_len)
    z = cache.prefill(i32(tok), i32(plen)).cpu().numpy().astype(np.float64)
    ref_cache = kv_cache_empty(oc, batch, max_len)
    z_ref = prefill(p32, oc, ref_cache, tok, plen)
    tol = 1e-4 if mode == 1 else 2e-2
    assert rel_err(z, z_ref) <= tol
    pos = plen.copy()
    for step in range(6):
        t_step = inputs.uniform_tokens(batch, 1, vocab_real, seed=100 + step)[0][:, 0]
        z = cache.step(i32(t_step), i32(pos)).cpu().numpy().astype(np.float64)
        z_ref = decode_step(p32, oc, ref_cache, t_step, pos)
        assert rel_err(z, z_ref) <= tol, step
        pos = pos + 1
    torch.cuda.synchronize()
    assert model.status() == 0


def test_decode_equals_forward_logits_full_context():
    # a row decoded up to the last position of a small cache: the attention
    # covers several 32-key tiles per warp; checked against the oracle forward
    oc = HD64
    params = params_for(oc, seed=44)
    model = make_model(oc, oc.vocab, 2, 1)
    p32 = load_params(model, params, oc)
    T = oc.n_ctx
    tok, _ = inputs.uniform_tokens(2, T, oc.vocab, seed=45)
    cache = gp.KVCache(model, 2, T)
    plen = np.array([T - 3, 40], dtype=np.int32)
    cache.prefill(i32(tok), i32(plen))
    pos = plen.copy()
    ref = forward(p32, oc, tok, np.full(tok.shape, G.IGNORE))[1]["z"]
    for _ in range(3):
        z = cache.step(i32(tok[np.arange(2), pos]), i32(pos)).cpu().numpy().astype(np.float64)
        for b in range(2):
            assert rel_err(z[b], ref[b, pos[b]]) <= 1e-4
        pos = pos + 1


def test_greedy_next_ties_padding_nan_and_advance():
    model = make_model(TINY, 500, 4, 0)
    rng = np.random.default_rng(46)
    z = rng.standard_normal((5, TINY.vocab)).astype(np.float32)
    z[0, [17, 301]] = 9.0              # tie: lowest id
    z[1, 505] = 50.0                   # padded id (vocab_real 500): not eligible
    z[2, :] = -np.inf
    z[2, 499] = -1e30
    z[3, [7, 400]] = np.nan            # first NaN
    z[4, :] = -np.inf                  # all equal: id 0
    nxt = torch.full((5,), -7, dtype=torch.int32, device="cuda")
    pos = i32([3, 0, 9, 1, 5])
    gp.gpt2_greedy_next(model.ctx, torch.from_numpy(z).cuda(), 5, nxt, pos)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(nxt.cpu().numpy(), greedy_next(z.astype(np.float64), 500))
    np.testing.assert_array_equal(pos.cpu().numpy(), [4, 1, 10, 2, 6])


def test_graph_captured_decode_loop_matches_eager():
    oc = HD64
    model = make_model(oc, oc.vocab, 4, 0)
    load_params(model, params_for(oc, seed=47), oc)
    tok, _ = inputs.uniform_tokens(4, oc.n_ctx, oc.vocab, seed=48)
    plen = i32([5, 9, 1, 30])

    def run(graph):
        cache = gp.KVCache(model, 4, oc.n_ctx)
        cache.prefill(i32(tok), plen)
        outs = []
        if graph:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                cache.step()          # warm-up outside the capture (sets kernel attributes)
                cache.greedy_advance()
            torch.cuda.current_stream().wait_stream(s)
            cache.prefill(i32(tok), plen)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                cache.step()
                cache.greedy_advance()
            for _ in range(5):
                g.replay()
                outs.append((cache.logits.clone(), cache.tokens.clone()))
        else:
            for _ in range(5):
                cache.step()
                cache.greedy_advance()
                outs.append((cache.logits.clone(), cache.tokens.clone()))
        torch.cuda.synchronize()
        return outs

    eager, graphed = run(False), run(True)
    for (ze, te), (zg, tg) in zip(eager, graphed):
        assert torch.equal(ze, zg) and torch.equal(te, tg)
    assert model.status() == 0


def test_out_of_range_position_and_token_are_flagged():
    model = make_model(TINY, 500, 2, 0)
    load_params(model, params_for(TINY, seed=49), TINY)
    cache = gp.KVCache(model, 2, 16)
    cache.step(i32([3, 4]), i32([0, 16]))          # position == max_len
    torch.cuda.synchronize()
    assert model.status() == gp.ERRORS_BY_NAME["GPT2_ERR_POSITION_RANGE"]
    cache.step(i32([3, 500]), i32([0, 1]))         # id == vocab_real
    torch.cuda.synchronize()
    assert model.status() == gp.ERRORS_BY_NAME["GPT2_ERR_TOKEN_RANGE"]
    cache.step(i32([3, 4]), i32([1, 2]))
    torch.cuda.synchronize()
    assert model.status() == 0
    tok = torch.zeros(2, TINY.n_ctx, dtype=torch.int32, device="cuda")
    cache.prefill(tok, i32([0, 3]))                # empty prompt
    torch.cuda.synchronize()
    assert model.status() == gp.ERRORS_BY_NAME["GPT2_ERR_POSITION_RANGE"]


def test_invalid_cache_arguments():
    model = make_model(TINY, 500, 4, 0)
    assert gp.gpt2_kv_cache_bytes(model.cfg, 17, 8) == 0
    assert gp.gpt2_kv_cache_bytes(model.cfg, 2, TINY.n_ctx + 1) == 0
    cache = gp.KVCache(model, 2, 8)
    # each of these is rejected on the host before any launch: a larger
    # (batch, max_len) than the buffer holds, a misaligned buffer, a too-short one
    with pytest.raises(gp.Gpt2Error):
        gp.gpt2_decode_step(model.ctx, cache.buf, 2, 9, cache.tokens, cache.pos, cache.logits)
    with pytest.raises(gp.Gpt2Error):
        gp.gpt2_decode_step(model.ctx, cache.buf, 3, 8, cache.tokens, cache.pos, cache.logits)
    with pytest.raises(gp.Gpt2Error):
        gp.gpt2_decode_step(model.ctx, cache.buf[256:], 2, 8, cache.tokens, cache.pos, cache.logits)
    with pytest.raises(gp.Gpt2Error):
        gp.gpt2_decode_step(model.ctx, cache.buf[1:], 2, 8, cache.tokens, cache.pos, cache.logits)


def test_full_size_decode_in_bench_configuration():
    # GPT-2 124M, batch 8 after 128-token prompts (the bench's decode workload
    # and kernel variants), two teacher-forced steps: every row's logits
    # against the oracle forward over the same prefix
    from oracle_fixtures import GPT2_124M
    mc = gp.ModelConfig(12, 768, 12, 1024, 50257, 50304, 8, 0)
    model = gp.GPT2(mc)
    model.init_params(seed=0)
    p32 = oracle.unflatten(model.master.double().cpu().numpy(), GPT2_124M)
    B, P = 8, 128
    tok = inputs.zipf_tokens(B, 1024, n_ids=50257, seed=777)[0]
    cache = gp.KVCache(model, B, 1024)
    cache.prefill(i32(tok), i32(np.full(B, P)))
    for t in (P, P + 1):
        z = cache.step(i32(tok[:, t]), i32(np.full(B, t))).cpu().numpy().astype(np.float64)
    n = P + 2  # the logits after positions 0 .. n-1
    ref = forward(p32, GPT2_124M, tok[:, :n], np.full((B, n), G.IGNORE))[1]["z"][:, n - 1]
    for b in range(B):
        assert rel_err(z[b], ref[b]) <= 2e-2, b
    torch.cuda.synchronize()
    assert model.status() == 0


def test_full_size_training_forward_sampled_logits():
    # the training forward in the bench's launch configuration (GPT-2 124M,
    # 16 x 1024 tokens, all 12 layers) read through prefill: each row's logits
    # at one position against the oracle forward over that row's prefix
    # (causality: positions <= p depend on tokens 0..p only)
    from oracle_fixtures import GPT2_124M
    mc = gp.ModelConfig(12, 768, 12, 1024, 50257, 50304, 16, 0)
    model = gp.GPT2(mc)
    model.init_params(seed=3)
    p32 = oracle.unflatten(model.master.double().cpu().numpy(), GPT2_124M)
    B = 16
    tok = inputs.zipf_tokens(B, 1024, n_ids=50257, seed=1000)[0]
    plen = (np.arange(B, dtype=np.int32) * 3 + 5) % 48 + 1
    cache = gp.KVCache(model, B, 1024)
    z = cache.prefill(i32(tok), i32(plen)).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    assert model.status() == 0
    for b in range(B):
        n = int(plen[b])
        ref = forward(p32, GPT2_124M, tok[b:b + 1, :n], np.full((1, n), G.IGNORE))[1]["z"][0, n - 1]
        assert rel_err(z[b], ref) <= 2e-2, b


@pytest.mark.parametrize("batch", [5, 16])
def test_decode_wide_model_matches_oracle(batch):
    # d 1600 / 25 heads (the XL width): the LayerNorm staging's wide-row path
    # (rows over 1024 wide) and a 6400-deep k split in the MLP projection
    oc = Config(n_layer=1, d_model=1600, n_head=25, n_ctx=64, vocab=1024)
    params = params_for(oc, seed=51)
    model = make_model(oc, 1000, batch, 0)
    p32 = load_params(model, params, oc)
    max_len = 48
    plen = (np.arange(batch, dtype=np.int32) * 5) % 20 + 1
    tok, _ = inputs.uniform_tokens(batch, oc.n_ctx, 1000, seed=52)
    cache = gp.KVCache(model, batch, max_len)
    z = cache.prefill(i32(tok), i32(plen)).cpu().numpy().astype(np.float64)
    ref_cache = kv_cache_empty(oc, batch, max_len)
    assert rel_err(z, prefill(p32, oc, ref_cache, tok, plen)) <= 2e-2
    pos = plen.copy()
    for step in range(3):
        t_step = inputs.uniform_tokens(batch, 1, 1000, seed=200 + step)[0][:, 0]
        z = cache.step(i32(t_step), i32(pos)).cpu().numpy().astype(np.float64)
        assert rel_err(z, decode_step(p32, oc, ref_cache, t_step, pos)) <= 2e-2, step
        pos = pos + 1
    torch.cuda.synchronize()
    assert model.status() == 0


def test_decode_step_launch_count_and_repeatability():
    # one decode step = embedding, 5 kernels per layer (LN1 + QKV, attention,
    # attention projection, LN2 + fc, MLP projection), LN_f + LM head; every
    # sum in a fixed order, so the same step on the same cache is bitwise the same
    oc = Config(n_layer=2, d_model=128, n_head=2, n_ctx=64, vocab=1024)
    params = params_for(oc, seed=71)
    model = make_model(oc, 1000, 4, 0)
    load_params(model, params, oc)
    tok, _ = inputs.uniform_tokens(4, oc.n_ctx, 1000, seed=72)
    plen = np.array([3, 9, 1, 20], dtype=np.int32)
    cache = gp.KVCache(model, 4, 48)
    cache.prefill(i32(tok), i32(plen))
    t_step = i32(tok[:, 30])
    l0 = gp.gpt2_kernel_launches()
    a = cache.step(t_step, i32(plen)).clone()
    assert gp.gpt2_kernel_launches() - l0 == 2 + 5 * oc.n_layer
    b = cache.step(t_step, i32(plen)).clone()  # the same cache rows rewritten with the same values
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert model.status() == 0


@pytest.mark.parametrize("batch", [1, 8])
def test_tensor_core_gemv_matches_cuda_core_gemv_and_oracle(batch):
    # bf16 at up to 8 rows the decode GEMVs run on the tensor cores;
    # GPT2_DECODE_GEMV=simt selects the CUDA-core kernel.  Both against the
    # oracle's cache decoder and against each other (they differ only in
    # summation order) over steps with the rows at different positions.
    import os
    oc = Config(n_layer=2, d_model=256, n_head=4, n_ctx=128, vocab=2048)
    vocab_real = 2000
    params = params_for(oc, seed=61)
    model = make_model(oc, vocab_real, batch, 0)
    p32 = load_params(model, params, oc)
    max_len = 64
    plen = (np.arange(batch, dtype=np.int32) * 7) % 30 + 1
    tok, _ = inputs.uniform_tokens(batch, oc.n_ctx, vocab_real, seed=62)
    out = {}
    for kind in ("mma", "simt"):
        old = os.environ.pop("GPT2_DECODE_GEMV", None)
        if kind == "simt":
            os.environ["GPT2_DECODE_GEMV"] = "simt"
        try:
            cache = gp.KVCache(model, batch, max_len)
            cache.prefill(i32(tok), i32(plen))
            pos, zs = plen.copy(), []
            for step in range(4):
                t_step = inputs.uniform_tokens(batch, 1, vocab_real, seed=300 + step)[0][:, 0]
                zs.append(cache.step(i32(t_step), i32(pos)).cpu().numpy().astype(np.float64))
                pos = pos + 1
            torch.cuda.synchronize()
        finally:
            os.environ.pop("GPT2_DECODE_GEMV", None)
            if old is not None:
                os.environ["GPT2_DECODE_GEMV"] = old
        assert model.status() == 0
        out[kind] = zs
    ref_cache = kv_cache_empty(oc, batch, max_len)
    prefill(p32, oc, ref_cache, tok, plen)
    pos = plen.copy()
    for step in range(4):
        t_step = inputs.uniform_tokens(batch, 1, vocab_real, seed=300 + step)[0][:, 0]
        z_ref = decode_step(p32, oc, ref_cache, t_step, pos)
        assert rel_err(out["mma"][step], z_ref) <= 2e-2, step
        assert rel_err(out["simt"][step], z_ref) <= 2e-2, step
        assert rel_err(out["mma"][step], out["simt"][step]) <= 5e-3, step
        pos = pos + 1
