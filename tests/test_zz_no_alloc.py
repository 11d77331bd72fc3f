"""The allocation-free attention backward, for callers that cannot allocate
device memory (a plug-in host that passes only input/output buffers, a runtime
whose caching allocator holds the device memory, a loop that cannot afford
cudaMalloc's synchronisation): it keeps its scratch in an array compiled into
the library.  Called through the C ABI, twice in a row (the second call sees
the first call's leftovers in the shared array), it must agree with the entry
point that takes caller scratch, and with the oracle's attention backward on
the same bf16 inputs, within the attention tests' tolerance."""
import numpy as np
import pytest
import torch

import decoder_only_transformer_step_b200 as gp
from oracle import gpt2_oracle as G

pytestmark = pytest.mark.gpu


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).cuda()


def _compare(got, ref):
    g = got.double().cpu().numpy().ravel()
    r = ref.double().cpu().numpy().ravel()
    cos = float(g @ r / (np.linalg.norm(g) * np.linalg.norm(r)))
    rel = float(np.abs(g - r).max() / np.abs(r).max())
    assert cos >= 0.999 and rel <= 2e-2, (cos, rel)


@pytest.mark.parametrize("hd,T", [(64, 200), (16, 77)])
def test_noalloc_matches_scratch_entry_point(hd, T):
    B, H = 2, 3
    d = H * hd
    qkv = _rand((B * T, 3 * d), 1)
    dout = _rand((B * T, d), 2)
    o = torch.empty((B * T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    gp.gpt2_op_attention_fwd_bf16(qkv, o, lse, B, T, H, hd)
    ref = torch.empty((B * T, 3 * d), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(B * T * d + B * H * T, dtype=torch.float32, device="cuda")
    gp.gpt2_op_attention_bwd_bf16(qkv, o, lse, dout, ref, scratch, B, T, H, hd)
    x = qkv.double().cpu().numpy().reshape(B, T, 3, H, hd)
    q, k, v = [x[:, :, i].transpose(0, 2, 1, 3) for i in range(3)]
    _, p = G.attention_fwd(q, k, v, None)
    do = dout.double().cpu().numpy().reshape(B, T, H, hd).transpose(0, 2, 1, 3)
    dq, dk, dv = G.attention_bwd(do, q, k, v, p, None)
    oracle_dqkv = np.stack([dq, dk, dv], 2).transpose(0, 3, 2, 1, 4).reshape(B * T, 3 * d)
    for _ in range(2):
        got = torch.full((B * T, 3 * d), float("nan"), dtype=torch.bfloat16, device="cuda")
        gp.gpt2_op_attention_bwd_bf16_noalloc(qkv, o, lse, dout, got, B, T, H, hd)
        torch.cuda.synchronize()
        _compare(got, ref)
        _compare(got, torch.from_numpy(oracle_dqkv))


def test_noalloc_rejects_problems_beyond_its_scratch():
    # the smallest supported shape past the 4 Mi-float array: 4096 * 16 * 64
    # + 16 * 4096 floats.  Every buffer has its true size, so if the host-side
    # size check ever regressed the call would compute on valid memory and
    # this test would fail on its assertion, not on a memory fault.
    B, T, H, hd = 1, 4096, 16, 64
    d = H * hd
    qkv = torch.zeros((B * T, 3 * d), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros((B * T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, H, T), dtype=torch.float32, device="cuda")
    dout = torch.zeros((B * T, d), dtype=torch.bfloat16, device="cuda")
    dqkv = torch.zeros((B * T, 3 * d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gp.Gpt2Error) as e:
        gp.gpt2_op_attention_bwd_bf16_noalloc(qkv, o, lse, dout, dqkv, B, T, H, hd)
    assert e.value.code == gp.ERRORS_BY_NAME["GPT2_ERR_TOO_LARGE"]
