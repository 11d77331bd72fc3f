"""The allocation-free attention backward, for callers that cannot allocate
device memory (a plug-in host that passes only input/output buffers, a runtime
whose caching allocator holds the device memory, a loop that cannot afford
cudaMalloc's synchronisation): it keeps its scratch in an array compiled into
the library.  Called through the C ABI, twice in a row (the second call sees
the first call's leftovers in the shared array), it must agree with the entry
point that takes caller scratch, within the attention tests' tolerance."""
import numpy as np
import pytest
import torch

import decoder_only_transformer_step_b200 as gp

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
    for _ in range(2):
        got = torch.full((B * T, 3 * d), float("nan"), dtype=torch.bfloat16, device="cuda")
        gp.gpt2_op_attention_bwd_bf16_noalloc(qkv, o, lse, dout, got, B, T, H, hd)
        torch.cuda.synchronize()
        _compare(got, ref)


def test_noalloc_rejects_problems_beyond_its_scratch():
    B, T, H, hd = 64, 1024, 12, 64          # needs ~51 M floats > the 4 M-float array
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(gp.Gpt2Error) as e:
        gp.gpt2_op_attention_bwd_bf16_noalloc(x, x, f, x, x, B, T, H, hd)
    assert e.value.code == -9
