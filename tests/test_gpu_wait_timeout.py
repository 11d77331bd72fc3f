"""Hang detection on the GPU, without hanging it: every pipeline wait of the
tcgen05 kernels gives up after a limit and reports GPT2_ERR_TIMEOUT in a
device status word.  With the limit set to one nanosecond every wait that is
not already satisfied (after the hardware's own short suspension inside one
try-wait) gives up, so a long GEMM takes the abort path (copies and
MMAs in flight are drained, tensor memory is freed, the kernel returns);
afterwards, with the default limit, the same call on the same context
computes the right result."""
import numpy as np
import pytest
import torch

import decoder_only_transformer_step_b200 as gp

pytestmark = pytest.mark.gpu

DEV_ERR_TIMEOUT = 4


def _operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    return A, B


@pytest.mark.parametrize("bn", [256, 128])
def test_timeout_is_reported_and_the_context_recovers(bn):
    # single-CTA tiles with a 1024-k-block loop (about 0.3 ms of MMAs per
    # tile): the epilogue's wait for the accumulator cannot complete inside
    # the hardware's own suspension of a single try-wait
    M, N, K = 256, 256, 65536
    A, B = _operands(M, N, K, 7 + bn)
    C = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        gp.gpt2_set_wait_timeout_ns(1)
        gp.gpt2_op_gemm_bf16_status(A, 0, K, B, 0, K, C, 0, N, M, N, K, bn=bn, splits=1, status=status)
        torch.cuda.synchronize()
    finally:
        gp.gpt2_set_wait_timeout_ns(0)
    assert int(status.item()) & DEV_ERR_TIMEOUT
    status.zero_()
    gp.gpt2_op_gemm_bf16_status(A, 0, K, B, 0, K, C, 0, N, M, N, K, bn=bn, splits=1, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = A.float() @ B.float().t()
    assert (C.float() - ref).abs().max().item() <= 1e-2 * ref.abs().max().item()
