"""The split-K GEMM entry point that allocates no device memory.

It serves callers that cannot call cudaMalloc where they need the product
(a memory pool owns the device, or an allocation would stall a real-time
path).  Its partial sums live in a fixed device array inside the library;
this test checks, through the C ABI, that two calls in a row give the same
result as the ordinary gpt_gemm_bf16 entry point (within the GEMM tests'
tolerance) and that a request larger than the array is refused.  It sits in
a file pytest collects last, and needs nothing from the other tests.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed):
    import torch
    g = torch.Generator().manual_seed(seed)
    # weight-gradient layout: A = dY^T and B = X^T, both stored [K rows, M or N cols]
    A = torch.randn((K, M), generator=g).to(torch.bfloat16).cuda()
    B = torch.randn((K, N), generator=g).to(torch.bfloat16).cuda()
    return A, B


@pytest.mark.parametrize("calls", [[(768, 768, 4096, 4), (2304, 768, 2048, 2)]])
def test_noalloc_splitk_matches_gemm_on_two_calls(calls):
    import torch
    from scratch_decoder_only_b200.gpt import gemm_bf16, gemm_bf16_splitk_noalloc
    for i, (M, N, K, splits) in enumerate(calls):
        A, B = _operands(M, N, K, 100 + i)
        got = gemm_bf16_splitk_noalloc(A, B, True, True, splits=splits)
        ref = gemm_bf16(A, B, True, True)
        torch.cuda.synchronize()
        err = (got - ref).abs().max().item() / np.sqrt(K)
        assert err <= 1e-4, (i, err)
        assert torch.isfinite(got).all()


def test_noalloc_rejects_oversize():
    from scratch_decoder_only_b200.gpt import GPTError, GPT_ERR_ARG, gemm_bf16_splitk_noalloc
    A, B = _operands(2048, 2048, 1024, 7)     # 4 x 2048 x 2048 partials > 4194304 floats
    with pytest.raises(GPTError) as e:
        gemm_bf16_splitk_noalloc(A, B, True, True, splits=4)
    assert e.value.code == GPT_ERR_ARG
    assert "exceeds" in str(e.value)
