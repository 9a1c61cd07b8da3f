"""The split-K GEMM entry point that allocates no device memory.

It serves callers that cannot call cudaMalloc where they need the product
(a memory pool owns the device, or an allocation would stall a real-time
path).  Its partial sums live in a fixed device array inside the library.
Through the C ABI this file checks, on several calls in a row:

* each result against the fp64 product of the same bf16 operands (computed
  on the host, independent of every GPU kernel) and against the ordinary
  gpt_gemm_bf16 entry point, within the GEMM tests' tolerance;
* a call whose split count is reduced (too few k-blocks for the asked
  splits), a ragged call (M, N not multiples of the tile) and an N that is not
  a multiple of 4, each made right after a larger call, so leftover partials
  of the earlier call in the shared array would show up;
* that a request larger than the array is refused, and that the sticky
  status reads GPT_OK after calls whose waits all completed.

It sits in a file pytest collects last and needs nothing from other tests.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed):
    import torch
    g = torch.Generator().manual_seed(seed)
    # weight-gradient layout: A = dY^T and B = X^T, both stored [K rows, M or N
    # cols] with row strides rounded up to 8 elements (16 bytes, as TMA wants)
    A = torch.randn((K, (M + 7) // 8 * 8), generator=g).to(torch.bfloat16)
    B = torch.randn((K, (N + 7) // 8 * 8), generator=g).to(torch.bfloat16)
    return A, B


def _fp64_product(A, B, M, N):
    a = A.double().numpy()[:, :M]
    b = B.double().numpy()[:, :N]
    return a.T @ b           # C[m, n] = sum_k A[k, m] * B[k, n]


# (M, N, K, splits): a long-K call, a second long-K call, then a call whose
# splits get reduced (K = 192 is three k-blocks), a ragged call and an N that
# is not a multiple of 4, each after a larger one
CALLS = [(768, 768, 4096, 4), (2304, 768, 2048, 2), (256, 320, 192, 16), (200, 136, 1000, 3), (130, 66, 513, 2)]
# (the last call's operands are stored with row strides 136 and 72)


def test_noalloc_splitk_matches_fp64_and_gemm_on_calls_in_a_row():
    import torch
    from scratch_decoder_only_b200.gpt import GPT_OK, gemm_bf16, gemm_bf16_splitk_noalloc, noalloc_status
    for i, (M, N, K, splits) in enumerate(CALLS):
        A, B = _operands(M, N, K, 100 + i)
        Ad, Bd = A.cuda(), B.cuda()
        got = gemm_bf16_splitk_noalloc(Ad, Bd, True, True, splits=splits, M=M, N=N, K=K)
        torch.cuda.synchronize()
        want = _fp64_product(A, B, M, N)
        g = got.double().cpu().numpy()
        assert np.all(np.isfinite(g)), i
        # products of bf16 values are exact in fp32; the fp32 sums of K of them
        # stay within a few ulp of sqrt(K)-sized results
        err = np.max(np.abs(g - want)) / np.sqrt(K)
        assert err <= 1e-4, (i, err)
        if N % 8 == 0 and M % 8 == 0:
            ref = gemm_bf16(Ad, Bd, True, True)
            torch.cuda.synchronize()
            assert (got - ref).abs().max().item() / np.sqrt(K) <= 1e-4, i
    assert noalloc_status() == GPT_OK


def test_noalloc_rejects_oversize():
    from scratch_decoder_only_b200.gpt import GPTError, GPT_ERR_ARG, gemm_bf16_splitk_noalloc
    A, B = _operands(2048, 2048, 1024, 7)     # 4 x 2048 x 2048 partials > 4194304 floats
    with pytest.raises(GPTError) as e:
        gemm_bf16_splitk_noalloc(A.cuda(), B.cuda(), True, True, splits=4)
    assert e.value.code == GPT_ERR_ARG
    assert "exceeds" in str(e.value)
