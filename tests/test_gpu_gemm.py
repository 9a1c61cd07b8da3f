"""The tcgen05 GEMM alone, per operand layout, against a plain fp64 matmul of
the same bf16-rounded operands (sizes span several 128 x 256 tiles, ragged
tails in every dimension and K tails shorter than one 64-wide k-block)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

SHAPES = [(128, 256, 64), (300, 200, 136), (1000, 768, 3072), (257, 50304 // 8, 768), (64, 8, 24)]


def _operand(g, rows, cols):
    """bf16 [rows, cols] stored with a row stride rounded up to 8 (16 bytes);
    the padding holds NaN so a read of it would show."""
    import torch
    ld = (cols + 7) // 8 * 8
    X = torch.full((rows, ld), float("nan"), dtype=torch.bfloat16)
    X[:, :cols] = torch.randn((rows, cols), generator=g).to(torch.bfloat16)
    return X, ld


@pytest.mark.parametrize("a_t,b_t", [(False, False), (False, True), (True, True), (True, False)])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_layouts(M, N, K, a_t, b_t):
    import torch
    from scratch_decoder_only_b200.gpt import gemm_bf16
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    A, lda = _operand(g, *((K, M) if a_t else (M, K)))
    B, ldb = _operand(g, *((K, N) if b_t else (N, K)))
    C = gemm_bf16(A.cuda(), B.cuda(), a_t, b_t, M=M, N=N, K=K, lda=lda, ldb=ldb).cpu().numpy()
    a = A.float().numpy().astype(np.float64)
    b = B.float().numpy().astype(np.float64)
    a = a[:, :M].T if a_t else a[:, :K]
    b = b[:, :N].T if b_t else b[:, :K]
    ref = a @ b.T
    assert np.isfinite(C).all()
    # fp32 accumulation in the tensor core: ~2^-15 relative on sums of K unit
    # products (|sum| ~ sqrt(K)); a wrong layout or index gives O(1) errors
    err = np.abs(C - ref).max() / np.sqrt(K)
    assert err <= 1e-4, (err, np.argwhere(np.abs(C - ref) > 1e-2)[:5])


def test_gemm_padded_leading_dimension():
    import torch
    from scratch_decoder_only_b200.gpt import gemm_bf16
    M, N, K, ld = 200, 136, 257, 264        # K = 257 columns inside rows of 264
    g = torch.Generator().manual_seed(1)
    A = torch.randn((M, ld), generator=g).to(torch.bfloat16)
    A[:, K:] = float("nan")                 # padding must never be read
    B = torch.randn((N, ld), generator=g).to(torch.bfloat16)
    B[:, K:] = float("nan")
    C = gemm_bf16(A.cuda(), B.cuda(), False, False, M=M, N=N, K=K, lda=ld, ldb=ld).cpu().numpy()
    ref = A[:, :K].double().numpy() @ B[:, :K].double().numpy().T
    assert np.isfinite(C).all()
    assert np.abs(C - ref).max() <= 2e-5 * np.sqrt(K) * 4
