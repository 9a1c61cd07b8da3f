// SIMT GEMM (fp32 FFMA) used by the fp32 precision mode, where tf32/bf16
// tensor-core rounding would break the 1e-4 parity bar.  Computes
// C[M,N] = A(M x K) . B(N x K)^T for any operand majorness, with the shared
// epilogue (bias, residual, GELU, GELU', fp32 / split-K fp32 outputs).
#include "launch.h"

#define SG_BM 64
#define SG_BN 64
#define SG_BK 16

template <typename T>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(int M, int N, int K, const T* __restrict__ A, long lda, bool a_t, const T* __restrict__ B,
                 long ldb, bool b_t, EpiParams<T> epi, int kchunk) {
  __shared__ float As[SG_BK][SG_BM + 4];
  __shared__ float Bs[SG_BK][SG_BN + 4];
  int bm = blockIdx.y * SG_BM, bn = blockIdx.x * SG_BN;
  int split = blockIdx.z;
  int k0 = split * kchunk, k1 = min(K, k0 + kchunk);
  int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int kt = k0; kt < k1; kt += SG_BK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int e = threadIdx.x + i * 256;
      int r, kk;
      if (!a_t) { r = e / SG_BK; kk = e % SG_BK; } else { kk = e / SG_BM; r = e % SG_BM; }
      int gm = bm + r, gk = kt + kk;
      float v = 0.f;
      if (gm < M && gk < k1) v = to_f(a_t ? A[(long)gk * lda + gm] : A[(long)gm * lda + gk]);
      As[kk][r] = v;
      if (!b_t) { r = e / SG_BK; kk = e % SG_BK; } else { kk = e / SG_BN; r = e % SG_BN; }
      int gn = bn + r;
      gk = kt + kk;
      v = 0.f;
      if (gn < N && gk < k1) v = to_f(b_t ? B[(long)gk * ldb + gn] : B[(long)gn * ldb + gk]);
      Bs[kk][r] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int m = bm + ty * 4 + i, n = bn + tx + 16 * j;
      if (m < M && n < N) epi_apply1<T>(epi, m, n, acc[i][j], split);
    }
}

template <typename T>
cudaError_t launch_gemm_simt(int M, int N, int K, const T* A, long lda, bool a_t, const T* B, long ldb,
                             bool b_t, const EpiParams<T>& epi, int splits, cudaStream_t s) {
  if (splits < 1) splits = 1;
  int kchunk = (K + splits - 1) / splits;
  kchunk = ((kchunk + SG_BK - 1) / SG_BK) * SG_BK;
  splits = (K + kchunk - 1) / kchunk;
  if (splits < 1) splits = 1;
  dim3 grid((N + SG_BN - 1) / SG_BN, (M + SG_BM - 1) / SG_BM, splits);
  ++g_kernel_launches;
  gemm_simt_kernel<T><<<grid, 256, 0, s>>>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, kchunk);
  return cudaGetLastError();
}

template cudaError_t launch_gemm_simt<float>(int, int, int, const float*, long, bool, const float*, long, bool,
                                             const EpiParams<float>&, int, cudaStream_t);
template cudaError_t launch_gemm_simt<bf16>(int, int, int, const bf16*, long, bool, const bf16*, long, bool,
                                            const EpiParams<bf16>&, int, cudaStream_t);
template cudaError_t launch_gemm_simt<f16>(int, int, int, const f16*, long, bool, const f16*, long, bool,
                                           const EpiParams<f16>&, int, cudaStream_t);
