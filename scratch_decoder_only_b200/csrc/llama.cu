// Kernels of the Llama-style block ("NTransformer" page, "key features":
// Llama architecture with RoPE, GQA, SwiGLU, KV cache): rotary positions on
// the query and key heads, the SwiGLU activation and its gradient, and the
// sum of the per-query-head key / value gradients over the query heads that
// share a key / value head.  All are HBM-bound elementwise passes with
// 16-byte accesses of 16-bit (bf16 or fp16) tensors.
#include "launch.h"

// Rotary positions, in place.  Row r of x (row stride ld) holds nq query
// heads at columns [0, nq d) and nk key heads at [kcol, kcol + nk d); the
// consecutive pair (2i, 2i+1) of a head is rotated by the angle of the row's
// position p: (x0, x1) -> (x0 c - x1 s, x0 s + x1 c) with (c, s) =
// tab[p][i] (cos, sin of p * base^(-2i/d), tabulated in double precision on
// the host).  inverse: rotate by -angle (the transpose, for gradients).
// Position p = pos[r], or pos0 + *step when pos is null (one decode step).
template <typename T>
__global__ void rope_kernel(T* __restrict__ x, long ld, int rows, int nq, int kcol, int nk, int d,
                            const int* __restrict__ pos, int pos0, const int* __restrict__ step,
                            const float2* __restrict__ tab, int max_seq, int inverse) {
  griddep_wait();
  griddep_release();
  const int cpr = (nq + nk) * d / 8;   // 8-element chunks per row
  const long n = (long)rows * cpr;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const int r = (int)(i / cpr), c = (int)(i % cpr);
    const int e = c * 8;                  // element within the (q heads | k heads) span
    const int qspan = nq * d;
    const long col = e < qspan ? e : kcol + (e - qspan);
    const int within = (e < qspan ? e : e - qspan) % d;   // first dimension of the chunk inside its head
    int p = pos ? pos[r] : pos0 + *step;
    p = p < 0 ? 0 : (p >= max_seq ? max_seq - 1 : p);
    T* px = x + (long)r * ld + col;
    float v[8];
    Vec<T>::load(px, v);
    const float2* tr = tab + (long)p * (d / 2) + within / 2;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 cs = tr[k];
      const float sn = inverse ? -cs.y : cs.y;
      const float a = v[2 * k], b = v[2 * k + 1];
      v[2 * k] = a * cs.x - b * sn;
      v[2 * k + 1] = a * sn + b * cs.x;
    }
    Vec<T>::store(px, v);
  }
}

template <typename T>
cudaError_t launch_rope(T* x, long ld, int rows, int nq, int kcol, int nk, int d, const int* pos, int pos0,
                        const int* step, const float2* tab, int max_seq, bool inverse, cudaStream_t s) {
  if (d % 8 || (ld % 8) || (kcol % 8)) return cudaErrorInvalidValue;
  const long n = (long)rows * (nq + nk) * d / 8;
  long blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  ++g_kernel_launches;
  return launch_k(rope_kernel<T>, dim3((unsigned)blocks), dim3(256), 0, s, x, ld, rows, nq, kcol, nk, d, pos, pos0,
                  step, tab, max_seq, inverse ? 1 : 0);
}

// SwiGLU: a[r, f] = silu(gu[r, f]) * gu[r, F + f], silu(z) = z / (1 + e^-z);
// gu holds the gate half then the up half of each row (the two GEMM outputs
// as stored, 16-bit), a is rounded once.
__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

template <typename T>
__global__ void swiglu_fwd_kernel(const T* __restrict__ gu, T* __restrict__ a, int rows, int F) {
  griddep_wait();
  griddep_release();
  const int cpr = F / 8;
  const long n = (long)rows * cpr;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const long r = i / cpr;
    const int f = (int)(i % cpr) * 8;
    float g[8], u[8], o[8];
    Vec<T>::load(gu + r * 2 * F + f, g);
    Vec<T>::load(gu + r * 2 * F + F + f, u);
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = silu_f(g[k]) * u[k];
    Vec<T>::store(a + r * F + f, o);
  }
}

// Its gradient: dgate = da * up * silu'(gate), dup = da * silu(gate), with
// silu'(z) = s (1 + z (1 - s)), s = 1 / (1 + e^-z); written as [dgate | dup].
template <typename T>
__global__ void swiglu_bwd_kernel(const T* __restrict__ da, const T* __restrict__ gu, T* __restrict__ dgu, int rows,
                                  int F) {
  const int cpr = F / 8;
  const long n = (long)rows * cpr;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const long r = i / cpr;
    const int f = (int)(i % cpr) * 8;
    float d[8], g[8], u[8], dg[8], du[8];
    Vec<T>::load(da + r * F + f, d);
    Vec<T>::load(gu + r * 2 * F + f, g);
    Vec<T>::load(gu + r * 2 * F + F + f, u);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float sg = 1.0f / (1.0f + __expf(-g[k]));
      dg[k] = d[k] * u[k] * sg * (1.0f + g[k] * (1.0f - sg));
      du[k] = d[k] * g[k] * sg;
    }
    Vec<T>::store(dgu + r * 2 * F + f, dg);
    Vec<T>::store(dgu + r * 2 * F + F + f, du);
  }
}

template <typename T>
cudaError_t launch_swiglu(const T* gu, T* a, int rows, int F, cudaStream_t s) {
  if (F % 8) return cudaErrorInvalidValue;
  const long n = (long)rows * F / 8;
  long blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  ++g_kernel_launches;
  return launch_k(swiglu_fwd_kernel<T>, dim3((unsigned)blocks), dim3(256), 0, s, gu, a, rows, F);
}

template <typename T>
cudaError_t launch_swiglu_bwd(const T* da, const T* gu, T* dgu, int rows, int F, cudaStream_t s) {
  if (F % 8) return cudaErrorInvalidValue;
  const long n = (long)rows * F / 8;
  long blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  ++g_kernel_launches;
  swiglu_bwd_kernel<T><<<(unsigned)blocks, 256, 0, s>>>(da, gu, dgu, rows, F);
  return cudaGetLastError();
}

// Key / value head gradients of grouped attention: the attention backward
// writes one key and one value gradient per query head into kvq [rows, 2 H d]
// (keys, then values); key / value head j receives the sum over its G query
// heads jG .. jG+G-1 (fixed order), written to dkv [rows, ld] at columns
// [kcol, kcol + Hkv d) and [vcol, vcol + Hkv d).
template <typename T>
__global__ void gqa_reduce_kernel(const T* __restrict__ kvq, T* __restrict__ dkv, long ld, int kcol, int vcol,
                                  int rows, int Hkv, int G, int d) {
  const int H = Hkv * G;
  const int cpr = 2 * Hkv * d / 8;
  const long n = (long)rows * cpr;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const long r = i / cpr;
    const int e = (int)(i % cpr) * 8;
    const int part = e / (Hkv * d);          // 0 keys, 1 values
    const int j = (e % (Hkv * d)) / d, w = e % d;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int g = 0; g < G; ++g) {
      float v[8];
      Vec<T>::load(kvq + r * 2 * H * d + part * H * d + (j * G + g) * d + w, v);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] += v[k];
    }
    Vec<T>::store(dkv + r * ld + (part ? vcol : kcol) + j * d + w, acc);
  }
}

template <typename T>
cudaError_t launch_gqa_reduce(const T* kvq, T* dkv, long ld, int kcol, int vcol, int rows, int Hkv, int G, int d,
                              cudaStream_t s) {
  if (d % 8 || ld % 8 || kcol % 8 || vcol % 8) return cudaErrorInvalidValue;
  const long n = (long)rows * 2 * Hkv * d / 8;
  long blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  ++g_kernel_launches;
  gqa_reduce_kernel<T><<<(unsigned)blocks, 256, 0, s>>>(kvq, dkv, ld, kcol, vcol, rows, Hkv, G, d);
  return cudaGetLastError();
}

#define INSTL(T)                                                                                            \
  template cudaError_t launch_rope<T>(T*, long, int, int, int, int, int, const int*, int, const int*,       \
                                      const float2*, int, bool, cudaStream_t);                              \
  template cudaError_t launch_swiglu<T>(const T*, T*, int, int, cudaStream_t);                             \
  template cudaError_t launch_swiglu_bwd<T>(const T*, const T*, T*, int, int, cudaStream_t);               \
  template cudaError_t launch_gqa_reduce<T>(const T*, T*, long, int, int, int, int, int, int, cudaStream_t);
INSTL(bf16)
INSTL(f16)
