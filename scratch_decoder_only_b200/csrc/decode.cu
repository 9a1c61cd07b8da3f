// Greedy decoding with a per-layer KV cache ("RustGPT", "Technical
// implementation": greedy decoding; "NTransformer" page, "No PyTorch, no
// cuBLAS": KV cache).  One new token per row and step: the weights are read
// once per step, so every kernel here is HBM-bound (GEMV-shaped, B <= 32).
//
// KV cache layout: kc/vc [B][H][Tmax][d] per layer.
#include "launch.h"

// pos = pos0 + *step (the step counter lives on the device so that one
// captured decode step can be replayed).
template <typename T>
__global__ void dec_embed_kernel(const int* __restrict__ tok, const float* __restrict__ wte,
                                 const float* __restrict__ wpe, T* __restrict__ x, int C, int pos0,
                                 const int* __restrict__ step, int max_seq, unsigned* err) {
  int b = blockIdx.x;
  int pos = pos0 + *step;
  if (pos < 0 || pos >= max_seq) {
    if (b == 0 && threadIdx.x == 0) set_dev_err(err, GPT_DEVERR_POS);
    pos = pos < 0 ? 0 : max_seq - 1;
  }
  const float* a = wte + (long)tok[b] * C;
  const float* p = wpe + (long)pos * C;
  for (int c = threadIdx.x; c < C; c += blockDim.x) x[(long)b * C + c] = from_f<T>(a[c] + p[c]);
}

template <typename T>
cudaError_t launch_dec_embed(const int* tok, const float* wte, const float* wpe, T* x, int B, int C, int pos0,
                             const int* step, int max_seq, unsigned* err, cudaStream_t s) {
  ++g_kernel_launches;
  dec_embed_kernel<T><<<B, 256, 0, s>>>(tok, wte, wpe, x, C, pos0, step, max_seq, err);
  return cudaGetLastError();
}

// Y[b, n] = sum_k X[b, k] W[n, k]  (+ bias, + residual / GELU / fp32 out).
// One warp per output column; X staged in shared memory (fp32) in K chunks.
// mode 0: out = T(y + bias + resid); 1: out = T(u = y + bias), out2 = T(gelu(u));
// mode 2: outf = y (fp32, no bias).
#define GEMV_WARPS 8
template <typename T, int BB>
__global__ void __launch_bounds__(GEMV_WARPS * 32)
gemv_kernel(const T* __restrict__ X, int B, int K, const T* __restrict__ W, int N,
            const float* __restrict__ bias, const T* resid, int mode, T* out, T* out2, float* outf) {
  constexpr int KC = 8192 / BB;
  constexpr int NV = Vec<T>::N;
  __shared__ __align__(16) float xs[BB * KC];
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n = blockIdx.x * GEMV_WARPS + warp;
  float acc[BB];
#pragma unroll
  for (int b = 0; b < BB; ++b) acc[b] = 0.f;
  for (int k0 = 0; k0 < K; k0 += KC) {
    int kend = min(KC, K - k0);
    __syncthreads();
    for (int i = threadIdx.x; i < B * kend; i += blockDim.x) {
      int b = i / kend, kk = i % kend;
      xs[b * KC + kk] = to_f(X[(long)b * K + k0 + kk]);
    }
    __syncthreads();
    if (n < N) {
      const T* wr = W + (long)n * K + k0;
      for (int kk = lane * NV; kk < kend; kk += 32 * NV) {
        float w[NV];
        Vec<T>::load(wr + kk, w);
#pragma unroll
        for (int b = 0; b < BB; ++b) {
          if (b < B) {
            float a = 0.f;
#pragma unroll
            for (int j = 0; j < NV; ++j) a = fmaf(w[j], xs[b * KC + kk + j], a);
            acc[b] += a;
          }
        }
      }
    }
  }
  if (n >= N) return;
#pragma unroll
  for (int b = 0; b < BB; ++b) {
    if (b < B) {
      float y = warp_sum(acc[b]);
      if (lane == 0) {
        long o = (long)b * N + n;
        if (mode == 2) {
          outf[o] = y;
        } else if (mode == 1) {
          float u = y + bias[n];
          T uq = from_f<T>(u);
          out[o] = uq;
          out2[o] = from_f<T>(gelu_f(to_f(uq)));
        } else {
          float v = y + (bias ? bias[n] : 0.f) + (resid ? to_f(resid[o]) : 0.f);
          out[o] = from_f<T>(v);
        }
      }
    }
  }
}

template <typename T>
cudaError_t launch_gemv(const T* X, int B, int K, const T* W, int N, const float* bias, const T* resid,
                        int mode, T* out, T* out2, float* outf, cudaStream_t s) {
  unsigned g = (N + GEMV_WARPS - 1) / GEMV_WARPS;
  if (B <= 1) { ++g_kernel_launches; gemv_kernel<T, 1><<<g, GEMV_WARPS * 32, 0, s>>>(X, B, K, W, N, bias, resid, mode, out, out2, outf); }
  else if (B <= 8) { ++g_kernel_launches; gemv_kernel<T, 8><<<g, GEMV_WARPS * 32, 0, s>>>(X, B, K, W, N, bias, resid, mode, out, out2, outf); }
  else if (B <= 32) { ++g_kernel_launches; gemv_kernel<T, 32><<<g, GEMV_WARPS * 32, 0, s>>>(X, B, K, W, N, bias, resid, mode, out, out2, outf); }
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

// Copy the prompt's K and V (from the prefill's qkv [B*Tp, 3C]) into the cache.
template <typename T>
__global__ void kv_fill_kernel(const T* __restrict__ qkv, T* __restrict__ kc, T* __restrict__ vc, int B, int Tp,
                               int H, int d, int Tmax) {
  int C = H * d;
  long n = (long)B * Tp * C;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    int c = i % C;
    long bt = i / C;
    int t = bt % Tp, b = bt / Tp;
    int h = c / d, e = c % d;
    long dst = (((long)b * H + h) * Tmax + t) * d + e;
    kc[dst] = qkv[bt * 3 * C + C + c];
    vc[dst] = qkv[bt * 3 * C + 2 * C + c];
  }
}

template <typename T>
cudaError_t launch_kv_fill(const T* qkv, T* kc, T* vc, int B, int Tp, int H, int d, int Tmax, cudaStream_t s) {
  ++g_kernel_launches;
  kv_fill_kernel<T><<<148 * 4, 256, 0, s>>>(qkv, kc, vc, B, Tp, H, d, Tmax);
  return cudaGetLastError();
}

// One query per (row, head) against keys 0..pos; the new key/value (at pos)
// is appended to the cache by the same warp.
template <typename T, int D>
__global__ void dec_attn_kernel(const T* __restrict__ qkv, T* kc, T* vc, T* __restrict__ out, int B, int H,
                                int Tmax, int pos0, const int* __restrict__ step) {
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int pos = pos0 + *step;
  if (pos < 0) pos = 0;
  if (pos >= Tmax) pos = Tmax - 1;
  int bh = blockIdx.x * 4 + warp;
  if (bh >= B * H) return;
  int b = bh / H, h = bh % H;
  const int C = H * D;
  const T* q = qkv + (long)b * 3 * C + h * D;
  const T* knew = q + C;
  const T* vnew = q + 2 * C;
  T* kcb = kc + (long)bh * Tmax * D;
  T* vcb = vc + (long)bh * Tmax * D;
  for (int i = lane; i < D; i += 32) {
    kcb[(long)pos * D + i] = knew[i];
    vcb[(long)pos * D + i] = vnew[i];
  }
  const float scale = 1.0f / sqrtf((float)D);
  float qv[D];
#pragma unroll
  for (int i = 0; i < D; ++i) qv[i] = to_f(q[i]) * scale;
  float mloc = -INFINITY, sloc = 0.f, acc[D];
#pragma unroll
  for (int i = 0; i < D; ++i) acc[i] = 0.f;
  for (int j = lane; j <= pos; j += 32) {
    const T* kr = j == pos ? knew : kcb + (long)j * D;
    const T* vr = j == pos ? vnew : vcb + (long)j * D;
    float sc = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) sc = fmaf(qv[i], to_f(kr[i]), sc);
    float mn = fmaxf(mloc, sc);
    float corr = expf(mloc - mn), p = expf(sc - mn);
    sloc = sloc * corr + p;
#pragma unroll
    for (int i = 0; i < D; ++i) acc[i] = acc[i] * corr + p * to_f(vr[i]);
    mloc = mn;
  }
  float mw = warp_max(mloc);
  float f = mloc == -INFINITY ? 0.f : expf(mloc - mw);
  float ssum = warp_sum(sloc * f);
#pragma unroll
  for (int i = 0; i < D; ++i) {
    float v = warp_sum(acc[i] * f);
    if ((i & 31) == lane) out[(long)b * C + h * D + i] = from_f<T>(v / ssum);
  }
}

template <typename T>
cudaError_t launch_dec_attn(const T* qkv, T* kc, T* vc, T* out, int B, int H, int d, int Tmax, int pos0,
                            const int* step, cudaStream_t s) {
  unsigned g = (B * H + 3) / 4;
  switch (d) {
    case 16: ++g_kernel_launches; dec_attn_kernel<T, 16><<<g, 128, 0, s>>>(qkv, kc, vc, out, B, H, Tmax, pos0, step); break;
    case 32: ++g_kernel_launches; dec_attn_kernel<T, 32><<<g, 128, 0, s>>>(qkv, kc, vc, out, B, H, Tmax, pos0, step); break;
    case 64: ++g_kernel_launches; dec_attn_kernel<T, 64><<<g, 128, 0, s>>>(qkv, kc, vc, out, B, H, Tmax, pos0, step); break;
    case 128: ++g_kernel_launches; dec_attn_kernel<T, 128><<<g, 128, 0, s>>>(qkv, kc, vc, out, B, H, Tmax, pos0, step); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Greedy choice: argmax over the real vocabulary of fp32 logits, lowest
// index on ties.  Writes tok[b] and out[b * out_ld + col].
__global__ void argmax_kernel(const float* __restrict__ logits, int V, int Vp, int* tok, int32_t* out,
                              int out_ld, const int* __restrict__ step) {
  int b = blockIdx.x;
  const int col = step ? *step : 0;
  const float* z = logits + (long)b * Vp;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int c = threadIdx.x; c < V; c += blockDim.x) {
    float v = z[c];
    if (v > best || (v == best && c < bi)) { best = v; bi = c; }
  }
  __shared__ float sv[32];
  __shared__ int si[32];
  for (int o = 16; o > 0; o >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, best, o);
    int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
  }
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sv[warp] = best; si[warp] = bi; }
  __syncthreads();
  if (warp == 0) {
    int nw = blockDim.x / 32;
    best = lane < nw ? sv[lane] : -INFINITY;
    bi = lane < nw ? si[lane] : 0x7fffffff;
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, best, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
    }
    if (lane == 0) {
      if (bi < 0 || bi >= V) bi = 0;   // all-NaN row: fall back to id 0
      tok[b] = bi;
      out[(long)b * out_ld + col] = bi;
    }
  }
}

cudaError_t launch_argmax(const float* logits, int B, int V, int Vp, int* tok, int32_t* out, int out_ld,
                          const int* step, cudaStream_t s) {
  ++g_kernel_launches;
  argmax_kernel<<<B, 1024, 0, s>>>(logits, V, Vp, tok, out, out_ld, step);
  return cudaGetLastError();
}

__global__ void step_advance_kernel(int* step) { *step += 1; }
cudaError_t launch_step_advance(int* step, cudaStream_t s) {
  ++g_kernel_launches;
  step_advance_kernel<<<1, 1, 0, s>>>(step);
  return cudaGetLastError();
}

template <typename T>
__global__ void gather_last_kernel(const T* __restrict__ x, int Tp, int C, T* __restrict__ out) {
  int b = blockIdx.x;
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    out[(long)b * C + c] = x[((long)b * Tp + Tp - 1) * C + c];
}
template <typename T>
cudaError_t launch_gather_last(const T* x, int B, int Tp, int C, T* out, cudaStream_t s) {
  ++g_kernel_launches;
  gather_last_kernel<T><<<B, 256, 0, s>>>(x, Tp, C, out);
  return cudaGetLastError();
}

#define INSTD(T)                                                                                         \
  template cudaError_t launch_dec_embed<T>(const int*, const float*, const float*, T*, int, int, int,      \
                                           const int*, int, unsigned*, cudaStream_t);                    \
  template cudaError_t launch_gemv<T>(const T*, int, int, const T*, int, const float*, const T*, int, T*, T*, \
                                      float*, cudaStream_t);                                             \
  template cudaError_t launch_kv_fill<T>(const T*, T*, T*, int, int, int, int, int, cudaStream_t);         \
  template cudaError_t launch_dec_attn<T>(const T*, T*, T*, T*, int, int, int, int, int, const int*,      \
                                          cudaStream_t);                                                 \
  template cudaError_t launch_gather_last<T>(const T*, int, int, int, T*, cudaStream_t);
INSTD(float)
INSTD(bf16)
