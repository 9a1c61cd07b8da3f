// Greedy decoding with a per-layer KV cache ("RustGPT", "Technical
// implementation": greedy decoding; "NTransformer" page, "No PyTorch, no
// cuBLAS": KV cache).  One new token per row and step: the weights are read
// once per step, so every kernel here is HBM-bound (GEMV-shaped, B <= 32).
//
// KV cache layout: kc/vc [B][H][Tmax][d] per layer.
#include "launch.h"

// pos = pos0 + *step (the step counter lives on the device so that one
// captured decode step can be replayed).  st (C % 16 == 0, or null): per
// 16-column group g of row b, st[g B + b] = (mean, sum of squared
// deviations) of the stored values, for the LayerNorm of the next projection.
template <typename T>
__global__ void dec_embed_kernel(const int* __restrict__ tok, const float* __restrict__ wte,
                                 const float* __restrict__ wpe, T* __restrict__ x, int C, int pos0,
                                 const int* __restrict__ step, int max_seq, unsigned* err, float2* st) {
  griddep_wait();
  griddep_release();
  int b = blockIdx.x;
  int pos = pos0 + *step;
  if (pos < 0 || pos >= max_seq) {
    if (b == 0 && threadIdx.x == 0) set_dev_err(err, GPT_DEVERR_POS);
    pos = pos < 0 ? 0 : max_seq - 1;
  }
  const float* a = wte + (long)tok[b] * C;
  const float* p = wpe ? wpe + (long)pos * C : nullptr;
  // blockDim.x is a multiple of 32: a group's 16 columns sit in 16 consecutive lanes
  for (int c0 = 0; c0 < C; c0 += blockDim.x) {
    const int c = c0 + threadIdx.x;
    const bool ok = c < C;
    float v = 0.f;
    if (ok) {
      const T t = from_f<T>(a[c] + (p ? p[c] : 0.f));
      x[(long)b * C + c] = t;
      v = to_f(t);
    }
    if (st) {
      float sm = v;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
      const float mean = sm * (1.f / 16.f), d = ok ? v - mean : 0.f;
      float q = d * d;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      if (ok && (threadIdx.x & 15) == 0) st[(long)(c / 16) * gridDim.x + b] = make_float2(mean, q);
    }
  }
}

template <typename T>
cudaError_t launch_dec_embed(const int* tok, const float* wte, const float* wpe, T* x, int B, int C, int pos0,
                             const int* step, int max_seq, unsigned* err, cudaStream_t s, float2* st) {
  if (st && C % 16) return cudaErrorInvalidValue;
  ++g_kernel_launches;
  cudaError_t e = launch_k(dec_embed_kernel<T>, dim3(B), dim3(256), 0, s, tok, wte, wpe, x, C, pos0, step, max_seq, err,
                           st);
  if (e != cudaSuccess) return e;
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
  griddep_wait();
  griddep_release();
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

// Small-batch form (B <= 8): each warp computes R consecutive outputs for all
// rows, every lane streaming 16-byte chunks of the R weight rows and of X
// straight from global memory (no staging, no block barrier), so a warp has
// R weight chunks in flight per step of the k loop.
template <typename T, int BB, int R>
__global__ void __launch_bounds__(GEMV_WARPS * 32)
gemv_rows_kernel(const T* __restrict__ X, int B, int K, const T* __restrict__ W, int N,
                 const float* __restrict__ bias, const T* resid, int mode, T* out, T* out2, float* outf) {
  griddep_wait();
  griddep_release();
  constexpr int NV = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = (blockIdx.x * GEMV_WARPS + warp) * R;
  if (n0 >= N) return;
  float acc[R][BB];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < BB; ++b) acc[r][b] = 0.f;
#pragma unroll 4
  for (int kk = lane * NV; kk < K; kk += 32 * NV) {
    float w[R][NV];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (n0 + r < N) Vec<T>::load(W + (long)(n0 + r) * K + kk, w[r]);
      else
#pragma unroll
        for (int j = 0; j < NV; ++j) w[r][j] = 0.f;
    }
#pragma unroll
    for (int b = 0; b < BB; ++b) {
      if (b < B) {
        float x[NV];
        Vec<T>::load(X + (long)b * K + kk, x);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int j = 0; j < NV; ++j) acc[r][b] = fmaf(w[r][j], x[j], acc[r][b]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int n = n0 + r;
#pragma unroll
    for (int b = 0; b < BB; ++b) {
      if (b < B) {
        const float y = warp_sum(acc[r][b]);
        if (lane == 0 && n < N) {
          const long o = (long)b * N + n;
          if (mode == 2) {
            outf[o] = y;
          } else if (mode == 1) {
            const float u = y + bias[n];
            const T uq = from_f<T>(u);
            out[o] = uq;
            out2[o] = from_f<T>(gelu_f(to_f(uq)));
          } else {
            const float v = y + (bias ? bias[n] : 0.f) + (resid ? to_f(resid[o]) : 0.f);
            out[o] = from_f<T>(v);
          }
        }
      }
    }
  }
}

template <typename T>
cudaError_t launch_gemv(const T* X, int B, int K, const T* W, int N, const float* bias, const T* resid,
                        int mode, T* out, T* out2, float* outf, cudaStream_t s) {
  unsigned g = (N + GEMV_WARPS - 1) / GEMV_WARPS;
  cudaError_t e;
  const dim3 gb(GEMV_WARPS * 32);
  const bool chunks = K % Vec<T>::N == 0 && ((uintptr_t)X & 15) == 0 && ((uintptr_t)W & 15) == 0;
  const unsigned g2 = (N + GEMV_WARPS * 2 - 1) / (GEMV_WARPS * 2), g4 = (N + GEMV_WARPS * 4 - 1) / (GEMV_WARPS * 4);
  if (chunks && B <= 1 && N >= 4096)
    e = launch_k(gemv_rows_kernel<T, 1, 4>, dim3(g4), gb, 0, s, X, B, K, W, N, bias, resid, mode, out, out2, outf);
  else if (chunks && B <= 1)
    e = launch_k(gemv_rows_kernel<T, 1, 2>, dim3(g2), gb, 0, s, X, B, K, W, N, bias, resid, mode, out, out2, outf);
  else if (chunks && B <= 8 && N >= 4096)
    e = launch_k(gemv_rows_kernel<T, 8, 4>, dim3(g4), gb, 0, s, X, B, K, W, N, bias, resid, mode, out, out2, outf);
  else if (chunks && B <= 8)
    e = launch_k(gemv_rows_kernel<T, 8, 2>, dim3(g2), gb, 0, s, X, B, K, W, N, bias, resid, mode, out, out2, outf);
  else if (B <= 1) e = launch_k(gemv_kernel<T, 1>, dim3(g), gb, 0, s, X, B, K, W, N, bias, resid, mode, out, out2, outf);
  else if (B <= 8) e = launch_k(gemv_kernel<T, 8>, dim3(g), gb, 0, s, X, B, K, W, N, bias, resid, mode, out, out2, outf);
  else if (B <= 32) e = launch_k(gemv_kernel<T, 32>, dim3(g), gb, 0, s, X, B, K, W, N, bias, resid, mode, out, out2, outf);
  else return cudaErrorInvalidValue;
  ++g_kernel_launches;
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Copy the prompt's K and V (from the prefill's qkv [B*Tp, 3C]) into the cache.
template <typename T>
__global__ void kv_fill_kernel(const T* __restrict__ qkv, T* __restrict__ kc, T* __restrict__ vc, int B, int Tp,
                               int d, int Tmax, DecLayout L) {
  const int KC = L.Hkv * d;
  long n = (long)B * Tp * KC;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    int c = i % KC;
    long bt = i / KC;
    int t = bt % Tp, b = bt / Tp;
    int h = c / d, e = c % d;
    long dst = (((long)b * L.Hkv + h) * Tmax + t) * d + e;
    kc[dst] = qkv[bt * L.qw + L.kcol + c];
    vc[dst] = qkv[bt * L.qw + L.vcol + c];
  }
}

template <typename T>
cudaError_t launch_kv_fill(const T* qkv, T* kc, T* vc, int B, int Tp, int d, int Tmax, const DecLayout& L,
                           cudaStream_t s) {
  ++g_kernel_launches;
  kv_fill_kernel<T><<<148 * 4, 256, 0, s>>>(qkv, kc, vc, B, Tp, d, Tmax, L);
  return cudaGetLastError();
}

// Decode attention of the new query over the cache ("NTransformer" page,
// KV cache; "Feste", scaled dot-product attention with the causal mask):
// o = softmax(q K^T / sqrt(D)) V over keys 0 .. pos of the (row, head).
// Grid (B*H, S): the key range of a (row, head) is cut into act <= S
// contiguous pieces (act grows with the context, one per 256 keys), one CTA
// each; S is chosen so that about two CTAs per SM have work.  A CTA's NW
// warps (8 while the (row, head) pairs do not fill the SMs, else 4) take
// NW * (32 / (D / 8)) * U consecutive keys per pass (256 or 128 for D = 64 in
// 16 bits), a lane group of D / 8 lanes per key and U keys per lane group
// in flight (each lane one load of 8 values of a key and of a value row,
// kept packed until used), with an online softmax (max, sum, output) per lane
// group updated once per U keys.  The lane groups and warps
// merge in a fixed order; with act = 1 the CTA writes the output, otherwise
// its partial (m, l, o[D]) goes to part and the last CTA of the (row, head)
// (an arrival counter that it resets) merges the act partials in key order.
// The new key / value of this step come from qkv and are written to the
// cache by piece 0; the first pass's cached rows load before the
// programmatic-dependent-launch wait, while the q / k / v projection runs.
#define DA_SPLITS 16
template <typename T>
__device__ __forceinline__ void load8(const T* p, float* v) {
#pragma unroll
  for (int i = 0; i < 8; i += Vec<T>::N) Vec<T>::load(p + i, v + i);
}
__device__ __forceinline__ int dec_attn_act(int pos, int S) { return min(S, (pos + 256) / 256); }
// 8 values of T kept packed in registers
template <typename T>
struct Pack8 {
  uint4 w[sizeof(T) / 2];
};
template <typename T>
__device__ __forceinline__ Pack8<T> ld_pack8(const T* p) {
  Pack8<T> r;
#pragma unroll
  for (int i = 0; i < (int)(sizeof(T) / 2); ++i) r.w[i] = reinterpret_cast<const uint4*>(p)[i];
  return r;
}
template <typename T>
__device__ __forceinline__ void unpack8(const Pack8<T>& r, float* v) {
  load8(reinterpret_cast<const T*>(r.w), v);
}

template <typename T, int D, int NW>
__global__ void __launch_bounds__(NW * 32)
dec_attn_kernel(const T* __restrict__ qkv, T* kc, T* vc, T* __restrict__ out, float* part, unsigned* cnt, int B,
                int H, int Tmax, int pos0, const int* __restrict__ step, DecLayout Ly) {
  static_assert(D % 8 == 0 && D <= 256, "head size");
  constexpr int LPK = D / 8;            // lanes per key row (16 bytes each)
  constexpr int KPW = 32 / LPK;         // lane groups (keys) per warp
  constexpr int U = sizeof(T) == 2 ? 8 : 4;   // keys per lane group in flight
  constexpr int KPP = NW * KPW * U;           // keys per CTA pass
  int pos = pos0 + *step;
  if (pos < 0) pos = 0;
  if (pos >= Tmax) pos = Tmax - 1;
  const int bh = blockIdx.x, sp = blockIdx.y;
  const int act = dec_attn_act(pos, gridDim.y);
  if (sp >= act) return;
  const int b = bh / H, h = bh % H;
  const int G = H / Ly.Hkv, hk = h / G;   // query head h reads key/value head hk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / LPK, sub = lane % LPK;
  const T* q = qkv + (long)b * Ly.qw + h * D;
  const T* knew = qkv + (long)b * Ly.qw + Ly.kcol + hk * D;
  const T* vnew = qkv + (long)b * Ly.qw + Ly.vcol + hk * D;
  T* kcb = kc + ((long)b * Ly.Hkv + hk) * Tmax * D;
  T* vcb = vc + ((long)b * Ly.Hkv + hk) * Tmax * D;
  // this piece's keys [j_lo, j_hi); this warp's first pass starts at jb0
  const int per = (pos + act) / act;   // ceil((pos + 1) / act)
  const int j_lo = sp * per, j_hi = min(pos + 1, j_lo + per);
  const int jb0 = j_lo + warp * KPW * U;
  // The step counter, the beam source table and the cached keys before pos
  // come from earlier steps: the first pass's cached rows load before the
  // wait, while the q / k / v projection still runs.
  auto load_kv = [&](int jb, Pack8<T>* kp, Pack8<T>* vp, bool cached, bool fresh) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = jb + u * KPW + grp;
      const bool take = j < j_hi && ((j < pos && cached) || (j == pos && fresh));
      if (take) {
        long row = (long)j * D;
        if (Ly.src && j < pos) row += ((long)Ly.src[(long)b * Tmax + j] - b) * Ly.Hkv * Tmax * D;
        kp[u] = ld_pack8((j == pos ? knew : kcb + row) + sub * 8);
        vp[u] = ld_pack8((j == pos ? vnew : vcb + row) + sub * 8);
      } else if (cached) {
#pragma unroll
        for (int i = 0; i < (int)(sizeof(T) / 2); ++i) { kp[u].w[i] = make_uint4(0u, 0u, 0u, 0u); vp[u].w[i] = kp[u].w[i]; }
      }
    }
  };
  Pack8<T> kp[U], vp[U];
  load_kv(jb0, kp, vp, true, false);
  // q, k, v of this step belong to the previous kernel until here
  griddep_wait();
  griddep_release();
  if (sp == 0 && h % G == 0 && threadIdx.x < D) {
    kcb[(long)pos * D + threadIdx.x] = knew[threadIdx.x];
    vcb[(long)pos * D + threadIdx.x] = vnew[threadIdx.x];
  }
  const float scale = rsqrtf((float)D);
  float qv[8];
  load8(q + sub * 8, qv);
#pragma unroll
  for (int i = 0; i < 8; ++i) qv[i] *= scale;
  float m = -INFINITY, l = 0.f, o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0.f;
  for (int jb = jb0; jb < j_hi; jb += KPP) {
    if (jb == jb0) load_kv(jb, kp, vp, false, true);   // the new key of this step
    else load_kv(jb, kp, vp, true, true);
    float sc[U];
    float mn = m;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float kv[8];
      unpack8(kp[u], kv);
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) t = fmaf(qv[i], kv[i], t);
#pragma unroll
      for (int o2 = LPK / 2; o2 > 0; o2 >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o2);
      sc[u] = jb + u * KPW + grp < j_hi ? t : -INFINITY;
      mn = fmaxf(mn, sc[u]);
    }
    if (mn != -INFINITY) {
      const float corr = expf(m - mn);
      l *= corr;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] *= corr;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float p = expf(sc[u] - mn);
        l += p;
        float vv[8];
        unpack8(vp[u], vv);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = fmaf(p, vv[i], o[i]);
      }
      m = mn;
    }
  }
  // merge the lane groups of the warp (lanes with the same sub hold the same dimensions)
#pragma unroll
  for (int o2 = LPK; o2 < 32; o2 <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o2);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o2);
    const float mn = fmaxf(m, m2);
    const float f1 = m == -INFINITY ? 0.f : expf(m - mn), f2 = m2 == -INFINITY ? 0.f : expf(m2 - mn);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = o[i] * f1 + __shfl_xor_sync(0xffffffffu, o[i], o2) * f2;
    l = l * f1 + l2 * f2;
    m = mn;
  }
  // merge the warps through shared memory
  __shared__ float sm_m[NW], sm_l[NW], sm_o[NW][D];
  __shared__ int s_last;
  if (lane < LPK) {
    if (lane == 0) { sm_m[warp] = m; sm_l[warp] = l; }
#pragma unroll
    for (int i = 0; i < 8; ++i) sm_o[warp][sub * 8 + i] = o[i];
  }
  __syncthreads();
  float mm = -INFINITY, ll = 0.f, oo = 0.f;
  if (threadIdx.x < D) {
#pragma unroll
    for (int w = 0; w < NW; ++w) mm = fmaxf(mm, sm_m[w]);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = sm_m[w] == -INFINITY ? 0.f : expf(sm_m[w] - mm);
      ll += sm_l[w] * f;
      oo += sm_o[w][threadIdx.x] * f;
    }
  }
  T* orow = out + (long)b * H * D + h * D;
  if (act == 1) {
    if (threadIdx.x < D) orow[threadIdx.x] = from_f<T>(oo / ll);
    return;
  }
  float* pb = part + (long)bh * DA_SPLITS * (D + 2);
  if (threadIdx.x < D) {
    pb[sp * (D + 2) + 2 + threadIdx.x] = oo;
    if (threadIdx.x == 0) { pb[sp * (D + 2)] = mm; pb[sp * (D + 2) + 1] = ll; }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&cnt[bh], 1u);
    s_last = prev == (unsigned)(act - 1);
    if (s_last) atomicExch(&cnt[bh], 0u);   // ready for the next launch
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x < D) {
    float gm = -INFINITY;
    for (int s2 = 0; s2 < act; ++s2) gm = fmaxf(gm, __ldcg(pb + s2 * (D + 2)));
    float gl = 0.f, go = 0.f;
    for (int s2 = 0; s2 < act; ++s2) {
      const float ms = __ldcg(pb + s2 * (D + 2));
      const float f = ms == -INFINITY ? 0.f : expf(ms - gm);
      gl += __ldcg(pb + s2 * (D + 2) + 1) * f;
      go += __ldcg(pb + s2 * (D + 2) + 2 + threadIdx.x) * f;
    }
    orow[threadIdx.x] = from_f<T>(go / gl);
  }
}

size_t dec_attn_part_floats(int B, int H, int d) { return (size_t)B * H * DA_SPLITS * (d + 2); }

static int g_da_sms = 0;

template <typename T>
cudaError_t launch_dec_attn(const T* qkv, T* kc, T* vc, T* out, float* part, unsigned* cnt, int B, int H, int d,
                            int Tmax, int pos0, const int* step, const DecLayout& L, cudaStream_t s) {
  if (!g_da_sms) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_da_sms = n > 0 ? n : 148;
  }
  // pieces per (row, head): about two working CTAs per SM (a split costs a
  // fence, an arrival and a merge, more than one more pass over the keys)
  int S = (2 * g_da_sms + B * H - 1) / (B * H);
  if (S > DA_SPLITS) S = DA_SPLITS;
  if (S < 1) S = 1;
  dim3 g(B * H, S);
  // eight warps (one pass per 256-key piece at d = 64) while the (row, head)
  // pairs do not fill the SMs, else four (more CTAs resident per SM)
  const bool wide = B * H <= g_da_sms;
  cudaError_t e = cudaSuccess;
  switch (d) {
#define DA_CASE(DD)                                                                                               \
  case DD:                                                                                                        \
    g_kernel_launches += 1;                                                                                       \
    if (wide)                                                                                                     \
      e = launch_k(dec_attn_kernel<T, DD, 8>, g, dim3(256), 0, s, qkv, kc, vc, out, part, cnt, B, H, Tmax, pos0, \
                   step, L);                                                                                      \
    else                                                                                                          \
      e = launch_k(dec_attn_kernel<T, DD, 4>, g, dim3(128), 0, s, qkv, kc, vc, out, part, cnt, B, H, Tmax, pos0, \
                   step, L);                                                                                      \
    break;
    DA_CASE(16)
    DA_CASE(32)
    DA_CASE(64)
    DA_CASE(128)
#undef DA_CASE
    default: return cudaErrorInvalidValue;
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Greedy choice: argmax over the real vocabulary of fp32 logits, lowest
// index on ties.  Writes tok[b] and out[b * out_ld + col].  With nx.x (a
// replayed greedy step) the CTA also embeds its row's chosen token at the
// next position into x (with its LayerNorm group statistics), and the last
// CTA to finish (an arrival counter it resets) advances the step counter: the
// embedding and step-advance kernels of the step fold into this one.
template <typename T>
__global__ void argmax_kernel(const float* __restrict__ logits, int V, int Vp, int* tok, int32_t* out,
                              int out_ld, const int* __restrict__ step, GreedyNext<T> nx) {
  griddep_wait();
  griddep_release();
  int b = blockIdx.x;
  const int col = step ? *step : 0;
  const float* z = logits + (long)b * Vp;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  auto take = [&](float v, int c) {
    if (c < V && (v > best || (v == best && c < bi))) { best = v; bi = c; }
  };
  // 16-byte aligned rows (Vp % 4 == 0, so 4 ceil(V / 4) <= Vp): four columns
  // per load and four loads in flight per thread; columns from V on are padding
  const bool vec = (Vp & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0;
  const int nv = vec ? (V + 3) >> 2 : 0;
  const float4* z4 = reinterpret_cast<const float4*>(z);
  if (!vec)
    for (int c = threadIdx.x; c < V; c += blockDim.x) take(z[c], c);
  int q = threadIdx.x;
  for (; q + 3 * (int)blockDim.x < nv; q += 4 * blockDim.x) {
    float4 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) w[u] = z4[q + u * blockDim.x];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = 4 * (q + u * blockDim.x);
      take(w[u].x, c); take(w[u].y, c + 1); take(w[u].z, c + 2); take(w[u].w, c + 3);
    }
  }
  for (; q < nv; q += blockDim.x) {
    const float4 w = z4[q];
    take(w.x, 4 * q); take(w.y, 4 * q + 1); take(w.z, 4 * q + 2); take(w.w, 4 * q + 3);
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
      si[0] = bi;
    }
  }
  if (!nx.x) return;
  __syncthreads();
  const int t = si[0];
  // the next step's input row: token t at position pos0 + col + 1 (the last
  // replay embeds a position nobody reads; it is clamped, not flagged)
  int pos = nx.pos0 + col + 1;
  pos = pos < 0 ? 0 : pos >= nx.max_seq ? nx.max_seq - 1 : pos;
  const float* a = nx.wte + (long)t * nx.C;
  const float* p = nx.wpe ? nx.wpe + (long)pos * nx.C : nullptr;
  for (int c0 = 0; c0 < nx.C; c0 += blockDim.x) {
    const int c = c0 + threadIdx.x;
    const bool ok = c < nx.C;
    float v = 0.f;
    if (ok) {
      const T w = from_f<T>(a[c] + (p ? p[c] : 0.f));
      nx.x[(long)b * nx.C + c] = w;
      v = to_f(w);
    }
    if (nx.st) {
      float sm = v;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
      const float mean = sm * (1.f / 16.f), d = ok ? v - mean : 0.f;
      float q = d * d;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      if (ok && (threadIdx.x & 15) == 0) nx.st[(long)(c / 16) * gridDim.x + b] = make_float2(mean, q);
    }
  }
  // every CTA read the step counter at its start: the last one advances it
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(nx.cnt, 1u) == gridDim.x - 1) {
      *nx.step += 1;
      *nx.cnt = 0;
    }
  }
}

template <typename T>
cudaError_t launch_argmax(const float* logits, int B, int V, int Vp, int* tok, int32_t* out, int out_ld,
                          const int* step, cudaStream_t s, const GreedyNext<T>* nx) {
  GreedyNext<T> n{};
  if (nx) {
    if (!nx->x || !nx->wte || !nx->cnt || !nx->step || nx->step != step || (nx->st && nx->C % 16))
      return cudaErrorInvalidValue;
    n = *nx;
  }
  ++g_kernel_launches;
  cudaError_t e = launch_k(argmax_kernel<T>, dim3(B), dim3(1024), 0, s, logits, V, Vp, tok, out, out_ld, step, n);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ sampling
// Sampled choice of the next token ("RustGPT" roadmap: temperature scaling,
// top-k, top-p; "LucilleAI": sampler), one CTA per row, the row's values in
// shared memory.  In order: x = z / temperature over the real vocabulary;
// top-k keeps the k largest x (ties at the cut to the lower index); weights
// w = exp(x - max x) over the kept tokens; top-p keeps the shortest prefix,
// in (w descending, index ascending) order, whose weight reaches top_p times
// the kept total; the token is the first kept one, in ascending token order,
// at which the running weight exceeds u times the kept total.  Thresholds
// are found by bisection over order-preserving 32-bit keys, every sum by a
// fixed-order block reduction (deterministic).  temperature <= 0: greedy.
#define SMP_THREADS 1024
#define SMP_WARPS (SMP_THREADS / 32)

__device__ __forceinline__ uint32_t smp_key(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
// Fixed-order block sums (the same thread-to-element map every call).
__device__ __forceinline__ float smp_bsum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < SMP_WARPS ? red[lane] : 0.f;
  return warp_sum(t);
}
__device__ __forceinline__ int smp_bcount(int v, int* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int t = lane < SMP_WARPS ? red[lane] : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}
// Exclusive block scan of one value per thread (in thread order).
__device__ __forceinline__ float smp_bscan_excl(float v, float* red, float* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  __syncthreads();
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  float wsum = lane < SMP_WARPS ? red[lane] : 0.f, winc = wsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t = __shfl_up_sync(0xffffffffu, winc, o);
    if (lane >= o) winc += t;
  }
  const float wex = __shfl_sync(0xffffffffu, winc - wsum, warp);
  *total = __shfl_sync(0xffffffffu, winc, SMP_WARPS - 1);
  return wex + inc - v;
}
__device__ __forceinline__ int smp_bscan_excl_i(int v, int* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  __syncthreads();
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  int wsum = lane < SMP_WARPS ? red[lane] : 0, winc = wsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, winc, o);
    if (lane >= o) winc += t;
  }
  const int wex = __shfl_sync(0xffffffffu, winc - wsum, warp);
  return wex + inc - v;
}

__global__ void __launch_bounds__(SMP_THREADS) sample_kernel(const float* __restrict__ logits, int V, int Vp,
                                                             float temp, int top_k, float top_p,
                                                             const float* __restrict__ uni, int u_ld, int* tok,
                                                             int32_t* out, int out_ld, const int* __restrict__ step) {
  griddep_wait();
  griddep_release();
  extern __shared__ float w[];   // [V]
  __shared__ float redf[SMP_WARPS];
  __shared__ int redi[SMP_WARPS];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int col = step ? *step : 0;
  const float* z = logits + (long)b * Vp;
  // thread tid owns the contiguous indices [c0, c1)
  const int chunk = (V + SMP_THREADS - 1) / SMP_THREADS;
  const int c0 = min(V, tid * chunk), c1 = min(V, c0 + chunk);
  int choice = 0;
  if (!(temp > 0.f)) {
    // greedy: largest logit, lowest index on ties
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = c0; i < c1; ++i) {
      const float v = z[i];
      if (v > best) { best = v; bi = i; }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
    }
    __shared__ float sv[SMP_WARPS];
    __shared__ int si[SMP_WARPS];
    if ((tid & 31) == 0) { sv[tid >> 5] = best; si[tid >> 5] = bi; }
    __syncthreads();
    if (tid < 32) {
      best = sv[tid];
      bi = si[tid];
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
      }
      if (tid == 0) choice = (bi >= 0 && bi < V) ? bi : 0;
    }
  } else {
    const float it = 1.0f / temp;
    float mx = -INFINITY;
    for (int i = c0; i < c1; ++i) {
      const float x = z[i] * it;
      w[i] = x;
      mx = fmaxf(mx, x);
    }
    {
      mx = warp_max(mx);
      __syncthreads();
      if ((tid & 31) == 0) redf[tid >> 5] = mx;
      __syncthreads();
      mx = warp_max((tid & 31) < SMP_WARPS ? redf[tid & 31] : -INFINITY);
    }
    // top-k: the largest key tk with count(key >= tk) >= k
    const bool use_k = top_k > 0 && top_k < V;
    uint32_t tk = 0;
    int need_k = 0;
    if (use_k) {
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = tk | (1u << bit);
        int cnt = 0;
        for (int i = c0; i < c1; ++i) cnt += smp_key(w[i]) >= cand;
        if (smp_bcount(cnt, redi) >= top_k) tk = cand;
      }
      int gt = 0;
      for (int i = c0; i < c1; ++i) gt += smp_key(w[i]) > tk;
      need_k = top_k - smp_bcount(gt, redi);
    }
    // weights of the kept tokens (ties at the top-k cut: lower indices first)
    {
      int eq = 0;
      if (use_k)
        for (int i = c0; i < c1; ++i) eq += smp_key(w[i]) == tk;
      int rank = use_k ? smp_bscan_excl_i(eq, redi) : 0;
      for (int i = c0; i < c1; ++i) {
        bool keep = true;
        if (use_k) {
          const uint32_t k = smp_key(w[i]);
          keep = k > tk || (k == tk && rank++ < need_k);
        }
        w[i] = keep ? __expf(w[i] - mx) : 0.f;
      }
    }
    float part = 0.f;
    for (int i = c0; i < c1; ++i) part += w[i];
    const float Z = smp_bsum(part, redf);
    if (top_p < 1.f) {
      // the largest weight threshold tp with mass(w >= tp) >= top_p Z
      const float target = top_p * Z;
      uint32_t tp = 0;
      for (int bit = 30; bit >= 0; --bit) {
        const uint32_t cand = tp | (1u << bit);
        float m = 0.f;
        for (int i = c0; i < c1; ++i) m += __float_as_uint(w[i]) >= cand ? w[i] : 0.f;
        if (smp_bsum(m, redf) >= target) tp = cand;
      }
      const float pstar = __uint_as_float(tp);
      float gt = 0.f;
      int eq = 0;
      for (int i = c0; i < c1; ++i) {
        gt += w[i] > pstar ? w[i] : 0.f;
        eq += w[i] == pstar;
      }
      const float mgt = smp_bsum(gt, redf);
      const int neq = smp_bcount(eq, redi);
      int need = pstar > 0.f ? (int)ceilf((target - mgt) / pstar) : neq;
      need = max(1, min(need, neq));
      int rank = smp_bscan_excl_i(eq, redi);
      for (int i = c0; i < c1; ++i) {
        const bool keep = w[i] > pstar || (w[i] == pstar && rank++ < need);
        if (!keep) w[i] = 0.f;
      }
    }
    // inverse CDF in ascending token order
    part = 0.f;
    int last = -1;
    for (int i = c0; i < c1; ++i) {
      part += w[i];
      if (w[i] > 0.f) last = i;
    }
    float Z2;
    const float before = smp_bscan_excl(part, redf, &Z2);
    const float u = uni[(long)b * u_ld + col];
    const float target = u * Z2;
    __shared__ int s_choice, s_last;
    if (tid == 0) { s_choice = -1; s_last = -1; }
    __syncthreads();
    if (last >= 0) atomicMax(&s_last, last);
    if (before <= target && target < before + part) {
      float run = before;
      for (int i = c0; i < c1; ++i) {
        run += w[i];
        if (w[i] > 0.f && run > target) { s_choice = i; break; }
      }
    }
    __syncthreads();
    if (tid == 0) {
      int c = s_choice >= 0 ? s_choice : s_last;
      choice = (c >= 0 && c < V) ? c : 0;
    }
  }
  if (tid == 0) {
    tok[b] = choice;
    out[(long)b * out_ld + col] = choice;
  }
}

cudaError_t launch_sample(const float* logits, int B, int V, int Vp, float temp, int top_k, float top_p,
                          const float* uni, int u_ld, int* tok, int32_t* out, int out_ld, const int* step,
                          cudaStream_t s) {
  const size_t smem = (size_t)V * 4;
  static size_t attr = 0;
  if (smem > attr) {
    cudaError_t e = cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = smem;
  }
  ++g_kernel_launches;
  cudaError_t e = launch_k(sample_kernel, dim3(B), dim3(SMP_THREADS), smem, s, logits, V, Vp, temp, top_k, top_p,
                           uni, u_ld, tok, out, out_ld, step);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

__global__ void step_advance_kernel(int* step) { griddep_wait(); griddep_release(); *step += 1; }
cudaError_t launch_step_advance(int* step, cudaStream_t s) {
  ++g_kernel_launches;
  cudaError_t e = launch_k(step_advance_kernel, dim3(1), dim3(1), 0, s, step);
  if (e != cudaSuccess) return e;
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
  template cudaError_t launch_argmax<T>(const float*, int, int, int, int*, int32_t*, int, const int*,     \
                                        cudaStream_t, const GreedyNext<T>*);                             \
  template cudaError_t launch_dec_embed<T>(const int*, const float*, const float*, T*, int, int, int,      \
                                           const int*, int, unsigned*, cudaStream_t, float2*);           \
  template cudaError_t launch_gemv<T>(const T*, int, int, const T*, int, const float*, const T*, int, T*, T*, \
                                      float*, cudaStream_t);                                             \
  template cudaError_t launch_kv_fill<T>(const T*, T*, T*, int, int, int, int, const DecLayout&, cudaStream_t); \
  template cudaError_t launch_dec_attn<T>(const T*, T*, T*, T*, float*, unsigned*, int, int, int, int, int, const int*,      \
                                          const DecLayout&, cudaStream_t);                               \
  template cudaError_t launch_gather_last<T>(const T*, int, int, int, T*, cudaStream_t);
INSTD(float)
INSTD(bf16)
INSTD(f16)
