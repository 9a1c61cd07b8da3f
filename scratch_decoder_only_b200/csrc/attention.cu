// Causal / block-diagonal multi-head attention, forward and backward.
//
// Scores s_ij = q_i . k_j / sqrt(d) for allowed keys j: j <= i and j in the
// same document as i (dstart[i] <= j), all others masked to -inf before the
// softmax ("Feste", "Model Architecture mirrors GPT-2": masked_fill with
// -inf; "LucilleAI": sequence packing).  The forward keeps the row
// log-sum-exp; the backward recomputes P from it.
//
// qkv is [B*T, 3C] (q | k | v, head h at columns h*d..h*d+d-1 of each part),
// out / dout are [B*T, C], lse / D are [B, H, T].
//
// SIMT kernels here (fp32 FFMA, online softmax per lane, merged across the
// warp) serve the fp32 mode and any head size; the bf16 tensor-core kernels
// live in attention_mma.cu.
#include "launch.h"

#define ATT_WARPS 4

template <typename T, int D>
__global__ void __launch_bounds__(ATT_WARPS * 32)
attn_fwd_simt(const T* __restrict__ qkv, T* __restrict__ out, float* __restrict__ lse,
              const int* __restrict__ dstart, int B, int T_, int H) {
  __shared__ float qs[ATT_WARPS][D];
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long gw = (long)blockIdx.x * ATT_WARPS + warp;
  if (gw >= (long)B * H * T_) return;
  int t = gw % T_;
  int bh = gw / T_;
  int h = bh % H, b = bh / H;
  const int C = H * D;
  const long C3 = 3L * C;
  const float scale = 1.0f / sqrtf((float)D);
  long mrow = (long)b * T_ + t;
  for (int i = lane; i < D; i += 32) qs[warp][i] = to_f(qkv[mrow * C3 + h * D + i]) * scale;
  __syncwarp();
  int j0 = dstart[mrow];
  float mloc = -INFINITY, sloc = 0.f;
  float acc[D];
#pragma unroll
  for (int i = 0; i < D; ++i) acc[i] = 0.f;
  for (int j = j0 + lane; j <= t; j += 32) {
    const T* kr = qkv + ((long)b * T_ + j) * C3 + C + h * D;
    const T* vr = kr + C;
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) s = fmaf(qs[warp][i], to_f(kr[i]), s);
    float mn = fmaxf(mloc, s);
    float corr = expf(mloc - mn);
    float p = expf(s - mn);
    sloc = sloc * corr + p;
#pragma unroll
    for (int i = 0; i < D; ++i) acc[i] = acc[i] * corr + p * to_f(vr[i]);
    mloc = mn;
  }
  float mw = warp_max(mloc);
  float f = (mloc == -INFINITY) ? 0.f : expf(mloc - mw);
  float ssum = warp_sum(sloc * f);
  float inv = 1.0f / ssum;
#pragma unroll
  for (int i = 0; i < D; ++i) {
    float v = warp_sum(acc[i] * f);
    if ((i & 31) == lane) out[mrow * C + h * D + i] = from_f<T>(v * inv);
  }
  if (lane == 0) lse[(long)bh * T_ + t] = mw + logf(ssum);
}

// dQ (and D_i = dO_i . O_i) for query row i.
template <typename T, int D>
__global__ void __launch_bounds__(ATT_WARPS * 32)
attn_bwd_dq_simt(const T* __restrict__ qkv, const T* __restrict__ out, const T* __restrict__ dout,
                 const float* __restrict__ lse, float* __restrict__ Dbuf, const int* __restrict__ dstart,
                 T* __restrict__ dqkv, int B, int T_, int H) {
  __shared__ float qs[ATT_WARPS][D], dos[ATT_WARPS][D];
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long gw = (long)blockIdx.x * ATT_WARPS + warp;
  if (gw >= (long)B * H * T_) return;
  int t = gw % T_;
  int bh = gw / T_;
  int h = bh % H, b = bh / H;
  const int C = H * D;
  const long C3 = 3L * C;
  const float scale = 1.0f / sqrtf((float)D);
  long mrow = (long)b * T_ + t;
  float dd = 0.f;
  for (int i = lane; i < D; i += 32) {
    float dov = to_f(dout[mrow * C + h * D + i]);
    qs[warp][i] = to_f(qkv[mrow * C3 + h * D + i]) * scale;
    dos[warp][i] = dov;
    dd += dov * to_f(out[mrow * C + h * D + i]);
  }
  dd = warp_sum(dd);
  __syncwarp();
  float L = lse[(long)bh * T_ + t];
  if (lane == 0) Dbuf[(long)bh * T_ + t] = dd;
  int j0 = dstart[mrow];
  float acc[D];
#pragma unroll
  for (int i = 0; i < D; ++i) acc[i] = 0.f;
  for (int j = j0 + lane; j <= t; j += 32) {
    const T* kr = qkv + ((long)b * T_ + j) * C3 + C + h * D;
    const T* vr = kr + C;
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) {
      s = fmaf(qs[warp][i], to_f(kr[i]), s);
      dp = fmaf(dos[warp][i], to_f(vr[i]), dp);
    }
    float p = expf(s - L);
    float ds = p * (dp - dd);
#pragma unroll
    for (int i = 0; i < D; ++i) acc[i] = fmaf(ds, to_f(kr[i]), acc[i]);
  }
#pragma unroll
  for (int i = 0; i < D; ++i) {
    float v = warp_sum(acc[i]);
    if ((i & 31) == lane) dqkv[mrow * C3 + h * D + i] = from_f<T>(v * scale);
  }
}

// dK, dV for key row j: sum over the queries i >= j of the same document.
template <typename T, int D>
__global__ void __launch_bounds__(ATT_WARPS * 32)
attn_bwd_dkdv_simt(const T* __restrict__ qkv, const T* __restrict__ dout, const float* __restrict__ lse,
                   const float* __restrict__ Dbuf, const int* __restrict__ dstart, T* __restrict__ dqkv,
                   int B, int T_, int H) {
  __shared__ float ks[ATT_WARPS][D], vs[ATT_WARPS][D];
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long gw = (long)blockIdx.x * ATT_WARPS + warp;
  if (gw >= (long)B * H * T_) return;
  int j = gw % T_;
  int bh = gw / T_;
  int h = bh % H, b = bh / H;
  const int C = H * D;
  const long C3 = 3L * C;
  const float scale = 1.0f / sqrtf((float)D);
  long mj = (long)b * T_ + j;
  for (int i = lane; i < D; i += 32) {
    ks[warp][i] = to_f(qkv[mj * C3 + C + h * D + i]);
    vs[warp][i] = to_f(qkv[mj * C3 + 2 * C + h * D + i]);
  }
  __syncwarp();
  int ds_j = dstart[mj];
  float dk[D], dv[D];
#pragma unroll
  for (int i = 0; i < D; ++i) { dk[i] = 0.f; dv[i] = 0.f; }
  for (int i0 = j; i0 < T_; i0 += 32) {
    int i = i0 + lane;
    bool ok = i < T_ && dstart[(long)b * T_ + (i < T_ ? i : 0)] == ds_j;
    if (!__any_sync(0xffffffffu, ok)) break;
    if (ok) {
      long mi = (long)b * T_ + i;
      const T* qr = qkv + mi * C3 + h * D;
      const T* dor = dout + mi * C + h * D;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) {
        s = fmaf(to_f(qr[c]), ks[warp][c], s);
        dp = fmaf(to_f(dor[c]), vs[warp][c], dp);
      }
      float p = expf(s * scale - lse[(long)bh * T_ + i]);
      float dsv = p * (dp - Dbuf[(long)bh * T_ + i]);
#pragma unroll
      for (int c = 0; c < D; ++c) {
        dv[c] = fmaf(p, to_f(dor[c]), dv[c]);
        dk[c] = fmaf(dsv, to_f(qr[c]), dk[c]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < D; ++c) {
    float a = warp_sum(dk[c]);
    float v = warp_sum(dv[c]);
    if ((c & 31) == lane) {
      dqkv[mj * C3 + C + h * D + c] = from_f<T>(a * scale);
      dqkv[mj * C3 + 2 * C + h * D + c] = from_f<T>(v);
    }
  }
}

template <typename T, int D>
static cudaError_t attn_fwd_simt_launch(const T* qkv, T* out, float* lse, const int* dstart, int B, int T_,
                                        int H, cudaStream_t s) {
  long rows = (long)B * H * T_;
  ++g_kernel_launches;
  attn_fwd_simt<T, D><<<(unsigned)((rows + ATT_WARPS - 1) / ATT_WARPS), ATT_WARPS * 32, 0, s>>>(
      qkv, out, lse, dstart, B, T_, H);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t attn_bwd_simt_launch(const T* qkv, const T* out, const T* dout, const float* lse,
                                        float* Dbuf, const int* dstart, T* dqkv, int B, int T_, int H,
                                        cudaStream_t s) {
  long rows = (long)B * H * T_;
  unsigned g = (unsigned)((rows + ATT_WARPS - 1) / ATT_WARPS);
  ++g_kernel_launches;
  attn_bwd_dq_simt<T, D><<<g, ATT_WARPS * 32, 0, s>>>(qkv, out, dout, lse, Dbuf, dstart, dqkv, B, T_, H);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ++g_kernel_launches;
  attn_bwd_dkdv_simt<T, D><<<g, ATT_WARPS * 32, 0, s>>>(qkv, dout, lse, Dbuf, dstart, dqkv, B, T_, H);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_attn_fwd_simt(const T* qkv, T* out, float* lse, const int* dstart, int B, int T_, int H,
                                 int d, cudaStream_t s) {
  switch (d) {
    case 16: return attn_fwd_simt_launch<T, 16>(qkv, out, lse, dstart, B, T_, H, s);
    case 32: return attn_fwd_simt_launch<T, 32>(qkv, out, lse, dstart, B, T_, H, s);
    case 64: return attn_fwd_simt_launch<T, 64>(qkv, out, lse, dstart, B, T_, H, s);
    case 128: return attn_fwd_simt_launch<T, 128>(qkv, out, lse, dstart, B, T_, H, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_attn_bwd_simt(const T* qkv, const T* out, const T* dout, const float* lse, float* Dbuf,
                                 const int* dstart, T* dqkv, int B, int T_, int H, int d, cudaStream_t s) {
  switch (d) {
    case 16: return attn_bwd_simt_launch<T, 16>(qkv, out, dout, lse, Dbuf, dstart, dqkv, B, T_, H, s);
    case 32: return attn_bwd_simt_launch<T, 32>(qkv, out, dout, lse, Dbuf, dstart, dqkv, B, T_, H, s);
    case 64: return attn_bwd_simt_launch<T, 64>(qkv, out, dout, lse, Dbuf, dstart, dqkv, B, T_, H, s);
    case 128: return attn_bwd_simt_launch<T, 128>(qkv, out, dout, lse, Dbuf, dstart, dqkv, B, T_, H, s);
  }
  return cudaErrorInvalidValue;
}

template cudaError_t launch_attn_fwd_simt<float>(const float*, float*, float*, const int*, int, int, int, int,
                                                 cudaStream_t);
template cudaError_t launch_attn_fwd_simt<bf16>(const bf16*, bf16*, float*, const int*, int, int, int, int,
                                                cudaStream_t);
template cudaError_t launch_attn_bwd_simt<float>(const float*, const float*, const float*, const float*, float*,
                                                 const int*, float*, int, int, int, int, cudaStream_t);
template cudaError_t launch_attn_bwd_simt<bf16>(const bf16*, const bf16*, const bf16*, const float*, float*,
                                                const int*, bf16*, int, int, int, int, cudaStream_t);
template cudaError_t launch_attn_fwd_simt<f16>(const f16*, f16*, float*, const int*, int, int, int, int,
                                               cudaStream_t);
template cudaError_t launch_attn_bwd_simt<f16>(const f16*, const f16*, const f16*, const float*, float*,
                                               const int*, f16*, int, int, int, int, cudaStream_t);
