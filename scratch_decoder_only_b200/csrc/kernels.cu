// Memory-bound kernels of the training step: input preparation, embedding
// gather / scatter, LayerNorm forward / backward, fused softmax
// cross-entropy with its logits gradient, deterministic row reductions,
// global-norm clip and AdamW.  All are HBM-bound: 16-byte vector loads, one
// warp per row where a row is reduced, no fp32 copies of bf16 tensors.
#include <algorithm>
#include "launch.h"
#include "tc_common.cuh"

unsigned long long g_kernel_launches = 0;
bool g_pdl = true;

#define LN_MAXC 1024   // largest d_model the register-resident LayerNorm handles

// ---------------------------------------------------------------------------
// Input preparation: clamp ids, positions inside packed documents, targets.
// Position restarts at 0 at the first token of each document ("LucilleAI",
// sequence packing); dstart[m] = row index of the first token of m's document.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) prep_kernel(const int32_t* __restrict__ tokens,
                                                    const int32_t* __restrict__ targets,
                                                    const int32_t* __restrict__ seg, int B, int T, int V,
                                                    int* tok_out, int* tgt_out, int* pos_out, int* dstart_out,
                                                    DevScalars* sc) {
  griddep_wait();
  griddep_release();
  // one block per row; the document start of t is the largest run start <= t
  // (an inclusive max-scan of "t if a document starts at t"), carried across
  // chunks of blockDim.x positions
  __shared__ int wscan[32];
  __shared__ int carry_s;
  __shared__ int nv_s[32];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  unsigned err = 0;
  int nv = 0;
  unsigned long long pairs = 0;   // keys each query may attend to, summed (packed rows)
  int carry = 0;
  for (int t0 = 0; t0 < T; t0 += blockDim.x) {
    const int t = t0 + threadIdx.x;
    int start = 0;
    if (t < T) {
      const long m = (long)b * T + t;
      int tok = tokens[m];
      if (tok < 0 || tok >= V) { err |= GPT_DEVERR_TOKEN; tok = tok < 0 ? 0 : V - 1; }
      tok_out[m] = tok;
      if (targets) {
        int tg = targets[m];
        if (tg < -1 || tg >= V) { err |= GPT_DEVERR_TARGET; tg = -1; }
        tgt_out[m] = tg;
        nv += (tg >= 0);
      }
      if (seg) {
        const int sg = seg[m];
        if (t > 0) {
          const int pv = seg[m - 1];
          if (sg < pv) err |= GPT_DEVERR_SEGMENT;
          if (sg != pv) start = t;
        }
      }
    }
    // inclusive max-scan over the chunk
    int v = start;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v = max(v, u);
    }
    if (lane == 31) wscan[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int w = lane < nw ? wscan[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w = max(w, u);
      }
      if (lane < nw) wscan[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v = max(v, wscan[warp - 1]);
    v = max(v, carry);
    if (t < T) {
      const long m = (long)b * T + t;
      const int ds = seg ? v : 0;
      dstart_out[m] = ds;
      pos_out[m] = t - ds;
      pairs += (unsigned long long)(t - ds + 1);
    }
    if (threadIdx.x == blockDim.x - 1) carry_s = v;
    __syncthreads();
    carry = carry_s;
    __syncthreads();
  }
  if (err) atomicOr(&sc->err, err);
  for (int o = 16; o > 0; o >>= 1) nv += __shfl_xor_sync(0xffffffffu, nv, o);
  if (lane == 0) nv_s[warp] = nv;
  __syncthreads();
  if (threadIdx.x == 0 && targets) {
    int tot = 0;
    for (int w = 0; w < nw; ++w) tot += nv_s[w];
    atomicAdd(&sc->n_valid, tot);   // cleared before the launch
  }
  if (seg) {
    for (int o = 16; o > 0; o >>= 1) pairs += __shfl_xor_sync(0xffffffffu, pairs, o);
    if (lane == 0) atomicAdd(&sc->attn_pairs, pairs);   // cleared before the launch
  }
}

// ---------------------------------------------------------------------------
// Zero fill inside the dependent-launch chain (a memset node would end the
// overlap of its neighbours).  The buffer belongs to no kernel still running
// (the caller's contract), so the fill starts at once and overlaps the
// previous kernel; the wait sits at the end, so this kernel completes only
// after its predecessor and the chain's order holds for the next kernel.
// ---------------------------------------------------------------------------
__global__ void zero_fill_kernel(uint8_t* p, size_t bytes) {
  griddep_release();
  const size_t head = (16 - (reinterpret_cast<uintptr_t>(p) & 15)) & 15;
  const size_t pre = head < bytes ? head : bytes;
  const size_t n16 = (bytes - pre) / 16, tail0 = pre + n16 * 16;
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x, nth = (size_t)gridDim.x * blockDim.x;
  if (tid < pre) p[tid] = 0;
  uint4* q = reinterpret_cast<uint4*>(p + pre);
  for (size_t i = tid; i < n16; i += nth) q[i] = make_uint4(0u, 0u, 0u, 0u);
  if (tid < bytes - tail0) p[tail0 + tid] = 0;
  griddep_wait();
}

static int g_zero_sms = 0;

cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t s) {
  if (!bytes) return cudaSuccess;
  if (!g_zero_sms) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_zero_sms = n > 0 ? n : 148;
  }
  size_t blocks = (bytes / 16 + 255) / 256;
  if (blocks > (size_t)g_zero_sms * 4) blocks = (size_t)g_zero_sms * 4;
  if (blocks < 1) blocks = 1;
  ++g_kernel_launches;
  return launch_k(zero_fill_kernel, dim3((unsigned)blocks), dim3(256), 0, s, (uint8_t*)p, bytes);
}

cudaError_t launch_prep(const int32_t* tokens, const int32_t* targets, const int32_t* seg, int B, int T,
                        int V, int* tok_out, int* tgt_out, int* pos_out, int* dstart_out,
                        DevScalars* sc, cudaStream_t s) {
  if (targets) {
    cudaError_t e = launch_zero(&sc->n_valid, sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  if (seg) {
    cudaError_t e = launch_zero(&sc->attn_pairs, sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
  }
  int th = T >= 1024 ? 1024 : ((T + 31) / 32) * 32;
  ++g_kernel_launches;
  return launch_k(prep_kernel, dim3(B), dim3(th), 0, s,
                  tokens, targets, seg, B, T, V, tok_out, tgt_out, pos_out, dstart_out, sc);
}

// ---------------------------------------------------------------------------
// Embedding: x[m] = wte[tok[m]] + wpe[pos[m]] ("Feste", "Model Architecture
// mirrors GPT-2": the position embedding is added directly).  fp32 sources.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void embed_fwd_kernel(const int* __restrict__ tok, const int* __restrict__ pos,
                                 const float* __restrict__ wte, const float* __restrict__ wpe,
                                 T* __restrict__ x, int M, int C) {
  griddep_wait();
  griddep_release();
  int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* a = wte + (long)tok[row] * C;
  const float* b = wpe ? wpe + (long)pos[row] * C : nullptr;
  T* o = x + (long)row * C;
  constexpr int NV = Vec<T>::N;
  for (int c = lane * NV; c < C; c += 32 * NV) {
    float va[NV], vb[NV];
#pragma unroll
    for (int i = 0; i < NV; i += 4) {
      Vec<float>::load(a + c + i, va + i);
      if (b) Vec<float>::load(b + c + i, vb + i);
    }
    if (b) {
#pragma unroll
      for (int i = 0; i < NV; ++i) va[i] += vb[i];
    }
    Vec<T>::store(o + c, va);
  }
}

template <typename T>
cudaError_t launch_embed_fwd(const int* tok, const int* pos, const float* wte, const float* wpe, T* x,
                             int M, int C, cudaStream_t s) {
  ++g_kernel_launches;
  return launch_k(embed_fwd_kernel<T>, dim3((M + 7) / 8), dim3(256), 0, s, tok, pos, wte, wpe, x, M, C);
}

// ---------------------------------------------------------------------------
// LayerNorm forward: one warp per row, the row kept in registers.  Biased
// variance, y = (x - mean) * rstd * g + b; mean and rstd kept for backward.
// ---------------------------------------------------------------------------
template <typename T, int NCH>
__global__ void __launch_bounds__(256, (NCH * Vec<T>::N <= 24 ? 4 : 2)) ln_fwd_kernel(const T* __restrict__ x, const float* __restrict__ g,
                                                        const float* __restrict__ b, T* __restrict__ y,
                                                        float* __restrict__ mean, float* __restrict__ rstd, int M,
                                                        int C, float eps) {
  // one warp per row, warps walk rows with a grid stride over a grid of one
  // resident wave; the next row's x is loaded before the current row is
  // reduced, so each warp keeps two rows in flight.  gamma and beta are read
  // per row through L1 (a few KB, always resident) rather than held in
  // registers: for rows of up to 24 values per lane (C = 768 in bf16) the
  // kernel fits in 64 registers and four 256-thread blocks share an SM, which
  // is what keeps enough bytes in flight to cover HBM latency.
  constexpr int NV = Vec<T>::N;
  griddep_wait();
  griddep_release();
  const int lane = threadIdx.x & 31;
  const int nch = C / NV;
  const float inv_c = 1.0f / C;
  const int stride = gridDim.x * (blockDim.x >> 5);
  int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  uint4 nxt[NCH];
  auto fetch = [&](int r) {
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int ch = lane + i * 32;
      if (r < M && ch < nch) nxt[i] = *reinterpret_cast<const uint4*>(x + (long)r * C + ch * NV);
    }
  };
  fetch(row);
  for (; row < M; row += stride) {
    float v[NCH][NV];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      if (lane + i * 32 < nch) Vec<T>::load(reinterpret_cast<const T*>(&nxt[i]), v[i]);
      else
#pragma unroll
        for (int j = 0; j < NV; ++j) v[i][j] = 0.f;
    }
    fetch(row + stride);
    // two interleaved partial sums per lane halve the dependent-add chains;
    // the row normalises as x * rs + (-mu * rs), then gamma and beta by one FMA
    float sum2[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int j = 0; j < NV; ++j) sum2[j & 1] += v[i][j];
    const bool rms = b == nullptr;   // RMSNorm: no mean, no shift
    const float mu = rms ? 0.f : warp_sum(sum2[0] + sum2[1]) * inv_c;
    float sq2[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      if (lane + i * 32 < nch) {
#pragma unroll
        for (int j = 0; j < NV; ++j) { const float d = v[i][j] - mu; sq2[j & 1] = fmaf(d, d, sq2[j & 1]); }
      }
    }
    const float rs = 1.0f / sqrtf(warp_sum(sq2[0] + sq2[1]) * inv_c + eps);
    const float nb = -mu * rs;
    T* yr = y + (long)row * C;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int ch = lane + i * 32;
      if (ch < nch) {
        float o[NV];
#pragma unroll
        for (int j = 0; j < NV; j += 4) {
          const float4 gv = __ldg(reinterpret_cast<const float4*>(g + ch * NV + j));
          const float4 bv = rms ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldg(reinterpret_cast<const float4*>(b + ch * NV + j));
          o[j] = fmaf(fmaf(v[i][j], rs, nb), gv.x, bv.x);
          o[j + 1] = fmaf(fmaf(v[i][j + 1], rs, nb), gv.y, bv.y);
          o[j + 2] = fmaf(fmaf(v[i][j + 2], rs, nb), gv.z, bv.z);
          o[j + 3] = fmaf(fmaf(v[i][j + 3], rs, nb), gv.w, bv.w);
        }
        Vec<T>::store(yr + ch * NV, o);
      }
    }
    if (lane == 0) { mean[row] = mu; rstd[row] = rs; }
  }
}

// Blocks of one resident wave for a kernel of 256-thread blocks (occupancy
// queried once per kernel).
template <auto KERN>
static int resident_blocks(int want) {
  static int per_sm = 0, sms = 0;
  if (!per_sm) {
    int dev = 0, n = 0, occ = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, KERN, 256, 0);
    sms = n > 0 ? n : 148;
    per_sm = occ > 0 ? occ : 1;
  }
  const int cap = per_sm * sms;
  return want < cap ? want : cap;
}

template <typename T>
cudaError_t launch_ln_fwd(const T* x, const float* g, const float* b, T* y, float* mean, float* rstd,
                          int M, int C, float eps, cudaStream_t s) {
  constexpr int NV = Vec<T>::N;
  const int per = (C / NV + 31) / 32;   // 16-byte chunks per lane
  const int want = (M + 7) / 8;
  ++g_kernel_launches;
  cudaError_t e = cudaSuccess;
#define LNF_CASE(K)                                                                                  \
  case K:                                                                                            \
    e = launch_k(ln_fwd_kernel<T, K>, dim3(resident_blocks<ln_fwd_kernel<T, K>>(want)), dim3(256), 0, s, x, g, b, \
                 y, mean, rstd, M, C, eps);                                                          \
    break;
  switch (per) {
    LNF_CASE(1)
    LNF_CASE(2)
    LNF_CASE(3)
    LNF_CASE(4)
    default:
      if constexpr (NV >= 8) return cudaErrorInvalidValue;
      else {
        e = launch_k(ln_fwd_kernel<T, 8>, dim3(resident_blocks<ln_fwd_kernel<T, 8>>(want)), dim3(256), 0, s, x, g, b,
                     y, mean, rstd, M, C, eps);
        break;
      }
  }
#undef LNF_CASE
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ---------------------------------------------------------------------------
// LayerNorm backward, fused with the residual-gradient add:
//   dx = rstd (gh - mean(gh) - xhat mean(gh xhat)),  gh = dy * g
//   dres_out = dres_in + dx (fp32) and its T copy (the next GEMM operand);
// per-block partial sums of dg = sum dy*xhat and db = sum dy go to
// partials[block][0..C) and [C..2C).
// ---------------------------------------------------------------------------
#define LNB_WARPS 4
// NCH = 16-byte chunks per lane (C <= 32 * NCH * Vec<T>::N): the row and the
// warp's column accumulators stay in registers.
template <typename T, int NCH>
__global__ void __launch_bounds__(LNB_WARPS * 32)
ln_bwd_kernel(const T* __restrict__ dy, const T* __restrict__ x, const float* __restrict__ mean,
              const float* __restrict__ rstd, const float* __restrict__ g, const float* dres_in,
              float* dres_out, T* __restrict__ dres_out_t, float* __restrict__ partials, int M, int C) {
  // partial row of this block: [dg (C) | db (C) | column sums of dres_out (C)]
  constexpr int NV = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = C / NV;
  float dg[NCH][NV], db[NCH][NV], dsm[NCH][NV];
#pragma unroll
  for (int i = 0; i < NCH; ++i)
#pragma unroll
    for (int j = 0; j < NV; ++j) { dg[i][j] = 0.f; db[i][j] = 0.f; dsm[i][j] = 0.f; }
  for (int row = blockIdx.x * LNB_WARPS + warp; row < M; row += gridDim.x * LNB_WARPS) {
    const float mu = mean[row], rs = rstd[row];
    const T* dyr = dy + (long)row * C;
    const T* xr = x + (long)row * C;
    // every load of the row is issued before the first use (one memory latency
    // per row); dy and x stay packed until they are used
    uint4 dyp[NCH], xp[NCH];
    float o[NCH][NV];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int ch = lane + i * 32;
      if (ch < nch) {
        dyp[i] = *reinterpret_cast<const uint4*>(dyr + ch * NV);
        xp[i] = *reinterpret_cast<const uint4*>(xr + ch * NV);
        if (dres_in) {
#pragma unroll
          for (int j = 0; j < NV; j += 4) Vec<float>::load(dres_in + (long)row * C + ch * NV + j, o[i] + j);
        } else {
#pragma unroll
          for (int j = 0; j < NV; ++j) o[i][j] = 0.f;
        }
      }
    }
    float xh[NCH][NV], gh[NCH][NV];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int ch = lane + i * 32;
      if (ch < nch) {
        float dv[NV], gg[NV];
        Vec<T>::load(reinterpret_cast<const T*>(&dyp[i]), dv);
        Vec<T>::load(reinterpret_cast<const T*>(&xp[i]), xh[i]);
#pragma unroll
        for (int j = 0; j < NV; j += 4) Vec<float>::load(g + ch * NV + j, gg + j);
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          xh[i][j] = (xh[i][j] - mu) * rs;
          gh[i][j] = dv[j] * gg[j];
          s1 += gh[i][j];
          s2 += gh[i][j] * xh[i][j];
          dg[i][j] += dv[j] * xh[i][j];
          db[i][j] += dv[j];
        }
      }
    }
    s1 = warp_sum(s1) / C;
    s2 = warp_sum(s2) / C;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int ch = lane + i * 32;
      if (ch < nch) {
        const long off = (long)row * C + ch * NV;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          o[i][j] += rs * (gh[i][j] - s1 - xh[i][j] * s2);
          dsm[i][j] += o[i][j];
        }
#pragma unroll
        for (int j = 0; j < NV; j += 4) Vec<float>::store(dres_out + off + j, o[i] + j);
        Vec<T>::store(dres_out_t + off, o[i]);
      }
    }
  }
  // sum the warps' accumulators through shared memory, one section at a time
  extern __shared__ float red_sm[];   // [LNB_WARPS][C]
  for (int sec = 0; sec < 3; ++sec) {
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int ch = lane + i * 32;
      if (ch < nch) {
#pragma unroll
        for (int j = 0; j < NV; ++j)
          red_sm[warp * C + ch * NV + j] = sec == 0 ? dg[i][j] : (sec == 1 ? db[i][j] : dsm[i][j]);
      }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < LNB_WARPS; ++w) acc += red_sm[w * C + c];
      partials[(long)blockIdx.x * 3 * C + sec * C + c] = acc;
    }
    __syncthreads();
  }
}

template <typename T, int NCH>
static cudaError_t ln_bwd_launch(const T* dy, const T* x, const float* mean, const float* rstd, const float* g,
                                 const float* dres_in, float* dres_out, T* dres_out_t, float* partials, int M,
                                 int C, int nblk, cudaStream_t s) {
  size_t smem = (size_t)LNB_WARPS * C * sizeof(float);
  ++g_kernel_launches;
  ln_bwd_kernel<T, NCH><<<nblk, LNB_WARPS * 32, smem, s>>>(dy, x, mean, rstd, g, dres_in, dres_out, dres_out_t,
                                                           partials, M, C);
  return cudaGetLastError();
}

// LayerNorm backward, row-group form: TPR = C / NV threads (one 16-byte chunk
// each) share a row, G groups per block walk rows with a stride; the next
// row's loads are issued before the current row's reduction, and the row sums
// go through a per-group named barrier with double-buffered slots.  Column
// accumulators (dgamma, dbeta, column sums of the residual gradient) are 24
// registers per thread, summed over groups into one partial row per block.
#define LNB2_THREADS 288
template <typename T>
__global__ void __launch_bounds__(LNB2_THREADS, 2)
ln_bwd2_kernel(const T* __restrict__ dy, const T* __restrict__ x, const float* __restrict__ mean,
               const float* __restrict__ rstd, const float* __restrict__ g, const float* dres_in, float* dres_out,
               T* __restrict__ dres_out_t, float* __restrict__ partials, int M, int C, int TPR, int G, int rms) {
  griddep_wait();
  griddep_release();
  constexpr int NV = Vec<T>::N;
  __shared__ float2 slot[2][LNB2_THREADS / 32];
  const int grp = threadIdx.x / TPR, t = threadIdx.x % TPR;
  const int nch = C / NV;
  const bool act = grp < G && t < nch;
  const int wpg = TPR / 32, wig = t / 32, lane = threadIdx.x & 31;
  const int col = t * NV;
  float gg[NV], dg[NV], db[NV], dsm[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) { gg[j] = 0.f; dg[j] = 0.f; db[j] = 0.f; dsm[j] = 0.f; }
  if (act) {
#pragma unroll
    for (int j = 0; j < NV; j += 4) Vec<float>::load(g + col + j, gg + j);
  }
  const int stride = gridDim.x * G;
  int row = blockIdx.x * G + grp;
  // prefetch of a row: dy, x packed, the residual gradient in fp32, mean, rstd
  uint4 dyp = make_uint4(0, 0, 0, 0), xp = make_uint4(0, 0, 0, 0);
  float dr[NV], mu = 0.f, rs = 0.f;
  auto fetch = [&](int r) {
    if (act && r < M) {
      dyp = *reinterpret_cast<const uint4*>(dy + (long)r * C + col);
      xp = *reinterpret_cast<const uint4*>(x + (long)r * C + col);
      if (dres_in) {
#pragma unroll
        for (int j = 0; j < NV; j += 4) Vec<float>::load(dres_in + (long)r * C + col + j, dr + j);
      } else {
#pragma unroll
        for (int j = 0; j < NV; ++j) dr[j] = 0.f;
      }
      mu = mean[r];
      rs = rstd[r];
    }
  };
  fetch(row);
  int it = 0;
  // every group runs the same number of iterations (rows past M are idle) so
  // its named barrier always sees all of its threads
  const int iters = (M + stride - 1) / stride;
  for (; it < iters; ++it, row += stride) {
    float dv[NV], xh[NV], o[NV];
    Vec<T>::load(reinterpret_cast<const T*>(&dyp), dv);
    Vec<T>::load(reinterpret_cast<const T*>(&xp), xh);
#pragma unroll
    for (int j = 0; j < NV; ++j) o[j] = dr[j];
    const float mu_r = mu, rs_r = rs;
    const bool live = act && row < M;
    fetch(row + stride);
    float s1 = 0.f, s2 = 0.f, gh[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      xh[j] = (xh[j] - mu_r) * rs_r;
      gh[j] = dv[j] * gg[j];
      s1 += gh[j];
      s2 += gh[j] * xh[j];
      if (live) { dg[j] += dv[j] * xh[j]; db[j] += dv[j]; }
    }
    s1 = warp_sum(live ? s1 : 0.f);
    s2 = warp_sum(live ? s2 : 0.f);
    if (lane == 0 && grp < G) slot[it & 1][grp * wpg + wig] = make_float2(s1, s2);
    if (grp < G) asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(TPR) : "memory");
    s1 = 0.f; s2 = 0.f;
    for (int w = 0; w < wpg; ++w) {
      const float2 v = slot[it & 1][grp * wpg + w];
      s1 += v.x;
      s2 += v.y;
    }
    s1 = rms ? 0.f : s1 / C;   // RMSNorm: no mean term
    s2 /= C;
    if (live) {
      const long off = (long)row * C + col;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        o[j] += rs_r * (gh[j] - s1 - xh[j] * s2);
        dsm[j] += o[j];
      }
#pragma unroll
      for (int j = 0; j < NV; j += 4) Vec<float>::store(dres_out + off + j, o + j);
      Vec<T>::store(dres_out_t + off, o);
    }
  }
  // sum the groups' accumulators: [dg | db | dsm] per block
  __syncthreads();
  extern __shared__ float red2[];   // [G][3C]
  if (act) {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      red2[grp * 3 * C + col + j] = dg[j];
      red2[grp * 3 * C + C + col + j] = db[j];
      red2[grp * 3 * C + 2 * C + col + j] = dsm[j];
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 3 * C; c += blockDim.x) {
    float acc = 0.f;
    for (int gi = 0; gi < G; ++gi) acc += red2[gi * 3 * C + c];
    partials[(long)blockIdx.x * 3 * C + c] = acc;
  }
}

// The same row-group backward with the next LNB3_NS rows of every group (dy,
// x and the incoming residual gradient) in a ring of shared-memory slots
// filled by bulk copies: each group keeps LNB3_NS rows in flight without
// holding them in registers, so a block moves three times the bytes of the
// register-prefetch form per memory latency.  A slot is refilled by the
// group's first thread once the group's named barrier shows that every thread
// has read it; the arithmetic and its order are those of ln_bwd2_kernel, so the
// results are the same bits.  Needs 16-byte aligned rows (C * sizeof(T) % 16
// == 0 and aligned bases).
#define LNB3_NS 2
template <typename T>
__global__ void __launch_bounds__(LNB2_THREADS, 2)
ln_bwd3_kernel(const T* __restrict__ dy, const T* __restrict__ x, const float* __restrict__ mean,
               const float* __restrict__ rstd, const float* __restrict__ g, const float* dres_in, float* dres_out,
               T* __restrict__ dres_out_t, float* __restrict__ partials, int M, int C, int TPR, int G, int rms,
               unsigned* __restrict__ err) {
  constexpr int NV = Vec<T>::N;
  extern __shared__ __align__(16) uint8_t lb3_raw[];
  __shared__ __align__(8) uint64_t full[LNB2_THREADS / 32][LNB3_NS];
  __shared__ float2 slot[2][LNB2_THREADS / 32];
  const int grp = threadIdx.x / TPR, t = threadIdx.x % TPR;
  const int nch = C / NV;
  const bool act = grp < G && t < nch;
  const int wpg = TPR / 32, wig = t / 32, lane = threadIdx.x & 31;
  const int col = t * NV;
  // one slot: dy | x | incoming residual gradient (absent for the first backward)
  const uint32_t tb = (uint32_t)C * sizeof(T), fb = dres_in ? (uint32_t)C * 4u : 0u;
  const uint32_t sb = 2 * tb + fb;
  const uint32_t ring = smem_u32(lb3_raw) + grp * LNB3_NS * sb;
  const int stride = gridDim.x * G;
  int row = blockIdx.x * G + grp;
  auto fbar = [&](int s) { return smem_u32(&full[grp][s]); };
  auto issue = [&](int r, int s) {
    const uint32_t bar = fbar(s), dst = ring + s * sb;
    mbar_expect_tx(bar, sb);
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(dy + (long)r * C)), "r"(tb), "r"(bar) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst + tb), "l"(reinterpret_cast<uint64_t>(x + (long)r * C)), "r"(tb), "r"(bar) : "memory");
    if (fb)
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(dst + 2 * tb), "l"(reinterpret_cast<uint64_t>(dres_in + (long)r * C)), "r"(fb), "r"(bar)
                   : "memory");
  };
  if (grp < G && t == 0) {
    for (int s = 0; s < LNB3_NS; ++s) mbar_init(fbar(s), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  griddep_wait();
  griddep_release();
  if (grp < G && t == 0)
    for (int s = 0; s < LNB3_NS; ++s)
      if (row + s * stride < M) issue(row + s * stride, s);
  float gg[NV], dg[NV], db[NV], dsm[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) { gg[j] = 0.f; dg[j] = 0.f; db[j] = 0.f; dsm[j] = 0.f; }
  if (act) {
#pragma unroll
    for (int j = 0; j < NV; j += 4) Vec<float>::load(g + col + j, gg + j);
  }
  float mu = 0.f, rs = 0.f;
  if (act && row < M) { mu = mean[row]; rs = rstd[row]; }
  __syncthreads();   // the barriers are initialised before any thread waits on them
  // every issued copy is waited for, each wait bounded (a wait that gives up
  // flags the step and the kernel still ends)
  volatile int never = 0;
  const int iters = (M + stride - 1) / stride;
  for (int it = 0; it < iters; ++it, row += stride) {
    const int s = it % LNB3_NS;
    const bool live = act && row < M;
    float dv[NV], xh[NV], o[NV];
    if (grp < G && row < M && !mbar_wait(fbar(s), (it / LNB3_NS) & 1, &never, 1ll << 28) && t == 0)
      atomicOr(err, GPT_DEVERR_TIMEOUT);
    if (live) {
      const uint32_t src = ring + s * sb + col * (uint32_t)sizeof(T);
      uint4 q;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(q.x), "=r"(q.y), "=r"(q.z), "=r"(q.w) : "r"(src));
      Vec<T>::load(reinterpret_cast<const T*>(&q), dv);
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(q.x), "=r"(q.y), "=r"(q.z), "=r"(q.w) : "r"(src + tb));
      Vec<T>::load(reinterpret_cast<const T*>(&q), xh);
      if (fb) {
        const uint32_t fsrc = ring + s * sb + 2 * tb + col * 4u;
#pragma unroll
        for (int j = 0; j < NV; j += 4)
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(o[j]), "=f"(o[j + 1]), "=f"(o[j + 2]), "=f"(o[j + 3]) : "r"(fsrc + 4u * j));
      } else {
#pragma unroll
        for (int j = 0; j < NV; ++j) o[j] = 0.f;
      }
    } else {
#pragma unroll
      for (int j = 0; j < NV; ++j) { dv[j] = 0.f; xh[j] = 0.f; o[j] = 0.f; }
    }
    const float mu_r = mu, rs_r = rs;
    if (act && row + stride < M) { mu = mean[row + stride]; rs = rstd[row + stride]; }
    float s1 = 0.f, s2 = 0.f, gh[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      xh[j] = (xh[j] - mu_r) * rs_r;
      gh[j] = dv[j] * gg[j];
      s1 += gh[j];
      s2 += gh[j] * xh[j];
      if (live) { dg[j] += dv[j] * xh[j]; db[j] += dv[j]; }
    }
    s1 = warp_sum(live ? s1 : 0.f);
    s2 = warp_sum(live ? s2 : 0.f);
    if (lane == 0 && grp < G) slot[it & 1][grp * wpg + wig] = make_float2(s1, s2);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // slot reads before the refill's writes
    if (grp < G) asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(TPR) : "memory");
    if (grp < G && t == 0 && row + LNB3_NS * stride < M) issue(row + LNB3_NS * stride, s);
    s1 = 0.f; s2 = 0.f;
    for (int w = 0; w < wpg; ++w) {
      const float2 v = slot[it & 1][grp * wpg + w];
      s1 += v.x;
      s2 += v.y;
    }
    s1 = rms ? 0.f : s1 / C;   // RMSNorm: no mean term
    s2 /= C;
    if (live) {
      const long off = (long)row * C + col;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        o[j] += rs_r * (gh[j] - s1 - xh[j] * s2);
        dsm[j] += o[j];
      }
#pragma unroll
      for (int j = 0; j < NV; j += 4) Vec<float>::store(dres_out + off + j, o + j);
      Vec<T>::store(dres_out_t + off, o);
    }
  }
  // every issued copy has been waited for (each group consumes the rows it
  // prefetched), so the ring is free for the group sums: [dg | db | dsm] per block
  __syncthreads();
  float* red2 = reinterpret_cast<float*>(lb3_raw);
  if (act) {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      red2[grp * 3 * C + col + j] = dg[j];
      red2[grp * 3 * C + C + col + j] = db[j];
      red2[grp * 3 * C + 2 * C + col + j] = dsm[j];
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 3 * C; c += blockDim.x) {
    float acc = 0.f;
    for (int gi = 0; gi < G; ++gi) acc += red2[gi * 3 * C + c];
    partials[(long)blockIdx.x * 3 * C + c] = acc;
  }
}

template <typename T>
cudaError_t launch_ln_bwd(const T* dy, const T* x, const float* mean, const float* rstd, const float* g,
                          const float* dres_in, float* dres_out, T* dres_out_t, float* partials,
                          int M, int C, int* nblk_out, cudaStream_t s, bool rms, unsigned* err) {
  constexpr int NV = Vec<T>::N;
  {
    // row-group kernel: C / NV threads per row (whole warps), several rows per block
    const int tpr = ((C / NV + 31) / 32) * 32;
    if (C % NV == 0 && tpr <= LNB2_THREADS) {
      const int G = LNB2_THREADS / tpr;
      int nblk = (M + G - 1) / G;
      if (nblk > 148 * 2) nblk = 148 * 2;
      *nblk_out = nblk;
      // bulk-copied rows when every row starts on a 16-byte boundary
      const bool bulk = err && (C * sizeof(T)) % 16 == 0 && ((uintptr_t)dy & 15) == 0 && ((uintptr_t)x & 15) == 0 &&
                        ((uintptr_t)dres_in & 15) == 0;
      if (bulk) {
        const size_t sb = (size_t)C * (2 * sizeof(T) + (dres_in ? 4 : 0));
        const size_t smem3 = std::max((size_t)G * LNB3_NS * sb, (size_t)G * 3 * C * sizeof(float));
        static size_t attr3 = 0;
        if (smem3 > 48 * 1024 && smem3 > attr3) {
          cudaError_t e = cudaFuncSetAttribute(ln_bwd3_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3);
          if (e != cudaSuccess) return e;
          attr3 = smem3;
        }
        ++g_kernel_launches;
        return launch_k(ln_bwd3_kernel<T>, dim3(nblk), dim3(G * tpr), smem3, s, dy, x, mean, rstd, g, dres_in,
                        dres_out, dres_out_t, partials, M, C, tpr, G, rms ? 1 : 0, err);
      }
      const size_t smem = (size_t)G * 3 * C * sizeof(float);
      static size_t attr = 0;
      if (smem > 48 * 1024 && smem > attr) {
        cudaError_t e = cudaFuncSetAttribute(ln_bwd2_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = smem;
      }
      ++g_kernel_launches;
      return launch_k(ln_bwd2_kernel<T>, dim3(nblk), dim3(G * tpr), smem, s,
                      dy, x, mean, rstd, g, dres_in, dres_out, dres_out_t, partials, M, C, tpr, G, rms ? 1 : 0);
    }
  }
  if (rms) return cudaErrorNotSupported;   // the register-row form has no RMSNorm variant
  int nblk = (M + LNB_WARPS - 1) / LNB_WARPS;
  if (nblk > 148 * 3) nblk = 148 * 3;
  *nblk_out = nblk;
  int per_lane = (C / NV + 31) / 32;   // 16-byte chunks per lane
  switch (per_lane) {
    case 1: return ln_bwd_launch<T, 1>(dy, x, mean, rstd, g, dres_in, dres_out, dres_out_t, partials, M, C, nblk, s);
    case 2: return ln_bwd_launch<T, 2>(dy, x, mean, rstd, g, dres_in, dres_out, dres_out_t, partials, M, C, nblk, s);
    case 3: return ln_bwd_launch<T, 3>(dy, x, mean, rstd, g, dres_in, dres_out, dres_out_t, partials, M, C, nblk, s);
    case 4: return ln_bwd_launch<T, 4>(dy, x, mean, rstd, g, dres_in, dres_out, dres_out_t, partials, M, C, nblk, s);
    default:   // C <= 1024: at most 4 chunks of 8 bf16 or 8 chunks of 4 fp32
      if constexpr (NV >= 8) return cudaErrorInvalidValue;
      else return ln_bwd_launch<T, 8>(dy, x, mean, rstd, g, dres_in, dres_out, dres_out_t, partials, M, C, nblk, s);
  }
}

// Deferred column reductions: every segment is dst[n] = sum over r < rows of
// src[r * ld + n], n < cols, summed in a fixed order (deterministic).  All
// the per-block partial rows a backward pass leaves (LayerNorm dg/db, bias
// gradients) are reduced by one launch instead of one small launch each.
// A block takes 128 columns of one segment: 32 column quads x 8 row groups,
// row group g summing rows g, g+8, ...; the groups are then added in order.
__global__ void __launch_bounds__(256) reduce_segs_kernel(RedSegList L) {
  griddep_wait();
  griddep_release();
  __shared__ float red[8][129];
  int si = 0;
  while (si + 1 < L.n && (int)blockIdx.x >= L.seg[si + 1].blk0) ++si;
  const RedSeg& sg = L.seg[si];
  const int q = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int c = ((int)blockIdx.x - sg.blk0) * 128 + 4 * q;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  if (c < sg.cols) {
    const bool vec = c + 4 <= sg.cols && (sg.ld & 3) == 0 && ((uintptr_t)sg.src & 15) == 0;
    if (vec) {
#pragma unroll 4
      for (int r = grp; r < sg.rows; r += 8) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(sg.src + (long)r * sg.ld + c));
        a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
      }
    } else {
      for (int r = grp; r < sg.rows; r += 8)
        for (int j = 0; j < 4 && c + j < sg.cols; ++j) a[j] += sg.src[(long)r * sg.ld + c + j];
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) red[grp][4 * q + j] = a[j];
  __syncthreads();
  if (threadIdx.x < 128) {
    const int n = ((int)blockIdx.x - sg.blk0) * 128 + threadIdx.x;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += red[w][threadIdx.x];
    if (n < sg.cols) sg.dst[n] = L.add ? sg.dst[n] + acc : acc;
  }
}

cudaError_t launch_reduce_segs(const RedSeg* segs, int n, bool add, cudaStream_t s) {
  for (int i0 = 0; i0 < n; i0 += RED_MAX_SEGS) {
    RedSegList L;
    L.add = add ? 1 : 0;
    L.n = n - i0 < RED_MAX_SEGS ? n - i0 : RED_MAX_SEGS;
    int blk = 0;
    for (int i = 0; i < L.n; ++i) {
      L.seg[i] = segs[i0 + i];
      L.seg[i].blk0 = blk;
      blk += (L.seg[i].cols + 127) / 128;
    }
    if (blk == 0) continue;
    ++g_kernel_launches;
    cudaError_t e = launch_k(reduce_segs_kernel, dim3(blk), dim3(256), 0, s, L);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Column sums of x [M, N] (bias gradients): blocks of 128 columns x 256 rows
// (4 columns per lane, 8 warps x 32 rows) write per-row-chunk partials; a
// deferred reduction segment sums the chunks.
#define CS_ROWS 256
template <typename Tin>
__global__ void __launch_bounds__(256) colsum_kernel(const Tin* __restrict__ x, long ldx, int M, int N,
                                                     float* __restrict__ partials) {
  __shared__ float red[8][128];
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int c0 = blockIdx.x * 128 + lane * 4;
  int r0 = blockIdx.y * CS_ROWS + warp * (CS_ROWS / 8);
  int r1 = min(M, r0 + CS_ROWS / 8);
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  if (c0 < N) {
    bool full = c0 + 4 <= N && (ldx & 3) == 0;
    for (int r = r0; r < r1; ++r) {
      const Tin* row = x + (long)r * ldx + c0;
      if (full) {
#pragma unroll
        for (int j = 0; j < 4; ++j) a[j] += to_f(row[j]);
      } else {
        for (int j = 0; j < 4 && c0 + j < N; ++j) a[j] += to_f(row[j]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) red[warp][lane * 4 + j] = a[j];
  __syncthreads();
  if (threadIdx.x < 128) {
    int c = blockIdx.x * 128 + threadIdx.x;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += red[w][threadIdx.x];
    if (c < N) partials[(long)blockIdx.y * N + c] = acc;
  }
}

// 16-bit (bf16 or fp16) column sums with 16-byte loads: a block covers 256 columns (32 lanes
// x 8 columns) and CS2_ROWS rows split over 8 warps, four rows in flight per
// thread; one partial row per block row-chunk.
#define CS2_ROWS 256
template <typename T16>
__global__ void __launch_bounds__(256) colsum16_kernel(const T16* __restrict__ x, long ldx, int M, int N,
                                                       float* __restrict__ partials) {
  griddep_wait();
  griddep_release();
  __shared__ float red[8][257];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * 256 + lane * 8;
  const int rb = blockIdx.y * CS2_ROWS, re = min(M, rb + CS2_ROWS);
  float a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = 0.f;
  if (c0 < N) {
    int r = rb + warp;
    for (; r + 24 < re; r += 32) {
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) w[u] = *reinterpret_cast<const uint4*>(x + (long)(r + 8 * u) * ldx + c0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float v[8];
        Vec<T16>::load(reinterpret_cast<const T16*>(&w[u]), v);
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] += v[j];
      }
    }
    for (; r < re; r += 8) {
      float v[8];
      Vec<T16>::load(x + (long)r * ldx + c0, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] += v[j];
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[warp][lane * 8 + j] = a[j];
  __syncthreads();
  const int c = blockIdx.x * 256 + threadIdx.x;
  float acc = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) acc += red[w][threadIdx.x];
  if (c < N) partials[(long)blockIdx.y * N + c] = acc;
}

template <typename Tin>
cudaError_t launch_colsum(const Tin* x, long ldx, int M, int N, float* partials, int* rows_out, cudaStream_t s) {
  if constexpr (sizeof(Tin) == 2) {
    if (N % 8 == 0 && ldx % 8 == 0 && ((uintptr_t)x & 15) == 0) {
      dim3 g2((N + 255) / 256, (M + CS2_ROWS - 1) / CS2_ROWS);
      *rows_out = (int)g2.y;
      ++g_kernel_launches;
      return launch_k(colsum16_kernel<Tin>, g2, dim3(256), 0, s, x, ldx, M, N, partials);
    }
  }
  dim3 grid((N + 127) / 128, (M + CS_ROWS - 1) / CS_ROWS);
  *rows_out = (int)grid.y;
  ++g_kernel_launches;
  colsum_kernel<Tin><<<grid, 256, 0, s>>>(x, ldx, M, N, partials);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Fused softmax cross-entropy and its gradient, in place over the logits.
// Per row: lse over the real vocabulary 0..V-1 (online max / sum), loss =
// lse - z[target]; then dz = (softmax - onehot) * loss_scale * loss_weight / N_valid for
// c < V, 0 for the padded columns and for ignored rows.  No fp32
// probability tensor is written.  ("RustGPT", "Technical implementation":
// cross-entropy loss.)
// ---------------------------------------------------------------------------
#define XENT_THREADS 512
template <typename T>
__global__ void __launch_bounds__(XENT_THREADS)
xent_kernel(T* __restrict__ logits, long ldl, const int* __restrict__ tgt, int V, int Vp,
            float* __restrict__ rowloss, const DevScalars* __restrict__ sc) {
  constexpr int NV = Vec<T>::N;
  int row = blockIdx.x;
  T* z = logits + (long)row * ldl;
  int tg = tgt[row];
  float m = -INFINITY, ssum = 0.f;
  int nvec = V / NV;
  for (int i = threadIdx.x; i < nvec; i += XENT_THREADS) {
    float v[NV];
    Vec<T>::load(z + i * NV, v);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      if (v[j] > m) { ssum = ssum * expf(m - v[j]) + 1.f; m = v[j]; }
      else ssum += expf(v[j] - m);
    }
  }
  for (int c = nvec * NV + threadIdx.x; c < V; c += XENT_THREADS) {
    float v = to_f(z[c]);
    if (v > m) { ssum = ssum * expf(m - v) + 1.f; m = v; }
    else ssum += expf(v - m);
  }
  // merge (m, s) across the block
  __shared__ float sm[XENT_THREADS / 32], ss[XENT_THREADS / 32];
  __shared__ float s_lse, s_ztg;
  float wm = warp_max(m);
  float ws = warp_sum(m == -INFINITY ? 0.f : ssum * expf(m - wm));
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sm[warp] = wm; ss[warp] = ws; }
  __syncthreads();
  if (warp == 0) {
    float mm = lane < XENT_THREADS / 32 ? sm[lane] : -INFINITY;
    float s2 = lane < XENT_THREADS / 32 ? ss[lane] : 0.f;
    float gm = warp_max(mm);
    float gs = warp_sum(mm == -INFINITY ? 0.f : s2 * expf(mm - gm));
    if (lane == 0) {
      s_lse = gm + logf(gs);
      s_ztg = tg >= 0 ? to_f(z[tg]) : 0.f;
    }
  }
  __syncthreads();
  float lse = s_lse;
  if (threadIdx.x == 0) rowloss[row] = tg >= 0 ? lse - s_ztg : 0.f;
  int nv = sc->n_valid;
  float scale = tg >= 0 ? sc->loss_scale * sc->loss_weight / (float)(nv > 0 ? nv : 1) : 0.f;
  int nvp = Vp / NV;
  for (int i = threadIdx.x; i < nvp; i += XENT_THREADS) {
    float v[NV];
    Vec<T>::load(z + i * NV, v);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      int c = i * NV + j;
      float p = c < V ? expf(v[j] - lse) : 0.f;
      v[j] = (p - (c == tg ? 1.f : 0.f)) * scale;
    }
    Vec<T>::store(z + i * NV, v);
  }
  for (int c = nvp * NV + threadIdx.x; c < Vp; c += XENT_THREADS) {
    float p = c < V ? expf(to_f(z[c]) - lse) : 0.f;
    z[c] = from_f<T>((p - (c == tg ? 1.f : 0.f)) * scale);
  }
}

// Same computation with the row staged in shared memory: one HBM read and
// one HBM write per logit (used when the padded row fits, e.g. 100 KB bf16).
__device__ __forceinline__ float block_reduce(float v, bool is_max, float* red) {
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = is_max ? warp_max(v) : warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float x = lane < (int)(blockDim.x >> 5) ? red[lane] : (is_max ? -INFINITY : 0.f);
    x = is_max ? warp_max(x) : warp_sum(x);
    if (lane == 0) red[32] = x;
  }
  __syncthreads();
  return red[32];
}

template <typename T>
__global__ void __launch_bounds__(XENT_THREADS)
xent_smem_kernel(T* __restrict__ logits, long ldl, const int* __restrict__ tgt, int V, int Vp,
                 float* __restrict__ rowloss, const DevScalars* __restrict__ sc) {
  constexpr int NV = Vec<T>::N;
  extern __shared__ __align__(16) uint8_t xent_raw[];
  T* zs = reinterpret_cast<T*>(xent_raw);
  __shared__ float red[33];
  const int row = blockIdx.x;
  T* z = logits + (long)row * ldl;
  const int tg = tgt[row];
  const int nvec = (Vp + NV - 1) / NV;   // ldl >= nvec * NV
  float m = -INFINITY;
  for (int i = threadIdx.x; i < nvec; i += XENT_THREADS) {
    uint4 raw = *reinterpret_cast<const uint4*>(z + i * NV);
    *reinterpret_cast<uint4*>(zs + i * NV) = raw;
    float v[NV];
    Vec<T>::load(zs + i * NV, v);
#pragma unroll
    for (int j = 0; j < NV; ++j)
      if (i * NV + j < V) m = fmaxf(m, v[j]);
  }
  m = block_reduce(m, true, red);
  // e = exp(z - max), kept in place of z (z[target] is read first); the
  // second pass only scales: dz = e / sum - onehot
  const float zt = tg >= 0 ? to_f(zs[tg]) : 0.f;
  __syncthreads();
  float ssum = 0.f;
  for (int i = threadIdx.x; i < nvec; i += XENT_THREADS) {
    float v[NV];
    Vec<T>::load(zs + i * NV, v);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      v[j] = i * NV + j < V ? exp2f((v[j] - m) * 1.4426950408889634f) : 0.f;
      ssum += v[j];
    }
    Vec<T>::store(zs + i * NV, v);
  }
  ssum = block_reduce(ssum, false, red);
  if (threadIdx.x == 0) rowloss[row] = tg >= 0 ? m + logf(ssum) - zt : 0.f;
  const int nv = sc->n_valid;
  const float scale = tg >= 0 ? sc->loss_scale * sc->loss_weight / (float)(nv > 0 ? nv : 1) : 0.f;
  const float inv = scale / ssum;
  for (int i = threadIdx.x; i < nvec; i += XENT_THREADS) {
    float v[NV];
    Vec<T>::load(zs + i * NV, v);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      int c = i * NV + j;
      v[j] = v[j] * inv - (c == tg ? scale : 0.f);
    }
    Vec<T>::store(z + i * NV, v);
  }
}

// 16-bit logits: the row moves between HBM and shared memory as one bulk copy
// each way (the copy engine keeps the whole row in flight); the three passes
// over it (max, exp and sum, scale) run on shared memory.  exp(z - max) is
// kept in place as 16-bit values and summed in fp32.
#define XB_THREADS 512
template <typename T16>
__global__ void __launch_bounds__(XB_THREADS, 2)
xent_bulk_kernel(T16* __restrict__ logits, long ldl, const int* __restrict__ tgt, int V, int Vp,
                 float* __restrict__ rowloss, DevScalars* __restrict__ sc) {
  griddep_wait();
  griddep_release();
  extern __shared__ __align__(128) uint8_t xb_raw[];
  __shared__ float red[33];
  __shared__ __align__(8) uint64_t bar;
  T16* zs = reinterpret_cast<T16*>(xb_raw);
  const int row = blockIdx.x;
  T16* z = logits + (long)row * ldl;
  const int tg = tgt[row];
  const int nvec = Vp / 8;
  const uint32_t bytes = (uint32_t)nvec * 16;
  const uint32_t sbar = smem_u32(&bar), sz = smem_u32(zs);
  if (threadIdx.x == 0) {
    mbar_init(sbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_expect_tx(sbar, bytes);
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(sz),
                 "l"(reinterpret_cast<uint64_t>(z)), "r"(bytes), "r"(sbar)
                 : "memory");
  }
  __syncthreads();
  {
    volatile int never = 0;
    if (!mbar_wait(sbar, 0, &never, 1ll << 30)) atomicOr(&sc->err, GPT_DEVERR_TIMEOUT);
  }
  const uint4* zv = reinterpret_cast<const uint4*>(zs);
  float m = -INFINITY;
  for (int i = threadIdx.x; i < nvec; i += XB_THREADS) {
    float v[8];
    const uint4 w = zv[i];
    Vec<T16>::load(reinterpret_cast<const T16*>(&w), v);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (i * 8 + j < V) m = fmaxf(m, v[j]);
  }
  m = block_reduce(m, true, red);
  const float zt = tg >= 0 ? to_f(zs[tg]) : 0.f;
  __syncthreads();   // z[target] is read before the exp pass overwrites it
  const float ml2 = m * 1.4426950408889634f;
  float ssum = 0.f;
  for (int i = threadIdx.x; i < nvec; i += XB_THREADS) {
    float v[8];
    uint4 w = zv[i];
    Vec<T16>::load(reinterpret_cast<const T16*>(&w), v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float e;
      asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(fmaf(v[j], 1.4426950408889634f, -ml2)));
      v[j] = i * 8 + j < V ? e : 0.f;
      ssum += v[j];
    }
    Vec<T16>::store(reinterpret_cast<T16*>(&w), v);
    reinterpret_cast<uint4*>(zs)[i] = w;
  }
  ssum = block_reduce(ssum, false, red);
  if (threadIdx.x == 0) rowloss[row] = tg >= 0 ? m + logf(ssum) - zt : 0.f;
  const int nv = sc->n_valid;
  const float scale = tg >= 0 ? sc->loss_scale * sc->loss_weight / (float)(nv > 0 ? nv : 1) : 0.f;
  const float inv = scale / ssum;
  for (int i = threadIdx.x; i < nvec; i += XB_THREADS) {
    float v[8];
    uint4 w = zv[i];
    Vec<T16>::load(reinterpret_cast<const T16*>(&w), v);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = v[j] * inv - (i * 8 + j == tg ? scale : 0.f);
    Vec<T16>::store(reinterpret_cast<T16*>(&w), v);
    reinterpret_cast<uint4*>(zs)[i] = w;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(z)),
                 "r"(sz), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // shared memory stays live until read
  }
}

template <typename T>
cudaError_t launch_xent(T* logits, long ldl, const int* tgt, int M, int V, int Vp, float* rowloss,
                        DevScalars* sc, cudaStream_t s) {
  constexpr int NV = Vec<T>::N;
  if constexpr (NV == 8) {
    // bulk copies: 16-byte aligned rows, whole row within 110 KB (two blocks per SM)
    const size_t bytes = (size_t)Vp * 2;
    if (Vp % 8 == 0 && ldl % 8 == 0 && bytes <= 110 * 1024) {
      static size_t attr = 0;
      if (bytes > attr) {
        cudaError_t e = cudaFuncSetAttribute(xent_bulk_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        attr = bytes;
      }
      ++g_kernel_launches;
      return launch_k(xent_bulk_kernel<T>, dim3(M), dim3(XB_THREADS), bytes, s, logits, ldl, tgt, V, Vp, rowloss, sc);
    }
  }
  size_t smem = (size_t)((Vp + NV - 1) / NV) * NV * sizeof(T);
  if (smem <= 200 * 1024 && (ldl % NV) == 0) {
    static size_t attr = 0;
    if (smem > attr) {
      cudaError_t e = cudaFuncSetAttribute(xent_smem_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
      attr = smem;
    }
    ++g_kernel_launches;
    xent_smem_kernel<T><<<M, XENT_THREADS, smem, s>>>(logits, ldl, tgt, V, Vp, rowloss, sc);
    return cudaGetLastError();
  }
  ++g_kernel_launches;
  xent_kernel<T><<<M, XENT_THREADS, 0, s>>>(logits, ldl, tgt, V, Vp, rowloss, sc);
  return cudaGetLastError();
}

__global__ void loss_finalize_kernel(const float* __restrict__ rowloss, int M, DevScalars* sc, float* loss_out) {
  griddep_wait();
  griddep_release();
  __shared__ float red[32];
  float acc = 0.f;
  for (int i = threadIdx.x; i < M; i += blockDim.x) acc += rowloss[i];
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) {
      int nv = sc->n_valid;
      float loss = nv > 0 ? v / (float)nv : 0.f;
      sc->loss = loss;
      if (loss_out) *loss_out = loss;
    }
  }
}

cudaError_t launch_loss_finalize(const float* rowloss, int M, DevScalars* sc, float* loss_out, cudaStream_t s) {
  ++g_kernel_launches;
  return launch_k(loss_finalize_kernel, dim3(1), dim3(1024), 0, s, rowloss, M, sc, loss_out);
}

// ---------------------------------------------------------------------------
// Embedding backward: scatter-add of the residual gradient into the token
// rows of dwte and the position rows of dwpe (fp32 atomics).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void embed_bwd_kernel(const float* __restrict__ dres, const int* __restrict__ tok,
                                 const int* __restrict__ pos, float* gwte, float* gwpe, int M, int C) {
  griddep_wait();
  griddep_release();
  // one warp per row; the row's fp32 gradient is loaded whole (up to 8
  // 16-byte vectors per lane in flight), then added into the token's and the
  // position's gradient rows with 16-byte vector atomics (a row's additions
  // land in no fixed order among the rows that share a token or position)
  int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float4* d = reinterpret_cast<const float4*>(dres + (long)row * C);
  float4* a = reinterpret_cast<float4*>(gwte + (long)tok[row] * C);
  float4* b = gwpe ? reinterpret_cast<float4*>(gwpe + (long)pos[row] * C) : nullptr;
  const int n4 = C / 4;
  float4 v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (lane + 32 * k < n4) v[k] = __ldcs(d + lane + 32 * k);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (lane + 32 * k < n4) {
      atomicAdd(a + lane + 32 * k, v[k]);
      if (b) atomicAdd(b + lane + 32 * k, v[k]);
    }
  }
}

template <typename T>
cudaError_t launch_embed_bwd(const float* dres, const int* tok, const int* pos, float* gwte, float* gwpe,
                             int M, int C, cudaStream_t s) {
  ++g_kernel_launches;
  return launch_k(embed_bwd_kernel<T>, dim3((M + 7) / 8), dim3(256), 0, s, dres, tok, pos, gwte, gwpe, M, C);
}

// ---------------------------------------------------------------------------
// Global L2 norm, clip, dynamic loss scale and AdamW over the flat fp32
// parameter vector (one tensor: the canonical layout is contiguous).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void sumsq_block(const float* __restrict__ g, size_t n, double* __restrict__ partials) {
  float acc = 0.f;
  size_t n4 = n / 4;
  const float4* g4 = reinterpret_cast<const float4*>(g);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    float4 v = g4[i];
    acc += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  if (blockIdx.x == 0)
    for (size_t i = n4 * 4 + threadIdx.x; i < n; i += blockDim.x) acc += g[i] * g[i];
  double d = acc;
  for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
  __shared__ double red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = d;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)blockDim.x / 32; ++w) t += red[w];
    partials[blockIdx.x] = t;
  }
}
__global__ void sumsq_kernel(const float* __restrict__ g, size_t n, double* __restrict__ partials) {
  sumsq_block(g, n, partials);
}

cudaError_t launch_sumsq(const float* g, size_t n, double* partials, int nblk, cudaStream_t s) {
  ++g_kernel_launches;
  sumsq_kernel<<<nblk, 512, 0, s>>>(g, n, partials);
  return cudaGetLastError();
}

// Learning rate of AdamW step s (0-based count of steps taken before it)
// under the schedule in sc (cosine with linear warm-up and a floor).
__device__ double sched_lr(const DevScalars* sc, int s, double lr_const) {
  if (sc->sched_kind != 1) return lr_const;
  const double mx = sc->sched_max_lr, mn = sc->sched_min_lr;
  if (s < sc->sched_warmup) return mx * (double)(s + 1) / (double)sc->sched_warmup;
  if (s >= sc->sched_total) return mn;
  const double r = (double)(s - sc->sched_warmup) / (double)(sc->sched_total - sc->sched_warmup);
  return mn + 0.5 * (mx - mn) * (1.0 + cos(3.14159265358979323846 * r));
}

// One block: the global norm from the per-block partials, the clip
// coefficient, the skip decision, the loss-scale update and the bias
// corrections, all into sc (thread 0 writes).
__device__ __forceinline__ void opt_finalize_block(const double* partials, int nblk, float clip, float beta1,
                                                   float beta2, float lr, DevScalars* sc, float* norm_out,
                                                   int32_t* skipped_out) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int i = threadIdx.x; i < nblk; i += blockDim.x) acc += __ldcg(partials + i);
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x != 0) return;
  double tot = 0.0;
  for (int w = 0; w < (int)blockDim.x / 32; ++w) tot += red[w];
  double inv = 1.0 / (double)sc->loss_scale;
  double norm = sqrt(tot) * inv;
  bool finite = isfinite(norm);
  sc->grad_norm = (float)norm;
  if (!finite) {
    sc->skipped = 1;
    if (sc->loss_scaling) sc->loss_scale *= 0.5f;
    sc->good_steps = 0;
  } else {
    sc->skipped = 0;
    double coef = (double)clip / (norm + 1e-6);
    if (coef > 1.0) coef = 1.0;
    sc->coef = (float)(coef * inv);
    sc->lr = (float)sched_lr(sc, sc->step, (double)lr);
    int t = sc->step + 1;
    sc->step = t;
    sc->bc1 = (float)(1.0 - pow((double)beta1, (double)t));
    sc->bc2 = (float)(1.0 - pow((double)beta2, (double)t));
    if (sc->loss_scaling) {
      sc->good_steps += 1;
      if (sc->good_steps >= 2000) { sc->loss_scale *= 2.0f; sc->good_steps = 0; }
    }
  }
  if (norm_out) *norm_out = (float)norm;
  if (skipped_out) *skipped_out = sc->skipped;
}
__global__ void opt_finalize_kernel(const double* __restrict__ partials, int nblk, float clip, float beta1,
                                    float beta2, float lr, DevScalars* sc, float* norm_out, int32_t* skipped_out) {
  opt_finalize_block(partials, nblk, clip, beta1, beta2, lr, sc, norm_out, skipped_out);
}

cudaError_t launch_opt_finalize(const double* partials, int nblk, float clip, float beta1, float beta2, float lr,
                                DevScalars* sc, float* norm_out, int32_t* skipped_out, cudaStream_t s) {
  ++g_kernel_launches;
  opt_finalize_kernel<<<1, 1024, 0, s>>>(partials, nblk, clip, beta1, beta2, lr, sc, norm_out, skipped_out);
  return cudaGetLastError();
}

// AdamW ("Feste", "Manual Backpropagation from scratch": decoupled weight
// decay) on the clipped, unscaled gradient g * coef, with lr = sc->lr:
//   m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;
//   p -= lr (m / bc1 / (sqrt(v / bc2) + eps) + wd p);  pw = T(p).
template <typename T>
__device__ __forceinline__ void adamw_body(float* __restrict__ p, const float* __restrict__ g, float* __restrict__ m,
                                           float* __restrict__ v, T* __restrict__ pw, size_t n, float beta1,
                                           float beta2, float eps, float wd, const DevScalars* sc) {
  // the scalars are read from L2: in the fused form another block wrote them
  // in this kernel
  if (__ldcg(&sc->skipped)) return;
  const float lr = __ldcg(&sc->lr);
  float coef = __ldcg(&sc->coef), bc1 = __ldcg(&sc->bc1), bc2 = __ldcg(&sc->bc2);
  float ib1 = 1.0f / bc1, ib2 = 1.0f / bc2;
  size_t n4 = n / 4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    float pp[4], gg[4], mm[4], vv[4];
    Vec<float>::load(p + 4 * i, pp);
    Vec<float>::load(g + 4 * i, gg);
    Vec<float>::load(m + 4 * i, mm);
    Vec<float>::load(v + 4 * i, vv);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float gj = gg[j] * coef;
      mm[j] = beta1 * mm[j] + (1.f - beta1) * gj;
      vv[j] = beta2 * vv[j] + (1.f - beta2) * gj * gj;
      float upd = (mm[j] * ib1) / (sqrtf(vv[j] * ib2) + eps) + wd * pp[j];
      pp[j] = pp[j] - lr * upd;
    }
    Vec<float>::store(p + 4 * i, pp);
    Vec<float>::store(m + 4 * i, mm);
    Vec<float>::store(v + 4 * i, vv);
    if (pw) {
#pragma unroll
      for (int j = 0; j < 4; ++j) pw[4 * i + j] = from_f<T>(pp[j]);
    }
  }
  if (blockIdx.x == 0) {
    for (size_t i = n4 * 4 + threadIdx.x; i < n; i += blockDim.x) {
      float gj = g[i] * coef;
      float mj = beta1 * m[i] + (1.f - beta1) * gj;
      float vj = beta2 * v[i] + (1.f - beta2) * gj * gj;
      float pj = p[i] - lr * ((mj * ib1) / (sqrtf(vj * ib2) + eps) + wd * p[i]);
      p[i] = pj; m[i] = mj; v[i] = vj;
      if (pw) pw[i] = from_f<T>(pj);
    }
  }
}

template <typename T>
__global__ void adamw_kernel(float* __restrict__ p, const float* __restrict__ g, float* __restrict__ m,
                             float* __restrict__ v, T* __restrict__ pw, size_t n, float beta1,
                             float beta2, float eps, float wd, const DevScalars* __restrict__ sc) {
  adamw_body<T>(p, g, m, v, pw, n, beta1, beta2, eps, wd, sc);
}

// The whole optimiser step in one cooperative launch ("a single multi-tensor
// kernel"): every block sums the squares of its share of the gradient (fp64
// partials), a grid barrier, block 0 finalises the norm / clip / skip /
// loss-scale / bias corrections, a second barrier, and every block updates
// its share of p, m, v and the 16-bit copy.  The barriers count on
// sc->opt_bar (zeroed before the launch) and give up after about a second,
// setting GPT_DEVERR_TIMEOUT (no update then happens).
__device__ __forceinline__ bool opt_grid_sync(DevScalars* sc, unsigned k) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    atomicAdd(&sc->opt_bar, 1u);
    const unsigned target = k * gridDim.x;
    const long long t0 = clock64();
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&sc->opt_bar) : "memory");
      if (v >= target) break;
      if (*(volatile unsigned*)&sc->opt_abort) { ok = 0; break; }
      if (clock64() - t0 > (1ll << 31)) {
        atomicOr(&sc->err, GPT_DEVERR_TIMEOUT);
        atomicExch(&sc->opt_abort, 1u);
        ok = 0;
        break;
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

template <typename T>
__global__ void __launch_bounds__(512) clip_adamw_fused_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                              float* __restrict__ m, float* __restrict__ v,
                                                              T* __restrict__ pw, size_t n, double* partials,
                                                              float clip, float beta1, float beta2, float eps,
                                                              float wd, float lr, DevScalars* sc, float* norm_out,
                                                              int32_t* skipped_out) {
  sumsq_block(g, n, partials);
  if (!opt_grid_sync(sc, 1)) return;
  if (blockIdx.x == 0) opt_finalize_block(partials, gridDim.x, clip, beta1, beta2, lr, sc, norm_out, skipped_out);
  if (!opt_grid_sync(sc, 2)) return;
  adamw_body<T>(p, g, m, v, pw, n, beta1, beta2, eps, wd, sc);
}

template <typename T>
cudaError_t launch_clip_adamw_fused(float* p, const float* g, float* m, float* v, T* pw, size_t n, double* partials,
                                    int max_blocks, float clip, float beta1, float beta2, float eps, float wd,
                                    float lr, DevScalars* sc, float* norm_out, int32_t* skipped_out,
                                    cudaStream_t s) {
  static int grid = 0;
  if (!grid) {
    int dev = 0, sms = 0, per = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, clip_adamw_fused_kernel<T>, 512, 0);
    if (e != cudaSuccess) return e;
    if (per > 4) per = 4;
    grid = sms * per;
  }
  const int G = grid < max_blocks ? grid : max_blocks;
  if (G < 1) return cudaErrorNotSupported;
  cudaError_t e = launch_zero(&sc->opt_bar, 2 * sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
  void* args[] = {&p, (void*)&g, &m, &v, &pw, &n, &partials, &clip, &beta1, &beta2, &eps, &wd, &lr, &sc, &norm_out,
                  &skipped_out};
  ++g_kernel_launches;
  return cudaLaunchCooperativeKernel((void*)clip_adamw_fused_kernel<T>, dim3(G), dim3(512), args, 0, s);
}

template <typename T>
cudaError_t launch_adamw(float* p, const float* g, float* m, float* v, T* pw, size_t n,
                         float beta1, float beta2, float eps, float wd, const DevScalars* sc,
                         cudaStream_t s) {
  ++g_kernel_launches;
  adamw_kernel<T><<<148 * 8, 256, 0, s>>>(p, g, m, v, pw, n, beta1, beta2, eps, wd, sc);
  return cudaGetLastError();
}

template <typename T>
__global__ void cast_kernel(const float* __restrict__ src, T* __restrict__ dst, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = from_f<T>(src[i]);
}
template <typename T>
cudaError_t launch_cast(const float* src, T* dst, size_t n, cudaStream_t s) {
  ++g_kernel_launches;
  cast_kernel<T><<<148 * 8, 256, 0, s>>>(src, dst, n);
  return cudaGetLastError();
}

template <typename T>
__global__ void to_f32_kernel(const T* __restrict__ src, long ld, int rows, int cols, float* __restrict__ dst) {
  size_t n = (size_t)rows * cols;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    size_t r = i / cols, c = i % cols;
    dst[i] = to_f(src[r * ld + c]);
  }
}
template <typename T>
cudaError_t launch_to_f32(const T* src, long ld, int rows, int cols, float* dst, cudaStream_t s) {
  ++g_kernel_launches;
  to_f32_kernel<T><<<148 * 8, 256, 0, s>>>(src, ld, rows, cols, dst);
  return cudaGetLastError();
}


// A bounded wait that cannot complete: an mbarrier nobody arrives on.  The
// waiting thread gives up after timeout_cycles, records GPT_DEVERR_TIMEOUT
// and returns, leaving the context usable.
__global__ void wait_timeout_probe_kernel(unsigned* err, long long timeout_cycles) {
  __shared__ __align__(8) uint64_t bar;
  uint32_t a = (uint32_t)__cvta_generic_to_shared(&bar);
  if (threadIdx.x == 0) asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(1));
  __syncthreads();
  if (threadIdx.x == 0) {
    long long t0 = clock64();
    uint32_t done = 0;
    while (!done) {
      asm volatile("{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
                   : "=r"(done) : "r"(a), "r"(0u));
      if (!done && clock64() - t0 > timeout_cycles) { atomicOr(err, GPT_DEVERR_TIMEOUT); break; }
    }
  }
}
cudaError_t launch_wait_timeout_probe(unsigned* err, long long timeout_cycles, cudaStream_t s) {
  ++g_kernel_launches;
  wait_timeout_probe_kernel<<<1, 32, 0, s>>>(err, timeout_cycles);
  return cudaGetLastError();
}

// ---- explicit instantiations
#define INST(T)                                                                                          \
  template cudaError_t launch_embed_fwd<T>(const int*, const int*, const float*, const float*, T*, int, int, \
                                           cudaStream_t);                                                \
  template cudaError_t launch_ln_fwd<T>(const T*, const float*, const float*, T*, float*, float*, int, int, \
                                        float, cudaStream_t);                                            \
  template cudaError_t launch_ln_bwd<T>(const T*, const T*, const float*, const float*, const float*,      \
                                        const float*, float*, T*, float*, int, int, int*, cudaStream_t,   \
                                        bool, unsigned*);                                                \
  template cudaError_t launch_colsum<T>(const T*, long, int, int, float*, int*, cudaStream_t);            \
  template cudaError_t launch_xent<T>(T*, long, const int*, int, int, int, float*, DevScalars*, cudaStream_t); \
  template cudaError_t launch_embed_bwd<T>(const float*, const int*, const int*, float*, float*, int, int,  \
                                           cudaStream_t);                                                \
  template cudaError_t launch_adamw<T>(float*, const float*, float*, float*, T*, size_t, float, float,     \
                                       float, float, const DevScalars*, cudaStream_t);                   \
  template cudaError_t launch_cast<T>(const float*, T*, size_t, cudaStream_t);                            \
  template cudaError_t launch_clip_adamw_fused<T>(float*, const float*, float*, float*, T*, size_t, double*, int, \
                                                  float, float, float, float, float, float, DevScalars*, float*, \
                                                  int32_t*, cudaStream_t);                               \
  template cudaError_t launch_to_f32<T>(const T*, long, int, int, float*, cudaStream_t);
INST(float)
INST(bf16)
INST(f16)
