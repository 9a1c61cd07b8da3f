// Beam search over the decode rows ("RustGPT", roadmap "high-priority
// feature requests": beam search beside top-k / top-p and temperature).
// Per prompt, W beams occupy decode rows b W .. b W + W - 1; each keeps the
// sum of its tokens' log-probabilities (log-softmax over the real
// vocabulary).  A step extends every beam by every token and keeps the W
// best (score descending, ties to the lower parent * V + token, the parent
// counted by its place in the previous order).  The key / value cache is
// never copied: a table src[row][t] names the cache row that holds position
// t of the row's sequence, reordered with the beams (the attention kernel
// reads through it), and the token history is reordered the same way.
#include "launch.h"

#define BM_THREADS 1024
#define BM_WARPS (BM_THREADS / 32)

__global__ void beam_init_kernel(int* src, int Tmax, float* scores, int B, int W, int Tp) {
  const long n = (long)B * W * Tp;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const int r = (int)(i / Tp), t = (int)(i % Tp);
    src[(long)r * Tmax + t] = r / W;
  }
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < (long)B * W; i += (long)gridDim.x * blockDim.x)
    scores[i] = (i % W) == 0 ? 0.f : -INFINITY;
}

cudaError_t launch_beam_init(int* src, int Tmax, float* scores, int B, int W, int Tp, cudaStream_t s) {
  ++g_kernel_launches;
  beam_init_kernel<<<148, 256, 0, s>>>(src, Tmax, scores, B, W, Tp);
  return cudaGetLastError();
}

// (x, i) precedes (y, j) in the candidate order: larger value first, then the lower index.
__device__ __forceinline__ bool bm_before(float x, int i, float y, int j) { return x > y || (x == y && i < j); }

__global__ void __launch_bounds__(BM_THREADS)
beam_topk_kernel(const float* __restrict__ logits, int Vp, int V, int W, int first,
                 const float* __restrict__ scores, float* __restrict__ cand_s, int* __restrict__ cand_t) {
  griddep_wait();
  griddep_release();
  extern __shared__ float zs[];   // [V]
  __shared__ float redf[BM_WARPS], redg[BM_WARPS];
  __shared__ int redi[BM_WARPS];
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = r / W, w = r % W;
  const float sc = scores[r];
  if (first ? w != 0 : !(sc > -INFINITY)) {
    // no live beam here: its candidates can never be chosen
    if (tid < W) { cand_s[(long)r * W + tid] = -INFINITY; cand_t[(long)r * W + tid] = tid; }
    return;
  }
  const float* z = logits + (long)(first ? b : r) * Vp;
  // thread tid owns the contiguous indices [c0, c1): a fixed summation order
  const int chunk = (V + BM_THREADS - 1) / BM_THREADS;
  const int c0 = min(V, tid * chunk), c1 = min(V, c0 + chunk);
  float mx = -INFINITY;
  for (int i = c0; i < c1; ++i) {
    const float v = z[i];
    zs[i] = v;
    mx = fmaxf(mx, v);
  }
  mx = warp_max(mx);
  if (lane == 0) redf[warp] = mx;
  __syncthreads();
  mx = warp_max(lane < BM_WARPS ? redf[lane] : -INFINITY);
  float part = 0.f;
  for (int i = c0; i < c1; ++i) part += expf(zs[i] - mx);
  part = warp_sum(part);
  if (lane == 0) redg[warp] = part;
  __syncthreads();
  const float lse = mx + logf(warp_sum(lane < BM_WARPS ? redg[lane] : 0.f));
  // W rounds: the best candidate strictly after the previous pick in the order
  float pv = INFINITY;
  int pi = -1;
  for (int k = 0; k < W; ++k) {
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = c0; i < c1; ++i) {
      const float v = zs[i];
      if (bm_before(pv, pi, v, i) && bm_before(v, i, best, bi)) { best = v; bi = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (bm_before(ov, oi, best, bi)) { best = ov; bi = oi; }
    }
    __syncthreads();
    if (lane == 0) { redf[warp] = best; redi[warp] = bi; }
    __syncthreads();
    best = lane < BM_WARPS ? redf[lane] : -INFINITY;
    bi = lane < BM_WARPS ? redi[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (bm_before(ov, oi, best, bi)) { best = ov; bi = oi; }
    }
    if (tid == 0) {
      const bool ok = bi >= 0 && bi < V;   // false only for a row of NaNs
      cand_s[(long)r * W + k] = ok ? sc + (best - lse) : -INFINITY;
      cand_t[(long)r * W + k] = ok ? bi : 0;
    }
    pv = best;
    pi = bi;
  }
}

cudaError_t launch_beam_topk(const float* logits, int Vp, int V, int B, int W, bool first, const float* scores,
                             float* cand_s, int* cand_t, cudaStream_t s) {
  if (W < 1 || W > BEAM_MAX_WIDTH || V < W || V > SMP_MAX_VOCAB) return cudaErrorInvalidValue;
  const size_t smem = (size_t)V * 4;
  static size_t attr = 0;
  if (smem > attr) {
    cudaError_t e = cudaFuncSetAttribute(beam_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = smem;
  }
  ++g_kernel_launches;
  cudaError_t e = launch_k(beam_topk_kernel, dim3(B * W), dim3(BM_THREADS), smem, s, logits, Vp, V, W,
                           first ? 1 : 0, scores, cand_s, cand_t);
  return e != cudaSuccess ? e : cudaGetLastError();
}

#define BMM_THREADS 256
#define BMM_CHUNK 512
__global__ void __launch_bounds__(BMM_THREADS)
beam_merge_kernel(const float* __restrict__ cand_s, const int* __restrict__ cand_t, int W, int V, int Tp,
                  int* __restrict__ src, int Tmax, float* __restrict__ scores, int* __restrict__ tok,
                  int32_t* __restrict__ out, int out_ld, const int* __restrict__ step) {
  griddep_wait();
  griddep_release();
  __shared__ int par[BEAM_MAX_WIDTH], ctok[BEAM_MAX_WIDTH];
  __shared__ float csc[BEAM_MAX_WIDTH];
  __shared__ int stage[BEAM_MAX_WIDTH * BMM_CHUNK];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int col = step ? *step : 0;
  const long r0 = (long)b * W;
  if (tid == 0) {
    // the W best of the W x W candidates; a row's own candidates arrive in
    // order, so the order over all of them is (score desc, parent V + token asc)
    float ps = INFINITY;
    long pk = -1;
    for (int k = 0; k < W; ++k) {
      float bs = -INFINITY;
      long bk = 0x7fffffffffffffffL;
      int bw = 0, bt = 0;
      for (int i = 0; i < W * W; ++i) {
        const float v = cand_s[r0 * W + i];
        const int pw = i / W, t = cand_t[r0 * W + i];
        const long key = (long)pw * V + t;
        const bool after = v < ps || (v == ps && key > pk);
        const bool better = v > bs || (v == bs && key < bk);
        if (after && better) { bs = v; bk = key; bw = pw; bt = t; }
      }
      par[k] = bw;
      ctok[k] = bt;
      csc[k] = bs;
      ps = bs;
      pk = bk;
    }
  }
  __syncthreads();
  // token history: columns [0, col) follow the parent, column col is the new token
  for (int c0 = 0; c0 < col; c0 += BMM_CHUNK) {
    const int n = min(BMM_CHUNK, col - c0);
    for (int i = tid; i < W * n; i += BMM_THREADS)
      stage[(i / n) * BMM_CHUNK + i % n] = out[(r0 + i / n) * out_ld + c0 + i % n];
    __syncthreads();
    for (int i = tid; i < W * n; i += BMM_THREADS)
      out[(r0 + i / n) * out_ld + c0 + i % n] = stage[par[i / n] * BMM_CHUNK + i % n];
    __syncthreads();
  }
  // source rows of the generated positions Tp .. Tp + col - 1: those before
  // the latest follow the parent's table; the latest (fed this step) lies in
  // the parent's own row
  const int g0 = Tp, g1 = Tp + col;    // [g0, g1)
  for (int c0 = g0; c0 < g1; c0 += BMM_CHUNK) {
    const int n = min(BMM_CHUNK, g1 - c0);
    for (int i = tid; i < W * n; i += BMM_THREADS) {
      const int t = c0 + i % n;
      stage[(i / n) * BMM_CHUNK + i % n] = t == g1 - 1 ? (int)(r0 + i / n) : src[(r0 + i / n) * Tmax + t];
    }
    __syncthreads();
    for (int i = tid; i < W * n; i += BMM_THREADS)
      src[(r0 + i / n) * Tmax + c0 + i % n] = stage[par[i / n] * BMM_CHUNK + i % n];
    __syncthreads();
  }
  if (tid < W) {
    out[(r0 + tid) * out_ld + col] = ctok[tid];
    tok[r0 + tid] = ctok[tid];
    scores[r0 + tid] = csc[tid];
  }
}

cudaError_t launch_beam_merge(const float* cand_s, const int* cand_t, int B, int W, int V, int Tp, int* src,
                              int Tmax, float* scores, int* tok, int32_t* out, int out_ld, const int* step,
                              cudaStream_t s) {
  if (W < 1 || W > BEAM_MAX_WIDTH) return cudaErrorInvalidValue;
  ++g_kernel_launches;
  cudaError_t e = launch_k(beam_merge_kernel, dim3(B), dim3(BMM_THREADS), 0, s, cand_s, cand_t, W, V, Tp, src, Tmax,
                           scores, tok, out, out_ld, step);
  return e != cudaSuccess ? e : cudaGetLastError();
}
