// Greedy decoding for small batches (B <= 4) as one persistent kernel that
// runs every remaining decode step of a gpt_greedy_decode call ("RustGPT",
// "Technical implementation": greedy decoding; "NTransformer" page, "No
// PyTorch, no cuBLAS": per-layer KV cache).
//
// Why one kernel: a decode step at batch 1 reads the 247 MB of bf16 weights
// of GPT-2 124M once, about 38 us at HBM speed, but as ~100 separate launches
// of a few microseconds each it is bound by launch and ramp latency.  Here
// one CTA per SM (a cooperative launch, so all CTAs are resident) walks the
// step as a sequence of phases separated by a grid-wide barrier:
//
//   per layer  A  LN1 of the residual row (every CTA, redundantly), then the
//                 CTA's 16-row units of the qkv projection (+ bias)
//              B  attention of the new query over the cache, split over
//                 (row, head, key range) units; the new key and value are
//                 written into the cache
//              C  merge of the key-range partials, then 16-row units of the
//                 output projection (+ bias + residual)
//              D  LN2 (every CTA), 16-row units of fc (+ bias, GELU)
//              E  row units of fc2 (+ bias + residual)
//   then       F  final LN (every CTA), the LM head (fp32 logits) in 4-row
//                 chunks that every warp streams on its own (two in flight
//                 per warp, no block barrier) with a per-CTA argmax;
//                 after the barrier every CTA
//                 reduces the per-CTA maxima (lowest index on ties) into the
//                 next token and embeds it for the next step.
//
// Weight rows of a unit are contiguous in the bf16 working copy; each CTA
// moves its units of the next phase into shared memory with bulk copies
// (cp.async.bulk, completion on an mbarrier) issued before it waits at the
// barrier, so the weight stream overlaps the barrier, and it asks L2 to
// prefetch its share of the next layer's weights at the start of a layer.
// LayerNorm gamma / beta and the bias rows of the CTA's units travel the
// same way into two small parameter areas, one phase ahead.  The key-range
// partials of phase B are merged by the CTAs of phase C that need the
// attention rows (no atomics, no fences).
// Rounding points are those of the training forward: the residual stream,
// LN outputs, q/k/v, the attention output, u and GELU(u) are bf16; all dot
// products, LN statistics and the softmax are fp32; the logits are fp32.
//
// Every wait is bounded: a barrier or mbarrier wait that exceeds its limit
// sets GPT_DEVERR_TIMEOUT and an abort word that makes every CTA leave.
#include "launch.h"
#include "tc_common.cuh"

#define DF_THREADS 256
#define DF_WARPS (DF_THREADS / 32)
#define DF_WBUF (48 * 1024)             // bytes of each of the two weight buffers
#define DF_MAX_SPLITS 16
#define DF_BAR_LIMIT (1ll << 31)         // clock cycles (about a second)
#define DF_WSLOT (DF_WBUF / DF_WARPS)   // bytes of one LM-head slot (two per warp)
#define DF_PRM_BIAS 256                  // bias floats of one CTA's units in one phase (at most)
#define DF_PRM(C) (2 * (C) + DF_PRM_BIAS)  // floats of one parameter area

// DecFusedParams is declared in launch.h.

// ------------------------------------------------------------------ barrier
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier number `k` (1, 2, ...): false if the kernel must abort.
// One thread per CTA arrives with a release reduction (the CTA's writes,
// ordered before it by the block barrier, become visible with it) and polls
// the counter with acquire loads; the abort word and the clock are looked at
// only every 64 polls so that the pollers add little traffic.
__device__ __forceinline__ bool df_grid_sync(const DecFusedParams& p, unsigned k, int* s_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ab = 0;
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.bar) : "memory");
    const unsigned target = k * gridDim.x;
    const long long t0 = clock64();
    for (unsigned it = 1;; ++it) {
      if (ld_acquire_u32(p.bar) >= target) break;
      if ((it & 63) == 0) {
        if (*(volatile unsigned*)p.abortf) { ab = 1; break; }
        if (clock64() - t0 > DF_BAR_LIMIT) {
          atomicOr(p.err, GPT_DEVERR_TIMEOUT);
          atomicExch(p.abortf, 1u);
          ab = 1;
          break;
        }
      }
    }
    *s_flag = ab;
  }
  __syncthreads();
  return *s_flag == 0;
}

// Bounded wait for an mbarrier phase by one thread: the global abort word is
// read only every 64 polls (every thread of every CTA reading it on each
// poll made one L2 line a hot spot and delayed each wake-up by a round trip).
__device__ __forceinline__ bool df_mbar_wait(uint32_t bar, uint32_t parity, const unsigned* abortf) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*(volatile const unsigned*)abortf) return false;
      if (clock64() - t0 > DF_BAR_LIMIT) return false;
    }
  }
}

// ------------------------------------------------------------------ weight buffers
// Two 48 KB buffers (slots 0 and 1); the LM-head phase splits them into four
// 24 KB slots, slot s at buffer s & 1, half s >> 1.  Slot s completes on bar[s].
struct WBufs {
  uint8_t* buf[2];
  uint32_t bar[4];
  uint32_t parity[4];
  int inflight[4];   // a queued copy not yet waited for (same value in every thread)
};

// Thread 0 queues `n` contiguous byte ranges into buffer `i` (total <= DF_WBUF);
// every thread must later call wbuf_wait(i).
__device__ __forceinline__ void wbuf_issue_begin(WBufs& w, int i, uint32_t total) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_expect_tx(w.bar[i], total);
}
__device__ __forceinline__ void wbuf_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}
// Every thread of the CTA calls this; thread 0 waits and the block barrier
// hands the data to the others; the outcome is the same in all of them.
__device__ __forceinline__ bool wbuf_wait(WBufs& w, int i, const DecFusedParams& p) {
  int ok = 1;
  if (threadIdx.x == 0) ok = df_mbar_wait(w.bar[i], w.parity[i], p.abortf);
  if (!__syncthreads_or(!ok)) {
    w.parity[i] ^= 1u;
    w.inflight[i] = 0;
    return true;
  }
  if (threadIdx.x == 0) {
    atomicOr(p.err, GPT_DEVERR_TIMEOUT);
    atomicExch(p.abortf, 1u);
  }
  return false;
}
// Before leaving on an abort: wait (bounded, ignoring the abort word) for the
// copies still in flight into this CTA's shared memory.
__device__ __forceinline__ void wbuf_drain(WBufs& w) {
  volatile int never = 0;
  for (int i = 0; i < 4; ++i)
    if (w.inflight[i]) mbar_wait(w.bar[i], w.parity[i], &never, 1ll << 28);
}

__device__ __forceinline__ void l2_prefetch(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
               : "memory");
}

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ float bfr(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// LayerNorm of BB rows of C fp32 values in smem `x` into smem `y` (bf16-rounded
// values kept as fp32), one warp per row; two-pass statistics as in training.
// g and b are in shared memory (staged by a bulk copy one phase ahead).
template <int BB>
__device__ __forceinline__ void df_layernorm(const float* x, float* y, const float* g, const float* b, int B, int C,
                                             float eps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < B; r += DF_WARPS) {
    const float* xr = x + r * C;
    float s = 0.f;
    for (int c = lane; c < C; c += 32) s += xr[c];
    const float mu = warp_sum(s) / C;
    float q = 0.f;
    for (int c = lane; c < C; c += 32) { const float d = xr[c] - mu; q += d * d; }
    const float rs = 1.0f / sqrtf(warp_sum(q) / C + eps);
    for (int c = lane; c < C; c += 32) y[r * C + c] = bfr((xr[c] - mu) * rs * g[c] + b[c]);
  }
}

// y[b][r] = sum_k ws[r][k] * xin[b][k] for r < R, b < B; epi(r, b, y) runs on
// lane 0 of the warp that owns row r.  ws: bf16 [R][K] in smem; xin fp32.
template <int BB, typename Epi>
__device__ __forceinline__ void df_project(const bf16* ws, int R, int K, const float* xin, int ldx, int B, Epi epi) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < R; r += DF_WARPS) {
    float acc[BB];
#pragma unroll
    for (int b = 0; b < BB; ++b) acc[b] = 0.f;
    const bf16* wr = ws + (long)r * K;
    for (int k = lane * 8; k < K; k += 256) {
      float w[8];
      Vec<bf16>::load(wr + k, w);
#pragma unroll
      for (int b = 0; b < BB; ++b) {
        if (b < B) {
          const float4 x0 = *reinterpret_cast<const float4*>(xin + b * ldx + k);
          const float4 x1 = *reinterpret_cast<const float4*>(xin + b * ldx + k + 4);
          float a = acc[b];
          a = fmaf(w[0], x0.x, a); a = fmaf(w[1], x0.y, a); a = fmaf(w[2], x0.z, a); a = fmaf(w[3], x0.w, a);
          a = fmaf(w[4], x1.x, a); a = fmaf(w[5], x1.y, a); a = fmaf(w[6], x1.z, a); a = fmaf(w[7], x1.w, a);
          acc[b] = a;
        }
      }
    }
#pragma unroll
    for (int b = 0; b < BB; ++b) {
      if (b < B) {
        const float y = warp_sum(acc[b]);
        if (lane == 0) epi(r, b, y);
      }
    }
  }
}

// Load BB rows of n bf16 values from global memory written earlier in this
// kernel (L2 only: another SM's L1 copy may be stale) into fp32 smem.
__device__ __forceinline__ void df_load_rows(const bf16* src, float* dst, int B, int n) {
  const int tot = B * n / 8;
  for (int i = threadIdx.x; i < tot; i += DF_THREADS) {
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(src) + i);
    float f[8];
    Vec<bf16>::load(reinterpret_cast<const bf16*>(&v), f);
    *reinterpret_cast<float4*>(dst + i * 8) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4*>(dst + i * 8 + 4) = make_float4(f[4], f[5], f[6], f[7]);
  }
}

// ------------------------------------------------------------------ the kernel
template <int BB>
__global__ void __launch_bounds__(DF_THREADS, 1) decode_fused_kernel(const DecFusedParams p) {
  extern __shared__ __align__(128) uint8_t df_smem[];
  __shared__ __align__(8) uint64_t wbars[4];
  __shared__ __align__(8) uint64_t pbars[2];
  __shared__ __align__(8) uint64_t hbars[2 * DF_WARPS];   // LM head: two slots per warp
  __shared__ int s_flag;
  __shared__ float s_rv[DF_WARPS][BB];
  __shared__ int s_ri[DF_WARPS][BB];
  __shared__ int s_tok[BB];

  const int C = p.C, F = p.F, H = p.H, D = p.D, B = p.B, G = gridDim.x;
  const int cta = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WBufs wb;
  wb.buf[0] = df_smem;
  wb.buf[1] = df_smem + DF_WBUF;
  float* xs = reinterpret_cast<float*>(df_smem + 2 * DF_WBUF);   // [BB][C] residual row (bf16 values)
  float* xm = xs + BB * C;                                        // [BB][C] x_mid
  float* xin = xm + BB * C;                                       // [BB][KX] projection input
  // two parameter areas of DF_PRM(C) floats: LayerNorm gamma and beta (2C),
  // then the bias slices of the CTA's units, staged one phase ahead
  float* prm[2];
  prm[0] = xin + BB * (C > F ? C : F);
  prm[1] = prm[0] + DF_PRM(C);
  uint32_t pbar[2] = {smem_u32(&pbars[0]), smem_u32(&pbars[1])};
  uint32_t ppar[2] = {0u, 0u};
  int pinf[2] = {0, 0};
  for (int i = 0; i < 4; ++i) {
    wb.bar[i] = smem_u32(&wbars[i]);
    wb.parity[i] = 0;
    wb.inflight[i] = 0;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(wb.bar[i], 1);
    for (int i = 0; i < 2 * DF_WARPS; ++i) mbar_init(smem_u32(&hbars[i]), 1);
    mbar_init(pbar[0], 1);
    mbar_init(pbar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x < BB) s_tok[threadIdx.x] = threadIdx.x < B ? __ldcg(p.tok + threadIdx.x) : 0;
  __syncthreads();

  // unit geometry (rows per unit): qkv, out-proj and fc take 16 rows, fc2
  // takes as many rows as fit a buffer, the head 32-row chunks
  const int nu_qkv = 3 * C / 16, nu_o = C / 16, nu_fc = F / 16;
  int rows_e = DF_WBUF / (F * 2);
  if (rows_e > 16) rows_e = 16;
  rows_e &= ~3;   // bias slices of whole 16-byte groups
  const int nu_e = (C + rows_e - 1) / rows_e;
  // LM head: warp-chunks of hw rows, each warp streaming its own through two
  // DF_WSLOT-byte slots in the weight buffers (free during the head phase)
  int hw = DF_WSLOT / (2 * C);
  if (hw > 8) hw = 8;
  const int n_wc = (p.Vp + hw - 1) / hw;
  uint32_t hpar = 0;    // bit s: parity of this warp's next wait on slot s
  int hpend = 0;        // this warp's slots with a copy in flight (bit s)
  const int S = p.S, nu_att = B * H * S;
  const float* P32 = p.p32;
  const bf16* PW = p.pw;
  unsigned nbar = 0;

  // queue this CTA's units of a projection phase into buffer i; returns the
  // number of units queued (0: nothing queued, no wait needed)
  auto issue_units = [&](int i, const bf16* W, int nunits, int rows_per_unit, int nrows, int K) -> int {
    int cnt = 0;
    uint32_t total = 0;
    for (int u = cta; u < nunits; u += G) {
      const int r0 = u * rows_per_unit;
      const int rr = min(rows_per_unit, nrows - r0);
      total += (uint32_t)rr * K * 2;
      ++cnt;
    }
    if (cnt) wb.inflight[i] = 1;
    if (cnt && threadIdx.x == 0) {
      wbuf_issue_begin(wb, i, total);
      uint32_t off = 0;
      for (int u = cta; u < nunits; u += G) {
        const int r0 = u * rows_per_unit;
        const int rr = min(rows_per_unit, nrows - r0);
        const uint32_t bytes = (uint32_t)rr * K * 2;
        wbuf_copy(smem_u32(wb.buf[i] + off), W + (long)r0 * K, bytes, wb.bar[i]);
        off += bytes;
      }
    }
    return cnt;
  };
  auto lw = [&](long off0, int l) -> long { return off0 + (long)l * p.l_stride; };
  // queue parameter area k: gamma and beta (2C contiguous floats at ln, or
  // none) and the bias rows of this CTA's units (rows_per_unit each)
  auto issue_params = [&](int k, long ln, long bias, int nunits, int rows_per_unit, int nrows) {
    pinf[k] = 1;
    if (threadIdx.x == 0) {
      uint32_t total = ln >= 0 ? (uint32_t)(2 * C * 4) : 0u;
      for (int u = cta; u < nunits; u += G) total += (uint32_t)min(rows_per_unit, nrows - u * rows_per_unit) * 4;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(pbar[k], total);
      uint32_t off = 0;
      if (ln >= 0) {
        wbuf_copy(smem_u32(prm[k]), P32 + ln, (uint32_t)(2 * C * 4), pbar[k]);
        off = (uint32_t)(2 * C * 4);
      }
      for (int u = cta; u < nunits; u += G) {
        const int r0 = u * rows_per_unit;
        const uint32_t bytes = (uint32_t)min(rows_per_unit, nrows - r0) * 4;
        wbuf_copy(smem_u32(prm[k]) + off, P32 + bias + r0, bytes, pbar[k]);
        off += bytes;
      }
    }
  };
  auto wait_params = [&](int k) -> bool {
    int ok = 1;
    if (threadIdx.x == 0) ok = df_mbar_wait(pbar[k], ppar[k], p.abortf);
    if (__syncthreads_or(!ok)) {
      if (threadIdx.x == 0) {
        atomicOr(p.err, GPT_DEVERR_TIMEOUT);
        atomicExch(p.abortf, 1u);
      }
      return false;
    }
    ppar[k] ^= 1u;
    pinf[k] = 0;
    return true;
  };

  // weights and parameters of layer 0's phase A go first
  int pend_a = issue_units(0, PW + lw(p.l_w_qkv, 0), nu_qkv, 16, 3 * C, C);
  issue_params(0, lw(p.l_ln1_g, 0), lw(p.l_b_qkv, 0), nu_qkv, 16, 3 * C);
  int pend_c = 0, pend_d = 0, pend_e = 0;

  for (int st = 0; st < p.n_steps; ++st) {
    const int pos = p.pos_first + st;
    // ---- embedding of the current tokens: x = bf16(wte[tok] + wpe[pos])
    for (int i = threadIdx.x; i < B * C; i += DF_THREADS) {
      const int b = i / C, c = i % C;
      const float* we = P32 + p.o_wte + (long)s_tok[b] * C;
      const float* pe = P32 + p.o_wpe + (long)pos * C;
      xs[i] = bfr(we[c] + pe[c]);
    }
    __syncthreads();
    for (int l = 0; l < p.NL; ++l) {
      // ---- L2 prefetch of this CTA's share of the next layer (or the head)
      if (threadIdx.x == 0) {
        const bf16* nb;
        long n;
        if (l + 1 < p.NL) { nb = PW + lw(p.l_ln1_g, l + 1); n = p.l_stride; }
        else { nb = PW + p.o_head; n = (long)p.Vp * C; }
        long share = (n + G - 1) / G;
        share = (share + 7) & ~7L;
        long a = (long)cta * share, e = a + share;
        if (e > n) e = n;
        for (long o = a; o < e; o += 32768) {
          const long len = e - o < 32768 ? e - o : 32768;
          if (len >= 8) l2_prefetch(nb + o, (uint32_t)(len & ~7L) * 2);
        }
      }
      // ---- phase A: LN1, qkv units
      if (!wait_params(0)) goto abort;
      df_layernorm<BB>(xs, xin, prm[0], prm[0] + C, B, C, p.eps);
      __syncthreads();
      if (pend_a) {
        if (!wbuf_wait(wb, 0, p)) goto abort;
        const float* bq = prm[0] + 2 * C;
        int slot = 0;
        for (int u = cta; u < nu_qkv; u += G, ++slot) {
          const int r0 = u * 16;
          df_project<BB>(reinterpret_cast<const bf16*>(wb.buf[0]) + (long)slot * 16 * C, 16, C, xin, C, B,
                         [&](int r, int b, float y) {
                           p.qkv[(long)b * 3 * C + r0 + r] = __float2bfloat16_rn(y + bq[slot * 16 + r]);
                         });
        }
      }
      __syncthreads();
      // the out-projection's weights and bias can move while the barrier and attention run
      pend_c = issue_units(1, PW + lw(p.l_w_o, l), nu_o, 16, C, C);
      issue_params(1, -1, lw(p.l_b_o, l), nu_o, 16, C);
      if (!df_grid_sync(p, ++nbar, &s_flag)) goto abort;

      // ---- phase B: attention units (row b, head h, key range s)
      {
        const int LPK = D / 8, KPW = 32 / LPK;
        const int L = pos + 1;
        const float scale = rsqrtf((float)D);
        float* sm = xin;                       // [DF_WARPS][D + 2] warp partials
        bf16* kcl = p.kc + (long)l * p.kvl;
        bf16* vcl = p.vc + (long)l * p.kvl;
        for (int u = cta; u < nu_att; u += G) {
          const int bh = u / S, s = u % S, b = bh / H, h = bh % H;
          const int j0 = (int)((long)s * L / S), j1 = (int)((long)(s + 1) * L / S);
          const bf16* q = p.qkv + (long)b * 3 * C + h * D;
          const bf16* knew = q + C;
          const bf16* vnew = q + 2 * C;
          bf16* kcb = kcl + ((long)b * H + h) * p.Tmax * D;
          bf16* vcb = vcl + ((long)b * H + h) * p.Tmax * D;
          if (s == 0 && threadIdx.x < D) {
            kcb[(long)pos * D + threadIdx.x] = __ldcg(knew + threadIdx.x);
            vcb[(long)pos * D + threadIdx.x] = __ldcg(vnew + threadIdx.x);
          }
          const int grp = lane / LPK, sub = lane % LPK;
          float qv[8];
          {
            const uint4 t = __ldcg(reinterpret_cast<const uint4*>(q + sub * 8));
            Vec<bf16>::load(reinterpret_cast<const bf16*>(&t), qv);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) qv[i] *= scale;
          float m = -INFINITY, lsum = 0.f, o[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = 0.f;
          for (int jb = j0 + warp * KPW; jb < j1; jb += DF_WARPS * KPW) {
            const int j = jb + grp;
            const bool live = j < j1;
            float kv[8], vv[8];
            if (live) {
              const bf16* kr = j == pos ? knew : kcb + (long)j * D;
              const bf16* vr = j == pos ? vnew : vcb + (long)j * D;
              const uint4 tk = __ldcg(reinterpret_cast<const uint4*>(kr + sub * 8));
              const uint4 tv = __ldcg(reinterpret_cast<const uint4*>(vr + sub * 8));
              Vec<bf16>::load(reinterpret_cast<const bf16*>(&tk), kv);
              Vec<bf16>::load(reinterpret_cast<const bf16*>(&tv), vv);
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) { kv[i] = 0.f; vv[i] = 0.f; }
            }
            float sc = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) sc = fmaf(qv[i], kv[i], sc);
            for (int o2 = LPK / 2; o2 > 0; o2 >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o2);
            if (live) {
              const float mn = fmaxf(m, sc);
              const float corr = __expf(m - mn), pe = __expf(sc - mn);
              lsum = lsum * corr + pe;
#pragma unroll
              for (int i = 0; i < 8; ++i) o[i] = o[i] * corr + pe * vv[i];
              m = mn;
            }
          }
          // merge the key groups of the warp, then the warps
          for (int o2 = LPK; o2 < 32; o2 <<= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o2);
            const float l2 = __shfl_xor_sync(0xffffffffu, lsum, o2);
            const float mn = fmaxf(m, m2);
            const float f1 = m == -INFINITY ? 0.f : __expf(m - mn), f2 = m2 == -INFINITY ? 0.f : __expf(m2 - mn);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = o[i] * f1 + __shfl_xor_sync(0xffffffffu, o[i], o2) * f2;
            lsum = lsum * f1 + l2 * f2;
            m = mn;
          }
          if (lane < LPK) {
            float* w = sm + warp * (D + 2);
            if (lane == 0) { w[0] = m; w[1] = lsum; }
#pragma unroll
            for (int i = 0; i < 8; ++i) w[2 + sub * 8 + i] = o[i];
          }
          __syncthreads();
          float* dst = p.part + ((long)bh * S + s) * (D + 2);
          if (threadIdx.x < D) {
            float mm = -INFINITY;
            for (int w2 = 0; w2 < DF_WARPS; ++w2) mm = fmaxf(mm, sm[w2 * (D + 2)]);
            float ll = 0.f, oo = 0.f;
            for (int w2 = 0; w2 < DF_WARPS; ++w2) {
              const float mw = sm[w2 * (D + 2)];
              const float f = mw == -INFINITY ? 0.f : __expf(mw - mm);
              ll += sm[w2 * (D + 2) + 1] * f;
              oo += sm[w2 * (D + 2) + 2 + threadIdx.x] * f;
            }
            dst[2 + threadIdx.x] = oo;
            if (threadIdx.x == 0) { dst[0] = mm; dst[1] = ll; }
          }
          __syncthreads();
        }
      }
      if (!df_grid_sync(p, ++nbar, &s_flag)) goto abort;

      // ---- phase C: out-projection units over the merged attention rows
      if (!wait_params(1)) goto abort;
      if (pend_c) {
        // merge the key-range partials of every (row, head) into the
        // attention rows: partials into shared memory (buffer 0 is free in
        // this phase), then one output element per thread
        {
          float* ps = reinterpret_cast<float*>(wb.buf[0]);
          const int npart = B * H * S * (D + 2), np4 = npart / 4;
          for (int i = threadIdx.x; i < np4; i += DF_THREADS)
            reinterpret_cast<float4*>(ps)[i] = __ldcg(reinterpret_cast<const float4*>(p.part) + i);
          for (int i = np4 * 4 + threadIdx.x; i < npart; i += DF_THREADS) ps[i] = __ldcg(p.part + i);
          __syncthreads();
          for (int i = threadIdx.x; i < B * C; i += DF_THREADS) {
            const int bh = i / D, d = i % D;
            const float* pp = ps + (long)bh * S * (D + 2);
            float mm = -INFINITY;
            for (int s2 = 0; s2 < S; ++s2) mm = fmaxf(mm, pp[s2 * (D + 2)]);
            float ll = 0.f, oo = 0.f;
            for (int s2 = 0; s2 < S; ++s2) {
              const float ms = pp[s2 * (D + 2)];
              const float f = ms == -INFINITY ? 0.f : __expf(ms - mm);
              ll += pp[s2 * (D + 2) + 1] * f;
              oo += pp[s2 * (D + 2) + 2 + d] * f;
            }
            xin[i] = bfr(oo / ll);   // the attention output is rounded to bf16 as in training
          }
        }
        __syncthreads();
        if (!wbuf_wait(wb, 1, p)) goto abort;
        const float* bo = prm[1];
        int slot = 0;
        for (int u = cta; u < nu_o; u += G, ++slot) {
          const int r0 = u * 16;
          df_project<BB>(reinterpret_cast<const bf16*>(wb.buf[1]) + (long)slot * 16 * C, 16, C, xin, C, B,
                         [&](int r, int b, float y) {
                           const int n = r0 + r;
                           p.xmid[(long)b * C + n] = __float2bfloat16_rn(y + bo[slot * 16 + r] + xs[b * C + n]);
                         });
        }
      }
      __syncthreads();
      pend_d = issue_units(0, PW + lw(p.l_w_fc, l), nu_fc, 16, F, C);
      issue_params(0, lw(p.l_ln2_g, l), lw(p.l_b_fc, l), nu_fc, 16, F);
      if (!df_grid_sync(p, ++nbar, &s_flag)) goto abort;

      // ---- phase D: LN2, fc units (u and GELU(u))
      df_load_rows(p.xmid, xm, B, C);
      __syncthreads();
      if (!wait_params(0)) goto abort;
      df_layernorm<BB>(xm, xin, prm[0], prm[0] + C, B, C, p.eps);
      __syncthreads();
      if (pend_d) {
        if (!wbuf_wait(wb, 0, p)) goto abort;
        const float* bf = prm[0] + 2 * C;
        int slot = 0;
        for (int u = cta; u < nu_fc; u += G, ++slot) {
          const int r0 = u * 16;
          df_project<BB>(reinterpret_cast<const bf16*>(wb.buf[0]) + (long)slot * 16 * C, 16, C, xin, C, B,
                         [&](int r, int b, float y) {
                           const int n = r0 + r;
                           const float uq = bfr(y + bf[slot * 16 + r]);
                           p.abuf[(long)b * F + n] = __float2bfloat16_rn(gelu_f(uq));
                         });
        }
      }
      __syncthreads();
      pend_e = issue_units(1, PW + lw(p.l_w_fc2, l), nu_e, rows_e, C, F);
      issue_params(1, -1, lw(p.l_b_fc2, l), nu_e, rows_e, C);
      if (!df_grid_sync(p, ++nbar, &s_flag)) goto abort;

      // ---- phase E: fc2 units (+ bias + residual)
      if (!wait_params(1)) goto abort;
      if (pend_e) {
        df_load_rows(p.abuf, xin, B, F);
        __syncthreads();
        if (!wbuf_wait(wb, 1, p)) goto abort;
        const float* b2 = prm[1];
        int slot = 0;
        for (int u = cta; u < nu_e; u += G, ++slot) {
          const int r0 = u * rows_e;
          const int rr = min(rows_e, C - r0);
          df_project<BB>(reinterpret_cast<const bf16*>(wb.buf[1]) + (long)slot * rows_e * F, rr, F, xin, F, B,
                         [&](int r, int b, float y) {
                           const int n = r0 + r;
                           p.xbuf[(long)b * C + n] = __float2bfloat16_rn(y + b2[slot * rows_e + r] + xm[b * C + n]);
                         });
        }
      }
      __syncthreads();
      if (l + 1 < p.NL) {
        pend_a = issue_units(0, PW + lw(p.l_w_qkv, l + 1), nu_qkv, 16, 3 * C, C);
        issue_params(0, lw(p.l_ln1_g, l + 1), lw(p.l_b_qkv, l + 1), nu_qkv, 16, 3 * C);
      } else {
        issue_params(0, p.o_lnf_g, 0, 0, 1, 1);   // the final LayerNorm's gamma and beta
      }
      if (!df_grid_sync(p, ++nbar, &s_flag)) goto abort;
      df_load_rows(p.xbuf, xs, B, C);
      __syncthreads();
    }

    // ---- phase F: final LN, LM head chunks with a per-CTA argmax
    {
      if (!wait_params(0)) goto abort;
      df_layernorm<BB>(xs, xin, prm[0], prm[0] + C, B, C, p.eps);
      float bv[BB];
      int bi[BB];
#pragma unroll
      for (int b = 0; b < BB; ++b) { bv[b] = -INFINITY; bi[b] = 0x7fffffff; }
      const bf16* Wh = PW + p.o_head;
      // layer 0 of the next step into L2 while the head streams
      if (threadIdx.x == 0 && st + 1 < p.n_steps) {
        long share = (p.l_stride + G - 1) / G;
        share = (share + 7) & ~7L;
        long a = (long)cta * share, e = a + share;
        if (e > p.l_stride) e = p.l_stride;
        for (long o = a; o < e; o += 32768) {
          const long len = e - o < 32768 ? e - o : 32768;
          if (len >= 8) l2_prefetch(PW + p.l_ln1_g + o, (uint32_t)(len & ~7L) * 2);
        }
      }
      // warp-chunk k of this warp is cta * DF_WARPS + warp + k * G * DF_WARPS
      // (hw rows), in the warp's slot k & 1; each warp waits for its own copies
      // and syncs only its own lanes, so warps stream independently
      int nkw = 0;
      for (int c2 = cta * DF_WARPS + warp; c2 < n_wc; c2 += G * DF_WARPS) ++nkw;
      uint8_t* wsl = df_smem + warp * 2 * DF_WSLOT;
      auto issue_w = [&](int k) {
        const int sl = k & 1, wc = cta * DF_WARPS + warp + k * G * DF_WARPS;
        const int r0 = wc * hw, rr = min(hw, p.Vp - r0);
        hpend |= 1 << sl;
        if (lane == 0) {
          const uint32_t hb = smem_u32(&hbars[warp * 2 + sl]);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_expect_tx(hb, (uint32_t)rr * C * 2);
          wbuf_copy(smem_u32(wsl + sl * DF_WSLOT), Wh + (long)r0 * C, (uint32_t)rr * C * 2, hb);
        }
      };
      __syncthreads();   // the weight buffers are no longer read by the last layer
      if (nkw > 0) issue_w(0);
      if (nkw > 1) issue_w(1);
      bool hok = true;
      for (int k = 0; k < nkw; ++k) {
        const int sl = k & 1, wc = cta * DF_WARPS + warp + k * G * DF_WARPS;
        const int r0 = wc * hw, rr = min(hw, p.Vp - r0);
        {
          const uint32_t hb = smem_u32(&hbars[warp * 2 + sl]);
          bool okw = true;
          const long long t0 = clock64();
          for (unsigned it = 1; !mbar_try_wait(hb, (hpar >> sl) & 1); ++it) {
            if ((it & 63) == 0 && (*(volatile const unsigned*)p.abortf || clock64() - t0 > DF_BAR_LIMIT)) {
              okw = false;
              break;
            }
          }
          if (!__all_sync(0xffffffffu, okw)) { hok = false; break; }
          hpar ^= 1u << sl;
          hpend &= ~(1 << sl);
        }
        const bf16* ws = reinterpret_cast<const bf16*>(wsl + sl * DF_WSLOT);
        for (int r = 0; r < rr; ++r) {
          float acc[BB];
#pragma unroll
          for (int b = 0; b < BB; ++b) acc[b] = 0.f;
          for (int kk = lane * 8; kk < C; kk += 256) {
            float w[8];
            Vec<bf16>::load(ws + (long)r * C + kk, w);
#pragma unroll
            for (int b = 0; b < BB; ++b) {
              if (b < B) {
                const float4 x0 = *reinterpret_cast<const float4*>(xin + b * C + kk);
                const float4 x1 = *reinterpret_cast<const float4*>(xin + b * C + kk + 4);
                float a = acc[b];
                a = fmaf(w[0], x0.x, a); a = fmaf(w[1], x0.y, a); a = fmaf(w[2], x0.z, a); a = fmaf(w[3], x0.w, a);
                a = fmaf(w[4], x1.x, a); a = fmaf(w[5], x1.y, a); a = fmaf(w[6], x1.z, a); a = fmaf(w[7], x1.w, a);
                acc[b] = a;
              }
            }
          }
#pragma unroll
          for (int b = 0; b < BB; ++b) {
            if (b < B) {
              const float y = warp_sum(acc[b]);
              const int n = r0 + r;
              if (lane == 0) {
                p.logits[(long)b * p.Vp + n] = y;
                if (n < p.V && (y > bv[b] || (y == bv[b] && n < bi[b]))) { bv[b] = y; bi[b] = n; }
              }
            }
          }
        }
        __syncwarp();   // every lane is done with the slot before it is refilled
        if (k + 2 < nkw) issue_w(k + 2);
      }
      if (!hok && lane == 0) {
        atomicOr(p.err, GPT_DEVERR_TIMEOUT);
        atomicExch(p.abortf, 1u);
      }
      if (__syncthreads_or(!hok)) {
        // leave with none of this warp's copies in flight
        volatile int never = 0;
        if (lane == 0)
          for (int sl = 0; sl < 2; ++sl)
            if (hpend & (1 << sl)) mbar_wait(smem_u32(&hbars[warp * 2 + sl]), (hpar >> sl) & 1, &never, 1ll << 28);
        goto abort;
      }
      // per-CTA maxima (lane 0 of every warp holds its own)
      if (lane == 0) {
#pragma unroll
        for (int b = 0; b < BB; ++b) { s_rv[warp][b] = bv[b]; s_ri[warp][b] = bi[b]; }
      }
      __syncthreads();
      if (threadIdx.x < B) {
        const int b = threadIdx.x;
        float v = -INFINITY;
        int ix = 0x7fffffff;
        for (int w2 = 0; w2 < DF_WARPS; ++w2) {
          const float v2 = s_rv[w2][b];
          const int i2 = s_ri[w2][b];
          if (v2 > v || (v2 == v && i2 < ix)) { v = v2; ix = i2; }
        }
        p.am_v[(long)b * G + cta] = v;
        p.am_i[(long)b * G + cta] = ix;
      }
      __syncthreads();
      // the next step's (or the next layer 0's) qkv weights
      if (st + 1 < p.n_steps) {
        pend_a = issue_units(0, PW + lw(p.l_w_qkv, 0), nu_qkv, 16, 3 * C, C);
        issue_params(0, lw(p.l_ln1_g, 0), lw(p.l_b_qkv, 0), nu_qkv, 16, 3 * C);
      } else {
        pend_a = 0;
      }
      if (!df_grid_sync(p, ++nbar, &s_flag)) goto abort;
      // every CTA reduces the maxima: warp b takes row b
      if (warp < B) {
        const int b = warp;
        float v = -INFINITY;
        int ix = 0x7fffffff;
        for (int c2 = lane; c2 < G; c2 += 32) {
          const float v2 = __ldcg(p.am_v + (long)b * G + c2);
          const int i2 = __ldcg(p.am_i + (long)b * G + c2);
          if (v2 > v || (v2 == v && i2 < ix)) { v = v2; ix = i2; }
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) {
          const float v2 = __shfl_xor_sync(0xffffffffu, v, o2);
          const int i2 = __shfl_xor_sync(0xffffffffu, ix, o2);
          if (v2 > v || (v2 == v && i2 < ix)) { v = v2; ix = i2; }
        }
        if (lane == 0) {
          if (ix < 0 || ix >= p.V) ix = 0;   // all-NaN logits: fall back to id 0
          s_tok[b] = ix;
          if (cta == 0) {
            p.out[(long)b * p.out_ld + p.out_col0 + st] = ix;
            p.tok[b] = ix;
          }
        }
      }
      __syncthreads();
    }
  }
  return;
abort:
  // leave with no bulk copy in flight into this CTA's shared memory
  wbuf_drain(wb);
  {
    volatile int never = 0;
    for (int k = 0; k < 2; ++k)
      if (pinf[k]) mbar_wait(pbar[k], ppar[k], &never, 1ll << 28);
  }
}

// ------------------------------------------------------------------ host side
static int g_df_sms = 0;

static int df_sms() {
  if (!g_df_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&g_df_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      g_df_sms = 0;
    }
  }
  return g_df_sms;
}

// Key-range splits of the attention phase: about one unit per SM.
static int df_splits(int B, int H) {
  int S = df_sms() / (B * H);
  return S < 1 ? 1 : (S > DF_MAX_SPLITS ? DF_MAX_SPLITS : S);
}

// Shapes the fused decode kernel takes: every phase's units of one CTA fit a
// weight buffer, and the shared memory fits one CTA per SM.
bool dec_fused_supported(int B, int C, int H, int F, int Vp) {
  const int G = df_sms();
  if (G < 1 || G > DF_MAX_GRID || B < 1 || B > 4 || H < 1 || C % H) return false;
  const int D = C / H;
  if (D % 8 || D > 128 || 32 % (D / 8) || C % 16 || F % 16 || Vp < 1) return false;
  auto per_cta = [G](long units) { return (units + G - 1) / G; };
  if (per_cta(3 * C / 16) * 16L * C * 2 > DF_WBUF) return false;   // qkv
  if (per_cta(C / 16) * 16L * C * 2 > DF_WBUF) return false;       // out-projection
  if (per_cta(F / 16) * 16L * C * 2 > DF_WBUF) return false;       // fc
  if (DF_WSLOT / (2L * C) < 1) return false;                        // head warp-chunks of at least a row
  long rows_e = DF_WBUF / (F * 2L);
  if (rows_e > 16) rows_e = 16;
  rows_e &= ~3L;
  if (rows_e < 4) return false;
  if (per_cta((C + rows_e - 1) / rows_e) * rows_e * F * 2 > DF_WBUF) return false;   // fc2
  // bias slices of one CTA's units in one parameter area
  if (per_cta(3 * C / 16) * 16 > DF_PRM_BIAS || per_cta(F / 16) * 16 > DF_PRM_BIAS ||
      per_cta(C / 16) * 16 > DF_PRM_BIAS || per_cta((C + rows_e - 1) / rows_e) * rows_e > DF_PRM_BIAS)
    return false;
  const int KX = C > F ? C : F;
  if (DF_WARPS * (D + 2) > KX) return false;                        // attention partials in xin
  if ((long)B * H * df_splits(B, H) * (D + 2) * 4 > DF_WBUF) return false;   // the partials in buffer 0
  const size_t smem = 2 * DF_WBUF + (size_t)4 * (2 * 4 * C + 4 * KX + 2 * DF_PRM(C));
  return smem <= 227 * 1024;
}

cudaError_t launch_decode_fused(const DecFusedParams& prm, cudaStream_t s) {
  const int BB = prm.B <= 1 ? 1 : prm.B <= 2 ? 2 : 4;
  const int KX = prm.C > prm.F ? prm.C : prm.F;
  const size_t smem = 2 * DF_WBUF + (size_t)4 * (2 * BB * prm.C + BB * KX + 2 * DF_PRM(prm.C));
  void* fn = BB == 1 ? (void*)decode_fused_kernel<1> : BB == 2 ? (void*)decode_fused_kernel<2>
                                                                 : (void*)decode_fused_kernel<4>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (df_sms() < 1) return cudaErrorNotSupported;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, DF_THREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorNotSupported;
  DecFusedParams q = prm;
  const int G = g_df_sms;
  q.S = df_splits(q.B, q.H);
  void* args[] = {(void*)&q};
  ++g_kernel_launches;
  return cudaLaunchCooperativeKernel(fn, dim3(G), dim3(DF_THREADS), args, smem, s);
}
