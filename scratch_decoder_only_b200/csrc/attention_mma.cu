// bf16 flash attention on tensor cores (mma.sync m16n8k16, fp32 accumulate),
// causal with the block-diagonal mask of packed documents.
//
// A query i sees the keys j with dstart[i] <= j <= i (its own document, up to
// itself).  Because document starts never decrease along a row, a 64-query
// block needs only the key blocks from dstart[first query] to the diagonal,
// and a 64-key block is seen only by query blocks up to the end of the
// documents it belongs to: all other tiles are skipped, not masked.
//
// Forward: one CTA = (64 queries, batch row, head), 4 warps x 16 query rows;
// scores S = Q K^T / sqrt(d) in registers, online softmax in the exp2 domain,
// O += P V with P taken straight from the score registers; O and the row
// log-sum-exp are written.
// Backward (deterministic, no atomics): a dQ kernel over query blocks
// (P recomputed from lse, dP = dO V^T, dS = P (dP - D), dQ = dS K, with
// D_i = dO_i . O_i computed there) and a dK/dV kernel over key blocks
// (P^T, dV = P^T dO, dP^T = V dO^T, dK = dS^T Q).
#include "launch.h"

#define FA_BLK 64
#define FA_THREADS 128
#define LOG2E 1.4426950408889634f
#define LN2 0.6931471805599453f

__device__ __forceinline__ uint32_t sm_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// Load rows r0..r0+63 (of T) of a [*, ld] bf16 matrix, columns col..col+D-1,
// into smem [64][D+8]; rows past T are zero-filled.
template <int D>
__device__ __forceinline__ void load_tile(bf16* sm, const bf16* base, int r0, int T, long ld, int col) {
  constexpr int LDS = D + 8, CH = D / 8;
  for (int i = threadIdx.x; i < FA_BLK * CH; i += FA_THREADS) {
    int r = i / CH, c = (i % CH) * 8;
    bool ok = r0 + r < T;
    const bf16* src = ok ? base + (long)(r0 + r) * ld + col + c : base;
    cp_async16(sm_addr(sm + r * LDS + c), src, ok);
  }
}

// A fragments (16 rows x D) of rows w*16.. of a smem tile.
template <int D>
__device__ __forceinline__ void load_afrag(const bf16* sm, int w, int lane, uint32_t (*f)[4]) {
  constexpr int LDS = D + 8;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    int row = w * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
    int col = kk * 16 + 8 * (lane >> 4);
    ldsm_x4(sm_addr(sm + row * LDS + col), f[kk][0], f[kk][1], f[kk][2], f[kk][3]);
  }
}

// acc[8][4] (16 x 64) = A(16 x D, fragments) . Bsm(64 rows x D)^T
template <int D>
__device__ __forceinline__ void mma_abt(float (*acc)[4], const uint32_t (*a)[4], const bf16* bsm, int lane) {
  constexpr int LDS = D + 8;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
  for (int np = 0; np < 4; ++np) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      int row = np * 16 + (lane & 7) + 8 * (lane >> 4);
      int col = kk * 16 + 8 * ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sm_addr(bsm + row * LDS + col), b0, b1, b2, b3);
      mma16816(acc[2 * np], a[kk], b0, b1);
      mma16816(acc[2 * np + 1], a[kk], b2, b3);
    }
  }
}

// acc[D/8][4] (16 x D) += P(16 x 64, from score registers) . Bsm(64 rows x D)
template <int D>
__device__ __forceinline__ void mma_pb(float (*acc)[4], const float (*p)[4], const bf16* bsm, int lane) {
  constexpr int LDS = D + 8;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = pack2(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack2(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack2(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack2(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int dp = 0; dp < D / 16; ++dp) {
      int row = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
      int col = dp * 16 + 8 * (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sm_addr(bsm + row * LDS + col), b0, b1, b2, b3);
      mma16816(acc[2 * dp], a, b0, b1);
      mma16816(acc[2 * dp + 1], a, b2, b3);
    }
  }
}

__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

// Double-buffered 64-row tiles: stage `buf` holds two 64 x (D+8) tiles.
template <int D>
__device__ __forceinline__ bf16* stage_ptr(bf16* base, int buf, int which) {
  return base + (buf * 2 + which) * FA_BLK * (D + 8);
}

// ---------------------------------------------------------------- forward
// One CTA = WARPS x 16 queries of one (batch row, head); key blocks of 64.
template <int D, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
attn_fwd_mma(const bf16* __restrict__ qkv, bf16* __restrict__ out, float* __restrict__ lse,
             const int* __restrict__ dstart, int T, int H) {
  constexpr int LDS = D + 8, QROWS = WARPS * 16;
  extern __shared__ __align__(16) bf16 fa_sm[];
  bf16* Qs = fa_sm;                        // QROWS rows, then reused: K/V double buffer
  bf16* KV = fa_sm + QROWS * LDS;          // 2 stages x (K, V) x 64 rows
  const int nqb = (T + QROWS - 1) / QROWS;
  const int qb = nqb - 1 - blockIdx.x;     // heaviest (latest) query blocks first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * D;
  const long C3 = 3L * C;
  const int q0 = qb * QROWS;
  const bf16* base = qkv + (long)b * T * C3;
  const int* dsr = dstart + (long)b * T;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb_lo = dsr[q0] / FA_BLK, kb_hi = min(q0 + QROWS - 1, T - 1) / FA_BLK;

  for (int i = threadIdx.x; i < QROWS * (D / 8); i += WARPS * 32) {
    int r = i / (D / 8), c = (i % (D / 8)) * 8;
    bool ok = q0 + r < T;
    cp_async16(sm_addr(Qs + r * LDS + c), ok ? base + (long)(q0 + r) * C3 + h * D + c : base, ok);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // first K/V block
  for (int i = threadIdx.x; i < FA_BLK * (D / 8); i += WARPS * 32) {
    int r = i / (D / 8), c = (i % (D / 8)) * 8;
    int j = kb_lo * FA_BLK + r;
    bool ok = j < T;
    const bf16* src = ok ? base + (long)j * C3 + C + h * D + c : base;
    cp_async16(sm_addr(stage_ptr<D>(KV, 0, 0) + r * LDS + c), src, ok);
    cp_async16(sm_addr(stage_ptr<D>(KV, 0, 1) + r * LDS + c), ok ? src + C : base, ok);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 1;" ::: "memory");
  __syncthreads();
  uint32_t qf[D / 16][4];
  {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      int row = w * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
      int col = kk * 16 + 8 * (lane >> 4);
      ldsm_x4(sm_addr(Qs + row * LDS + col), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
  }
  const int wr0 = q0 + w * 16;
  const int r_lo = wr0 + (lane >> 2), r_hi = r_lo + 8;
  const int ds_lo = r_lo < T ? dsr[r_lo] : 0, ds_hi = r_hi < T ? dsr[r_hi] : 0;
  const int ds_w = wr0 < T ? dsr[wr0] : T;   // smallest document start among the warp's rows
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
  const float sl2 = rsqrtf((float)D) * LOG2E;

  for (int kb = kb_lo, st = 0; kb <= kb_hi; ++kb, st ^= 1) {
    const int j0 = kb * FA_BLK;
    if (kb < kb_hi) {   // prefetch the next block into the other stage
      for (int i = threadIdx.x; i < FA_BLK * (D / 8); i += WARPS * 32) {
        int r = i / (D / 8), c = (i % (D / 8)) * 8;
        int j = j0 + FA_BLK + r;
        bool ok = j < T;
        const bf16* src = ok ? base + (long)j * C3 + C + h * D + c : base;
        cp_async16(sm_addr(stage_ptr<D>(KV, st ^ 1, 0) + r * LDS + c), src, ok);
        cp_async16(sm_addr(stage_ptr<D>(KV, st ^ 1, 1) + r * LDS + c), ok ? src + C : base, ok);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const bf16* Ks = stage_ptr<D>(KV, st, 0);
    const bf16* Vs = stage_ptr<D>(KV, st, 1);
    // skip a 16 x 64 sub-tile that is entirely masked for this warp
    const bool live = j0 <= wr0 + 15 && j0 + FA_BLK - 1 >= ds_w && wr0 < T;
    if (live) {
      float s[8][4];
      mma_abt<D>(s, qf, Ks, lane);
      float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int j = j0 + nt * 8 + (lane & 3) * 2 + (e & 1);
          int r = e < 2 ? r_lo : r_hi, ds = e < 2 ? ds_lo : ds_hi;
          float v = (j > r || j < ds) ? -INFINITY : s[nt][e] * sl2;
          s[nt][e] = v;
          if (e < 2) mx_lo = fmaxf(mx_lo, v); else mx_hi = fmaxf(mx_hi, v);
        }
      mx_lo = quad_max(mx_lo);
      mx_hi = quad_max(mx_hi);
      const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
      const float use_lo = mn_lo == -INFINITY ? 0.f : mn_lo, use_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
      const float c_lo = exp2f(m_lo - use_lo), c_hi = exp2f(m_hi - use_hi);
      float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][0] = exp2f(s[nt][0] - use_lo);
        s[nt][1] = exp2f(s[nt][1] - use_lo);
        s[nt][2] = exp2f(s[nt][2] - use_hi);
        s[nt][3] = exp2f(s[nt][3] - use_hi);
        ps_lo += s[nt][0] + s[nt][1];
        ps_hi += s[nt][2] + s[nt][3];
      }
      l_lo = l_lo * c_lo + ps_lo;
      l_hi = l_hi * c_hi + ps_hi;
      m_lo = mn_lo;
      m_hi = mn_hi;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[i][0] *= c_lo; o[i][1] *= c_lo;
        o[i][2] *= c_hi; o[i][3] *= c_hi;
      }
      mma_pb<D>(o, s, Vs, lane);
    }
    __syncthreads();   // stage st is refilled by the next iteration's prefetch
  }
  l_lo = quad_sum(l_lo);
  l_hi = quad_sum(l_hi);
  const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    int col = h * D + i * 8 + (lane & 3) * 2;
    if (r_lo < T)
      *reinterpret_cast<uint32_t*>(out + ((long)b * T + r_lo) * C + col) = pack2(o[i][0] * inv_lo, o[i][1] * inv_lo);
    if (r_hi < T)
      *reinterpret_cast<uint32_t*>(out + ((long)b * T + r_hi) * C + col) = pack2(o[i][2] * inv_hi, o[i][3] * inv_hi);
  }
  if ((lane & 3) == 0) {
    if (r_lo < T) lse[(long)bh * T + r_lo] = (m_lo + log2f(l_lo)) * LN2;
    if (r_hi < T) lse[(long)bh * T + r_hi] = (m_hi + log2f(l_hi)) * LN2;
  }
}

// ---------------------------------------------------------------- backward: dQ
template <int D, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
attn_bwd_dq_mma(const bf16* __restrict__ qkv, const bf16* __restrict__ out, const bf16* __restrict__ dout,
                const float* __restrict__ lse, float* __restrict__ Dbuf, const int* __restrict__ dstart,
                bf16* __restrict__ dqkv, int T, int H) {
  constexpr int LDS = D + 8, QROWS = WARPS * 16;
  extern __shared__ __align__(16) bf16 fa_sm[];
  bf16* Qs = fa_sm;
  bf16* dOs = fa_sm + QROWS * LDS;
  bf16* KV = fa_sm + 2 * QROWS * LDS;
  float* Dsm = reinterpret_cast<float*>(fa_sm + 2 * QROWS * LDS + 4 * FA_BLK * LDS);
  const int nqb = (T + QROWS - 1) / QROWS;
  const int qb = nqb - 1 - blockIdx.x;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * D;
  const long C3 = 3L * C;
  const int q0 = qb * QROWS;
  const bf16* base = qkv + (long)b * T * C3;
  const int* dsr = dstart + (long)b * T;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb_lo = dsr[q0] / FA_BLK, kb_hi = min(q0 + QROWS - 1, T - 1) / FA_BLK;

  for (int i = threadIdx.x; i < QROWS * (D / 8); i += WARPS * 32) {
    int r = i / (D / 8), c = (i % (D / 8)) * 8;
    bool ok = q0 + r < T;
    cp_async16(sm_addr(Qs + r * LDS + c), ok ? base + (long)(q0 + r) * C3 + h * D + c : base, ok);
    cp_async16(sm_addr(dOs + r * LDS + c), ok ? dout + ((long)b * T + q0 + r) * C + h * D + c : dout, ok);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int i = threadIdx.x; i < FA_BLK * (D / 8); i += WARPS * 32) {
    int r = i / (D / 8), c = (i % (D / 8)) * 8;
    int j = kb_lo * FA_BLK + r;
    bool ok = j < T;
    const bf16* src = ok ? base + (long)j * C3 + C + h * D + c : base;
    cp_async16(sm_addr(stage_ptr<D>(KV, 0, 0) + r * LDS + c), src, ok);
    cp_async16(sm_addr(stage_ptr<D>(KV, 0, 1) + r * LDS + c), ok ? src + C : base, ok);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // D_i = dO_i . O_i (two threads per row for QROWS rows, looping)
  for (int rr = threadIdx.x >> 1; rr < QROWS; rr += WARPS * 16) {
    int half = threadIdx.x & 1;
    float acc = 0.f;
    if (q0 + rr < T) {
      const bf16* a = dout + ((long)b * T + q0 + rr) * C + h * D + half * (D / 2);
      const bf16* c = out + ((long)b * T + q0 + rr) * C + h * D + half * (D / 2);
      for (int i = 0; i < D / 2; i += 8) {
        float x[8], y[8];
        Vec<bf16>::load(a + i, x);
        Vec<bf16>::load(c + i, y);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc += x[k] * y[k];
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (half == 0) {
      Dsm[rr] = acc;
      if (q0 + rr < T) Dbuf[(long)bh * T + q0 + rr] = acc;
    }
  }
  asm volatile("cp.async.wait_group 1;" ::: "memory");
  __syncthreads();
  uint32_t qf[D / 16][4], df[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    int row = w * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
    int col = kk * 16 + 8 * (lane >> 4);
    ldsm_x4(sm_addr(Qs + row * LDS + col), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    ldsm_x4(sm_addr(dOs + row * LDS + col), df[kk][0], df[kk][1], df[kk][2], df[kk][3]);
  }
  const int wr0 = q0 + w * 16;
  const int rl_lo = w * 16 + (lane >> 2), rl_hi = rl_lo + 8;
  const int r_lo = q0 + rl_lo, r_hi = q0 + rl_hi;
  const int ds_lo = r_lo < T ? dsr[r_lo] : 0, ds_hi = r_hi < T ? dsr[r_hi] : 0;
  const int ds_w = wr0 < T ? dsr[wr0] : T;
  const float L_lo = r_lo < T ? lse[(long)bh * T + r_lo] * LOG2E : 0.f;
  const float L_hi = r_hi < T ? lse[(long)bh * T + r_hi] * LOG2E : 0.f;
  const float D_lo = Dsm[rl_lo], D_hi = Dsm[rl_hi];
  const float scale = rsqrtf((float)D), sl2 = scale * LOG2E;
  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[i][e] = 0.f;
  for (int kb = kb_lo, st = 0; kb <= kb_hi; ++kb, st ^= 1) {
    const int j0 = kb * FA_BLK;
    if (kb < kb_hi) {
      for (int i = threadIdx.x; i < FA_BLK * (D / 8); i += WARPS * 32) {
        int r = i / (D / 8), c = (i % (D / 8)) * 8;
        int j = j0 + FA_BLK + r;
        bool ok = j < T;
        const bf16* src = ok ? base + (long)j * C3 + C + h * D + c : base;
        cp_async16(sm_addr(stage_ptr<D>(KV, st ^ 1, 0) + r * LDS + c), src, ok);
        cp_async16(sm_addr(stage_ptr<D>(KV, st ^ 1, 1) + r * LDS + c), ok ? src + C : base, ok);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const bf16* Ks = stage_ptr<D>(KV, st, 0);
    const bf16* Vs = stage_ptr<D>(KV, st, 1);
    const bool live = j0 <= wr0 + 15 && j0 + FA_BLK - 1 >= ds_w && wr0 < T;
    if (live) {
      float s[8][4], dp[8][4];
      mma_abt<D>(s, qf, Ks, lane);
      mma_abt<D>(dp, df, Vs, lane);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int j = j0 + nt * 8 + (lane & 3) * 2 + (e & 1);
          int r = e < 2 ? r_lo : r_hi, ds = e < 2 ? ds_lo : ds_hi;
          float p = (j > r || j < ds) ? 0.f : exp2f(s[nt][e] * sl2 - (e < 2 ? L_lo : L_hi));
          s[nt][e] = p * (dp[nt][e] - (e < 2 ? D_lo : D_hi));   // dS
        }
      mma_pb<D>(dq, s, Ks, lane);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    int col = h * D + i * 8 + (lane & 3) * 2;
    if (r_lo < T)
      *reinterpret_cast<uint32_t*>(dqkv + ((long)b * T + r_lo) * C3 + col) = pack2(dq[i][0] * scale, dq[i][1] * scale);
    if (r_hi < T)
      *reinterpret_cast<uint32_t*>(dqkv + ((long)b * T + r_hi) * C3 + col) = pack2(dq[i][2] * scale, dq[i][3] * scale);
  }
}

// ---------------------------------------------------------------- backward: dK, dV
template <int D, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
attn_bwd_dkdv_mma(const bf16* __restrict__ qkv, const bf16* __restrict__ dout, const float* __restrict__ lse,
                  const float* __restrict__ Dbuf, const int* __restrict__ dstart, bf16* __restrict__ dqkv, int T,
                  int H) {
  constexpr int LDS = D + 8, KROWS = WARPS * 16;
  extern __shared__ __align__(16) bf16 fa_sm[];
  bf16* Ks = fa_sm;
  bf16* Vs = fa_sm + KROWS * LDS;
  bf16* QD = fa_sm + 2 * KROWS * LDS;     // 2 stages x (Q, dO) x 64 rows
  float* aux = reinterpret_cast<float*>(QD + 4 * FA_BLK * LDS);   // 2 stages x (L, D, dstart) x 64
  const int kb = blockIdx.x;   // earliest key blocks see the most queries: launched first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * D;
  const long C3 = 3L * C;
  const int j0 = kb * KROWS;
  const bf16* base = qkv + (long)b * T * C3;
  const bf16* dbase = dout + (long)b * T * C;
  const int* dsr = dstart + (long)b * T;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + FA_BLK - 1) / FA_BLK;
  const int last_key = min(j0 + KROWS - 1, T - 1);
  const int qb_lo = j0 / FA_BLK;

  auto issue_q = [&](int qb, int st) {
    const int q0 = qb * FA_BLK;
    for (int i = threadIdx.x; i < FA_BLK * (D / 8); i += WARPS * 32) {
      int r = i / (D / 8), c = (i % (D / 8)) * 8;
      bool ok = q0 + r < T;
      cp_async16(sm_addr(stage_ptr<D>(QD, st, 0) + r * LDS + c), ok ? base + (long)(q0 + r) * C3 + h * D + c : base, ok);
      cp_async16(sm_addr(stage_ptr<D>(QD, st, 1) + r * LDS + c), ok ? dbase + (long)(q0 + r) * C + h * D + c : dbase, ok);
    }
    float* L = aux + st * 3 * FA_BLK;
    for (int i = threadIdx.x; i < FA_BLK; i += WARPS * 32) {
      int q = q0 + i;
      bool ok = q < T;
      L[i] = ok ? lse[(long)bh * T + q] * LOG2E : 0.f;
      L[FA_BLK + i] = ok ? Dbuf[(long)bh * T + q] : 0.f;
      reinterpret_cast<int*>(L)[2 * FA_BLK + i] = ok ? dsr[q] : 0x7fffffff;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  for (int i = threadIdx.x; i < KROWS * (D / 8); i += WARPS * 32) {
    int r = i / (D / 8), c = (i % (D / 8)) * 8;
    bool ok = j0 + r < T;
    const bf16* src = ok ? base + (long)(j0 + r) * C3 + C + h * D + c : base;
    cp_async16(sm_addr(Ks + r * LDS + c), src, ok);
    cp_async16(sm_addr(Vs + r * LDS + c), ok ? src + C : base, ok);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  issue_q(qb_lo, 0);
  asm volatile("cp.async.wait_group 1;" ::: "memory");
  __syncthreads();
  uint32_t kf[D / 16][4], vf[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    int row = w * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
    int col = kk * 16 + 8 * (lane >> 4);
    ldsm_x4(sm_addr(Ks + row * LDS + col), kf[kk][0], kf[kk][1], kf[kk][2], kf[kk][3]);
    ldsm_x4(sm_addr(Vs + row * LDS + col), vf[kk][0], vf[kk][1], vf[kk][2], vf[kk][3]);
  }
  const int wk0 = j0 + w * 16;
  const int k_lo = wk0 + (lane >> 2), k_hi = k_lo + 8;
  const float scale = rsqrtf((float)D), sl2 = scale * LOG2E;
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) { dk[i][e] = 0.f; dv[i][e] = 0.f; }
  int st = 0;
  for (int qb = qb_lo; qb < nqb; ++qb, st ^= 1) {
    const int q0 = qb * FA_BLK;
    if (dsr[q0] > last_key) break;   // every later query lives in a later document
    const bool more = qb + 1 < nqb && dsr[q0 + FA_BLK] <= last_key;
    if (more) {
      issue_q(qb + 1, st ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const bf16* Qs = stage_ptr<D>(QD, st, 0);
    const bf16* dOs = stage_ptr<D>(QD, st, 1);
    const float* Lsm = aux + st * 3 * FA_BLK;
    const float* Dsm = Lsm + FA_BLK;
    const int* DSs = reinterpret_cast<const int*>(Lsm + 2 * FA_BLK);
    // skip a 16-key x 64-query sub-tile that is entirely masked for this warp
    const bool live = q0 + FA_BLK - 1 >= wk0 && DSs[0] <= wk0 + 15 && wk0 < T;
    if (live) {
      float st_[8][4], dpt[8][4];
      mma_abt<D>(st_, kf, Qs, lane);     // S^T: keys x queries
      mma_abt<D>(dpt, vf, dOs, lane);    // dP^T = V dO^T
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int il = nt * 8 + (lane & 3) * 2 + (e & 1);
          int i = q0 + il;
          int j = e < 2 ? k_lo : k_hi;
          bool ok = i < T && i >= j && DSs[il] <= j;
          float p = ok ? exp2f(st_[nt][e] * sl2 - Lsm[il]) : 0.f;
          st_[nt][e] = p;
          dpt[nt][e] = p * (dpt[nt][e] - Dsm[il]);   // dS^T
        }
      mma_pb<D>(dv, st_, dOs, lane);
      mma_pb<D>(dk, dpt, Qs, lane);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    int col = h * D + i * 8 + (lane & 3) * 2;
    if (k_lo < T) {
      bf16* row = dqkv + ((long)b * T + k_lo) * C3;
      *reinterpret_cast<uint32_t*>(row + C + col) = pack2(dk[i][0] * scale, dk[i][1] * scale);
      *reinterpret_cast<uint32_t*>(row + 2 * C + col) = pack2(dv[i][0], dv[i][1]);
    }
    if (k_hi < T) {
      bf16* row = dqkv + ((long)b * T + k_hi) * C3;
      *reinterpret_cast<uint32_t*>(row + C + col) = pack2(dk[i][2] * scale, dk[i][3] * scale);
      *reinterpret_cast<uint32_t*>(row + 2 * C + col) = pack2(dv[i][2], dv[i][3]);
    }
  }
}

// ---------------------------------------------------------------- launchers
// head sizes up to 64 (register-resident fragments of one 16-row slice)
bool attn_mma_supported(int d) { return d == 16 || d == 32 || d == 64; }

#define FWD_WARPS 8
#define DQ_WARPS 4
#define DKV_WARPS 4

template <typename K>
static cudaError_t set_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int D>
static cudaError_t fwd_launch(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T, int H,
                              cudaStream_t s) {
  constexpr int LDS = D + 8;
  size_t smem = (size_t)(FWD_WARPS * 16 + 4 * FA_BLK) * LDS * 2;
  static bool attr = false;
  if (!attr) { cudaError_t e = set_smem(attn_fwd_mma<D, FWD_WARPS>, smem); if (e) return e; attr = true; }
  dim3 grid((T + FWD_WARPS * 16 - 1) / (FWD_WARPS * 16), B * H);
  ++g_kernel_launches;
  attn_fwd_mma<D, FWD_WARPS><<<grid, FWD_WARPS * 32, smem, s>>>(qkv, out, lse, dstart, T, H);
  return cudaGetLastError();
}

template <int D>
static cudaError_t bwd_launch(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dbuf,
                              const int* dstart, bf16* dqkv, int B, int T, int H, cudaStream_t s) {
  constexpr int LDS = D + 8;
  size_t smem_q = (size_t)(2 * DQ_WARPS * 16 + 4 * FA_BLK) * LDS * 2 + DQ_WARPS * 16 * 4;
  size_t smem_k = (size_t)(2 * DKV_WARPS * 16 + 4 * FA_BLK) * LDS * 2 + 6 * FA_BLK * 4;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = set_smem(attn_bwd_dq_mma<D, DQ_WARPS>, smem_q);
    if (e == cudaSuccess) e = set_smem(attn_bwd_dkdv_mma<D, DKV_WARPS>, smem_k);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 gq((T + DQ_WARPS * 16 - 1) / (DQ_WARPS * 16), B * H);
  ++g_kernel_launches;
  attn_bwd_dq_mma<D, DQ_WARPS><<<gq, DQ_WARPS * 32, smem_q, s>>>(qkv, out, dout, lse, Dbuf, dstart, dqkv, T, H);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 gk((T + DKV_WARPS * 16 - 1) / (DKV_WARPS * 16), B * H);
  ++g_kernel_launches;
  attn_bwd_dkdv_mma<D, DKV_WARPS><<<gk, DKV_WARPS * 32, smem_k, s>>>(qkv, dout, lse, Dbuf, dstart, dqkv, T, H);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_mma(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T, int H,
                                int d, cudaStream_t s) {
  switch (d) {
    case 16: return fwd_launch<16>(qkv, out, lse, dstart, B, T, H, s);
    case 32: return fwd_launch<32>(qkv, out, lse, dstart, B, T, H, s);
    case 64: return fwd_launch<64>(qkv, out, lse, dstart, B, T, H, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd_mma(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dbuf,
                                const int* dstart, bf16* dqkv, int B, int T, int H, int d, cudaStream_t s) {
  switch (d) {
    case 16: return bwd_launch<16>(qkv, out, dout, lse, Dbuf, dstart, dqkv, B, T, H, s);
    case 32: return bwd_launch<32>(qkv, out, dout, lse, Dbuf, dstart, dqkv, B, T, H, s);
    case 64: return bwd_launch<64>(qkv, out, dout, lse, Dbuf, dstart, dqkv, B, T, H, s);
  }
  return cudaErrorInvalidValue;
}
