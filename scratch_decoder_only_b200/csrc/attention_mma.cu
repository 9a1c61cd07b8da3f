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

// ---------------------------------------------------------------- forward
template <int D>
__global__ void __launch_bounds__(FA_THREADS)
attn_fwd_mma(const bf16* __restrict__ qkv, bf16* __restrict__ out, float* __restrict__ lse,
             const int* __restrict__ dstart, int T, int H) {
  constexpr int LDS = D + 8;
  __shared__ __align__(16) bf16 Qs[FA_BLK * LDS], Ks[FA_BLK * LDS], Vs[FA_BLK * LDS];
  const int nqb = (T + FA_BLK - 1) / FA_BLK;
  const int qb = nqb - 1 - blockIdx.x;   // heaviest (latest) query blocks first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * D;
  const long C3 = 3L * C;
  const int q0 = qb * FA_BLK;
  const bf16* base = qkv + (long)b * T * C3;
  const int* dsr = dstart + (long)b * T;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;

  load_tile<D>(Qs, base, q0, T, C3, h * D);
  cp_async_wait_all();
  __syncthreads();
  uint32_t qf[D / 16][4];
  load_afrag<D>(Qs, w, lane, qf);

  const int r_lo = q0 + w * 16 + (lane >> 2), r_hi = r_lo + 8;
  const int ds_lo = r_lo < T ? dsr[r_lo] : 0, ds_hi = r_hi < T ? dsr[r_hi] : 0;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
  const float sl2 = rsqrtf((float)D) * LOG2E;
  const int kb_lo = dsr[q0] / FA_BLK, kb_hi = min(q0 + FA_BLK - 1, T - 1) / FA_BLK;

  for (int kb = kb_lo; kb <= kb_hi; ++kb) {
    const int j0 = kb * FA_BLK;
    __syncthreads();
    load_tile<D>(Ks, base, j0, T, C3, C + h * D);
    load_tile<D>(Vs, base, j0, T, C3, 2 * C + h * D);
    cp_async_wait_all();
    __syncthreads();
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
  l_lo = quad_sum(l_lo);
  l_hi = quad_sum(l_hi);
  const float inv_lo = 1.f / l_lo, inv_hi = 1.f / l_hi;
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
template <int D>
__global__ void __launch_bounds__(FA_THREADS)
attn_bwd_dq_mma(const bf16* __restrict__ qkv, const bf16* __restrict__ out, const bf16* __restrict__ dout,
                const float* __restrict__ lse, float* __restrict__ Dbuf, const int* __restrict__ dstart,
                bf16* __restrict__ dqkv, int T, int H) {
  constexpr int LDS = D + 8;
  __shared__ __align__(16) bf16 Qs[FA_BLK * LDS], dOs[FA_BLK * LDS], Ks[FA_BLK * LDS], Vs[FA_BLK * LDS];
  __shared__ float Dsm[FA_BLK];
  const int nqb = (T + FA_BLK - 1) / FA_BLK;
  const int qb = nqb - 1 - blockIdx.x;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * D;
  const long C3 = 3L * C;
  const int q0 = qb * FA_BLK;
  const bf16* base = qkv + (long)b * T * C3;
  const int* dsr = dstart + (long)b * T;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;

  load_tile<D>(Qs, base, q0, T, C3, h * D);
  load_tile<D>(dOs, dout + (long)b * T * C, q0, T, C, h * D);
  // D_i = dO_i . O_i for the 64 rows (two threads per row)
  {
    int r = threadIdx.x >> 1, half = threadIdx.x & 1;
    float acc = 0.f;
    if (q0 + r < T) {
      const bf16* a = dout + ((long)b * T + q0 + r) * C + h * D + half * (D / 2);
      const bf16* c = out + ((long)b * T + q0 + r) * C + h * D + half * (D / 2);
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
      Dsm[r] = acc;
      if (q0 + r < T) Dbuf[(long)bh * T + q0 + r] = acc;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  uint32_t qf[D / 16][4], df[D / 16][4];
  load_afrag<D>(Qs, w, lane, qf);
  load_afrag<D>(dOs, w, lane, df);

  const int rl_lo = w * 16 + (lane >> 2), rl_hi = rl_lo + 8;
  const int r_lo = q0 + rl_lo, r_hi = q0 + rl_hi;
  const int ds_lo = r_lo < T ? dsr[r_lo] : 0, ds_hi = r_hi < T ? dsr[r_hi] : 0;
  const float L_lo = r_lo < T ? lse[(long)bh * T + r_lo] * LOG2E : 0.f;
  const float L_hi = r_hi < T ? lse[(long)bh * T + r_hi] * LOG2E : 0.f;
  const float D_lo = Dsm[rl_lo], D_hi = Dsm[rl_hi];
  const float scale = rsqrtf((float)D), sl2 = scale * LOG2E;
  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[i][e] = 0.f;
  const int kb_lo = dsr[q0] / FA_BLK, kb_hi = min(q0 + FA_BLK - 1, T - 1) / FA_BLK;
  for (int kb = kb_lo; kb <= kb_hi; ++kb) {
    const int j0 = kb * FA_BLK;
    __syncthreads();
    load_tile<D>(Ks, base, j0, T, C3, C + h * D);
    load_tile<D>(Vs, base, j0, T, C3, 2 * C + h * D);
    cp_async_wait_all();
    __syncthreads();
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
template <int D>
__global__ void __launch_bounds__(FA_THREADS)
attn_bwd_dkdv_mma(const bf16* __restrict__ qkv, const bf16* __restrict__ dout, const float* __restrict__ lse,
                  const float* __restrict__ Dbuf, const int* __restrict__ dstart, bf16* __restrict__ dqkv, int T,
                  int H) {
  constexpr int LDS = D + 8;
  __shared__ __align__(16) bf16 Ks[FA_BLK * LDS], Vs[FA_BLK * LDS], Qs[FA_BLK * LDS], dOs[FA_BLK * LDS];
  __shared__ float Lsm[FA_BLK], Dsm[FA_BLK];
  __shared__ int DSs[FA_BLK];
  const int nkb = (T + FA_BLK - 1) / FA_BLK;
  const int kb = blockIdx.x;   // earliest key blocks see the most queries: launched first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * D;
  const long C3 = 3L * C;
  const int j0 = kb * FA_BLK;
  const bf16* base = qkv + (long)b * T * C3;
  const bf16* dbase = dout + (long)b * T * C;
  const int* dsr = dstart + (long)b * T;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  (void)nkb;

  load_tile<D>(Ks, base, j0, T, C3, C + h * D);
  load_tile<D>(Vs, base, j0, T, C3, 2 * C + h * D);
  cp_async_wait_all();
  __syncthreads();
  uint32_t kf[D / 16][4], vf[D / 16][4];
  load_afrag<D>(Ks, w, lane, kf);
  load_afrag<D>(Vs, w, lane, vf);

  const int k_lo = j0 + w * 16 + (lane >> 2), k_hi = k_lo + 8;
  const float scale = rsqrtf((float)D), sl2 = scale * LOG2E;
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) { dk[i][e] = 0.f; dv[i][e] = 0.f; }
  const int nqb = (T + FA_BLK - 1) / FA_BLK;
  const int last_key = min(j0 + FA_BLK - 1, T - 1);
  for (int qb = kb; qb < nqb; ++qb) {
    const int q0 = qb * FA_BLK;
    if (dsr[q0] > last_key) break;   // every later query lives in a later document
    __syncthreads();
    load_tile<D>(Qs, base, q0, T, C3, h * D);
    load_tile<D>(dOs, dbase, q0, T, C, h * D);
    if (threadIdx.x < FA_BLK) {
      int i = q0 + threadIdx.x;
      bool ok = i < T;
      Lsm[threadIdx.x] = ok ? lse[(long)bh * T + i] * LOG2E : 0.f;
      Dsm[threadIdx.x] = ok ? Dbuf[(long)bh * T + i] : 0.f;
      DSs[threadIdx.x] = ok ? dsr[i] : 0x7fffffff;
    }
    cp_async_wait_all();
    __syncthreads();
    float st[8][4], dpt[8][4];
    mma_abt<D>(st, kf, Qs, lane);     // S^T: keys x queries
    mma_abt<D>(dpt, vf, dOs, lane);   // dP^T = V dO^T
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int il = nt * 8 + (lane & 3) * 2 + (e & 1);
        int i = q0 + il;
        int j = e < 2 ? k_lo : k_hi;
        bool ok = i < T && i >= j && DSs[il] <= j;
        float p = ok ? exp2f(st[nt][e] * sl2 - Lsm[il]) : 0.f;
        st[nt][e] = p;
        dpt[nt][e] = p * (dpt[nt][e] - Dsm[il]);   // dS^T
      }
    mma_pb<D>(dv, st, dOs, lane);
    mma_pb<D>(dk, dpt, Qs, lane);
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
// head sizes up to 64 fit four 64-row tiles in static shared memory
bool attn_mma_supported(int d) { return d == 16 || d == 32 || d == 64; }

template <int D>
static cudaError_t fwd_launch(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T, int H,
                              cudaStream_t s) {
  dim3 grid((T + FA_BLK - 1) / FA_BLK, B * H);
  ++g_kernel_launches;
  attn_fwd_mma<D><<<grid, FA_THREADS, 0, s>>>(qkv, out, lse, dstart, T, H);
  return cudaGetLastError();
}

template <int D>
static cudaError_t bwd_launch(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dbuf,
                              const int* dstart, bf16* dqkv, int B, int T, int H, cudaStream_t s) {
  dim3 grid((T + FA_BLK - 1) / FA_BLK, B * H);
  ++g_kernel_launches;
  attn_bwd_dq_mma<D><<<grid, FA_THREADS, 0, s>>>(qkv, out, dout, lse, Dbuf, dstart, dqkv, T, H);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ++g_kernel_launches;
  attn_bwd_dkdv_mma<D><<<grid, FA_THREADS, 0, s>>>(qkv, dout, lse, Dbuf, dstart, dqkv, T, H);
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
