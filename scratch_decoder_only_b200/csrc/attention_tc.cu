// Flash attention on tcgen05 tensor cores (sm_100a), head size 64, causal
// with the block-diagonal mask of packed documents (query i sees keys j with
// dstart[i] <= j <= i).  Same layouts as the other attention kernels: qkv
// [B*T, 3C], out / dout [B*T, C], lse / D [B, H, T].
//
// One 192-thread CTA per tile, warp-specialised like the GEMM:
//   warp 0     TMA producer (128-row tiles of Q, K, V, dO; 128-byte swizzle)
//   warp 1     MMA issuer (one thread; tcgen05.mma kind::f16, M = 128)
//   warps 2-5  "softmax" warps: thread t owns accumulator row t (TMEM lane t);
//              they read scores from TMEM, form P (and dS), write them to
//              shared memory as the next MMA's operand, and run the epilogues.
//
// Forward (CTA = 128 queries): per 128-key block, S = Q K^T into one of two
// TMEM buffers (the next block's S is computed while this one is being
// exponentiated), P = exp2(S log2e / sqrt(d) - m) to shared memory,
// O_blk = P V into TMEM, accumulated in registers with the online-softmax
// correction.  Writes O and the row log-sum-exp.
//
// Backward (CTA = 128 keys; K, V resident): per 128-query block, S^T = K Q^T
// and dP^T = V dO^T into TMEM; P^T = exp2(S^T ... - lse), dS^T = P^T (dP^T - D)
// to shared memory; dV += P^T dO and dK += dS^T Q accumulate in TMEM across
// query blocks; dQ_blk = dS K goes to TMEM and is added into an fp32 dQ
// accumulator in global memory with one TMA bulk reduce-add per tile (no
// per-element atomics).  The same shared-memory tiles serve as K-major and
// MN-major operands (a 64-wide bf16 row is exactly one 128-byte swizzle atom).
// Key / query blocks outside the document ranges are skipped, not masked.
#include "tc_common.cuh"

#define AT_D 64
#define AT_BLK 128
#define AT_THREADS 192
#define AT_TILE_BYTES (AT_BLK * AT_D * 2)   // 16 KB: 128 rows x 128 B
#define LOG2E_F 1.4426950408889634f
#define LN2_F 0.6931471805599453f

__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return smem_desc(addr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, uint32_t lbo) { return smem_desc(addr, lbo, 1024); }

__device__ __forceinline__ uint32_t pk_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Row r of a [128 rows x 128 bf16] K-major operand stored as two 16 KB
// 128-byte-swizzled column blocks; write 32 values at columns c0..c0+31.
__device__ __forceinline__ void st_row32_bf16(uint32_t base, int r, int c0, const float* v) {
  const uint32_t blk = base + (c0 >> 6) * AT_TILE_BYTES + r * 128;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int u = ((c0 & 63) >> 3) + q;
    uint32_t a = blk + ((u ^ (r & 7)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk_bf16(v[8 * q], v[8 * q + 1])),
                 "r"(pk_bf16(v[8 * q + 2], v[8 * q + 3])), "r"(pk_bf16(v[8 * q + 4], v[8 * q + 5])),
                 "r"(pk_bf16(v[8 * q + 6], v[8 * q + 7]))
                 : "memory");
  }
}

// Bounded barrier among the 128 softmax threads (an mbarrier with count 128):
// every thread arrives, then waits for the phase to complete.
__device__ __forceinline__ bool group_sync(uint32_t bar, uint32_t& phase, volatile int* abort_flag) {
  mbar_arrive(bar);
  bool ok = mbar_wait(bar, phase, abort_flag);
  phase ^= 1;
  return ok;
}

__device__ __forceinline__ void trap_timeout(volatile int* abort_flag, unsigned* err) {
  *abort_flag = 1;
  atomicOr(err, GPT_DEVERR_TIMEOUT);
}

// ============================================================== forward
struct FwdSmem {
  static constexpr int Q = 0;                              // 16 KB
  static constexpr int KV = Q + AT_TILE_BYTES;             // 2 stages x (K, V)
  static constexpr int P = KV + 4 * AT_TILE_BYTES;         // 32 KB (two column blocks)
  static constexpr int BAR = P + 2 * AT_TILE_BYTES;
  static constexpr int TOTAL = BAR + 256;
};

__global__ void __launch_bounds__(AT_THREADS, 1)
attn_fwd_tc(const __grid_constant__ CUtensorMap tmQKV, bf16* __restrict__ out, float* __restrict__ lse,
            const int* __restrict__ dstart, int T, int H, unsigned* err) {
  extern __shared__ __align__(1024) uint8_t at_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)at_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + FwdSmem::BAR);
  // bars: 0 q_full, 1-2 kv_full, 3-4 kv_empty, 5-6 s_full, 7-8 s_free, 9 p_full, 10 o_full, 11 o_free, 12 drain
  uint32_t* tmem_slot = (uint32_t*)(bars + 13);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  int* s_info = (int*)(tmem_slot + 2);
  const uint32_t b0 = smem_u32(bars);
  auto bar = [&](int i) { return b0 + 8u * i; };
  const uint32_t sQ = smem_u32(sm + FwdSmem::Q), sKV = smem_u32(sm + FwdSmem::KV), sP = smem_u32(sm + FwdSmem::P);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + AT_BLK - 1) / AT_BLK;
  const int qb = nqb - 1 - blockIdx.x;   // heaviest query blocks first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * AT_D;
  const int q0 = qb * AT_BLK;
  const long rowbase = (long)b * T;
  const int* dsr = dstart + rowbase;

  if (threadIdx.x == 0) {
    mbar_init(bar(0), 1);
    for (int i = 1; i <= 2; ++i) mbar_init(bar(i), 1);
    for (int i = 3; i <= 4; ++i) mbar_init(bar(i), 1);
    for (int i = 5; i <= 6; ++i) mbar_init(bar(i), 1);
    for (int i = 7; i <= 8; ++i) mbar_init(bar(i), 4);
    mbar_init(bar(9), 4);
    mbar_init(bar(10), 1);
    mbar_init(bar(11), 4);
    mbar_init(bar(12), 1);
    *abort_flag = 0;
    const int kb_lo = dsr[q0] / AT_BLK, kb_hi = min(q0 + AT_BLK - 1, T - 1) / AT_BLK;
    s_info[0] = kb_lo;
    s_info[1] = kb_hi - kb_lo + 1;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int kb_lo = s_info[0], nj = s_info[1];
  // TMEM columns: S[0] 0..127, S[1] 128..255, O 256..319

  if (warp == 0 && lane == 0) {
    // ---------------- producer
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQKV)) : "memory");
    mbar_expect_tx(bar(0), AT_TILE_BYTES);
    tma_load_2d(sQ, &tmQKV, bar(0), h * AT_D, (int)(rowbase + q0));
    bool ok = true;
    for (int j = 0; j < nj && ok; ++j) {
      const int st = j & 1;
      if (!mbar_wait(bar(3 + st), ((j >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
      mbar_expect_tx(bar(1 + st), 2 * AT_TILE_BYTES);
      const int k0 = (kb_lo + j) * AT_BLK;
      const uint32_t dst = sKV + st * 2 * AT_TILE_BYTES;
      tma_load_2d(dst, &tmQKV, bar(1 + st), C + h * AT_D, (int)(rowbase + k0));
      tma_load_2d(dst + AT_TILE_BYTES, &tmQKV, bar(1 + st), 2 * C + h * AT_D, (int)(rowbase + k0));
    }
    if (!ok) trap_timeout(abort_flag, err);
    volatile int never = 0;
    mbar_wait(bar(0), 0, &never, 1ll << 28);
    for (int j = max(0, nj - 2); j < nj; ++j) mbar_wait(bar(1 + (j & 1)), (j >> 1) & 1, &never, 1ll << 28);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t ID_S = instr_desc(128, false, false);   // S = Q K^T: 128 x 128, K = 64
    constexpr uint32_t ID_O = instr_desc(64, false, true);     // O = P V: 128 x 64, K = 128 (V MN-major)
    bool ok = mbar_wait(bar(0), 0, abort_flag);
    auto issue_s = [&](int j) -> bool {
      const int st = j & 1;
      if (!mbar_wait(bar(1 + st), (j >> 1) & 1, abort_flag)) return false;
      if (!mbar_wait(bar(7 + st), ((j >> 1) & 1) ^ 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t sK = sKV + st * 2 * AT_TILE_BYTES;
#pragma unroll
      for (int k = 0; k < AT_D / 16; ++k) umma_bf16(tmem + st * 128, kdesc(sQ + k * 32), kdesc(sK + k * 32), ID_S, k > 0);
      umma_commit(bar(5 + st));
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int j = 0; j < nj && ok; ++j) {
      if (j + 1 < nj && !issue_s(j + 1)) { ok = false; break; }
      if (!mbar_wait(bar(9), j & 1, abort_flag)) { ok = false; break; }
      if (!mbar_wait(bar(11), (j & 1) ^ 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sV = sKV + (j & 1) * 2 * AT_TILE_BYTES + AT_TILE_BYTES;
#pragma unroll
      for (int kk = 0; kk < AT_BLK / 16; ++kk) {
        const uint32_t pa = sP + (kk >> 2) * AT_TILE_BYTES + (kk & 3) * 32;
        umma_bf16(tmem + 256, kdesc(pa), mndesc(sV + kk * 2048, 8192), ID_O, kk > 0);
      }
      umma_commit(bar(10));
      umma_commit(bar(3 + (j & 1)));
    }
    if (!ok) trap_timeout(abort_flag, err);
    umma_commit(bar(12));
    volatile int never = 0;
    mbar_wait(bar(12), 0, &never, 1ll << 28);
  } else if (warp >= 2) {
    // ---------------- softmax warps: thread owns query row r
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int q = q0 + r;
    const bool qv = q < T;
    const int ds_q = qv ? dsr[q] : 0;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = 0.125f * LOG2E_F;   // 1/sqrt(64) in the exp2 domain
    float m = -INFINITY, l = 0.f;
    float o[AT_D];
#pragma unroll
    for (int i = 0; i < AT_D; ++i) o[i] = 0.f;
    for (int j = 0; j < nj; ++j) {
      const int st = j & 1;
      const int k0 = (kb_lo + j) * AT_BLK;
      if (!mbar_wait(bar(5 + st), (j >> 1) & 1, abort_flag)) { trap_timeout(abort_flag, err); break; }
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + st * 128;
      // pass 1: masked row maximum
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < AT_BLK; c += 32) {
        uint32_t rr[32];
        tmem_ld32(tS + c, rr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int k = k0 + c + i;
          if (k <= q && k >= ds_q) mx = fmaxf(mx, __uint_as_float(rr[i]) * sl2);
        }
      }
      const float mn = fmaxf(m, mx);
      const float mu = mn == -INFINITY ? 0.f : mn;
      const float corr = exp2f(m - mu);
      // pass 2: P = exp2(s - m) to shared memory (the previous P was consumed: o_full seen)
      float ps = 0.f;
#pragma unroll 1
      for (int c = 0; c < AT_BLK; c += 32) {
        uint32_t rr[32];
        tmem_ld32(tS + c, rr);
        tmem_wait_ld();
        float p[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int k = k0 + c + i;
          p[i] = (k <= q && k >= ds_q) ? exp2f(__uint_as_float(rr[i]) * sl2 - mu) : 0.f;
          ps += p[i];
        }
        st_row32_bf16(sP, r, c, p);
      }
      tc_fence_before();
      fence_async_smem();
      __syncwarp();
      if (lane == 0) { mbar_arrive(bar(7 + st)); mbar_arrive(bar(9)); }
      l = l * corr + ps;
      m = mn;
      // O_blk = P V
      if (!mbar_wait(bar(10), j & 1, abort_flag)) { trap_timeout(abort_flag, err); break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < AT_D; c += 32) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_off + 256 + c, rr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[c + i] = o[c + i] * corr + __uint_as_float(rr[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(11));
    }
    if (qv) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16* orow = out + (rowbase + q) * C + h * AT_D;
#pragma unroll
      for (int c = 0; c < AT_D; c += 8) {
        uint4 w;
        w.x = pk_bf16(o[c] * inv, o[c + 1] * inv);
        w.y = pk_bf16(o[c + 2] * inv, o[c + 3] * inv);
        w.z = pk_bf16(o[c + 4] * inv, o[c + 5] * inv);
        w.w = pk_bf16(o[c + 6] * inv, o[c + 7] * inv);
        *reinterpret_cast<uint4*>(orow + c) = w;
      }
      lse[(long)bh * T + q] = (m + log2f(l)) * LN2_F;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
}

// ============================================================== backward
struct BwdSmem {
  static constexpr int K = 0;                               // 16 KB
  static constexpr int V = K + AT_TILE_BYTES;               // 16 KB
  static constexpr int QD = V + AT_TILE_BYTES;              // 2 stages x (Q, dO)
  static constexpr int PT = QD + 4 * AT_TILE_BYTES;         // 32 KB
  static constexpr int DST = PT + 2 * AT_TILE_BYTES;        // 32 KB
  static constexpr int DQ = DST + 2 * AT_TILE_BYTES;        // 32 KB fp32 staging (two 32-column boxes)
  static constexpr int AUX = DQ + 2 * AT_TILE_BYTES;        // 2 x (lse2, D, dstart) x 128
  static constexpr int BAR = AUX + 2 * 3 * AT_BLK * 4;
  static constexpr int TOTAL = BAR + 256;
};

__global__ void __launch_bounds__(AT_THREADS, 1)
attn_bwd_tc(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
            const __grid_constant__ CUtensorMap tmDQ, const float* __restrict__ lse, const float* __restrict__ Dbuf,
            const int* __restrict__ dstart, bf16* __restrict__ dqkv, int T, int H, unsigned* err) {
  extern __shared__ __align__(1024) uint8_t at_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)at_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + BwdSmem::BAR);
  // bars: 0 kv_full, 1-2 q_full, 3-4 q_empty, 5 s_full, 6 p_full, 7 dq_full, 8 tm_free, 9 drain,
  //       10 softmax-group barrier
  uint32_t* tmem_slot = (uint32_t*)(bars + 11);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  int* s_info = (int*)(tmem_slot + 2);
  const uint32_t b0 = smem_u32(bars);
  auto bar = [&](int i) { return b0 + 8u * i; };
  const uint32_t sK = smem_u32(sm + BwdSmem::K), sV = smem_u32(sm + BwdSmem::V), sQD = smem_u32(sm + BwdSmem::QD);
  const uint32_t sPT = smem_u32(sm + BwdSmem::PT), sDST = smem_u32(sm + BwdSmem::DST), sDQ = smem_u32(sm + BwdSmem::DQ);
  float* aux = (float*)(sm + BwdSmem::AUX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x;   // earliest key blocks see the most queries: launched first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * AT_D;
  const int k0 = kb * AT_BLK;
  const long rowbase = (long)b * T;
  const int* dsr = dstart + rowbase;
  const int nqb = (T + AT_BLK - 1) / AT_BLK;

  if (threadIdx.x == 0) {
    mbar_init(bar(0), 1);
    for (int i = 1; i <= 4; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(5), 1);
    mbar_init(bar(6), 4);
    mbar_init(bar(7), 1);
    mbar_init(bar(8), 4);
    mbar_init(bar(9), 1);
    mbar_init(bar(10), 128);
    *abort_flag = 0;
    const int last_key = min(k0 + AT_BLK - 1, T - 1);
    int n = 0;
    for (int qb = kb; qb < nqb; ++qb) {
      if (dsr[qb * AT_BLK] > last_key) break;   // every later query lives in a later document
      ++n;
    }
    s_info[0] = n;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int niter = s_info[0];
  // TMEM columns: S^T 0..127, dP^T 128..255, dV 256..319, dK 320..383, dQ 384..447

  if (warp == 0 && lane == 0) {
    // ---------------- producer
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQKV)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmDO)) : "memory");
    mbar_expect_tx(bar(0), 2 * AT_TILE_BYTES);
    tma_load_2d(sK, &tmQKV, bar(0), C + h * AT_D, (int)(rowbase + k0));
    tma_load_2d(sV, &tmQKV, bar(0), 2 * C + h * AT_D, (int)(rowbase + k0));
    bool ok = true;
    for (int i = 0; i < niter && ok; ++i) {
      const int st = i & 1;
      if (!mbar_wait(bar(3 + st), ((i >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
      mbar_expect_tx(bar(1 + st), 2 * AT_TILE_BYTES);
      const int q0 = (kb + i) * AT_BLK;
      const uint32_t dst = sQD + st * 2 * AT_TILE_BYTES;
      tma_load_2d(dst, &tmQKV, bar(1 + st), h * AT_D, (int)(rowbase + q0));
      tma_load_2d(dst + AT_TILE_BYTES, &tmDO, bar(1 + st), h * AT_D, (int)(rowbase + q0));
    }
    if (!ok) trap_timeout(abort_flag, err);
    volatile int never = 0;
    mbar_wait(bar(0), 0, &never, 1ll << 28);
    for (int i = max(0, niter - 2); i < niter; ++i) mbar_wait(bar(1 + (i & 1)), (i >> 1) & 1, &never, 1ll << 28);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t ID_SS = instr_desc(128, false, false);   // S^T, dP^T: 128 keys x 128 queries, K = d
    constexpr uint32_t ID_KV = instr_desc(64, false, true);     // dV, dK: 128 keys x 64, K = queries
    constexpr uint32_t ID_Q = instr_desc(64, true, true);       // dQ: 128 queries x 64, K = keys
    bool ok = mbar_wait(bar(0), 0, abort_flag);
    for (int i = 0; i < niter && ok; ++i) {
      const int st = i & 1;
      if (!mbar_wait(bar(1 + st), (i >> 1) & 1, abort_flag)) { ok = false; break; }
      if (!mbar_wait(bar(8), (i & 1) ^ 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sQ = sQD + st * 2 * AT_TILE_BYTES, sDO = sQ + AT_TILE_BYTES;
#pragma unroll
      for (int k = 0; k < AT_D / 16; ++k) {
        umma_bf16(tmem + 0, kdesc(sK + k * 32), kdesc(sQ + k * 32), ID_SS, k > 0);
        umma_bf16(tmem + 128, kdesc(sV + k * 32), kdesc(sDO + k * 32), ID_SS, k > 0);
      }
      umma_commit(bar(5));
      if (!mbar_wait(bar(6), i & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < AT_BLK / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * AT_TILE_BYTES + (kk & 3) * 32;
        umma_bf16(tmem + 256, kdesc(sPT + koff), mndesc(sDO + kk * 2048, 8192), ID_KV, (i > 0 || kk > 0));
        umma_bf16(tmem + 320, kdesc(sDST + koff), mndesc(sQ + kk * 2048, 8192), ID_KV, (i > 0 || kk > 0));
      }
#pragma unroll
      for (int kk = 0; kk < AT_BLK / 16; ++kk)
        umma_bf16(tmem + 384, mndesc(sDST + kk * 2048, AT_TILE_BYTES), mndesc(sK + kk * 2048, 8192), ID_Q, kk > 0);
      umma_commit(bar(3 + st));
      umma_commit(bar(7));
    }
    if (!ok) trap_timeout(abort_flag, err);
    umma_commit(bar(9));
    volatile int never = 0;
    mbar_wait(bar(9), 0, &never, 1ll << 28);
  } else if (warp >= 2) {
    // ---------------- softmax warps: thread owns key row r (S^T, dP^T, dK, dV) and query row r (dQ)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int k = k0 + r;
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = 0.125f * LOG2E_F;
    bool ok = true;
    uint32_t gph = 0;
    for (int i = 0; i < niter; ++i) {
      const int q0 = (kb + i) * AT_BLK;
      float* L2 = aux + (i & 1) * 3 * AT_BLK;
      float* Dq = L2 + AT_BLK;
      int* DSq = reinterpret_cast<int*>(Dq + AT_BLK);
      {
        const int qq = q0 + tid;
        const bool v = qq < T;
        L2[tid] = v ? lse[(long)bh * T + qq] * LOG2E_F : 0.f;
        Dq[tid] = v ? Dbuf[(long)bh * T + qq] : 0.f;
        DSq[tid] = v ? dsr[qq] : 0x7fffffff;
      }
      if (!group_sync(bar(10), gph, abort_flag)) { ok = false; break; }
      if (!mbar_wait(bar(5), i & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < AT_BLK; c += 32) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tmem + lane_off + c, sr);
        tmem_ld32(tmem + lane_off + 128 + c, dr);
        tmem_wait_ld();
        float p[32], ds[32];
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int ql = c + jj, qq = q0 + ql;
          const bool allowed = qq < T && qq >= k && DSq[ql] <= k;
          const float pv = allowed ? exp2f(__uint_as_float(sr[jj]) * sl2 - L2[ql]) : 0.f;
          p[jj] = pv;
          ds[jj] = pv * (__uint_as_float(dr[jj]) - Dq[ql]);
        }
        st_row32_bf16(sPT, r, c, p);
        st_row32_bf16(sDST, r, c, ds);
      }
      tc_fence_before();
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(6));
      // dQ block (row r = query q0 + r): stage and add into the fp32 accumulator
      if (!mbar_wait(bar(7), i & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t qa[32], qb2[32];
      tmem_ld32(tmem + lane_off + 384, qa);
      tmem_ld32(tmem + lane_off + 416, qb2);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(8));   // S^T / dP^T / dQ tensor memory free
      if (tid == 0) bulk_wait_read<0>();    // the previous reduce has read the staging buffer
      if (!group_sync(bar(10), gph, abort_flag)) { ok = false; break; }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t* src = half ? qb2 : qa;
        const uint32_t boxb = sDQ + half * AT_TILE_BYTES + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t a = boxb + ((u ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(src[4 * u]), "r"(src[4 * u + 1]),
                       "r"(src[4 * u + 2]), "r"(src[4 * u + 3])
                       : "memory");
        }
      }
      fence_async_smem();
      if (!group_sync(bar(10), gph, abort_flag)) { ok = false; break; }
      if (tid == 0) {
        tma_reduce_add_2d(&tmDQ, sDQ, h * AT_D, (int)(rowbase + q0));
        tma_reduce_add_2d(&tmDQ, sDQ + AT_TILE_BYTES, h * AT_D + 32, (int)(rowbase + q0));
        bulk_commit();
      }
    }
    if (!ok) trap_timeout(abort_flag, err);
    if (ok && niter > 0) {
      // dK (scaled by 1/sqrt(d)) and dV rows, accumulated over all query blocks;
      // the tensor-memory loads are warp-collective, only the stores depend on k < T
      tc_fence_after();
      bf16* row = dqkv + (rowbase + k) * 3 * C;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const float sc = part == 0 ? 0.125f : 1.f;
        bf16* dst = row + (part == 0 ? C : 2 * C) + h * AT_D;
#pragma unroll
        for (int c = 0; c < AT_D; c += 32) {
          uint32_t rr[32];
          tmem_ld32(tmem + lane_off + (part == 0 ? 320 : 256) + c, rr);
          tmem_wait_ld();
          if (k < T) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 w;
              w.x = pk_bf16(__uint_as_float(rr[8 * u]) * sc, __uint_as_float(rr[8 * u + 1]) * sc);
              w.y = pk_bf16(__uint_as_float(rr[8 * u + 2]) * sc, __uint_as_float(rr[8 * u + 3]) * sc);
              w.z = pk_bf16(__uint_as_float(rr[8 * u + 4]) * sc, __uint_as_float(rr[8 * u + 5]) * sc);
              w.w = pk_bf16(__uint_as_float(rr[8 * u + 6]) * sc, __uint_as_float(rr[8 * u + 7]) * sc);
              *reinterpret_cast<uint4*>(dst + c + 8 * u) = w;
            }
          }
        }
      }
    }
    if (tid == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
}

// D[b, h, t] = dO[b*T+t, head h] . O[b*T+t, head h]   (one thread per (row, head))
__global__ void attn_rowdot_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout, float* __restrict__ Dbuf,
                                   int B, int T, int H) {
  long i = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (i >= (long)B * T * H) return;
  const int h = i % H;
  const long row = i / H;
  const int t = row % T, b = row / T;
  const long off = row * H * AT_D + h * AT_D;
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < AT_D; c += 8) {
    float x[8], y[8];
    Vec<bf16>::load(dout + off + c, x);
    Vec<bf16>::load(out + off + c, y);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc += x[k] * y[k];
  }
  Dbuf[((long)b * H + h) * T + t] = acc;
}

// dqkv[:, q part] = bf16(dQacc * 1/sqrt(d))
__global__ void dq_convert_kernel(const float* __restrict__ acc, bf16* __restrict__ dqkv, long rows, int C) {
  const long n8 = rows * C / 8;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n8; i += (long)gridDim.x * blockDim.x) {
    const long e = i * 8, row = e / C;
    const int c = e % C;
    float v[8];
    Vec<float>::load(acc + e, v);
    Vec<float>::load(acc + e + 4, v + 4);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] *= 0.125f;
    Vec<bf16>::store(dqkv + row * 3 * C + c, v);
  }
}

// ============================================================== launchers
bool attn_tc_supported(int d) { return d == AT_D && get_encode() != nullptr; }

cudaError_t launch_attn_fwd_tc(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T, int H,
                               unsigned* err, cudaStream_t s) {
  const int C = H * AT_D;
  CUtensorMap tm;
  if (!make_map_ex(&tm, MapKey{qkv, (long)B * T, 3L * C, 3L * C, 1, 0, AT_D, AT_BLK, 0, 128}))
    return cudaErrorInvalidValue;
  // more than half the shared memory: one CTA per SM, as each holds all 512 TMEM columns
  const int smem = FwdSmem::TOTAL + 1024 > 120 * 1024 ? FwdSmem::TOTAL + 1024 : 120 * 1024;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid((T + AT_BLK - 1) / AT_BLK, B * H);
  ++g_kernel_launches;
  attn_fwd_tc<<<grid, AT_THREADS, smem, s>>>(tm, out, lse, dstart, T, H, err);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dbuf,
                               float* dq_acc, const int* dstart, bf16* dqkv, int B, int T, int H, unsigned* err,
                               cudaStream_t s) {
  const int C = H * AT_D;
  const long rows = (long)B * T;
  CUtensorMap tq, tdo, tdq;
  if (!make_map_ex(&tq, MapKey{qkv, rows, 3L * C, 3L * C, 1, 0, AT_D, AT_BLK, 0, 128}) ||
      !make_map_ex(&tdo, MapKey{dout, rows, (long)C, (long)C, 1, 0, AT_D, AT_BLK, 0, 128}) ||
      !make_map_ex(&tdq, MapKey{dq_acc, rows, (long)C, (long)C, 1, 0, 32, AT_BLK, 1, 128}))
    return cudaErrorInvalidValue;
  const int smem = BwdSmem::TOTAL + 1024;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaError_t e = cudaMemsetAsync(dq_acc, 0, rows * C * sizeof(float), s);
  if (e != cudaSuccess) return e;
  long n = rows * H;
  ++g_kernel_launches;
  attn_rowdot_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(out, dout, Dbuf, B, T, H);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 grid((T + AT_BLK - 1) / AT_BLK, B * H);
  ++g_kernel_launches;
  attn_bwd_tc<<<grid, AT_THREADS, smem, s>>>(tq, tdo, tdq, lse, Dbuf, dstart, dqkv, T, H, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ++g_kernel_launches;
  dq_convert_kernel<<<148 * 4, 256, 0, s>>>(dq_acc, dqkv, rows, C);
  return cudaGetLastError();
}
