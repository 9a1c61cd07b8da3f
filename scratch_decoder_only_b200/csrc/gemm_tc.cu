// tcgen05 GEMM for sm_100a: C[M,N] = A(M x K) . B(N x K)^T, bf16 operands,
// fp32 accumulation in tensor memory, fused epilogues (bias, residual, GELU,
// GELU', fp32 / split-K fp32 outputs).  Every dense contraction of the
// training step runs here: the QKV, attention-out, MLP and LM-head
// projections forward (A and B K-major), their input gradients (B MN-major:
// the weight read transposed in place) and their weight gradients (A and B
// MN-major: both activations read transposed in place), so no transposed
// copy of any tensor is ever written.
//
// Structure (one 192-thread CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: 2-D tiled loads (128-byte swizzle) of A and B
//               k-blocks into a ring of shared-memory stages, completion
//               signalled on "full" mbarriers; also allocates tensor memory.
//   warp 1      MMA issuer: one thread issues tcgen05.mma (kind::f16,
//               M = 128, N = BN, K = 16) into a TMEM accumulator, and
//               tcgen05.commit frees each stage ("empty") and hands a finished
//               accumulator to the epilogue ("tfull").
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (one row per thread),
//               epilogue arithmetic, 16-byte global stores; "tempty" returns
//               the accumulator.  Two accumulators (2 x BN columns) let the
//               epilogue of one tile overlap the MMAs of the next.
// TMA loads never use cluster multicast.  Every mbarrier wait is bounded:
// on timeout the kernel records GPT_DEVERR_TIMEOUT, drains what it started,
// frees its tensor memory and returns.
#include <cuda.h>
#include <map>
#include <mutex>
#include <tuple>
#include "launch.h"

#define TC_BM 128
#define TC_BK 64
#define TC_THREADS 192
#define TC_TIMEOUT_CYCLES (4ll << 30)

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok;
}
// Bounded wait for the phase with the given parity; false on timeout / abort.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          long long limit = TC_TIMEOUT_CYCLES) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) return false;
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t gets lane (base + t),
// columns c..c+31.  No wait: pair with tmem_wait_ld().
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// TMA bulk-tensor store of a shared-memory box, tracked in the bulk async-group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y), "r"(z) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Hardware tanh (MUFU), relative error ~2^-11: below the bf16 rounding the
// epilogue applies to its outputs.
__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float gelu_fast(float u) {
  return 0.5f * u * (1.0f + tanh_fast(GELU_K * (u + GELU_C * u * u * u)));
}
__device__ __forceinline__ float gelu_grad_fast(float u) {
  float t = tanh_fast(GELU_K * (u + GELU_C * u * u * u));
  return 0.5f * (1.0f + t) + 0.5f * u * (1.0f - t * t) * GELU_K * (1.0f + 3.0f * GELU_C * u * u);
}

// Shared-memory matrix descriptor (tcgen05), 128-byte swizzle, version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Instruction descriptor: D fp32, A/B bf16, majorness, N >> 3, M >> 4.
__host__ __device__ constexpr uint32_t instr_desc(int bn, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(TC_BM >> 4) << 24);
}

// ------------------------------------------------------------------ epilogue
// Each epilogue warp owns 32 accumulator rows; it walks the tile in 32-column
// chunks: TMEM -> registers -> epilogue arithmetic -> a 32 x 32 box in its
// shared-memory staging buffer (swizzled like the TMA box) -> TMA store.
// Two staging buffers per output alternate so a store can drain while the
// next chunk is computed.
#define EPI_WARP_BYTES 8192   // per epilogue warp: 2 buffers x 4 KB

// Write 32 values of row r into a 32 x 32 bf16 box (64-byte rows, 64-byte swizzle).
__device__ __forceinline__ void stage_bf16(uint32_t buf, int r, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    uint32_t a = buf + r * 64 + ((q ^ ((r >> 1) & 3)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w)
                 : "memory");
  }
}
// Write 32 fp32 values of row r into a 32 x 32 fp32 box (128-byte rows, 128-byte swizzle).
__device__ __forceinline__ void stage_f32(uint32_t buf, int r, const float* v) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t a = buf + r * 128 + ((q ^ (r & 7)) << 4);
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v[4 * q]), "f"(v[4 * q + 1]),
                 "f"(v[4 * q + 2]), "f"(v[4 * q + 3])
                 : "memory");
  }
}

// 32 consecutive bf16 of one row into registers (16-byte loads), zero past N.
__device__ __forceinline__ void ld_row32(const bf16* src, int nvalid, uint4* raw) {
  if (nvalid >= 32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) raw[q] = *reinterpret_cast<const uint4*>(src + 8 * q);
  } else {
    bf16* h = reinterpret_cast<bf16*>(raw);
    for (int j = 0; j < 32; ++j) h[j] = j < nvalid ? src[j] : __float2bfloat16_rn(0.f);
  }
}
__device__ __forceinline__ float4 load_bias4(const float* bias, int c, int N) {
  if (c + 3 < N) return *reinterpret_cast<const float4*>(bias + c);
  float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
  if (c < N) b.x = bias[c];
  if (c + 1 < N) b.y = bias[c + 1];
  if (c + 2 < N) b.z = bias[c + 2];
  return b;
}
__device__ __forceinline__ void unpack_row32(const uint4* raw, float* x) {
#pragma unroll
  for (int q = 0; q < 4; ++q) Vec<bf16>::load(reinterpret_cast<const bf16*>(raw + q), x + 8 * q);
}

// ------------------------------------------------------------------ the kernel
template <int BN>
struct TcCfg {
  static constexpr int STAGES = BN >= 256 ? 4 : 6;
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 4 * EPI_WARP_BYTES + 256;
};

template <int BN, bool A_MN, bool B_MN, int KIND>
__global__ void __launch_bounds__(TC_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2, int M, int N,
               int K, int splits, EpiParams<bf16> epi, unsigned* err) {
  using Cfg = TcCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* tile_mem = smem;
  uint8_t* epi_mem = smem + STAGES * Cfg::STAGE_BYTES;   // 4 warps x EPI_WARP_BYTES, 1024-aligned
  uint64_t* bars = (uint64_t*)(epi_mem + 4 * EPI_WARP_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * STAGES + 5);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull_bar(a), 1); mbar_init(tempty_bar(a), 4); }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(Cfg::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int tiles_m = (M + TC_BM - 1) / TC_BM, tiles_n = (N + BN - 1) / BN;
  const int tiles = tiles_m * tiles_n;
  const int units = tiles * splits;
  const int kb_total = (K + TC_BK - 1) / TC_BK;
  const int kbs = (kb_total + splits - 1) / splits;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int split = u / tiles, t = u % tiles;
      const int m0 = (t % tiles_m) * TC_BM, n0 = (t / tiles_m) * BN;
      const int kb0 = split * kbs, kb1 = min(kb_total, kb0 + kbs);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1, abort_flag)) { ok = false; break; }
        const uint32_t fb = full_bar(stage);
        mbar_expect_tx(fb, Cfg::STAGE_BYTES);
        const uint32_t sa = smem_u32(tile_mem + stage * Cfg::STAGE_BYTES);
        const uint32_t sb = sa + Cfg::A_BYTES;
        const int k0 = kb * TC_BK;
        if (!A_MN) {
          tma_load_2d(sa, &tmA, fb, k0, m0);
        } else {
#pragma unroll
          for (int j = 0; j < TC_BM / 64; ++j) tma_load_2d(sa + j * 64 * TC_BK * 2, &tmA, fb, m0 + 64 * j, k0);
        }
        if (!B_MN) {
          tma_load_2d(sb, &tmB, fb, k0, n0);
        } else {
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) tma_load_2d(sb + j * 64 * TC_BK * 2, &tmB, fb, n0 + 64 * j, k0);
        }
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      atomicOr(err, GPT_DEVERR_TIMEOUT);
    }
    // drain: wait (bounded) for the most recent loads of every stage to land
    long nd = issued < STAGES ? issued : STAGES;
    int s = stage;
    uint32_t ph = phase;
    for (long i = 0; i < nd; ++i) {
      if (--s < 0) { s = STAGES - 1; ph ^= 1; }
      volatile int never = 0;
      mbar_wait(full_bar(s), ph, &never, 1ll << 28);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t IDESC = instr_desc(BN, A_MN, B_MN);
    // K-major: SBO = 8 rows x 128 B; k step (16 elements) = 32 B inside the swizzle row.
    // MN-major: LBO = one 64-element box (64 k-rows x 128 B), SBO = 8 k-rows x 128 B; k step = 16 rows.
    constexpr uint32_t A_LBO = A_MN ? 64 * TC_BK * 2 : 16, A_SBO = 1024, A_KSTEP = A_MN ? 16 * 128 : 32;
    constexpr uint32_t B_LBO = B_MN ? 64 * TC_BK * 2 : 16, B_SBO = 1024, B_KSTEP = B_MN ? 16 * 128 : 32;
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int split = u / tiles;
      const int kb0 = split * kbs, kb1 = min(kb_total, kb0 + kbs);
      if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tmem_d = tmem_base + (uint32_t)(acc * BN);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(tile_mem + stage * Cfg::STAGE_BYTES);
        const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
        for (int k = 0; k < TC_BK / 16; ++k) {
          uint64_t ad = smem_desc(sa + k * A_KSTEP, A_LBO, A_SBO);
          uint64_t bd = smem_desc(sb + k * B_KSTEP, B_LBO, B_SBO);
          umma_bf16(tmem_d, ad, bd, IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
        }
        umma_commit(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      umma_commit(tfull_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (!ok) {
      *abort_flag = 1;
      atomicOr(err, GPT_DEVERR_TIMEOUT);
    }
    // drain: all MMAs this thread issued have completed once this commit arrives
    umma_commit(drain_bar);
    volatile int never = 0;
    mbar_wait(drain_bar, 0, &never, 1ll << 28);
  } else if (warp >= 2) {
    // ---------------- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31
    const int quarter = warp & 3;
    const uint32_t sbuf = smem_u32(epi_mem + (warp - 2) * EPI_WARP_BYTES);
    constexpr bool F32OUT = (KIND == EPI_F32 || KIND == EPI_F32_SPLIT);
    constexpr uint32_t BOX_BYTES = F32OUT ? 4096 : 2048;   // one 32 x 32 box
    int acc = 0;
    uint32_t acc_phase = 0;
    int nbuf = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const int split = u / tiles, t = u % tiles;
      const int m0 = (t % tiles_m) * TC_BM, n0 = (t / tiles_m) * BN;
      const int rbase = m0 + quarter * 32;
      const int row = rbase + lane;
      const bool row_ok = row < M;
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
        *abort_flag = 1;
        atomicOr(err, GPT_DEVERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      // residual (STORE) or pre-activation (DGELU) row chunks, prefetched one chunk ahead
      const bf16* side = nullptr;
      long side_ld = 0;
      if (KIND == EPI_STORE && epi.resid) { side = epi.resid; side_ld = epi.ld_resid; }
      if (KIND == EPI_DGELU) { side = epi.aux; side_ld = epi.ld_aux; }
      uint4 nxt[4];
      if (side && row_ok) ld_row32(side + (long)row * side_ld + n0, N - n0, nxt);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        const int col0 = n0 + c;
        if (col0 >= N) break;
        uint32_t r[32];
        tmem_ld32(tbase + c, r);
        uint4 cur[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) cur[q] = nxt[q];
        if (side && row_ok && c + 32 < BN && col0 + 32 < N)
          ld_row32(side + (long)row * side_ld + col0 + 32, N - col0 - 32, nxt);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        // wait until the store that last used this staging buffer has read it
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        const uint32_t b0 = sbuf + nbuf * BOX_BYTES;
        if constexpr (KIND == EPI_STORE) {
          if (epi.bias) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float4 bb = load_bias4(epi.bias, col0 + 4 * q, N);
              v[4 * q] += bb.x; v[4 * q + 1] += bb.y; v[4 * q + 2] += bb.z; v[4 * q + 3] += bb.w;
            }
          }
          if (side) {
            float rr[32];
            unpack_row32(cur, rr);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += rr[j];
          }
          stage_bf16(b0, lane, v);
        } else if constexpr (KIND == EPI_GELU) {
          float a[32];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float4 bb = load_bias4(epi.bias, col0 + 4 * q, N);
            v[4 * q] += bb.x; v[4 * q + 1] += bb.y; v[4 * q + 2] += bb.z; v[4 * q + 3] += bb.w;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float uq = __bfloat162float(__float2bfloat16_rn(v[j]));
            v[j] = uq;
            a[j] = gelu_fast(uq);
          }
          stage_bf16(b0, lane, v);
          stage_bf16(b0 + 2 * BOX_BYTES, lane, a);
        } else if constexpr (KIND == EPI_DGELU) {
          float uu[32];
          unpack_row32(cur, uu);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= gelu_grad_fast(uu[j]);
          stage_bf16(b0, lane, v);
        } else {
          stage_f32(b0, lane, v);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (KIND == EPI_F32_SPLIT) {
            tma_store_3d(&tmC, b0, col0, rbase, split);
          } else {
            tma_store_2d(&tmC, b0, col0, rbase);
            if constexpr (KIND == EPI_GELU) tma_store_2d(&tmC2, b0 + 2 * BOX_BYTES, col0, rbase);
          }
          bulk_commit();
        }
        nbuf ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Cfg::TMEM_COLS));
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
    cudaGetLastError();
  });
  return fn;
}

// Tensor map of a row-major [depth][rows][cols] array (depth 1 = 2-D) with
// row stride ld elements and `depth_stride` elements between slabs.
struct MapKey {
  const void* base; long rows, cols, ld, depth, depth_stride; int box_cols, box_rows, f32, swz;
  bool operator<(const MapKey& o) const {
    return std::tie(base, rows, cols, ld, depth, depth_stride, box_cols, box_rows, f32, swz) <
           std::tie(o.base, o.rows, o.cols, o.ld, o.depth, o.depth_stride, o.box_cols, o.box_rows, o.f32, o.swz);
  }
};
static bool make_map_ex(CUtensorMap* map, const MapKey& k) {
  static std::mutex mu;
  static std::map<MapKey, CUtensorMap> cache;
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(k);
  if (it != cache.end()) { *map = it->second; return true; }
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const int es = k.f32 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)k.cols, (cuuint64_t)k.rows, (cuuint64_t)k.depth};
  cuuint64_t strides[2] = {(cuuint64_t)k.ld * es, (cuuint64_t)k.depth_stride * es};
  cuuint32_t box[3] = {(cuuint32_t)k.box_cols, (cuuint32_t)k.box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMapSwizzle swz = k.swz == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                           : k.swz == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = enc(map, k.f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   k.depth > 1 ? 3 : 2, const_cast<void*>(k.base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  if (cache.size() > 4096) cache.clear();
  cache[k] = *map;
  return true;
}
// 2-D bf16 operand [rows][cols], row stride ld; box = box_cols x box_rows, 128-byte swizzle.
static bool make_map(CUtensorMap* map, const void* base, long rows, long cols, long ld, int box_cols, int box_rows) {
  return make_map_ex(map, MapKey{base, rows, cols, ld, 1, 0, box_cols, box_rows, 0, 128});
}

bool gemm_tc_supported(int M, int N, int K, long lda, bool a_t, long ldb, bool b_t) {
  // operands and outputs move by TMA: 16-byte row strides
  if (M < 1 || N < 1 || K < 1) return false;
  if ((lda & 7) || (ldb & 7)) return false;   // 16-byte row strides for TMA
  (void)a_t; (void)b_t;
  return get_encode() != nullptr;
}

static int g_sms = 0;

template <int BN, bool A_MN, bool B_MN, int KIND>
static cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                             const CUtensorMap& tc2, int M, int N, int K, int splits, const EpiParams<bf16>& epi,
                             unsigned* err, cudaStream_t s) {
  using Cfg = TcCfg<BN>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, A_MN, B_MN, KIND>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  int units = ((M + TC_BM - 1) / TC_BM) * ((N + BN - 1) / BN) * splits;
  int grid = units < g_sms ? units : g_sms;
  ++g_kernel_launches;
  gemm_tc_kernel<BN, A_MN, B_MN, KIND><<<grid, TC_THREADS, Cfg::SMEM, s>>>(ta, tb, tc, tc2, M, N, K, splits, epi,
                                                                          err);
  return cudaGetLastError();
}

// The (layout, epilogue) combinations the training step and the stand-alone
// GEMM use; any other returns cudaErrorNotSupported.
template <int BN, bool A_MN, bool B_MN>
static cudaError_t launch_kind(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                               const CUtensorMap& tc2, int M, int N, int K, int splits, const EpiParams<bf16>& epi,
                               unsigned* err, cudaStream_t s) {
  if (epi.kind == EPI_F32) return launch_tc<BN, A_MN, B_MN, EPI_F32>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  if constexpr (!A_MN) {
    if (epi.kind == EPI_STORE) return launch_tc<BN, A_MN, B_MN, EPI_STORE>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    if constexpr (!B_MN) {
      if (epi.kind == EPI_GELU) return launch_tc<BN, A_MN, B_MN, EPI_GELU>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    } else {
      if (epi.kind == EPI_DGELU) return launch_tc<BN, A_MN, B_MN, EPI_DGELU>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    }
  } else if constexpr (B_MN) {
    if (epi.kind == EPI_F32_SPLIT)
      return launch_tc<BN, A_MN, B_MN, EPI_F32_SPLIT>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  }
  return cudaErrorNotSupported;
}

template <int BN>
static cudaError_t launch_bn(int M, int N, int K, const bf16* A, long lda, bool a_t, const bf16* B, long ldb,
                             bool b_t, const EpiParams<bf16>& epi, int splits, unsigned* err, cudaStream_t s) {
  CUtensorMap ta, tb, tc, tc2;
  bool ok;
  // A: K-major [M rows][K cols] (box 64 x 128) or MN-major [K rows][M cols] (box 64 x 64)
  ok = a_t ? make_map(&ta, A, K, M, lda, 64, TC_BK) : make_map(&ta, A, M, K, lda, TC_BK, TC_BM);
  if (!ok) return cudaErrorInvalidValue;
  ok = b_t ? make_map(&tb, B, K, N, ldb, 64, TC_BK) : make_map(&tb, B, N, K, ldb, TC_BK, BN);
  if (!ok) return cudaErrorInvalidValue;
  // output boxes: 32 x 32, bf16 with 64-byte swizzle or fp32 with 128-byte swizzle
  switch (epi.kind) {
    case EPI_STORE:
    case EPI_DGELU:
      ok = make_map_ex(&tc, MapKey{epi.out, M, N, epi.ld_out, 1, 0, 32, 32, 0, 64});
      tc2 = tc;
      break;
    case EPI_GELU:
      ok = make_map_ex(&tc, MapKey{epi.out, M, N, epi.ld_out, 1, 0, 32, 32, 0, 64}) &&
           make_map_ex(&tc2, MapKey{epi.out2, M, N, epi.ld_out2, 1, 0, 32, 32, 0, 64});
      break;
    case EPI_F32:
      ok = make_map_ex(&tc, MapKey{epi.outf, M, N, epi.ld_outf, 1, 0, 32, 32, 1, 128});
      tc2 = tc;
      break;
    case EPI_F32_SPLIT:
      ok = make_map_ex(&tc, MapKey{epi.outf, M, N, epi.ld_outf, splits, epi.split_stride, 32, 32, 1, 128});
      tc2 = tc;
      break;
    default:
      ok = false;
  }
  if (!ok) return cudaErrorInvalidValue;
  if (!a_t && !b_t) return launch_kind<BN, false, false>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  if (!a_t && b_t) return launch_kind<BN, false, true>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  if (a_t && b_t) return launch_kind<BN, true, true>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  return launch_kind<BN, true, false>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
}

cudaError_t launch_gemm_tc(int M, int N, int K, const bf16* A, long lda, bool a_t, const bf16* B, long ldb,
                           bool b_t, const EpiParams<bf16>& epi, int splits, unsigned* err, cudaStream_t s) {
  if (!g_sms) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sms = n > 0 ? n : 148;
  }
  if (((uintptr_t)A & 15) || ((uintptr_t)B & 15)) return cudaErrorInvalidValue;
  // outputs are written by TMA: 16-byte aligned bases and row strides
  const void* outs[2] = {epi.kind >= EPI_F32 ? (const void*)epi.outf : (const void*)epi.out,
                         epi.kind == EPI_GELU ? (const void*)epi.out2 : nullptr};
  for (const void* o : outs)
    if (o && ((uintptr_t)o & 15)) return cudaErrorInvalidValue;
  if (epi.kind >= EPI_F32 ? (epi.ld_outf & 3) : (epi.ld_out & 7)) return cudaErrorInvalidValue;
  if (splits < 1) splits = 1;
  // tile width: prefer 256 columns unless 128 fills the machine's waves better
  long tm = (M + TC_BM - 1) / TC_BM;
  long u256 = tm * ((N + 255) / 256) * splits, u128 = tm * ((N + 127) / 128) * splits;
  auto eff = [](long units, long per) {
    long waves = (units + g_sms - 1) / g_sms;
    return (double)units * per / ((double)waves * g_sms * 256);
  };
  bool use128 = N <= 128 || eff(u128, 128) > eff(u256, 256) * 1.15;
  if (use128) return launch_bn<128>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, splits, err, s);
  return launch_bn<256>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, splits, err, s);
}
