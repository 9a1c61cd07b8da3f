// tcgen05 GEMM for sm_100a: C[M,N] = A(M x K) . B(N x K)^T, bf16 operands,
// fp32 accumulation in tensor memory, fused epilogues (bias, residual, GELU,
// GELU', fp32 / split-K fp32 outputs).  Every dense contraction of the
// training step runs here: the QKV, attention-out, MLP and LM-head
// projections forward (A and B K-major), their input gradients (B MN-major:
// the weight read transposed in place) and their weight gradients (A and B
// MN-major: both activations read transposed in place), so no transposed
// copy of any tensor is ever written.
//
// Structure (192-thread CTAs, persistent over output tiles; a CTA alone or a
// cluster of two sharing one MMA stream):
//   warp 0      TMA producer: 2-D tiled loads (128-byte swizzle) of A and B
//               k-blocks into a ring of shared-memory stages, completion
//               signalled on "full" mbarriers; also allocates tensor memory.
//   warp 1      MMA issuer: one thread issues tcgen05.mma (kind::f16, M = 128
//               for a CTA, 256 for a pair, N = BN, K = 16) into a TMEM
//               accumulator, and tcgen05.commit frees each stage ("empty")
//               and hands a finished accumulator to the epilogue ("tfull").
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (one row per thread),
//               epilogue arithmetic into a swizzled staging buffer, one TMA
//               bulk-tensor store per 128-row sub-tile; "tempty" returns the
//               accumulator.  Two accumulators (2 x BN columns) let the
//               epilogue of one tile overlap the MMAs of the next.
// Every TMA load is a plain tile load into the issuing CTA's own shared
// memory.  Every mbarrier wait is bounded: on timeout the kernel records
// GPT_DEVERR_TIMEOUT, drains what it started, frees its tensor memory and
// returns.
#include "tc_common.cuh"

#define TC_BM 128
#define TC_BK 64
#define TC_THREADS 192

// ------------------------------------------------------------------ epilogue
// The four epilogue warps cooperate on 128-row sub-tiles of the accumulator
// (64 columns for bf16 outputs, 32 for fp32: 128-byte rows either way): each
// thread owns one row (its TMEM lane), applies the epilogue and writes the
// row into a 128-byte-swizzled staging buffer; after a barrier one thread
// stores the whole 16 KB sub-tile with a single TMA bulk-tensor store.  Two
// staging buffers per output alternate so a store drains while the next
// sub-tile is computed (the second output of GELU uses buffers 2 and 3).
#define EPI_BUF_BYTES 16384

// Row r (0..127) of a 128-row staging buffer: 8 x 16 bytes, 128-byte swizzle.
__device__ __forceinline__ void stage_row128(uint32_t buf, int r, const uint4* w) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t a = buf + r * 128 + ((q ^ (r & 7)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[q].x), "r"(w[q].y), "r"(w[q].z),
                 "r"(w[q].w)
                 : "memory");
  }
}
template <bool F16>
__device__ __forceinline__ void pack16x64(const float* v, uint4* w) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    w[q].x = pack16x2<F16>(v[8 * q + 0], v[8 * q + 1]);
    w[q].y = pack16x2<F16>(v[8 * q + 2], v[8 * q + 3]);
    w[q].z = pack16x2<F16>(v[8 * q + 4], v[8 * q + 5]);
    w[q].w = pack16x2<F16>(v[8 * q + 6], v[8 * q + 7]);
  }
}

// Column sums of a warp's 32 rows x 64 columns (lane = row, v = its 64 values):
// five halving exchange steps leave lane l with the sums of columns 2l, 2l+1.
__device__ __forceinline__ float2 warp_colsum64(const float* v, int lane) {
  float t[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) t[i] = v[i];
#pragma unroll
  for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
    const bool hi = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = hi ? t[i] : t[i + n];
      const float keep = hi ? t[i + n] : t[i];
      t[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return make_float2(t[0], t[1]);
}

// Bounded barrier of the 128 epilogue threads (an mbarrier with count 128).
__device__ __forceinline__ bool epi_sync(uint32_t bar, uint32_t& phase, volatile int* abort_flag) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase, abort_flag);
  phase ^= 1;
  return ok;
}

// Row r of a 128-row, 128-byte-swizzled 16-bit buffer (64 values) into fp32.
template <bool F16>
__device__ __forceinline__ void load_row128_16(uint32_t buf, int r, float* x) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint4 w;
    const uint32_t a = buf + r * 128 + ((q ^ (r & 7)) << 4);
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w) : "r"(a)
                 : "memory");
    unpack16x8<F16>(w, x + 8 * q);
  }
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a)
               : "memory");
  return v;
}
// ------------------------------------------------------------------ the kernel
// EPI_STORE with a residual is its own instantiation: its residual tiles come
// in by TMA like the DGELU pre-activations.
#define EPI_STORE_RES 7
// EPI_STORE with a row-dot output (the attention backward's D = dO . O per
// row and head, taken while the dO tile is in registers): its own
// instantiation, the second operand of the dot read by TMA as a side input.
#define EPI_STORE_DOT 8
// Added to an epilogue kind in the kernel's template argument: the 16-bit
// operands and outputs are fp16 instead of bf16.
#define KIND_F16 16
template <int KIND>
struct EpiTraits {
  static constexpr bool SIDE = (KIND == EPI_STORE_RES || KIND == EPI_DGELU || KIND == EPI_STORE_DOT);   // reads a bf16 [M, N] input
  static constexpr bool BIAS = (KIND == EPI_STORE || KIND == EPI_STORE_RES || KIND == EPI_GELU);
  static constexpr bool F32OUT = (KIND == EPI_F32 || KIND == EPI_F32_SPLIT || KIND == EPI_F32_ADD);
};

template <int BN, int KIND, int CG = 1>
struct TcCfg {
  // GELU's second output and the side input each take two more staging
  // buffers; the other kinds keep one more mainloop stage instead
  static constexpr bool WIDE = (KIND == EPI_GELU || EpiTraits<KIND>::SIDE);
  static constexpr int EPI_BYTES = (WIDE ? 4 : 2) * EPI_BUF_BYTES;
  // bias of the tile, or (GELU') the four row quarters' column sums of a sub-tile
  static constexpr int BIAS_BYTES = EpiTraits<KIND>::BIAS ? BN * 4 : (KIND == EPI_DGELU ? 4 * 64 * 4 : 0);
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = (BN / CG) * TC_BK * 2;   // a CTA pair splits B along N
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int FREE = 232448 - 1024 - EPI_BYTES - 256 - BIAS_BYTES;
  static constexpr int STAGES = FREE / STAGE_BYTES > 8 ? 8 : FREE / STAGE_BYTES;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + 256 + BIAS_BYTES;
  static_assert(SMEM <= 232448, "shared memory per block");
};

// CG = 2: a cluster of two CTAs computes a 256-row tile with one
// tcgen05.mma.cta_group::2 stream issued by the even CTA; each CTA loads its
// 128 rows of A and half of the tile's B columns, and holds its 128 rows of
// the accumulator in its own TMEM.
template <int BN, bool A_MN, bool B_MN, int KINDF, int CG>
__global__ void __launch_bounds__(TC_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2, int M, int N,
               int K, int splits, EpiParams<bf16> epi, unsigned* err) {
  constexpr int KIND = KINDF & (KIND_F16 - 1);
  constexpr bool F16 = (KINDF & KIND_F16) != 0;
  using Cfg = TcCfg<BN, KIND, CG>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* tile_mem = smem;
  uint8_t* epi_mem = smem + STAGES * Cfg::STAGE_BYTES;   // Cfg::EPI_BYTES of staging, 1024-aligned
  uint64_t* bars = (uint64_t*)(epi_mem + Cfg::EPI_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, epilogue group, side[2]
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * STAGES + 8);
  float* bias_s = (float*)((uint8_t*)bars + 256);   // BN bias values of the current tile
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  const uint32_t group_bar = bar0 + 8u * (2 * STAGES + 5);
  auto side_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 6 + b); };

  const uint32_t rank = CG == 2 ? cluster_rank() : 0u;   // CTA inside the pair; 0 issues the MMAs
  const int cid = CG == 2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x, ncl = CG == 2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull_bar(a), 1); mbar_init(tempty_bar(a), 4 * CG); }
    mbar_init(drain_bar, 1);
    mbar_init(group_bar, 128);
    mbar_init(side_bar(0), 1);
    mbar_init(side_bar(1), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    if constexpr (CG == 2) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(Cfg::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(Cfg::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync_all();   // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the set-up above overlaps the previous kernel's tail; operands, side
  // inputs and outputs are touched only after it has completed
  griddep_wait();
  griddep_release();

  constexpr int TM = TC_BM * CG;   // output rows per work unit
  const int tiles_m = (M + TM - 1) / TM, tiles_n = (N + BN - 1) / BN;
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
    for (int u = cid; u < units && ok; u += ncl) {
      const int split = u / tiles, t = u % tiles;
      const int m0 = (t % tiles_m) * TM + TC_BM * (int)rank, n0 = (t / tiles_m) * BN + (BN / CG) * (int)rank;
      const int kb0 = split * kbs, kb1 = min(kb_total, kb0 + kbs);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1, abort_flag)) { ok = false; break; }
        // a pair completes both CTAs' bytes on the even CTA's barrier
        const uint32_t fb = CG == 2 ? cluster_addr(full_bar(stage), 0) : full_bar(stage);
        if (rank == 0) mbar_expect_tx(full_bar(stage), CG * Cfg::STAGE_BYTES);
        const uint32_t sa = smem_u32(tile_mem + stage * Cfg::STAGE_BYTES);
        const uint32_t sb = sa + Cfg::A_BYTES;
        const int k0 = kb * TC_BK;
        auto load = [&](uint32_t dst, const CUtensorMap* map, int x, int y) {
          if constexpr (CG == 2) tma_load_2d_pair(dst, map, fb, x, y);
          else tma_load_2d(dst, map, fb, x, y);
        };
        if (!A_MN) {
          load(sa, &tmA, k0, m0);
        } else {
#pragma unroll
          for (int j = 0; j < TC_BM / 64; ++j) load(sa + j * 64 * TC_BK * 2, &tmA, m0 + 64 * j, k0);
        }
        if (!B_MN) {
          load(sb, &tmB, k0, n0);
        } else {
#pragma unroll
          for (int j = 0; j < BN / CG / 64; ++j) load(sb + j * 64 * TC_BK * 2, &tmB, n0 + 64 * j, k0);
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
    // (a pair's loads all complete on the even CTA's barriers)
    long nd = rank == 0 ? (issued < STAGES ? issued : STAGES) : 0;
    int s = stage;
    uint32_t ph = phase;
    for (long i = 0; i < nd; ++i) {
      if (--s < 0) { s = STAGES - 1; ph ^= 1; }
      volatile int never = 0;
      mbar_wait(full_bar(s), ph, &never, 1ll << 28);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------- MMA issuer (the even CTA of a pair issues for both)
    constexpr uint32_t IDESC = instr_desc_t(F16, BN, A_MN, B_MN, TM);
    // K-major: SBO = 8 rows x 128 B; k step (16 elements) = 32 B inside the swizzle row.
    // MN-major: LBO = one 64-element box (64 k-rows x 128 B), SBO = 8 k-rows x 128 B; k step = 16 rows.
    constexpr uint32_t A_LBO = A_MN ? 64 * TC_BK * 2 : 16, A_SBO = 1024, A_KSTEP = A_MN ? 16 * 128 : 32;
    constexpr uint32_t B_LBO = B_MN ? 64 * TC_BK * 2 : 16, B_SBO = 1024, B_KSTEP = B_MN ? 16 * 128 : 32;
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int u = cid; u < units && ok; u += ncl) {
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
          if constexpr (CG == 2) umma_bf16_pair(tmem_d, ad, bd, IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
          else umma_bf16(tmem_d, ad, bd, IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
        }
        if constexpr (CG == 2) umma_commit_pair_both(empty_bar(stage));
        else umma_commit(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if constexpr (CG == 2) umma_commit_pair_both(tfull_bar(acc));
      else umma_commit(tfull_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (!ok) {
      *abort_flag = 1;
      atomicOr(err, GPT_DEVERR_TIMEOUT);
    }
    // drain: all MMAs this thread issued have completed once this commit arrives
    if constexpr (CG == 2) umma_commit_pair_local(drain_bar);
    else umma_commit(drain_bar);
    volatile int never = 0;
    mbar_wait(drain_bar, 0, &never, 1ll << 28);
  } else if (warp >= 2) {
    // ---------------- epilogue: thread owns tile row 32*(warp%4) + lane (its TMEM lane)
    using Tr = EpiTraits<KIND>;
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const int etid = threadIdx.x - 64;
    constexpr int SW = Tr::F32OUT ? 32 : 64;   // sub-tile columns (128-byte rows)
    const uint32_t sbase = smem_u32(epi_mem);
    const uint32_t rbase = sbase + 2 * EPI_BUF_BYTES;   // side-input buffers
    const uint32_t bias_sa = smem_u32(bias_s);
    const bool has_bias = Tr::BIAS && epi.bias != nullptr;
    uint32_t gph = 0;
    int sub = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    // side input: thread 0 loads sub-tile k into buffer k&1 one sub-tile ahead
    int ld_u = cid, ld_c = 0, issued = 0;
    auto issue_side = [&]() {
      if (ld_u >= units) return;
      const int t = ld_u % tiles;
      const int m0 = (t % tiles_m) * TM + TC_BM * (int)rank, n0 = (t / tiles_m) * BN;
      const uint32_t sb = side_bar(issued & 1);
      mbar_expect_tx(sb, EPI_BUF_BYTES);
      tma_load_2d(rbase + (issued & 1) * EPI_BUF_BYTES, &tmC2, sb, n0 + ld_c, m0);
      ++issued;
      ld_c += SW;
      if (ld_c >= BN || n0 + ld_c >= N) { ld_c = 0; ld_u += ncl; }
    };
    if (Tr::SIDE && etid == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmC2)) : "memory");
      issue_side();
    }
    // the even CTA's barrier that frees an accumulator (both CTAs' epilogues arrive)
    auto tempty_arrive = [&](int a) {
      if constexpr (CG == 2) mbar_arrive_cluster(cluster_addr(tempty_bar(a), 0));
      else mbar_arrive(tempty_bar(a));
    };
    for (int u = cid; u < units && ok; u += ncl) {
      const int split = u / tiles, t = u % tiles;
      const int m0 = (t % tiles_m) * TM + TC_BM * (int)rank, n0 = (t / tiles_m) * BN;
      const bool rows_in = m0 < M;   // a pair's second half can lie past the last row
      // this tile's bias: fetched before the accumulator wait, written to shared
      // memory after it (every thread has finished the previous tile's reads:
      // they precede its last group barrier)
      float bv[BN / 128];
      if (has_bias) {
#pragma unroll
        for (int j = 0; j < BN / 128; ++j) {
          const int col = n0 + etid + 128 * j;
          bv[j] = col < N ? epi.bias[col] : 0.f;
        }
      }
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (has_bias) {
#pragma unroll
        for (int j = 0; j < BN / 128; ++j) bias_s[etid + 128 * j] = bv[j];
      }
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN; c += SW) {
        const int col0 = n0 + c;
        if (col0 >= N) break;
        uint32_t r[SW];
        tmem_ld32(tbase + c, r);
        if (SW == 64) tmem_ld32(tbase + c + 32, r + 32);
        tmem_wait_ld();
        if (c + SW >= BN || col0 + SW >= N) {   // last sub-tile: the accumulator can be reused
          tc_fence_before();
          __syncwarp();
          if (lane == 0) tempty_arrive(acc);
        }
        // the store that last used this staging buffer has read it
        if (etid == 0) bulk_wait_read<1>();
        if (!epi_sync(group_bar, gph, abort_flag)) { ok = false; break; }
        // every thread is past the previous sub-tile: its side buffer is free
        if (Tr::SIDE && etid == 0) issue_side();
        const uint32_t b0 = sbase + (sub & 1) * EPI_BUF_BYTES;
        float v[SW];
#pragma unroll
        for (int j = 0; j < SW; ++j) v[j] = __uint_as_float(r[j]);
        if (has_bias) {
#pragma unroll
          for (int q = 0; q < SW / 4; ++q) {
            const float4 bb = ld_shared_f4(bias_sa + (c + 4 * q) * 4);
            v[4 * q] += bb.x; v[4 * q + 1] += bb.y; v[4 * q + 2] += bb.z; v[4 * q + 3] += bb.w;
          }
        }
        if constexpr (Tr::SIDE) {
          if (!mbar_wait(side_bar(sub & 1), (sub >> 1) & 1, abort_flag)) { ok = false; break; }
        }
        uint4 w[8];
        if constexpr (KIND == EPI_STORE || KIND == EPI_STORE_RES) {
          if constexpr (KIND == EPI_STORE_RES) {
            float rr[64];
            load_row128_16<F16>(rbase + (sub & 1) * EPI_BUF_BYTES, rl, rr);
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] += rr[j];
          }
          pack16x64<F16>(v, w);
          stage_row128(b0, rl, w);
        } else if constexpr (KIND == EPI_STORE_DOT) {
          float oo[64];
          load_row128_16<F16>(rbase + (sub & 1) * EPI_BUF_BYTES, rl, oo);
          float dot = 0.f;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            v[j] = round16<F16>(v[j]);
            dot += v[j] * oo[j];
          }
          pack16x64<F16>(v, w);
          stage_row128(b0, rl, w);
          const int row = m0 + rl;
          if (rows_in && row < M) {
            const int Tq = epi.rd_T, b = row / Tq;
            epi.rowdot[((long)b * (N / 64) + col0 / 64) * Tq + (row - b * Tq)] = dot;
          }
        } else if constexpr (KIND == EPI_GELU) {
          float a[64];
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const float uq = round16<F16>(v[j]);
            v[j] = uq;
            a[j] = gelu_fast(uq);
          }
          pack16x64<F16>(v, w);
          stage_row128(b0, rl, w);
          pack16x64<F16>(a, w);
          stage_row128(b0 + 2 * EPI_BUF_BYTES, rl, w);
        } else if constexpr (KIND == EPI_DGELU) {
          float uu[64];
          load_row128_16<F16>(rbase + (sub & 1) * EPI_BUF_BYTES, rl, uu);
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] *= gelu_grad_fast(uu[j]);
          pack16x64<F16>(v, w);
          stage_row128(b0, rl, w);
          if (epi.colsum) {   // this warp's 32 rows, summed per column, to shared memory
            const float2 cs = warp_colsum64(v, lane);
            bias_s[quarter * 64 + 2 * lane] = cs.x;
            bias_s[quarter * 64 + 2 * lane + 1] = cs.y;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            w[q] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]), __float_as_uint(v[4 * q + 2]),
                              __float_as_uint(v[4 * q + 3]));
          stage_row128(b0, rl, w);
        }
        fence_async_smem();
        if (!epi_sync(group_bar, gph, abort_flag)) { ok = false; break; }
        if constexpr (KIND == EPI_DGELU) {
          // the sub-tile's column sums over its 128 rows: one partial row per row tile
          if (epi.colsum && etid < 64 && rows_in && col0 + etid < N)
            epi.colsum[(long)(m0 / TC_BM) * N + col0 + etid] =
                (bias_s[etid] + bias_s[64 + etid]) + (bias_s[128 + etid] + bias_s[192 + etid]);
        }
        if (etid == 0 && rows_in) {
          if constexpr (KIND == EPI_F32_SPLIT) {
            tma_store_3d(&tmC, b0, col0, m0, split);
          } else if constexpr (KIND == EPI_F32_ADD) {
            tma_reduce_add_2d(&tmC, b0, col0, m0);
          } else {
            tma_store_2d(&tmC, b0, col0, m0);
            if constexpr (KIND == EPI_GELU) tma_store_2d(&tmC2, b0 + 2 * EPI_BUF_BYTES, col0, m0);
          }
          bulk_commit();
        }
        ++sub;
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (!ok) {
      *abort_flag = 1;
      atomicOr(err, GPT_DEVERR_TIMEOUT);
    }
    if (etid == 0) {
      bulk_wait_all();
      // side loads issued but not consumed (only after an abort): let them land
      for (int k = sub; k < issued; ++k) {
        volatile int never = 0;
        mbar_wait(side_bar(k & 1), (k >> 1) & 1, &never, 1ll << 28);
      }
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  // a pair leaves together: the even CTA's MMAs read the odd CTA's shared
  // memory and write its TMEM until the drain above
  if constexpr (CG == 2) cluster_sync_all();
  tc_fence_after();
  if (warp == 0) {
    if constexpr (CG == 2)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Cfg::TMEM_COLS));
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Cfg::TMEM_COLS));
  }
}

// ------------------------------------------------------------------ host side
bool gemm_tc_supported(int M, int N, int K, long lda, bool a_t, long ldb, bool b_t) {
  // operands and outputs move by TMA: 16-byte row strides
  if (M < 1 || N < 1 || K < 1) return false;
  if ((lda & 7) || (ldb & 7)) return false;   // 16-byte row strides for TMA
  (void)a_t; (void)b_t;
  return get_encode() != nullptr;
}

static int g_sms = 0;

template <int BN, bool A_MN, bool B_MN, int KINDF, int CG>
static cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                             const CUtensorMap& tc2, int M, int N, int K, int splits, const EpiParams<bf16>& epi,
                             unsigned* err, cudaStream_t s) {
  using Cfg = TcCfg<BN, KINDF & (KIND_F16 - 1), CG>;
  auto kern = gemm_tc_kernel<BN, A_MN, B_MN, KINDF, CG>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int units = ((M + TC_BM * CG - 1) / (TC_BM * CG)) * ((N + BN - 1) / BN) * splits;
  const int slots = g_sms / CG;
  const int grid = CG * (units < slots ? units : slots);
  ++g_kernel_launches;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(TC_THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute la[2];
  int na = 0;
  if constexpr (CG == 2) {
    la[na].id = cudaLaunchAttributeClusterDimension;
    la[na].val.clusterDim.x = 2;
    la[na].val.clusterDim.y = 1;
    la[na].val.clusterDim.z = 1;
    ++na;
  }
  if (g_pdl) {   // the prologue may overlap the previous kernel's tail (the kernel waits before any access)
    la[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = la;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, tc2, M, N, K, splits, epi, err);
}

// The (layout, epilogue) combinations the training step and the stand-alone
// GEMM use; any other returns cudaErrorNotSupported.
template <int BN, bool A_MN, bool B_MN, int CG, bool F16>
static cudaError_t launch_kind(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                               const CUtensorMap& tc2, int M, int N, int K, int splits, const EpiParams<bf16>& epi,
                               unsigned* err, cudaStream_t s) {
  constexpr int FK = F16 ? KIND_F16 : 0;
  if (epi.kind == EPI_F32) return launch_tc<BN, A_MN, B_MN, EPI_F32 + FK, CG>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  if constexpr (!A_MN) {
    if (epi.kind == EPI_STORE && epi.resid)
      return launch_tc<BN, A_MN, B_MN, EPI_STORE_RES + FK, CG>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    if constexpr (B_MN) {
      if (epi.kind == EPI_STORE && epi.rowdot)
        return launch_tc<BN, A_MN, B_MN, EPI_STORE_DOT + FK, CG>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    }
    if (epi.rowdot) return cudaErrorNotSupported;
    if (epi.kind == EPI_STORE)
      return launch_tc<BN, A_MN, B_MN, EPI_STORE + FK, CG>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    if constexpr (!B_MN) {
      if (epi.kind == EPI_GELU)
        return launch_tc<BN, A_MN, B_MN, EPI_GELU + FK, CG>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    } else {
      if (epi.kind == EPI_DGELU)
        return launch_tc<BN, A_MN, B_MN, EPI_DGELU + FK, CG>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    }
  } else if constexpr (B_MN) {
    if (epi.kind == EPI_F32_SPLIT)
      return launch_tc<BN, A_MN, B_MN, EPI_F32_SPLIT + FK, CG>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    if (epi.kind == EPI_F32_ADD)
      return launch_tc<BN, A_MN, B_MN, EPI_F32_ADD + FK, CG>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  }
  return cudaErrorNotSupported;
}

template <int BN, int CG>
static cudaError_t launch_bn(int M, int N, int K, const bf16* A, long lda, bool a_t, const bf16* B, long ldb,
                             bool b_t, const EpiParams<bf16>& epi, int splits, unsigned* err, cudaStream_t s) {
  CUtensorMap ta, tb, tc, tc2;
  bool ok;
  // A: K-major [M rows][K cols] (box 64 x 128) or MN-major [K rows][M cols] (box 64 x 64)
  ok = a_t ? make_map(&ta, A, K, M, lda, 64, TC_BK) : make_map(&ta, A, M, K, lda, TC_BK, TC_BM);
  if (!ok) return cudaErrorInvalidValue;
  // B: K-major [N rows][K cols] (box 64 x BN/CG: a pair splits the tile's columns) or MN-major (box 64 x 64)
  ok = b_t ? make_map(&tb, B, K, N, ldb, 64, TC_BK) : make_map(&tb, B, N, K, ldb, TC_BK, BN / CG);
  if (!ok) return cudaErrorInvalidValue;
  // output boxes: 128 rows x 128 bytes (64 bf16 or 32 fp32 columns), 128-byte swizzle
  switch (epi.kind) {
    case EPI_STORE:
      ok = make_map_ex(&tc, MapKey{epi.out, M, N, epi.ld_out, 1, 0, 64, TC_BM, 0, 128});
      tc2 = tc;
      // the residual is read by TMA in the same 128 x 64 boxes
      if (ok && epi.resid) ok = make_map_ex(&tc2, MapKey{epi.resid, M, N, epi.ld_resid, 1, 0, 64, TC_BM, 0, 128});
      // so is the row-dot's second operand (heads of 64 columns, no bias or residual)
      if (ok && epi.rowdot)
        ok = !epi.resid && !epi.bias && N % 64 == 0 && epi.rd_T > 0 && epi.aux &&
             make_map_ex(&tc2, MapKey{epi.aux, M, N, epi.ld_aux, 1, 0, 64, TC_BM, 0, 128});
      break;
    case EPI_DGELU:
      ok = make_map_ex(&tc, MapKey{epi.out, M, N, epi.ld_out, 1, 0, 64, TC_BM, 0, 128}) &&
           make_map_ex(&tc2, MapKey{epi.aux, M, N, epi.ld_aux, 1, 0, 64, TC_BM, 0, 128});
      break;
    case EPI_GELU:
      ok = make_map_ex(&tc, MapKey{epi.out, M, N, epi.ld_out, 1, 0, 64, TC_BM, 0, 128}) &&
           make_map_ex(&tc2, MapKey{epi.out2, M, N, epi.ld_out2, 1, 0, 64, TC_BM, 0, 128});
      break;
    case EPI_F32:
    case EPI_F32_ADD:
      ok = make_map_ex(&tc, MapKey{epi.outf, M, N, epi.ld_outf, 1, 0, 32, TC_BM, 1, 128});
      tc2 = tc;
      break;
    case EPI_F32_SPLIT:
      ok = make_map_ex(&tc, MapKey{epi.outf, M, N, epi.ld_outf, splits, epi.split_stride, 32, TC_BM, 1, 128});
      tc2 = tc;
      break;
    default:
      ok = false;
  }
  if (!ok) return cudaErrorInvalidValue;
  if (epi.f16) {
    if (!a_t && !b_t) return launch_kind<BN, false, false, CG, true>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    if (!a_t && b_t) return launch_kind<BN, false, true, CG, true>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    if (a_t && b_t) return launch_kind<BN, true, true, CG, true>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
    return launch_kind<BN, true, false, CG, true>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  }
  if (!a_t && !b_t) return launch_kind<BN, false, false, CG, false>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  if (!a_t && b_t) return launch_kind<BN, false, true, CG, false>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  if (a_t && b_t) return launch_kind<BN, true, true, CG, false>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
  return launch_kind<BN, true, false, CG, false>(ta, tb, tc, tc2, M, N, K, splits, epi, err, s);
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
  // residual / pre-activation inputs are read by TMA too
  const bf16* side = epi.kind == EPI_STORE ? epi.resid : epi.kind == EPI_DGELU ? epi.aux : nullptr;
  const long side_ld = epi.kind == EPI_STORE ? epi.ld_resid : epi.ld_aux;
  if (side && (((uintptr_t)side & 15) || (side_ld & 7))) return cudaErrorInvalidValue;
  if (splits < 1) splits = 1;
  // tile width: prefer 256 columns unless 128 fills the machine's waves better
  long tm = (M + TC_BM - 1) / TC_BM;
  long u256 = tm * ((N + 255) / 256) * splits, u128 = tm * ((N + 127) / 128) * splits;
  auto eff = [](long units, long per) {
    long waves = (units + g_sms - 1) / g_sms;
    return (double)units * per / ((double)waves * g_sms * 256);
  };
  bool use128 = N <= 128 || eff(u128, 128) > eff(u256, 256) * 1.15;
  if (use128) return launch_bn<128, 1>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, splits, err, s);
  // 256-row tiles on CTA pairs: each SM streams half of B, so the MMA is not
  // held back by shared-memory bandwidth; taken unless the pairs fill the
  // machine much worse than single CTAs
  long u2 = ((M + 255) / 256) * ((N + 255) / 256) * splits;
  auto eff2 = [](long units) {
    long slots = g_sms / 2, waves = (units + slots - 1) / slots;
    return (double)units / ((double)waves * slots);
  };
  bool pair = M > 128 && eff2(u2) * 1.2 >= eff(u256, 256);
  if (pair) return launch_bn<256, 2>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, splits, err, s);
  return launch_bn<256, 1>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, splits, err, s);
}
