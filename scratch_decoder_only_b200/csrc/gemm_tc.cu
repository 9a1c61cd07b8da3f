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
#include "tc_common.cuh"

#define TC_BM 128
#define TC_BK 64
#define TC_THREADS 192

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
