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

// 32 lanes x 32 consecutive 32-bit columns: thread t gets lane (base + t), columns c..c+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor (tcgen05), 128-byte swizzle, version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: D fp32, A/B bf16, majorness, N >> 3, M >> 4.
__host__ __device__ constexpr uint32_t instr_desc(int bn, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(TC_BM >> 4) << 24);
}

// ------------------------------------------------------------------ epilogue (one row, 32 columns)
__device__ __forceinline__ void store_bf16x32(bf16* dst, const float* x, int nvalid, bool vec) {
  if (vec && nvalid == 32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) Vec<bf16>::store(dst + 8 * q, x + 8 * q);
  } else {
    for (int j = 0; j < nvalid; ++j) dst[j] = __float2bfloat16_rn(x[j]);
  }
}
__device__ __forceinline__ void load_bf16x32(const bf16* src, float* x, int nvalid, bool vec) {
  if (vec && nvalid == 32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) Vec<bf16>::load(src + 8 * q, x + 8 * q);
  } else {
    for (int j = 0; j < 32; ++j) x[j] = j < nvalid ? __bfloat162float(src[j]) : 0.f;
  }
}
__device__ __forceinline__ bool al16(const void* p) { return ((uintptr_t)p & 15) == 0; }

__device__ __forceinline__ void epi_row32(const EpiParams<bf16>& p, int row, int col0, int M, int N, float* v,
                                          int split) {
  if (row >= M || col0 >= N) return;
  const int nv = min(32, N - col0);
  switch (p.kind) {
    case EPI_STORE: {
      if (p.bias) {
        if (nv == 32) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float b4[4];
            Vec<float>::load(p.bias + col0 + 4 * q, b4);
#pragma unroll
            for (int j = 0; j < 4; ++j) v[4 * q + j] += b4[j];
          }
        } else {
          for (int j = 0; j < nv; ++j) v[j] += p.bias[col0 + j];
        }
      }
      if (p.resid) {
        const bf16* r = p.resid + (long)row * p.ld_resid + col0;
        float rr[32];
        load_bf16x32(r, rr, nv, (p.ld_resid & 7) == 0 && al16(r));
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += rr[j];
      }
      bf16* o = p.out + (long)row * p.ld_out + col0;
      store_bf16x32(o, v, nv, (p.ld_out & 7) == 0 && al16(o));
    } break;
    case EPI_GELU: {
      float a[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float u = v[j] + ((p.bias && j < nv) ? p.bias[col0 + j] : 0.f);
        float uq = __bfloat162float(__float2bfloat16_rn(u));
        v[j] = uq;
        a[j] = gelu_f(uq);
      }
      bf16* o = p.out + (long)row * p.ld_out + col0;
      store_bf16x32(o, v, nv, (p.ld_out & 7) == 0 && al16(o));
      bf16* o2 = p.out2 + (long)row * p.ld_out2 + col0;
      store_bf16x32(o2, a, nv, (p.ld_out2 & 7) == 0 && al16(o2));
    } break;
    case EPI_DGELU: {
      const bf16* u = p.aux + (long)row * p.ld_aux + col0;
      float uu[32];
      load_bf16x32(u, uu, nv, (p.ld_aux & 7) == 0 && al16(u));
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= gelu_grad_f(uu[j]);
      bf16* o = p.out + (long)row * p.ld_out + col0;
      store_bf16x32(o, v, nv, (p.ld_out & 7) == 0 && al16(o));
    } break;
    case EPI_F32:
    case EPI_F32_SPLIT: {
      float* o = p.outf + (p.kind == EPI_F32_SPLIT ? (long)split * p.split_stride : 0) + (long)row * p.ld_outf + col0;
      if (nv == 32 && (p.ld_outf & 3) == 0 && al16(o)) {
#pragma unroll
        for (int q = 0; q < 8; ++q) Vec<float>::store(o + 4 * q, v + 4 * q);
      } else {
        for (int j = 0; j < nv; ++j) o[j] = v[j];
      }
    } break;
  }
}

// ------------------------------------------------------------------ the kernel
template <int BN>
struct TcCfg {
  static constexpr int STAGES = BN >= 256 ? 4 : 6;
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 256;
};

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(TC_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
               int K, int splits, EpiParams<bf16> epi, unsigned* err) {
  using Cfg = TcCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* tile_mem = smem;
  uint64_t* bars = (uint64_t*)(smem + STAGES * Cfg::STAGE_BYTES);
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
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const int split = u / tiles, t = u % tiles;
      const int m0 = (t % tiles_m) * TC_BM, n0 = (t / tiles_m) * BN;
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
        *abort_flag = 1;
        atomicOr(err, GPT_DEVERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int row = m0 + quarter * 32 + lane;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tbase + c, v);
        epi_row32(epi, row, n0 + c, M, N, v, split);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
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

// 2-D bf16 tensor [rows][cols] with row stride ld (elements); box = box_cols x box_rows.
static bool make_map(CUtensorMap* map, const void* base, long rows, long cols, long ld, int box_cols, int box_rows) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, long, long, long, int, int>, CUtensorMap> cache;
  auto key = std::make_tuple(base, rows, cols, ld, box_cols, box_rows);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) { *map = it->second; return true; }
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  if (cache.size() > 4096) cache.clear();
  cache[key] = *map;
  return true;
}

bool gemm_tc_supported(int M, int N, int K, long lda, bool a_t, long ldb, bool b_t) {
  if (M < 1 || N < 1 || K < 1) return false;
  if ((lda & 7) || (ldb & 7)) return false;   // 16-byte row strides for TMA
  (void)a_t; (void)b_t;
  return get_encode() != nullptr;
}

static int g_sms = 0;

template <int BN, bool A_MN, bool B_MN>
static cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K, int splits,
                             const EpiParams<bf16>& epi, unsigned* err, cudaStream_t s) {
  using Cfg = TcCfg<BN>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  int units = ((M + TC_BM - 1) / TC_BM) * ((N + BN - 1) / BN) * splits;
  int grid = units < g_sms ? units : g_sms;
  ++g_kernel_launches;
  gemm_tc_kernel<BN, A_MN, B_MN><<<grid, TC_THREADS, Cfg::SMEM, s>>>(ta, tb, M, N, K, splits, epi, err);
  return cudaGetLastError();
}

template <int BN>
static cudaError_t launch_bn(int M, int N, int K, const bf16* A, long lda, bool a_t, const bf16* B, long ldb,
                             bool b_t, const EpiParams<bf16>& epi, int splits, unsigned* err, cudaStream_t s) {
  CUtensorMap ta, tb;
  bool ok;
  // A: K-major [M rows][K cols] (box 64 x 128) or MN-major [K rows][M cols] (box 64 x 64)
  ok = a_t ? make_map(&ta, A, K, M, lda, 64, TC_BK) : make_map(&ta, A, M, K, lda, TC_BK, TC_BM);
  if (!ok) return cudaErrorInvalidValue;
  ok = b_t ? make_map(&tb, B, K, N, ldb, 64, TC_BK) : make_map(&tb, B, N, K, ldb, TC_BK, BN);
  if (!ok) return cudaErrorInvalidValue;
  if (!a_t && !b_t) return launch_tc<BN, false, false>(ta, tb, M, N, K, splits, epi, err, s);
  if (!a_t && b_t) return launch_tc<BN, false, true>(ta, tb, M, N, K, splits, epi, err, s);
  if (a_t && b_t) return launch_tc<BN, true, true>(ta, tb, M, N, K, splits, epi, err, s);
  return launch_tc<BN, true, false>(ta, tb, M, N, K, splits, epi, err, s);
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
