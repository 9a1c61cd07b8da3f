// Decode projections for 9 to 32 rows ("RustGPT", "Technical implementation":
// greedy decoding; "NTransformer" page, "No PyTorch, no cuBLAS": per-token
// projections over a KV-cached step): y[b, n] = sum_k x[b, k] W[n, k] with
// the epilogues of the decode GEMV (bias + residual, bias + GELU, fp32
// logits).
//
// A decode step reads every weight once and multiplies it by a handful of
// rows, so the work is a weight stream: the tensor-core GEMM's 128-row tiles
// leave 3-12 CTAs busy on the 768-column projections at 32 rows.  Here the
// weights are cut into 16-row slices spread over every SM; each slice (16
// contiguous rows) moves into shared memory by one bulk copy, several slices
// in flight per CTA, and the CTA's eight warps split the slice's k range,
// each multiplying on the tensor cores with mma.sync m16n8k16 (A = 16 rows of
// x, read from global memory and L1; B = the slice from shared memory).  The
// warps' partial tiles are summed in a fixed order in shared memory before
// the epilogue, so results are deterministic.  Weight copies are issued
// before the programmatic-dependent-launch wait: the stream starts while the
// previous kernel drains.
#include "launch.h"
#include "tc_common.cuh"

#define DM_THREADS 256
#define DM_WARPS (DM_THREADS / 32)
#define DM_ROWS 16        // weight rows per slice
#define DM_MAXBUF 4       // slice buffers (at most)

template <bool F16>
__device__ __forceinline__ void dm_mma(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  if constexpr (F16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void dm_ldmatrix_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// MT = 16-row tiles of x (B <= 16 MT).  smem: nbuf slices of [16][K] 16-bit
// values, then the warps' partial tiles [DM_WARPS][16 MT][16] fp32.  (The
// ldmatrix reads of a slice meet bank conflicts, rows being K * 2 bytes
// apart; they are a few hundred cycles per slice against microseconds of
// copy, and one bulk copy per slice instead of one per padded row is what
// keeps the weight stream at HBM speed.)
template <typename T, int MT>
__global__ void __launch_bounds__(DM_THREADS)
dec_mma_kernel(const T* __restrict__ X, int B, int K, const T* __restrict__ W, int N, const float* __restrict__ bias,
               const T* resid, int mode, T* out, T* out2, float* outf, int nbuf, unsigned* err) {
  constexpr bool F16 = std::is_same<T, f16>::value;
  extern __shared__ __align__(128) uint8_t dm_smem[];
  __shared__ __align__(8) uint64_t bars[DM_MAXBUF];
  __shared__ int s_abort;
  const int ldw = K;
  const uint32_t slice_bytes = (uint32_t)DM_ROWS * ldw * 2;
  float* red = reinterpret_cast<float*>(dm_smem + nbuf * slice_bytes);
  const int nslices = (N + DM_ROWS - 1) / DM_ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  int nmine = 0;
  for (int sl = blockIdx.x; sl < nslices; sl += gridDim.x) ++nmine;
  const uint32_t smem0 = smem_u32(dm_smem);
  if (threadIdx.x == 0) {
    for (int i = 0; i < nbuf; ++i) mbar_init(smem_u32(&bars[i]), 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // thread 0: slice i of this CTA (rows r0 .. r0 + rr - 1, contiguous) into
  // buffer i % nbuf with one bulk copy
  auto issue = [&](int i) {
    const int r0 = (blockIdx.x + i * gridDim.x) * DM_ROWS, rr = min(DM_ROWS, N - r0);
    const uint32_t dst = smem0 + (i % nbuf) * slice_bytes, bar = smem_u32(&bars[i % nbuf]);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_expect_tx(bar, (uint32_t)rr * K * 2);
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(W + (long)r0 * K)), "r"((uint32_t)rr * K * 2), "r"(bar)
                 : "memory");
  };
  int issued = 0;
  if (threadIdx.x == 0)
    for (; issued < nbuf && issued < nmine; ++issued) issue(issued);
  // x, the residual and the outputs belong to the previous kernel until here
  griddep_wait();
  griddep_release();
  // ldmatrix.x4 row addresses: matrices (rows 0-7, k0), (rows 0-7, k0 + 8),
  // (rows 8-15, k0), (rows 8-15, k0 + 8) -> B fragments of two 8-row n tiles
  const int lrow = (lane & 7) + ((lane >> 4) << 3), lcol = ((lane >> 3) & 1) * 8;
  int i = 0;
  for (; i < nmine; ++i) {
    const int r0 = (blockIdx.x + i * gridDim.x) * DM_ROWS;
    // a timed-out wait is voted block-wide so that every thread leaves together
    const bool okw = mbar_wait(smem_u32(&bars[i % nbuf]), (i / nbuf) & 1, &s_abort);
    if (__syncthreads_or(!okw)) {
      if (threadIdx.x == 0) set_dev_err(err, GPT_DEVERR_TIMEOUT);
      break;
    }
    float acc[MT][2][4];
#pragma unroll
    for (int bt = 0; bt < MT; ++bt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[bt][nt][e] = 0.f;
    const uint32_t ws = smem0 + (i % nbuf) * slice_bytes + (uint32_t)(lrow * ldw + lcol) * 2;
#pragma unroll 2
    for (int ks = warp; ks < K / 16; ks += DM_WARPS) {
      const int k0 = ks * 16;
      uint32_t b[4];
      dm_ldmatrix_x4(b, ws + k0 * 2);
#pragma unroll
      for (int bt = 0; bt < MT; ++bt) {
        const int ra = bt * 16 + g, rb = ra + 8;
        uint32_t a[4];
        a[0] = ra < B ? *reinterpret_cast<const uint32_t*>(X + (long)ra * K + k0 + 2 * tig) : 0u;
        a[1] = rb < B ? *reinterpret_cast<const uint32_t*>(X + (long)rb * K + k0 + 2 * tig) : 0u;
        a[2] = ra < B ? *reinterpret_cast<const uint32_t*>(X + (long)ra * K + k0 + 2 * tig + 8) : 0u;
        a[3] = rb < B ? *reinterpret_cast<const uint32_t*>(X + (long)rb * K + k0 + 2 * tig + 8) : 0u;
        dm_mma<F16>(acc[bt][0], a, b[0], b[1]);
        dm_mma<F16>(acc[bt][1], a, b[2], b[3]);
      }
    }
    // this warp's partial tile: rows b = x rows, columns n = slice rows
#pragma unroll
    for (int bt = 0; bt < MT; ++bt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float* rw = red + ((warp * 16 * MT) + bt * 16 + g) * 16 + nt * 8 + 2 * tig;
        rw[0] = acc[bt][nt][0];
        rw[1] = acc[bt][nt][1];
        rw[8 * 16] = acc[bt][nt][2];
        rw[8 * 16 + 1] = acc[bt][nt][3];
      }
    __syncthreads();
    // every ldmatrix of this buffer is done: refill it
    if (threadIdx.x == 0 && issued < nmine) issue(issued++);
    for (int o = threadIdx.x; o < B * DM_ROWS; o += DM_THREADS) {
      const int bb = o / DM_ROWS, nn = o % DM_ROWS, n = r0 + nn;
      if (n >= N) continue;
      float y = 0.f;
#pragma unroll
      for (int w = 0; w < DM_WARPS; ++w) y += red[((w * 16 * MT) + bb) * 16 + nn];
      const long oi = (long)bb * N + n;
      if (mode == 2) {
        outf[oi] = y;
      } else if (mode == 1) {
        const T uq = from_f<T>(y + bias[n]);
        out[oi] = uq;
        out2[oi] = from_f<T>(gelu_f(to_f(uq)));
      } else {
        out[oi] = from_f<T>(y + (bias ? bias[n] : 0.f) + (resid ? to_f(resid[oi]) : 0.f));
      }
    }
    __syncthreads();   // the partial tiles are rewritten by the next slice
  }
  // after a timeout: let the copies still in flight land before leaving
  if (threadIdx.x == 0) {
    volatile int never = 0;
    for (int j = i; j < issued; ++j) mbar_wait(smem_u32(&bars[j % nbuf]), (j / nbuf) & 1, &never, 1ll << 28);
  }
}

static int g_dm_sms = 0;

bool dec_mma_supported(int B, int K, int N) {
  if (B < 1 || B > 32 || K < 16 || K % 16 || N < 1) return false;
  const size_t slice = (size_t)DM_ROWS * K * 2, red = (size_t)DM_WARPS * 32 * 16 * 4;
  return 2 * slice + red <= 227 * 1024;
}

template <typename T>
cudaError_t launch_dec_mma(const T* X, int B, int K, const T* W, int N, const float* bias, const T* resid, int mode,
                           T* out, T* out2, float* outf, unsigned* err, cudaStream_t s) {
  if (!dec_mma_supported(B, K, N)) return cudaErrorInvalidValue;
  if (((uintptr_t)X & 3) || ((uintptr_t)W & 15)) return cudaErrorInvalidValue;
  if (!g_dm_sms) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_dm_sms = n > 0 ? n : 148;
  }
  const int MT = B <= 16 ? 1 : 2;
  const size_t slice = (size_t)DM_ROWS * K * 2, red = (size_t)DM_WARPS * 16 * MT * 16 * 4;
  // buffers: up to four slices, two CTAs per SM where they fit in ~113 KB each
  int nbuf = (int)((113 * 1024 - red) / slice);
  if (nbuf > DM_MAXBUF) nbuf = DM_MAXBUF;
  if (nbuf < 2) nbuf = 2;
  const size_t smem = nbuf * slice + red;
  void (*kern)(const T*, int, int, const T*, int, const float*, const T*, int, T*, T*, float*, int, unsigned*) =
      MT == 1 ? dec_mma_kernel<T, 1> : dec_mma_kernel<T, 2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, DM_THREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidValue;
  const int nslices = (N + DM_ROWS - 1) / DM_ROWS;
  int grid = g_dm_sms * per_sm;
  if (grid > nslices) grid = nslices;
  ++g_kernel_launches;
  return launch_k(kern, dim3(grid), dim3(DM_THREADS), smem, s, X, B, K, W, N, bias, resid, mode, out, out2, outf,
                  nbuf, err);
}

template cudaError_t launch_dec_mma<bf16>(const bf16*, int, int, const bf16*, int, const float*, const bf16*, int,
                                          bf16*, bf16*, float*, unsigned*, cudaStream_t);
template cudaError_t launch_dec_mma<f16>(const f16*, int, int, const f16*, int, const float*, const f16*, int, f16*,
                                         f16*, float*, unsigned*, cudaStream_t);
