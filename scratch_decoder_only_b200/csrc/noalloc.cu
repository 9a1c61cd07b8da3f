// Split-K tensor-core GEMM that allocates no device memory.
//
// Some callers cannot call cudaMalloc at the point where they need a GEMM:
// code that runs while a framework's memory pool owns all of the device,
// real-time or serving paths where an allocation (which may synchronise the
// device) is not allowed, and plugins whose host application hands them only
// the operands.  This entry point keeps its split-K partial sums in a fixed
// file-scope __device__ array instead of a per-call workspace.
//
// The array is NOALLOC_SCRATCH_FLOATS fp32 values (16 MiB); every GPU that
// loads the library holds it until the process exits.  All calls share it:
// calls whose GPU work overlaps (different streams, no ordering between them)
// race on it, so order them (one stream, or events).
//
// The GEMM's bounded waits report a wait that gave up in a device error word
// of this file.  Word 0 belongs to the call in flight: each call clears it on
// its stream before the GEMM, and the summation kernel, seeing it set, writes
// NaN into C instead of a partial product and copies the bits into word 1,
// which stays set until gpt_noalloc_status reads and clears it.
#include <mutex>
#include "gpt.h"
#include "launch.h"

#define NOALLOC_SCRATCH_FLOATS (4u << 20)
#define NOALLOC_MAX_DEVICES 64

static __device__ __align__(256) float g_noalloc_scratch[NOALLOC_SCRATCH_FLOATS];
static __device__ __align__(16) unsigned g_noalloc_err[4];

// Device addresses of the two arrays, looked up once per device with that
// device current (the host-side names are only stand-ins, not device addresses).
static std::mutex g_noalloc_mu;
static float* g_scratch_dev[NOALLOC_MAX_DEVICES];
static unsigned* g_err_dev[NOALLOC_MAX_DEVICES];

static int noalloc_setup(int dev) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_scratch_dev[dev]) return GPT_OK;
  void* p = nullptr;
  void* e = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess ||
      cudaGetSymbolAddress(&e, g_noalloc_err) != cudaSuccess) {
    cudaGetLastError();
    set_global_error("gpt_gemm_bf16_splitk_noalloc: cudaGetSymbolAddress failed");
    return GPT_ERR_CUDA;
  }
  g_err_dev[dev] = (unsigned*)e;
  g_scratch_dev[dev] = (float*)p;
  return GPT_OK;
}

// C[m, n] = sum over splits of the partial slabs (fixed order: deterministic),
// or NaN everywhere when this call's GEMM recorded a wait that gave up.
__global__ void noalloc_splitk_sum(const float* __restrict__ ws, int splits, long slab, int ldw, int M, int N,
                                   float* __restrict__ C, long ldc, unsigned* __restrict__ errw) {
  const unsigned bad = *(volatile unsigned*)errw;
  if (bad && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(errw + 1, bad);
  const long total = (long)M * N;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const long r = i / N, c = i % N;
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += ws[s * slab + r * ldw + c];
    C[r * ldc + c] = bad ? __int_as_float(0x7fc00000) : acc;
  }
}

extern "C" int gpt_gemm_bf16_splitk_noalloc(int M, int N, int K, const void* A, long lda, int a_t, const void* B,
                                            long ldb, int b_t, int splits, float* C, long ldc, void* stream) {
  if (!A || !B || !C || M < 1 || N < 1 || K < 1 || ldc < N || splits < 1 || splits > 16) {
    set_global_error("gpt_gemm_bf16_splitk_noalloc: bad argument (NULL pointer, size < 1, ldc < N or splits "
                     "outside 1..16)");
    return GPT_ERR_ARG;
  }
  if (!gemm_tc_supported(M, N, K, lda, a_t != 0, ldb, b_t != 0)) {
    set_global_error("gpt_gemm_bf16_splitk_noalloc: lda and ldb must be multiples of 8");
    return GPT_ERR_ARG;
  }
  // every split gets at least one 64-wide k-block
  const int kb_total = (K + 63) / 64;
  const int kbs = (kb_total + splits - 1) / splits;
  splits = (kb_total + kbs - 1) / kbs;
  // partial slabs keep 16-byte rows (the GEMM stores them by TMA)
  const int ldw = (N + 3) & ~3;
  if ((unsigned long long)splits * M * ldw > NOALLOC_SCRATCH_FLOATS) {
    set_global_error("gpt_gemm_bf16_splitk_noalloc: splits * M * round_up(N, 4) exceeds the fixed scratch of "
                     "4194304 floats");
    return GPT_ERR_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES) {
    cudaGetLastError();
    set_global_error("gpt_gemm_bf16_splitk_noalloc: no usable current device");
    return GPT_ERR_CUDA;
  }
  int r = noalloc_setup(dev);
  if (r != GPT_OK) return r;
  float* ws = g_scratch_dev[dev];
  EpiParams<bf16> e;
  memset(&e, 0, sizeof(e));
  e.kind = EPI_F32_SPLIT;
  e.outf = ws;
  e.ld_outf = ldw;
  e.split_stride = (long)M * ldw;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned* errw = g_err_dev[dev];
  cudaError_t ce = cudaMemsetAsync(errw, 0, sizeof(unsigned), s);
  if (ce == cudaSuccess)
    ce = launch_gemm_tc(M, N, K, (const bf16*)A, lda, a_t != 0, (const bf16*)B, ldb, b_t != 0, e, splits, errw, s);
  if (ce == cudaSuccess) {
    noalloc_splitk_sum<<<148 * 4, 256, 0, s>>>(ws, splits, (long)M * ldw, ldw, M, N, C, ldc, errw);
    ce = cudaGetLastError();
    if (ce == cudaSuccess) ++g_kernel_launches;
  }
  if (ce != cudaSuccess) {
    set_global_error(cudaGetErrorString(ce));
    return GPT_ERR_CUDA;
  }
  return GPT_OK;
}

extern "C" int gpt_noalloc_status(void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES) {
    cudaGetLastError();
    set_global_error("gpt_noalloc_status: no usable current device");
    return GPT_ERR_CUDA;
  }
  int r = noalloc_setup(dev);
  if (r != GPT_OK) return r;
  unsigned bits = 0;
  cudaError_t ce = cudaStreamSynchronize((cudaStream_t)stream);
  if (ce == cudaSuccess) ce = cudaMemcpy(&bits, g_err_dev[dev] + 1, sizeof(bits), cudaMemcpyDeviceToHost);
  if (ce == cudaSuccess && bits) ce = cudaMemset(g_err_dev[dev] + 1, 0, sizeof(bits));
  if (ce != cudaSuccess) {
    set_global_error(cudaGetErrorString(ce));
    return GPT_ERR_CUDA;
  }
  if (bits) {
    set_global_error("gpt_gemm_bf16_splitk_noalloc: a bounded wait in the GEMM gave up; C was set to NaN");
    return GPT_ERR_TIMEOUT;
  }
  return GPT_OK;
}
