// Shared device helpers for libgpt: element types, 16-byte vector I/O,
// warp reductions, the GELU used by the MLP, the sticky error word and the
// GEMM epilogue description shared by the SIMT and tcgen05 GEMMs.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <math.h>

typedef __nv_bfloat16 bf16;
typedef __half f16;

#define GPT_DEVERR_TOKEN 1u
#define GPT_DEVERR_TARGET 2u
#define GPT_DEVERR_SEGMENT 4u
#define GPT_DEVERR_TIMEOUT 8u
#define GPT_DEVERR_POS 16u

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f(f16 x) { return __half2float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ f16 from_f<f16>(float x) { return __float2half_rn(x); }

// 16 bytes of T moved as one vector and widened to fp32.
template <typename T> struct Vec;
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* o) {
    float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  }
  __device__ __forceinline__ static void store(float* p, const float* i) {
    *reinterpret_cast<float4*>(p) = make_float4(i[0], i[1], i[2], i[3]);
  }
};
template <> struct Vec<bf16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const bf16* p, float* o) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x; o[2 * i + 1] = f.y;
    }
  }
  __device__ __forceinline__ static void store(bf16* p, const float* i) {
    uint4 v;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) h[k] = __floats2bfloat162_rn(i[2 * k], i[2 * k + 1]);
    *reinterpret_cast<uint4*>(p) = v;
  }
};

template <> struct Vec<f16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const f16* p, float* o) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __half22float2(h[i]);
      o[2 * i] = f.x; o[2 * i + 1] = f.y;
    }
  }
  __device__ __forceinline__ static void store(f16* p, const float* i) {
    uint4 v;
    __half2* h = reinterpret_cast<__half2*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) h[k] = __floats2half2_rn(i[2 * k], i[2 * k + 1]);
    *reinterpret_cast<uint4*>(p) = v;
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// GELU, tanh form of GPT-2: 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))).
#define GELU_K 0.7978845608028654f
#define GELU_C 0.044715f
__device__ __forceinline__ float gelu_f(float u) {
  return 0.5f * u * (1.0f + tanhf(GELU_K * (u + GELU_C * u * u * u)));
}
__device__ __forceinline__ float gelu_grad_f(float u) {
  float t = tanhf(GELU_K * (u + GELU_C * u * u * u));
  return 0.5f * (1.0f + t) + 0.5f * u * (1.0f - t * t) * GELU_K * (1.0f + 3.0f * GELU_C * u * u);
}

// Programmatic dependent launch: a kernel launched with the programmatic
// serialization attribute may start while its predecessor in the stream
// finishes; griddep_wait() holds it until the predecessor has completed and
// its writes are visible (a no-op for a normal launch), and
// griddep_release() lets the successor start launching.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Every kernel launched through launch_k (and the tensor-core GEMM) calls
// griddep_wait() before it touches global memory that another kernel writes,
// so each may be launched with programmatic dependent launch: its blocks are
// scheduled, and its set-up runs, while the previous kernel drains.  The
// chain stays ordered because every kernel waits for its predecessor, which
// waited for its own.  g_pdl (default on) turns the launch attribute on.
extern bool g_pdl;
template <typename... KArgs, typename... Args>
static cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  if (!g_pdl) {
    kern<<<grid, block, smem, s>>>(args...);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

__device__ __forceinline__ void set_dev_err(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

// What a GEMM does with its fp32 accumulator acc[m, n].
enum EpiKind {
  EPI_STORE = 0,   // out[m,n] = T(acc + bias[n] + resid[m,n])      (bias/resid optional)
  EPI_GELU = 1,    // u = acc + bias[n]; out[m,n] = T(u); out2[m,n] = T(gelu(u))
  EPI_DGELU = 2,   // out[m,n] = T(acc * gelu'(aux[m,n]))
  EPI_F32 = 3,     // outf[m,n] = acc                                 (fp32)
  EPI_F32_SPLIT = 4, // outf[split][m,n] = acc: split-K partial slab   (fp32)
  EPI_F32_ADD = 5    // outf[m,n] += acc (fp32; split-K slices added in no fixed order onto a zeroed output)
};

template <typename T>
struct EpiParams {
  int kind;
  const float* bias;
  const T* resid; long ld_resid;
  T* out; long ld_out;
  T* out2; long ld_out2;
  const T* aux; long ld_aux;
  float* outf; long ld_outf;
  long split_stride;
  float* colsum;   // GELU' epilogue of the tensor-core GEMM: [ceil(M/128)][N] column sums of out (fp32), or null
  // EPI_STORE on the tensor-core GEMM, no bias or residual: with rowdot set,
  // also rowdot[(b * N/64 + h) * rd_T + t] = out[row, head h] . aux[row, head h]
  // over 64-wide heads, row = b * rd_T + t (out rounded to T first)
  float* rowdot;
  int rd_T;
  int f16;   // tensor-core GEMM: the 16-bit operands and outputs are fp16 (0: bf16)
};

// Apply the epilogue to one element (used by the SIMT GEMM).
template <typename T>
__device__ __forceinline__ void epi_apply1(const EpiParams<T>& p, int m, int n, float acc, int split) {
  switch (p.kind) {
    case EPI_STORE: {
      float v = acc;
      if (p.bias) v += p.bias[n];
      if (p.resid) v += to_f(p.resid[(long)m * p.ld_resid + n]);
      p.out[(long)m * p.ld_out + n] = from_f<T>(v);
    } break;
    case EPI_GELU: {
      float u = acc + (p.bias ? p.bias[n] : 0.f);
      T uq = from_f<T>(u);
      p.out[(long)m * p.ld_out + n] = uq;
      // gelu of the stored pre-activation, so that forward and backward see the same u
      p.out2[(long)m * p.ld_out2 + n] = from_f<T>(gelu_f(to_f(uq)));
    } break;
    case EPI_DGELU: {
      float u = to_f(p.aux[(long)m * p.ld_aux + n]);
      p.out[(long)m * p.ld_out + n] = from_f<T>(acc * gelu_grad_f(u));
    } break;
    case EPI_F32:
      p.outf[(long)m * p.ld_outf + n] = acc;
      break;
    case EPI_F32_SPLIT:
      p.outf[(long)split * p.split_stride + (long)m * p.ld_outf + n] = acc;
      break;
    case EPI_F32_ADD:
      atomicAdd(&p.outf[(long)m * p.ld_outf + n], acc);
      break;
  }
}
