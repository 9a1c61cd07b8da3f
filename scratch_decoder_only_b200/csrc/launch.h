// Host-side launchers of the kernels in this directory (internal to libgpt).
// Every launcher enqueues on `s` and returns the cudaGetLastError() status.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include "common.cuh"

// Error text for calls without a model handle (gpt_last_error(NULL)); engine.cu.
void set_global_error(const char* msg);

// Kernels launched by this library since load (bench / tracing counter).
extern unsigned long long g_kernel_launches;

struct DevScalars {
  float loss;         // mean cross-entropy of the latest forward with targets
  float loss_scale;   // dynamic loss scale
  int good_steps;     // finite steps since the last scale change
  int step;           // AdamW steps taken
  float grad_norm;    // unscaled global L2 norm of the latest step
  int skipped;        // latest step skipped
  float coef;         // clip coefficient / loss_scale for the update
  float bc1, bc2;     // AdamW bias corrections 1 - beta^t
  int n_valid;        // valid targets of the latest forward
  int loss_scaling;   // 1: dynamic scale on
  unsigned err;       // sticky device error word
  int dec_step;       // decode step counter
};

// ---- kernels.cu: embedding, LayerNorm, cross-entropy, reductions, optimiser
cudaError_t launch_prep(const int32_t* tokens, const int32_t* targets, const int32_t* seg, int B, int T,
                        int V, int* tok_out, int* tgt_out, int* pos_out, int* dstart_out,
                        DevScalars* sc, cudaStream_t s);
template <typename T>
cudaError_t launch_embed_fwd(const int* tok, const int* pos, const float* wte, const float* wpe, T* x,
                             int M, int C, cudaStream_t s);
template <typename T>
cudaError_t launch_ln_fwd(const T* x, const float* g, const float* b, T* y, float* mean, float* rstd,
                          int M, int C, float eps, cudaStream_t s);
// partials: [nblk][3C] = dg | db | column sums of dres_out (the bias gradient of
// the layer whose output gradient dres_out is)
template <typename T>
cudaError_t launch_ln_bwd(const T* dy, const T* x, const float* mean, const float* rstd, const float* g,
                          const float* dres_in, float* dres_out, T* dres_out_t, float* partials,
                          int M, int C, int* nblk_out, cudaStream_t s);
// Deferred column reductions: for each segment, dst[n] = sum_r src[r * ld + n]
// (n < cols, r < rows, fixed summation order).  Segments are launched in
// lists of RED_MAX_SEGS (the list travels as the kernel parameter).
struct RedSeg {
  const float* src;
  float* dst;
  int rows, cols, ld, blk0;   // blk0: first block of the segment (set by the launcher)
};
#define RED_MAX_SEGS 96
struct RedSegList {
  int n;
  RedSeg seg[RED_MAX_SEGS];
};
cudaError_t launch_reduce_segs(const RedSeg* segs, int n, cudaStream_t s);
// Column sums of x [M, N] as partial rows: partials[r][0..N), *rows_out rows
// (at most (M + 127) / 128), to be summed by a reduction segment.
template <typename Tin>
cudaError_t launch_colsum(const Tin* x, long ldx, int M, int N, float* partials, int* rows_out, cudaStream_t s);
template <typename T>
cudaError_t launch_xent(T* logits, long ldl, const int* tgt, int M, int V, int Vp, float* rowloss,
                        DevScalars* sc, cudaStream_t s);
cudaError_t launch_loss_finalize(const float* rowloss, int M, DevScalars* sc, float* loss_out, cudaStream_t s);
template <typename T>
cudaError_t launch_embed_bwd(const float* dres, const int* tok, const int* pos, float* gwte, float* gwpe,
                             int M, int C, cudaStream_t s);
cudaError_t launch_sumsq(const float* g, size_t n, double* partials, int nblk, cudaStream_t s);
cudaError_t launch_opt_finalize(const double* partials, int nblk, float clip, float beta1, float beta2,
                                DevScalars* sc, float* norm_out, int32_t* skipped_out, cudaStream_t s);
template <typename T>
cudaError_t launch_adamw(float* p, const float* g, float* m, float* v, T* pw, size_t n, float lr,
                         float beta1, float beta2, float eps, float wd, const DevScalars* sc,
                         cudaStream_t s);
template <typename T>
cudaError_t launch_cast(const float* src, T* dst, size_t n, cudaStream_t s);
template <typename T>
cudaError_t launch_to_f32(const T* src, long ld, int rows, int cols, float* dst, cudaStream_t s);
cudaError_t launch_wait_timeout_probe(unsigned* err, long long timeout_cycles, cudaStream_t s);

// ---- gemm_simt.cu: C[M,N] = A(M x K) . B(N x K)^T with epilogue, SIMT FFMA
// A(m,k) = a_t ? A[k*lda + m] : A[m*lda + k];  B(n,k) = b_t ? B[k*ldb + n] : B[n*ldb + k]
template <typename T>
cudaError_t launch_gemm_simt(int M, int N, int K, const T* A, long lda, bool a_t, const T* B, long ldb,
                             bool b_t, const EpiParams<T>& epi, int splits, cudaStream_t s);

// ---- gemm_tc.cu: same contract on tcgen05 tensor cores (bf16 operands)
bool gemm_tc_supported(int M, int N, int K, long lda, bool a_t, long ldb, bool b_t);
cudaError_t launch_gemm_tc(int M, int N, int K, const bf16* A, long lda, bool a_t, const bf16* B, long ldb,
                           bool b_t, const EpiParams<bf16>& epi, int splits, unsigned* err, cudaStream_t s);

// ---- attention.cu (SIMT, any precision) and attention_mma.cu (bf16 tensor cores)
template <typename T>
cudaError_t launch_attn_fwd_simt(const T* qkv, T* out, float* lse, const int* dstart, int B, int T_, int H,
                                 int d, cudaStream_t s);
template <typename T>
cudaError_t launch_attn_bwd_simt(const T* qkv, const T* out, const T* dout, const float* lse, float* Dbuf,
                                 const int* dstart, T* dqkv, int B, int T_, int H, int d, cudaStream_t s);
bool attn_mma_supported(int d);
cudaError_t launch_attn_fwd_mma(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T_,
                                int H, int d, cudaStream_t s);
cudaError_t launch_attn_bwd_mma(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                                float* Dbuf, const int* dstart, bf16* dqkv, int B, int T_, int H, int d,
                                cudaStream_t s);

// ---- attention_tc.cu: head size 64 on tcgen05 (dq_acc: fp32 [B*T, C] scratch)
bool attn_tc_supported(int d);
cudaError_t launch_attn_fwd_tc(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T, int H,
                               unsigned* err, cudaStream_t s);
// d_ready: Dbuf [B, H, T] already holds rowsum(dO o O) (written by the GEMM
// epilogue that produced dO); otherwise a row-dot kernel computes it first
cudaError_t launch_attn_bwd_tc(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dbuf,
                               bool d_ready, float* dq_acc, const int* dstart, bf16* dqkv, int B, int T, int H,
                               unsigned* err, cudaStream_t s);

// ---- decode.cu
// decode kernels read the position as pos0 + *step (device counter)
template <typename T>
cudaError_t launch_dec_embed(const int* tok, const float* wte, const float* wpe, T* x, int B, int C, int pos0,
                             const int* step, int max_seq, unsigned* err, cudaStream_t s);
template <typename T>
cudaError_t launch_gemv(const T* X, int B, int K, const T* W, int N, const float* bias, const T* resid,
                        int mode, T* out, T* out2, float* outf, cudaStream_t s);
template <typename T>
cudaError_t launch_kv_fill(const T* qkv, T* kc, T* vc, int B, int Tp, int H, int d, int Tmax, cudaStream_t s);
size_t dec_attn_part_floats(int B, int H, int d);
template <typename T>
cudaError_t launch_dec_attn(const T* qkv, T* kc, T* vc, T* out, float* part, int B, int H, int d, int Tmax, int pos0,
                            const int* step, cudaStream_t s);
// out[b * out_ld + (*step or 0)] = argmax; tok[b] = argmax
cudaError_t launch_argmax(const float* logits, int B, int V, int Vp, int* tok, int32_t* out, int out_ld,
                          const int* step, cudaStream_t s);
cudaError_t launch_step_advance(int* step, cudaStream_t s);
template <typename T>
cudaError_t launch_gather_last(const T* x, int B, int Tp, int C, T* out, cudaStream_t s);
