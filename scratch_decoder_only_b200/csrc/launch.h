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
  unsigned dec_cnt;   // arrival counter of the greedy step's argmax CTAs (kept zero)
  unsigned long long attn_pairs;   // allowed (query, key) pairs of the latest packed forward
  float lr;           // learning rate of the latest taken step (set by the finalize kernel)
  float loss_weight;  // multiplies the loss gradient of later forwards (micro-batch weight)
  int sched_kind;     // GPT_LR_CONSTANT / GPT_LR_COSINE
  int sched_warmup, sched_total;
  float sched_max_lr, sched_min_lr;
  unsigned opt_bar, opt_abort;   // grid barrier of the fused optimiser step (zeroed per launch)
};

// ---- kernels.cu: embedding, LayerNorm, cross-entropy, reductions, optimiser
// zero `bytes` bytes at p as a kernel in the dependent-launch chain; p must
// not be in use by a kernel that may still run (the fill starts at once)
cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t s);
cudaError_t launch_prep(const int32_t* tokens, const int32_t* targets, const int32_t* seg, int B, int T,
                        int V, int* tok_out, int* tgt_out, int* pos_out, int* dstart_out,
                        DevScalars* sc, cudaStream_t s);
// wpe may be null (no position table)
template <typename T>
cudaError_t launch_embed_fwd(const int* tok, const int* pos, const float* wte, const float* wpe, T* x,
                             int M, int C, cudaStream_t s);
// b == nullptr: RMSNorm (no mean subtracted, no shift; mean is written as 0)
template <typename T>
cudaError_t launch_ln_fwd(const T* x, const float* g, const float* b, T* y, float* mean, float* rstd,
                          int M, int C, float eps, cudaStream_t s);
// partials: [nblk][3C] = dg | db | column sums of dres_out (the bias gradient of
// the layer whose output gradient dres_out is)
// rms: the RMSNorm backward (no mean term; the db partials are then unused)
// err: device error word for the bounded waits of the bulk-copy form (taken only when given)
template <typename T>
cudaError_t launch_ln_bwd(const T* dy, const T* x, const float* mean, const float* rstd, const float* g,
                          const float* dres_in, float* dres_out, T* dres_out_t, float* partials,
                          int M, int C, int* nblk_out, cudaStream_t s, bool rms = false, unsigned* err = nullptr);
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
  int add;   // 1: dst[n] += sum (gradient accumulation), 0: dst[n] = sum
  RedSeg seg[RED_MAX_SEGS];
};
cudaError_t launch_reduce_segs(const RedSeg* segs, int n, bool add, cudaStream_t s);
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
// also sets sc->lr: the schedule's value at the step counter, or `lr`
cudaError_t launch_opt_finalize(const double* partials, int nblk, float clip, float beta1, float beta2, float lr,
                                DevScalars* sc, float* norm_out, int32_t* skipped_out, cudaStream_t s);
template <typename T>
cudaError_t launch_adamw(float* p, const float* g, float* m, float* v, T* pw, size_t n,
                         float beta1, float beta2, float eps, float wd, const DevScalars* sc,
                         cudaStream_t s);
// norm, clip, skip / loss scale and AdamW in one cooperative launch (at most
// max_blocks blocks: partials holds one double per block)
template <typename T>
cudaError_t launch_clip_adamw_fused(float* p, const float* g, float* m, float* v, T* pw, size_t n, double* partials,
                                    int max_blocks, float clip, float beta1, float beta2, float eps, float wd,
                                    float lr, DevScalars* sc, float* norm_out, int32_t* skipped_out, cudaStream_t s);
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
// Column layout of the fused q/k/v rows and of the key / value gradients.
// One key / value head per query head: qkv rows [q | k | v] of C each.
// Grouped heads (G query heads per key / value head): qkv rows of width qw
// hold the H query heads at 0, the Hkv key heads at kcol and the Hkv value
// heads at vcol; query head h reads key / value head h / G.  The backward
// writes one key and one value gradient per query head: at dkv + row * ld_kv
// + h d (keys) and + v_off + h d (values); grouped heads send them to a
// scratch [rows, 2C] that a reduction sums into the shared heads.
struct AttnLayout {
  int qw, kcol, vcol, G;
  bf16* dkv;
  long ld_kv;
  int v_off;
};
AttnLayout attn_layout_mha(bf16* dqkv, int C);
// f16: the 16-bit tensors hold fp16 values (same layouts; bf16 otherwise);
// lay: null for one key / value head per query head
// lse of the tcgen05 pair is the base-2 log-sum-exp of the scaled scores
// (log2e / sqrt(d) units), the form its backward consumes; the SIMT and
// mma.sync pairs keep the natural log.
// d_real: the true head size of heads zero-padded to 64 columns (64: none)
cudaError_t launch_attn_fwd_tc(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T, int H,
                               unsigned* err, cudaStream_t s, bool f16 = false, const AttnLayout* lay = nullptr,
                               int d_real = 64);
// d_ready: Dbuf [B, H, T] already holds rowsum(dO o O) (written by the GEMM
// epilogue that produced dO); otherwise a row-dot kernel computes it first
// bias_part (plain 64-column heads only): also write the column sums of the
// q|k|v gradient as partial rows [B * ceil(T/128) * 4][3 H 64], one per 32 rows
// (rows b T + 128 kb + 32 q + [0, 32) below T -> row (b ceil(T/128) + kb) 4 + q)
cudaError_t launch_attn_bwd_tc(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dbuf,
                               bool d_ready, float* dq_acc, const int* dstart, bf16* dqkv, int B, int T, int H,
                               unsigned* err, cudaStream_t s, bool f16 = false, const AttnLayout* lay = nullptr,
                               int d_real = 64, float* bias_part = nullptr);
// heads of d < 64 columns (64 % d == 0) on the d = 64 tensor-core kernels:
// copies with every head widened to 64 columns by zeros (pad: src [rows]
// [groups][d] -> dst [rows][groups][64]; !pad: back, the extra columns dropped)
bool attn_tc_pad_supported(int d);
// D[b, h, t] = dO . O over head h's d columns of row b T + t ([rows][H][d])
cudaError_t launch_attn_rowdot(const bf16* out, const bf16* dout, float* Dbuf, int B, int T, int H, int d, bool f16,
                               cudaStream_t s);
cudaError_t launch_attn_pad(const bf16* src, bf16* dst, long rows, int groups, int d, bool pad, cudaStream_t s);

// ---- decode.cu
// decode kernels read the position as pos0 + *step (device counter)
// wpe may be null (no position table); st (optional, C % 16 == 0): per
// 16-column group g and row b, st[g B + b] = (mean, sum of squared
// deviations) of the stored row
template <typename T>
cudaError_t launch_dec_embed(const int* tok, const float* wte, const float* wpe, T* x, int B, int C, int pos0,
                             const int* step, int max_seq, unsigned* err, cudaStream_t s, float2* st = nullptr);
template <typename T>
cudaError_t launch_gemv(const T* X, int B, int K, const T* W, int N, const float* bias, const T* resid,
                        int mode, T* out, T* out2, float* outf, cudaStream_t s);
// q|k|v row layout of a decode step: rows of width qw, query heads at 0, Hkv
// key heads at kcol, Hkv value heads at vcol; the cache holds Hkv heads
// ([B][Hkv][Tmax][d] per layer).  One key/value head per query head:
// {3C, C, 2C, H}.
struct DecLayout {
  int qw, kcol, vcol, Hkv;
  // beam search: src[b * Tmax + t] = the cache row holding position t of
  // row b's sequence (positions before the current one); null: row b itself
  const int* src = nullptr;
};
template <typename T>
cudaError_t launch_kv_fill(const T* qkv, T* kc, T* vc, int B, int Tp, int d, int Tmax, const DecLayout& L,
                           cudaStream_t s);
size_t dec_attn_part_floats(int B, int H, int d);
template <typename T>
// part: dec_attn_part_floats floats; cnt: B * H counters, zero before the
// first launch (every launch leaves them zero)
cudaError_t launch_dec_attn(const T* qkv, T* kc, T* vc, T* out, float* part, unsigned* cnt, int B, int H, int d,
                            int Tmax, int pos0, const int* step, const DecLayout& L, cudaStream_t s);
// The next step's input of a replayed greedy step, made by the argmax kernel:
// x[b] = T(wte[token] + wpe[pos0 + *step + 1]) (wpe may be null), with the
// LayerNorm group statistics in st (optional, C % 16 == 0); the last CTA
// advances *step (== the argmax's step) and resets cnt (zero before use).
template <typename T>
struct GreedyNext {
  const float* wte = nullptr;
  const float* wpe = nullptr;
  T* x = nullptr;
  int C = 0, pos0 = 0, max_seq = 0;
  float2* st = nullptr;
  unsigned* cnt = nullptr;
  int* step = nullptr;
};
// out[b * out_ld + (*step or 0)] = argmax; tok[b] = argmax
template <typename T = float>
cudaError_t launch_argmax(const float* logits, int B, int V, int Vp, int* tok, int32_t* out, int out_ld,
                          const int* step, cudaStream_t s, const GreedyNext<T>* nx = nullptr);
cudaError_t launch_step_advance(int* step, cudaStream_t s);
// sampled choice (temperature, top-k, top-p; temp <= 0: greedy) with the
// uniform uni[b * u_ld + (*step or 0)]; writes tok[b] and out[b * out_ld + col].
// Needs V * 4 bytes of shared memory (at most SMP_MAX_VOCAB tokens).
#define SMP_MAX_VOCAB 55000
cudaError_t launch_sample(const float* logits, int B, int V, int Vp, float temp, int top_k, float top_p,
                          const float* uni, int u_ld, int* tok, int32_t* out, int out_ld, const int* step,
                          cudaStream_t s);
template <typename T>
cudaError_t launch_gather_last(const T* x, int B, int Tp, int C, T* out, cudaStream_t s);

// ---- decode_mma.cu: decode projections of 1-32 rows on mma.sync (16-bit T),
// same modes and outputs as the GEMV (0: + bias + residual, 1: + bias and
// GELU into out / out2, 2: fp32 logits).  X and W 16-byte aligned; K > 768
// runs as clusters of CTAs that split the k range.  With lng the kernel
// first applies LayerNorm (lnb: shift; none: RMSNorm) with eps to the rows
// of X, which then hold the raw residual (K <= 768), from the statistics
// st_in when given, else its own.  st_out (mode 0, N % 16 == 0): the kernel
// also writes, per 16-column group g and row b, st_out[g B + b] = (mean,
// sum of squared deviations) of the stored outputs.
bool dec_mma_supported(int B, int K, int N, bool ln = false);
template <typename T>
cudaError_t launch_dec_mma(const T* X, int B, int K, const T* W, int N, const float* bias, const T* resid, int mode,
                           T* out, T* out2, float* outf, unsigned* err, cudaStream_t s, const float* lng = nullptr,
                           const float* lnb = nullptr, float eps = 0.f, float2* st_out = nullptr,
                           const float2* st_in = nullptr);

// ---- beam.cu: beam search over the decode rows (row r = b * W + w)
#define BEAM_MAX_WIDTH 8
// scores[b W + w] = 0 for w = 0, -inf otherwise; src rows of every beam of
// prompt b point at prefill row b for the prompt's positions t < Tp.
cudaError_t launch_beam_init(int* src, int Tmax, float* scores, int B, int W, int Tp, cudaStream_t s);
// Per row: log-softmax over the real vocabulary (fp32) and the row's W best
// candidates scores[r] + log p (ties to the lower token), into cand_s /
// cand_t [B W][W].  first: the logits of beam (b, w) are row b and only w = 0
// takes part (the others' candidates are -inf).  V * 4 bytes of shared memory.
cudaError_t launch_beam_topk(const float* logits, int Vp, int V, int B, int W, bool first, const float* scores,
                             float* cand_s, int* cand_t, cudaStream_t s);
// Per prompt: the W best of the W x W candidates (score descending, ties to
// the lower parent * V + token); reorders the token history out [B W][out_ld]
// and the source-row table by parent, appends the chosen tokens at column
// (*step or 0), sets scores and the next input tokens tok[B W].
cudaError_t launch_beam_merge(const float* cand_s, const int* cand_t, int B, int W, int V, int Tp, int* src,
                              int Tmax, float* scores, int* tok, int32_t* out, int out_ld, const int* step,
                              cudaStream_t s);

// ---- llama.cu: the Llama-style block's elementwise kernels (16-bit T)
// rotary positions in place on nq query heads at columns [0, nq d) and nk key
// heads at [kcol, kcol + nk d) of rows of stride ld; position pos[r] (or
// pos0 + *step when pos is null); tab: [max_seq][d/2] (cos, sin)
template <typename T>
cudaError_t launch_rope(T* x, long ld, int rows, int nq, int kcol, int nk, int d, const int* pos, int pos0,
                        const int* step, const float2* tab, int max_seq, bool inverse, cudaStream_t s);
// a [rows, F] = silu(gate) * up of gu [rows, 2F] = [gate | up]
template <typename T>
cudaError_t launch_swiglu(const T* gu, T* a, int rows, int F, cudaStream_t s);
// dgu [rows, 2F] = [da * up * silu'(gate) | da * silu(gate)]
template <typename T>
cudaError_t launch_swiglu_bwd(const T* da, const T* gu, T* dgu, int rows, int F, cudaStream_t s);
// per-query-head key / value gradients kvq [rows, 2 H d] summed into the
// Hkv shared heads of dkv (row stride ld; keys at kcol, values at vcol)
template <typename T>
cudaError_t launch_gqa_reduce(const T* kvq, T* dkv, long ld, int kcol, int vcol, int rows, int Hkv, int G, int d,
                              cudaStream_t s);

