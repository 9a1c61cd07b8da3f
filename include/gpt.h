/*
 * gpt.h -- C ABI of libgpt.so: one training step of a GPT-style decoder-only
 * transformer, and greedy decoding with a KV cache, on one NVIDIA B200
 * (sm_100a).
 *
 * The calls follow the pages' statement of the problem: a language model is a
 * function from the start of a text to a probability for every next token;
 * generating means picking a token, appending it and repeating; training means
 * raising the probability of the token that really came next ("Smallem -- Le
 * projet et ses regles", section "Ce qu'est un modele de langage").
 *
 * Conventions for every call:
 *  - Return value: 0 (GPT_OK) or a negative GPT_ERR_* code.  On error the
 *    call has enqueued no work and gpt_last_error() describes the cause.
 *  - Pointers documented as "device" must point to CUDA device memory of the
 *    current device, owned by the caller, valid until the set stream reaches
 *    the call.  Pointers documented as "host" are ordinary host memory.
 *  - Work is enqueued asynchronously on the stream given to gpt_set_stream
 *    (the default stream until then).  Only gpt_create, gpt_get_*,
 *    gpt_set_*, gpt_status and gpt_greedy_decode's argument checks block.
 *  - The library owns parameters, fp32 master weights, AdamW moments,
 *    gradients, activations and the KV cache, in one device arena allocated
 *    by gpt_create and freed by gpt_destroy.
 *  - Bad token / target / segment ids found on the device are clamped (no
 *    memory fault) and recorded in a sticky device error word, which
 *    gpt_status reports (GPT_ERR_DEVICE) and clears.
 *  - A model handle is not thread safe: one host thread at a time.  Some
 *    launch state is process-wide (the decode-graph capture switches on
 *    programmatic dependent launch for the kernels it records; per-kernel
 *    occupancy and tensor-map caches), so drive all handles of a process
 *    from one host thread.
 */
#ifndef GPT_H_
#define GPT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPT_OK            0
#define GPT_ERR_ARG      -1  /* NULL pointer, size out of range, bad config  */
#define GPT_ERR_STATE    -2  /* call order violated (e.g. backward w/o loss) */
#define GPT_ERR_CUDA     -3  /* a CUDA runtime call failed                   */
#define GPT_ERR_TIMEOUT  -4  /* a bounded device-side wait gave up           */
#define GPT_ERR_DEVICE   -5  /* sticky device flag: bad ids were clamped     */
#define GPT_ERR_NOMEM    -6  /* the arena does not fit in device memory      */

#define GPT_PRECISION_FP32 0
#define GPT_PRECISION_BF16 1
#define GPT_PRECISION_FP16 2

/* Device error word bits (reported through gpt_status / gpt_device_error). */
#define GPT_DEVERR_TOKEN   1u   /* token id outside [0, vocab)                */
#define GPT_DEVERR_TARGET  2u   /* target id outside [-1, vocab)              */
#define GPT_DEVERR_SEGMENT 4u   /* seg_ids decrease inside a row              */
#define GPT_DEVERR_TIMEOUT 8u   /* a bounded wait in a kernel gave up         */
#define GPT_DEVERR_POS     16u  /* position beyond max_seq (decode)           */

/*
 * Model shape and numerics.  Architecture: token embedding plus a learned
 * position embedding added to it, n_layers pre-LayerNorm blocks (causal
 * multi-head attention, then a GELU MLP, each added back to the residual),
 * a final LayerNorm and a projection to the vocabulary ("Feste: GPT-2 from
 * scratch in Rust", section "Model Architecture mirrors GPT-2"; "LucilleAI",
 * section "Architecture (from source)").
 *
 *  vocab          real vocabulary size V (softmax / argmax over 0..V-1)
 *  vocab_padded   LM-head width Vp >= V; rows V..Vp-1 of the embedding and
 *                 head are zero-initialised and receive zero gradient
 *  d_model        C; must be a multiple of 8 and of n_heads, at most 1024
 *  n_heads        H; head size d = C / H must be 16, 32, 64 or 128
 *  d_mlp          F; multiple of 8
 *  n_layers       L >= 1
 *  max_seq        largest T (also the number of position-embedding rows)
 *  max_batch      largest B accepted by gpt_forward_loss / decode
 *  tied           1: the LM head reuses the token embedding matrix
 *  precision      GPT_PRECISION_FP32 (fp32 everywhere, SIMT FFMA),
 *                 GPT_PRECISION_BF16 (bf16 GEMM/attention operands and
 *                 activations, fp32 accumulate, fp32 master weights, moments
 *                 and weight gradients; tcgen05 tensor cores) or
 *                 GPT_PRECISION_FP16 (the same with fp16 in place of bf16:
 *                 the pages' FP16 AMP with a loss scaler, "LucilleAI",
 *                 "Architecture (from source)": autocast FP16 + GradScaler;
 *                 use loss_scaling = 1)
 *  loss_scaling   1: dynamic loss scale (x0.5 and skip on a non-finite
 *                 gradient, x2 after 2000 finite steps); 0: scale fixed at 1
 *                 (the non-finite skip stays on)
 *  init_loss_scale  starting scale when loss_scaling = 1 (e.g. 32768)
 *  ln_eps         LayerNorm epsilon (1e-5, biased variance)
 *  init_std       std of the N(0, init_std) initial weight matrices (0.02)
 *  arch           GPT_ARCH_GPT2 (the block above) or GPT_ARCH_LLAMA: a
 *                 Llama-style block ("NTransformer" page, "key features":
 *                 Llama architecture with RoPE, GQA, SwiGLU and a KV cache)
 *                 -- RMSNorm in place of LayerNorm (gains only), no position
 *                 table: queries and keys rotated by their position inside
 *                 the document (consecutive pairs (2i, 2i+1) by pos *
 *                 rope_base^(-2i/d)), n_kv_heads key/value heads shared by
 *                 n_heads / n_kv_heads query heads each, a SwiGLU MLP
 *                 (silu(x W_gate^T) * (x W_up^T)) W_down^T, no biases.
 *                 Needs 16-bit precision and head size 64.
 *  n_kv_heads     Llama: key/value heads, dividing n_heads (0: n_heads)
 *  rope_base      Llama: rotary base (10000)
 */
#define GPT_ARCH_GPT2  0
#define GPT_ARCH_LLAMA 1
typedef struct {
  int32_t vocab, vocab_padded, d_model, n_heads, d_mlp, n_layers, max_seq, max_batch;
  int32_t tied, precision, loss_scaling;
  float init_loss_scale;
  float ln_eps, init_std;
  int32_t arch, n_kv_heads;
  float rope_base;
} gpt_config;

/* AdamW with decoupled weight decay ("Feste", section "Manual
 * Backpropagation from scratch") after global L2 clipping to clip_norm
 * ("RustGPT", section "Technical implementation": L2 norm capped at 5.0):
 * coef = min(1, clip_norm / (||g|| + 1e-6)).  Weight decay applies to every
 * parameter. */
typedef struct {
  float lr, beta1, beta2, eps, weight_decay, clip_norm;
} gpt_adamw;

typedef struct gpt_model gpt_model;   /* opaque */

/* Optimiser / loss-scale scalars, read back by gpt_get_scalars. */
typedef struct {
  float loss_scale;      /* current dynamic loss scale                       */
  int32_t good_steps;    /* consecutive finite steps since the last change   */
  int32_t step;          /* AdamW steps taken (skipped steps do not count)   */
  float last_loss;       /* loss of the latest gpt_forward_loss with targets */
  float last_grad_norm;  /* unscaled global L2 norm of the latest step       */
  int32_t last_skipped;  /* 1 if the latest step was skipped (non-finite)    */
  float last_lr;         /* learning rate the latest taken step used         */
} gpt_scalars;

/* Learning-rate schedule evaluated on the device from the AdamW step counter
 * (the number of steps taken before the one being computed, s = 0, 1, ...;
 * skipped steps do not advance it), so that a step captured in a CUDA graph
 * still follows the schedule when replayed.  The pages' SFT recipe trains
 * with a cosine schedule, warm-up steps and a floor ("LucilleAI", "Getting
 * started": --lr-scheduler cosine --warmup-steps 100 --min-lr 0.00003):
 *   GPT_LR_CONSTANT  lr = gpt_adamw.lr of each gpt_clip_adamw_step call
 *   GPT_LR_COSINE    s <  warmup_steps: lr = max_lr * (s + 1) / warmup_steps
 *                    s >= total_steps:  lr = min_lr
 *                    otherwise, with r = (s - warmup_steps) / (total_steps -
 *                    warmup_steps): lr = min_lr + (max_lr - min_lr) *
 *                    (1 + cos(pi r)) / 2
 * With a cosine schedule set, gpt_adamw.lr is ignored. */
#define GPT_LR_CONSTANT 0
#define GPT_LR_COSINE   1
typedef struct {
  int32_t kind;            /* GPT_LR_CONSTANT or GPT_LR_COSINE             */
  int32_t warmup_steps;    /* >= 0                                          */
  int32_t total_steps;     /* > warmup_steps                                */
  float max_lr, min_lr;    /* 0 <= min_lr <= max_lr                         */
} gpt_lr_schedule;

/* Validate cfg, size and allocate the device arena, initialise parameters
 * from seed (weights N(0, init_std) drawn per canonical element from
 * SplitMix64 + Box-Muller, LayerNorm gains 1, biases and shifts 0, padded
 * vocabulary rows 0), and return a handle in *out.  Synchronous.
 * Errors: GPT_ERR_ARG (bad cfg / NULL), GPT_ERR_NOMEM, GPT_ERR_CUDA. */
int gpt_create(const gpt_config* cfg, uint64_t seed, gpt_model** out);

/* Free the arena and the handle.  NULL is ignored.  Synchronises. */
void gpt_destroy(gpt_model* m);

/* Enqueue all later work on this cudaStream_t (NULL = legacy default). */
int gpt_set_stream(gpt_model* m, void* cuda_stream);

/* Forward pass over tokens [B, T] (device int32, row-major).
 *  targets  device int32 [B, T]: next-token ids, -1 = ignored; NULL = no
 *           loss (the logits of the last forward stay readable through
 *           gpt_get_logits and no backward is possible).
 *  seg_ids  device int32 [B, T]: document id of each token, non-decreasing
 *           inside a row (sequence packing: a token attends only to earlier
 *           tokens of its own document and its position restarts at 0 at
 *           each document -- "LucilleAI", sections "What makes it special"
 *           and "Real measured numbers"); NULL = one document per row.
 *  loss_dev device float[1] receiving the mean cross-entropy over valid
 *           targets ("RustGPT", "Technical implementation": cross-entropy
 *           loss); may be NULL.
 * Requires 1 <= B <= max_batch, 1 <= T <= max_seq.
 * With targets the logits buffer is overwritten by the loss gradient. */
int gpt_forward_loss(gpt_model* m, const int32_t* tokens, const int32_t* targets,
                     const int32_t* seg_ids, int B, int T, float* loss_dev);

/* Backward pass by the chain rule ("Feste", section "Manual Backpropagation
 * from scratch") for the latest gpt_forward_loss with targets.  Overwrites
 * all parameter gradients (fp32, canonical layout, multiplied by the current
 * loss scale).  Errors: GPT_ERR_STATE if no forward with targets preceded. */
int gpt_backward(gpt_model* m);

/* Gradient accumulation over micro-batches.  gpt_backward_accumulate is
 * gpt_backward except that it adds this micro-batch's gradient to the stored
 * gradients instead of overwriting them; gpt_set_loss_weight(w) multiplies
 * the loss gradient of every later gpt_forward_loss by w (default 1; the
 * reported loss stays the plain mean).  With k micro-batches of equal valid
 * target counts, weight 1/k, one gpt_backward and k - 1 accumulating
 * backwards give the gradient of the mean loss over all of them, which one
 * gpt_clip_adamw_step then applies (the pages train with FP16 accumulation
 * and a loss scaler on a 4 GB GPU: "LucilleAI", "Why it matters",
 * "Architecture (from source)").  gpt_set_loss_weight synchronises.
 * Errors: GPT_ERR_STATE (no forward with targets), GPT_ERR_ARG (w <= 0 or
 * not finite). */
int gpt_backward_accumulate(gpt_model* m);
int gpt_set_loss_weight(gpt_model* m, float w);

/* Unscale, clip and update: g <- g / loss_scale; if any g is not finite the
 * step is skipped (parameters and moments unchanged, scale halved when
 * loss_scaling = 1); otherwise the global L2 norm is clipped and AdamW
 * updates the fp32 master weights and refreshes the bf16 working copy.
 *  grad_norm_dev  device float[1]: the unscaled global norm (may be NULL)
 *  skipped_dev    device int32[1]: 1 if skipped, else 0 (may be NULL) */
int gpt_clip_adamw_step(gpt_model* m, const gpt_adamw* hp, float* grad_norm_dev,
                        int32_t* skipped_dev);

/* Greedy decoding ("RustGPT", "Technical implementation": greedy decoding):
 * prefill over prompt [B, Tp] (device int32), then n_new tokens, each the
 * argmax (lowest index on ties) of the fp32 logits over 0..V-1 at the last
 * position, appended and fed back through a per-layer KV cache.
 *  out  device int32 [B, n_new].
 * Requires 1 <= B <= max_batch, Tp >= 1, n_new >= 1, Tp + n_new - 1 <= max_seq.
 * Errors: GPT_ERR_ARG, GPT_ERR_STATE (sequence too long). */
int gpt_greedy_decode(gpt_model* m, const int32_t* prompt, int B, int Tp, int n_new,
                      int32_t* out);

/* Sampling controls for gpt_sample_decode. */
typedef struct {
  float temperature;   /* > 0: logits divided by it; 0: greedy            */
  int32_t top_k;       /* keep the top_k largest logits (0: no top-k)     */
  float top_p;         /* keep the smallest top-probability prefix whose  */
                       /* mass reaches top_p (1: no top-p); 0 < top_p <= 1 */
} gpt_sampling;

/* Sampled decoding: as gpt_greedy_decode, but every new token is drawn from
 * the fp32 logits of the last position ("RustGPT", roadmap "high-priority
 * feature requests": temperature scaling, top-k, top-p; "LucilleAI" lists a
 * sampler in its GPU stack), in this order: x = z / temperature over the real
 * vocabulary; top-k keeps the top_k largest x (ties at the cut to the lower
 * index); weights w = exp(x - max x) over the kept tokens; top-p keeps the
 * shortest prefix, in (w descending, index ascending) order, whose weight
 * reaches top_p times the kept total; the token is the first kept one, in
 * ascending token order, at which the running weight exceeds u times the
 * kept total.  The random numbers are inputs:
 *  uniforms  device float [B, n_new], values in [0, 1): column s is the draw
 *            for new token s of each row.
 * Requires vocab <= 55000 (the row is held in shared memory).
 * Errors: as gpt_greedy_decode; GPT_ERR_ARG for bad controls. */
int gpt_sample_decode(gpt_model* m, const int32_t* prompt, int B, int Tp, int n_new, const gpt_sampling* sp,
                      const float* uniforms, int32_t* out);

/* Beam search ("RustGPT", roadmap "high-priority feature requests": beam
 * search): per prompt, the `width` continuations of n_new tokens with the
 * largest sum of next-token log-probabilities (fp32 log-softmax over the real
 * vocabulary).  Each step extends every kept beam by every token and keeps
 * the best `width` (score descending, ties to the lower parent * V + token,
 * parents counted by their place in the previous order); the first step
 * extends the prompt alone.  No end token, no length normalisation.
 *  prompt  device int32 [B, Tp]
 *  out     device int32 [B, width, n_new]: the beams' tokens, best first
 *  scores  device float [B, width]: their summed log-probabilities
 * The beams share the prompt's cache rows and never copy the key/value cache:
 * each reads its earlier positions through a table of source rows.
 * Requires 1 <= width <= 8, width <= vocab <= 55000, B * width <= max_batch
 * and <= 32, Tp + n_new - 1 <= max_seq.
 * Errors: GPT_ERR_ARG, GPT_ERR_STATE (sequence too long). */
int gpt_beam_decode(gpt_model* m, const int32_t* prompt, int B, int Tp, int n_new, int width, int32_t* out,
                    float* scores);

/* Number of parameters N in the canonical layout:
 *  wte[Vp,C], wpe[max_seq,C]; per layer ln1_g[C], ln1_b[C], w_qkv[3C,C]
 *  (rows: q, then k, then v; head h = rows h*d..h*d+d-1 of each), b_qkv[3C],
 *  w_o[C,C], b_o[C], ln2_g[C], ln2_b[C], w_fc[F,C], b_fc[F], w_fc2[C,F],
 *  b_fc2[C]; then lnf_g[C], lnf_b[C]; then w_head[Vp,C] only if untied.
 * Llama-style (Hkv key/value heads): wte[Vp,C]; per layer attn_norm_g[C],
 *  w_qkv[C + 2*Hkv*d, C] (q rows, then the key heads', then the value
 *  heads'), w_o[C,C], mlp_norm_g[C], w_gu[2F,C] (gate rows, then up rows),
 *  w_down[C,F]; then norm_g[C]; then w_head[Vp,C] only if untied. */
int gpt_num_params(const gpt_model* m, size_t* n);

/* Copy N fp32 values (canonical layout) between the library and dst/src,
 * which may be host or device memory (cudaMemcpyDefault).  Synchronous.
 * n must equal gpt_num_params.
 *  gpt_get_params / gpt_set_params : fp32 master weights (set also refreshes
 *                                    the bf16 working copy)
 *  gpt_get_grads  / gpt_set_grads  : gradients as stored (x loss scale)
 *  gpt_get_adam_m / gpt_set_adam_m, gpt_get_adam_v / gpt_set_adam_v : moments */
int gpt_get_params(gpt_model* m, float* dst, size_t n);
int gpt_set_params(gpt_model* m, const float* src, size_t n);
int gpt_get_grads(gpt_model* m, float* dst, size_t n);
int gpt_set_grads(gpt_model* m, const float* src, size_t n);
int gpt_get_adam_m(gpt_model* m, float* dst, size_t n);
int gpt_set_adam_m(gpt_model* m, const float* src, size_t n);
int gpt_get_adam_v(gpt_model* m, float* dst, size_t n);
int gpt_set_adam_v(gpt_model* m, const float* src, size_t n);

/* Copy the logits of the latest gpt_forward_loss called with targets = NULL,
 * as fp32 [B*T, Vp] row-major, to dst (host or device).  n = B*T*Vp.
 * Synchronous.  Errors: GPT_ERR_STATE if those logits were overwritten. */
int gpt_get_logits(gpt_model* m, float* dst, size_t n);

/* Copy the residual stream entering block `layer` of the latest forward
 * (layer 0: the embedding sum wte[tok] + wpe[pos]; layer = n_layers: the
 * input of the final LayerNorm) as fp32 [B*T, C] to dst (host or device).
 * n = B*T*C.  Synchronous.  Errors: GPT_ERR_ARG (layer or n out of range),
 * GPT_ERR_STATE (no forward yet). */
int gpt_get_residual(gpt_model* m, int layer, float* dst, size_t n);

/* Read / write the optimiser and loss-scale scalars.  Synchronous.
 * gpt_set_scalars writes loss_scale, good_steps and step only. */
int gpt_get_scalars(gpt_model* m, gpt_scalars* out);
int gpt_set_scalars(gpt_model* m, const gpt_scalars* in);

/* Set (or, with NULL, clear to GPT_LR_CONSTANT) the learning-rate schedule
 * used by later gpt_clip_adamw_step calls.  Synchronous.
 * Errors: GPT_ERR_ARG (kind unknown, warmup_steps < 0, total_steps <=
 * warmup_steps, or not 0 <= min_lr <= max_lr). */
int gpt_set_lr_schedule(gpt_model* m, const gpt_lr_schedule* sched);

/* One training step, gpt_forward_loss + gpt_backward + gpt_clip_adamw_step
 * with the same arguments and results, launched as one CUDA graph: the
 * step's kernels are captured once and the graph is replayed while the
 * pointers, B, T and the hyper-parameters match the captured call (any change
 * captures anew).  Device buffers are read when the step runs, so new tokens
 * written into the same buffers need no new capture.  Falls back to the three
 * calls when profiling is on or the runtime refuses the capture.
 *  tokens, targets  device int32 [B, T]; seg_ids device int32 [B, T] or NULL
 *  loss_dev, grad_norm_dev (device float [1]) and skipped_dev (device int32
 *  [1]) may be NULL.
 * Errors: as the three calls (GPT_ERR_ARG for NULL targets). */
int gpt_train_step(gpt_model* m, const int32_t* tokens, const int32_t* targets, const int32_t* seg_ids, int B, int T,
                   const gpt_adamw* hp, float* loss_dev, float* grad_norm_dev, int32_t* skipped_dev);

/* K training steps in one call, all enqueued without a host round trip:
 * for k = 0..K-1, gpt_forward_loss on tokens + k*B*T (targets, seg_ids
 * likewise; seg_ids may be NULL), gpt_backward and gpt_clip_adamw_step.
 *  tokens, targets  device int32 [K, B, T];  seg_ids device int32 [K, B, T] or NULL
 *  losses_dev       device float [K] (may be NULL): loss of each step
 *  grad_norms_dev   device float [K] (may be NULL): unscaled norm of each step
 *  skipped_dev      device int32 [K] (may be NULL): 1 where a step was skipped
 * Errors: as the three calls, GPT_ERR_ARG for K < 1 or NULL targets. */
int gpt_train_steps(gpt_model* m, const int32_t* tokens, const int32_t* targets, const int32_t* seg_ids, int K,
                    int B, int T, const gpt_adamw* hp, float* losses_dev, float* grad_norms_dev,
                    int32_t* skipped_dev);

/* Synchronise the stream, then return GPT_OK, GPT_ERR_CUDA, GPT_ERR_TIMEOUT
 * or GPT_ERR_DEVICE from the sticky device error word, which is cleared. */
int gpt_status(gpt_model* m);

/* The sticky device error word (GPT_DEVERR_* bits) without clearing it.
 * Synchronous. */
int gpt_device_error(gpt_model* m, uint32_t* bits);

/* Human-readable description of the last error on this handle ("" if none).
 * The string lives until the next call on the handle. */
const char* gpt_last_error(const gpt_model* m);

/* Stand-alone tensor-core GEMM (the library's tcgen05 path), enqueued on
 * `stream` (a cudaStream_t; NULL = legacy default):
 *   C[m, n] = sum_k A(m, k) * B(n, k),  fp32 C with row stride ldc >= N,
 * bf16 A and B in device memory.  A(m, k) = a_t ? A[k*lda + m] : A[m*lda + k];
 * B(n, k) = b_t ? B[k*ldb + n] : B[n*ldb + k].  lda and ldb must be multiples
 * of 8 and A, B 16-byte aligned.  Errors: GPT_ERR_ARG, GPT_ERR_CUDA. */
int gpt_gemm_bf16(int M, int N, int K, const void* A, long lda, int a_t, const void* B, long ldb, int b_t,
                  float* C, long ldc, void* stream);

/* Split-K variant of gpt_gemm_bf16 that allocates no device memory, for
 * callers that cannot call cudaMalloc where they need the product (a memory
 * pool owns the device, an allocation would synchronise a real-time path, or
 * a host application hands a plugin only the operands).  The paper has no
 * counterpart: this is a deployment convenience, not a step of the method.
 *
 * Same operands, layouts and result as gpt_gemm_bf16 (fp32 C[M, N], row
 * stride ldc >= N, any N >= 1); the K range is split into `splits` slices
 * (1..16, reduced so that no slice is empty) whose partial sums live in a
 * fixed file-scope device array of 4194304 floats (16 MiB, held on every GPU
 * that loads the library until the process exits), with rows padded to a
 * multiple of 4 floats, then summed into C in a fixed order.
 * Requires splits * M * round_up(N, 4) <= 4194304, else GPT_ERR_ARG with the
 * reason in gpt_last_error(NULL).  Calls no cudaMalloc / cudaFree.
 * The first call on a device looks up the array's device address with that
 * device current; make that first call before any stream capture.
 * All calls share the array (it keeps the last call's partials): calls whose
 * GPU work overlaps (unordered streams) race on it.
 * A bounded wait inside the GEMM that gives up makes that call write NaN to
 * every element of C and sets a sticky error word, read and cleared by
 * gpt_noalloc_status.
 * Errors: GPT_ERR_ARG, GPT_ERR_CUDA. */
int gpt_gemm_bf16_splitk_noalloc(int M, int N, int K, const void* A, long lda, int a_t, const void* B, long ldb,
                                 int b_t, int splits, float* C, long ldc, void* stream);

/* Status of gpt_gemm_bf16_splitk_noalloc on the current device: synchronises
 * `stream` (a cudaStream_t; NULL = legacy default), then returns
 * GPT_ERR_TIMEOUT if any call since the last gpt_noalloc_status had a bounded
 * device wait give up (its C holds NaN), else GPT_OK, and clears the word.
 * Allocates nothing.  Errors: GPT_ERR_CUDA. */
int gpt_noalloc_status(void* stream);

/* Number of kernels libgpt has launched in this process (all handles).
 * Benchmarks read it before and after a timed region. */
int gpt_kernel_launches(uint64_t* out);

/* Per-kernel-class device timing (tracing).  While enabled, every GEMM,
 * attention, cross-entropy, LayerNorm and optimiser launch of later calls on
 * this handle is bracketed by CUDA events recorded on the handle's stream,
 * together with its algorithmic FLOPs and HBM bytes.  gpt_profile_enable(m, 1)
 * starts a fresh record, (m, 0) stops recording and keeps the record. */
typedef struct {
  char name[24];      /* gemm_fwd, gemm_dgrad, gemm_wgrad, attn_fwd, attn_bwd,
                         xent, ln_fwd, ln_bwd, clip_adamw, bias_grad, embed   */
  int32_t launches;   /* bracketed calls                                      */
  double ms;          /* summed event time                                    */
  double flops;       /* summed algorithmic FLOPs (0 where not applicable)    */
  double bytes;       /* summed algorithmic HBM bytes (0 where not applicable) */
} gpt_prof_entry;
int gpt_profile_enable(gpt_model* m, int on);

/* Synchronise and summarise the record into out[0..max_entries), one entry
 * per class with launches > 0; *n_out receives the number written. */
int gpt_profile_read(gpt_model* m, gpt_prof_entry* out, int max_entries, int* n_out);

/* Fault injection for tests: write value into gradient element index
 * (e.g. +inf to exercise the skip path).  Synchronous, host-side. */
int gpt_debug_poison_grad(gpt_model* m, size_t index, float value);

/* Exercise a bounded device-side wait that can never complete: a kernel
 * waits on a shared-memory mbarrier that nothing arrives on, gives up after
 * about timeout_us microseconds, sets GPT_DEVERR_TIMEOUT and returns.  The
 * call synchronises and returns GPT_ERR_TIMEOUT when the wait gave up as
 * designed (the context stays usable).  For the failure-detection tests. */
int gpt_debug_wait_timeout(gpt_model* m, int timeout_us);

#ifdef __cplusplus
}
#endif
#endif /* GPT_H_ */
