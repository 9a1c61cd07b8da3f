// libgpt engine: the device arena, parameter initialisation, the forward /
// backward / optimiser schedule of one training step, greedy decoding, and
// the C ABI declared in include/gpt.h.
//
// Everything of a step is enqueued on one stream; nothing returns to the host
// during a step (loss, grad norm, skip flag and loss scale live in device
// scalars).  Layouts (row-major):
//   parameters  fp32 master p32[N] in canonical order (see gpt.h); gradients,
//               AdamW m and v share that layout; bf16 mode adds a bf16 working
//               copy pw[N] that every GEMM reads.
//   activations [B*T, C] per layer: x (residual input), h1 = LN1(x), qkv
//               [B*T, 3C], att, x_mid, h2 = LN2(x_mid), u = pre-GELU [B*T, F],
//               a = GELU(u); LayerNorm mean / rstd [B*T] fp32; lse [B, H, T].
//   logits      [B*T, ldl], ldl = Vp rounded up to 8 (16-byte rows for TMA);
//               overwritten in place by the loss gradient.
#include <string.h>
#include <math.h>
#include <string>
#include <vector>
#include <thread>
#include <algorithm>
#include <type_traits>
#include "gpt.h"
#include "launch.h"

struct LayerOff {
  size_t ln1_g, ln1_b, w_qkv, b_qkv, w_o, b_o, ln2_g, ln2_b, w_fc, b_fc, w_fc2, b_fc2;
};

struct gpt_model {
  gpt_config cfg;
  int device = 0;
  cudaStream_t stream = 0;
  bool lp = false;     // 16-bit operands and activations (bf16 or fp16)
  bool fp16 = false;   // ... and those are fp16
  // Llama-style block: RMSNorm, rotary positions, Hkv key/value heads, SwiGLU
  bool llama = false;
  int Hkv = 0, QW = 0, UW = 0;     // key/value heads; q|k|v row width; MLP up-projection width (F or 2F)
  float2* rope_tab = nullptr;      // [max_seq][d/2] (cos, sin)
  void* dkvq = nullptr;            // [Mmax, 2C] per-query-head key/value gradients (grouped heads)
  int V, Vp, C, H, d, F, NL, Tmax, Bmax, ldl;
  long Mmax;
  size_t N = 0;
  size_t o_wte, o_wpe, o_lnf_g, o_lnf_b, o_head;
  std::vector<LayerOff> L;
  char* arena = nullptr;
  size_t arena_bytes = 0;
  float *p32, *g32, *m32, *v32;
  void* pw;
  void *xs, *xmid, *h1, *h2, *qkv, *att, *u, *a, *xf, *logits;
  float *mu1, *rs1, *mu2, *rs2, *muf, *rsf, *lse;
  int *tok, *tgt, *pos, *dstart;
  float* dres32;
  void *dres_t, *dC, *dF, *dqkv;
  float *attD, *rowloss, *partials, *dq_acc;
  // heads of d < 64 on the tensor-core attention: q|k|v, O / dO and the
  // q|k|v gradient with every head zero-padded to 64 columns (16-bit)
  void *apad = nullptr, *opad = nullptr, *dqkvpad = nullptr;
  size_t dq_acc_n = 0;
  size_t partials_n;
  double* normpart;
  int normblk = 592;
  DevScalars* sc;
  void *kc, *vc, *dx, *dh, *dq, *datt, *du, *da, *dxf;
  float *dlogits, *dmu, *drs, *dpart;
  unsigned* dacnt = nullptr;    // decode attention: per-(row, head) arrival counters (kept zero)
  float2* dxst = nullptr;       // decode: LayerNorm statistics of the residual rows per 16-column group
  int* dtok;
  int fwd_B = 0, fwd_T = 0;
  bool have_targets = false, logits_valid = false;
  std::string err;
  // tracing: per-kernel-class CUDA-event brackets
  bool seg_used = false;
  // decode: one captured step replayed on an internal stream
  cudaStream_t cap_stream = nullptr;
  cudaEvent_t ev_a = nullptr, ev_b = nullptr;
  cudaGraphExec_t dec_graph = nullptr;
  // gpt_train_step: one captured training step, replayed while its inputs match
  cudaGraphExec_t train_graph = nullptr;
  struct TrainKey {
    const void *tok, *tgt, *seg, *loss, *gn, *skip;
    int B, T;
    float lr, beta1, beta2, eps, wd, clip;
    bool operator==(const TrainKey& o) const { return memcmp(this, &o, sizeof(TrainKey)) == 0; }
  } train_key;
  int train_kernels = 0;
  bool train_graph_ok = true;   // false once a capture failed: plain launches from then on
  int dec_B = 0, dec_Tp = 0, dec_nnew = 0, dec_kernels = 0;
  int32_t* dec_out = nullptr;
  // sampling decode (gpt_sample_decode); smp_on = false: greedy
  bool smp_on = false;
  float smp_temp = 0.f, smp_topp = 1.f;
  int smp_topk = 0;
  const float* smp_u = nullptr;
  // beam search (gpt_beam_decode); beam_w = 0: off.  dsrc [Bmax][Tmax]: the
  // cache row of each (row, position); dbcs / dbct: per-row candidates
  int beam_w = 0;
  float* beam_scores = nullptr;
  int* dsrc = nullptr;
  float* dbcs = nullptr;
  int* dbct = nullptr;
  int dec_beam_w = 0;
  float* dec_beam_scores = nullptr;
  bool dec_smp_on = false;   // the sampling state the captured graph was built with
  float dec_smp_temp = 0.f, dec_smp_topp = 1.f;
  int dec_smp_topk = 0;
  const float* dec_smp_u = nullptr;
  bool prof = false;
  // pair_mult: FLOPs per allowed (query, key) pair of the latest packed
  // forward, whose count the device holds (added at gpt_profile_read)
  struct ProfRec { int cls; cudaEvent_t a, b; double flops, bytes, pair_mult; };
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> evpool;
  size_t evused = 0;
  std::vector<RedSeg> redsegs;   // deferred column reductions of the current backward pass
  bool accum_now = false;        // the backward in progress adds to the stored gradients
};

enum ProfCls { PC_GEMM_FWD, PC_GEMM_DX, PC_GEMM_DW, PC_ATTN_FWD, PC_ATTN_BWD, PC_XENT, PC_LN_FWD, PC_LN_BWD,
               PC_OPT, PC_BIAS, PC_EMBED, PC_COUNT };
static const char* kProfNames[PC_COUNT] = {"gemm_fwd", "gemm_dgrad", "gemm_wgrad", "attn_fwd", "attn_bwd",
                                           "xent", "ln_fwd", "ln_bwd", "clip_adamw", "bias_grad", "embed"};

static cudaEvent_t prof_event(gpt_model* m) {
  if (m->evused == m->evpool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    m->evpool.push_back(e);
  }
  return m->evpool[m->evused++];
}

// Brackets the launches made during its lifetime with two events.
struct ProfScope {
  gpt_model* m;
  long idx = -1;
  ProfScope(gpt_model* mm, int cls, double flops, double bytes, double pair_mult = 0.0) : m(mm) {
    if (!m->prof) return;
    cudaEvent_t a = prof_event(m);
    if (!a) return;
    cudaEventRecord(a, m->stream);
    m->recs.push_back({cls, a, nullptr, flops, bytes, pair_mult});
    idx = (long)m->recs.size() - 1;
  }
  ~ProfScope() {
    if (idx < 0) return;
    cudaEvent_t b = prof_event(m);
    if (!b) { m->recs.pop_back(); return; }
    cudaEventRecord(b, m->stream);
    m->recs[idx].b = b;
  }
};

#define FAIL(code, msg)            \
  do {                             \
    m->err = (msg);                \
    return (code);                 \
  } while (0)
#define CK(x)                                                                       \
  do {                                                                              \
    cudaError_t e_ = (x);                                                           \
    if (e_ != cudaSuccess) {                                                        \
      m->err = std::string(#x) + ": " + cudaGetErrorString(e_);                     \
      return GPT_ERR_CUDA;                                                          \
    }                                                                               \
  } while (0)
#define CKI(x)                   \
  do {                           \
    int r_ = (x);                \
    if (r_ != GPT_OK) return r_; \
  } while (0)

// ---------------------------------------------------------------------------
// Parameter layout and initialisation
// ---------------------------------------------------------------------------
static void layout_params(gpt_model* m) {
  size_t o = 0;
  size_t C = m->C, F = m->F, Vp = m->Vp;
  if (m->llama) {
    // wte; per layer attn_norm_g, w_qkv [QW, C], w_o, mlp_norm_g, w_gu [2F, C],
    // w_down [C, F]; norm_g; head if untied (no position table, no biases:
    // the unused offsets are left at 0 and never read)
    m->o_wte = o; o += Vp * C;
    m->o_wpe = 0;
    m->L.assign(m->NL, LayerOff{});
    for (int l = 0; l < m->NL; ++l) {
      LayerOff& lo = m->L[l];
      lo.ln1_g = o; o += C;
      lo.w_qkv = o; o += (size_t)m->QW * C;
      lo.w_o = o; o += C * C;
      lo.ln2_g = o; o += C;
      lo.w_fc = o; o += 2 * F * C;
      lo.w_fc2 = o; o += C * F;
    }
    m->o_lnf_g = o; o += C;
    m->o_lnf_b = 0;
    if (m->cfg.tied) {
      m->o_head = m->o_wte;
    } else {
      m->o_head = o; o += Vp * C;
    }
    m->N = o;
    return;
  }
  m->o_wte = o; o += Vp * C;
  m->o_wpe = o; o += (size_t)m->Tmax * C;
  m->L.resize(m->NL);
  for (int l = 0; l < m->NL; ++l) {
    LayerOff& lo = m->L[l];
    lo.ln1_g = o; o += C;
    lo.ln1_b = o; o += C;
    lo.w_qkv = o; o += 3 * C * C;
    lo.b_qkv = o; o += 3 * C;
    lo.w_o = o; o += C * C;
    lo.b_o = o; o += C;
    lo.ln2_g = o; o += C;
    lo.ln2_b = o; o += C;
    lo.w_fc = o; o += F * C;
    lo.b_fc = o; o += F;
    lo.w_fc2 = o; o += C * F;
    lo.b_fc2 = o; o += C;
  }
  m->o_lnf_g = o; o += C;
  m->o_lnf_b = o; o += C;
  if (m->cfg.tied) {
    m->o_head = m->o_wte;
  } else {
    m->o_head = o; o += Vp * C;
  }
  m->N = o;
}

// SplitMix64 output k for a seed (Steele, Lea, Flood 2014; Vigna's reference
// splitmix64.c): state after k+1 golden-ratio increments, then the finaliser.
static inline uint64_t splitmix64_at(uint64_t seed, uint64_t k) {
  uint64_t z = seed + (k + 1) * 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// Box-Muller (1958) normal deviate for canonical element e, from draws 2e, 2e+1.
static inline double normal_at(uint64_t seed, uint64_t e) {
  uint64_t x1 = splitmix64_at(seed, 2 * e), x2 = splitmix64_at(seed, 2 * e + 1);
  double u1 = ((double)(x1 >> 11) + 1.0) * 0x1.0p-53;
  double u2 = (double)(x2 >> 11) * 0x1.0p-53;
  return sqrt(-2.0 * log(u1)) * cos(2.0 * M_PI * u2);
}

static void fill_normal(std::vector<float>& h, size_t off, size_t n, uint64_t seed, double stddev) {
  unsigned nt = std::max(1u, std::min(32u, std::thread::hardware_concurrency()));
  if (n < 65536) nt = 1;
  std::vector<std::thread> th;
  for (unsigned t = 0; t < nt; ++t) {
    size_t a = off + n * t / nt, b = off + n * (t + 1) / nt;
    th.emplace_back([&h, a, b, seed, stddev]() {
      for (size_t e = a; e < b; ++e) h[e] = (float)(stddev * normal_at(seed, e));
    });
  }
  for (auto& x : th) x.join();
}

static void init_host_params(gpt_model* m, uint64_t seed, std::vector<float>& h) {
  h.assign(m->N, 0.f);
  size_t C = m->C, F = m->F;
  double sd = m->cfg.init_std;
  auto zero_pad_rows = [&](size_t off) {
    for (size_t r = (size_t)m->V; r < (size_t)m->Vp; ++r)
      for (size_t c = 0; c < C; ++c) h[off + r * C + c] = 0.f;
  };
  if (m->llama) {
    fill_normal(h, m->o_wte, (size_t)m->Vp * C, seed, sd);
    zero_pad_rows(m->o_wte);
    for (auto& lo : m->L) {
      for (size_t i = 0; i < C; ++i) { h[lo.ln1_g + i] = 1.f; h[lo.ln2_g + i] = 1.f; }
      fill_normal(h, lo.w_qkv, (size_t)m->QW * C, seed, sd);
      fill_normal(h, lo.w_o, C * C, seed, sd);
      fill_normal(h, lo.w_fc, 2 * F * C, seed, sd);
      fill_normal(h, lo.w_fc2, C * F, seed, sd);
    }
    for (size_t i = 0; i < C; ++i) h[m->o_lnf_g + i] = 1.f;
    if (!m->cfg.tied) {
      fill_normal(h, m->o_head, (size_t)m->Vp * C, seed, sd);
      zero_pad_rows(m->o_head);
    }
    return;
  }
  fill_normal(h, m->o_wte, (size_t)m->Vp * C, seed, sd);
  zero_pad_rows(m->o_wte);
  fill_normal(h, m->o_wpe, (size_t)m->Tmax * C, seed, sd);
  for (auto& lo : m->L) {
    for (size_t i = 0; i < C; ++i) { h[lo.ln1_g + i] = 1.f; h[lo.ln2_g + i] = 1.f; }
    fill_normal(h, lo.w_qkv, 3 * C * C, seed, sd);
    fill_normal(h, lo.w_o, C * C, seed, sd);
    fill_normal(h, lo.w_fc, F * C, seed, sd);
    fill_normal(h, lo.w_fc2, C * F, seed, sd);
  }
  for (size_t i = 0; i < C; ++i) h[m->o_lnf_g + i] = 1.f;
  if (!m->cfg.tied) {
    fill_normal(h, m->o_head, (size_t)m->Vp * C, seed, sd);
    zero_pad_rows(m->o_head);
  }
}

// ---------------------------------------------------------------------------
// Arena
// ---------------------------------------------------------------------------
struct Carver {
  size_t off = 0;
  std::vector<std::pair<void**, size_t>> items;
  void add(void** p, size_t bytes) {
    off = (off + 255) & ~(size_t)255;
    items.push_back({p, off});
    off += bytes;
  }
};

static int build_arena(gpt_model* m) {
  size_t es = m->lp ? 2 : 4;
  size_t N = m->N, C = m->C, F = m->F, Mx = m->Mmax, NL = m->NL;
  Carver cv;
  cv.add((void**)&m->p32, N * 4);
  cv.add((void**)&m->g32, N * 4);
  cv.add((void**)&m->m32, N * 4);
  cv.add((void**)&m->v32, N * 4);
  if (m->lp) cv.add(&m->pw, N * es);
  cv.add(&m->xs, (NL + 1) * Mx * C * es);
  cv.add(&m->xmid, NL * Mx * C * es);
  cv.add(&m->h1, NL * Mx * C * es);
  cv.add(&m->h2, NL * Mx * C * es);
  cv.add(&m->qkv, NL * Mx * 3 * C * es);
  cv.add(&m->att, NL * Mx * C * es);
  cv.add(&m->u, NL * Mx * (size_t)m->UW * es);
  cv.add(&m->a, NL * Mx * F * es);
  cv.add(&m->xf, Mx * C * es);
  cv.add(&m->logits, Mx * (size_t)m->ldl * es);
  cv.add((void**)&m->mu1, NL * Mx * 4);
  cv.add((void**)&m->rs1, NL * Mx * 4);
  cv.add((void**)&m->mu2, NL * Mx * 4);
  cv.add((void**)&m->rs2, NL * Mx * 4);
  cv.add((void**)&m->muf, Mx * 4);
  cv.add((void**)&m->rsf, Mx * 4);
  cv.add((void**)&m->lse, NL * Mx * m->H * 4);
  cv.add((void**)&m->tok, Mx * 4);
  cv.add((void**)&m->tgt, Mx * 4);
  cv.add((void**)&m->pos, Mx * 4);
  cv.add((void**)&m->dstart, Mx * 4);
  cv.add((void**)&m->dres32, Mx * C * 4);
  cv.add(&m->dres_t, Mx * C * es);
  cv.add(&m->dC, Mx * C * es);
  cv.add(&m->dF, Mx * (size_t)(m->UW + (m->llama ? F : 0)) * es);   // llama: dgu [M, 2F] then da [M, F]
  if (m->llama) {
    cv.add((void**)&m->rope_tab, (size_t)m->Tmax * (m->d / 2) * sizeof(float2));
    if (m->Hkv < m->H) cv.add(&m->dkvq, Mx * 2 * C * es);
  }
  cv.add(&m->dqkv, Mx * 3 * C * es);
  cv.add((void**)&m->attD, Mx * m->H * 4);
  const bool pad_heads = m->lp && !m->llama && !attn_tc_supported(m->d) && attn_tc_pad_supported(m->d);
  m->dq_acc_n = m->lp ? Mx * (size_t)(pad_heads ? m->H * 64 : C) : 1;
  cv.add((void**)&m->dq_acc, m->dq_acc_n * 4);
  if (pad_heads) {
    cv.add(&m->apad, NL * Mx * 3 * m->H * 64 * es);   // per layer
    cv.add(&m->opad, Mx * m->H * 64 * es);
    cv.add(&m->dqkvpad, Mx * 3 * m->H * 64 * es);
  }
  cv.add((void**)&m->rowloss, Mx * 4);
  {
    // partial rows of every deferred column reduction of one backward pass:
    // LayerNorm blocks (at most 444 rows of 3C) and bias column sums (at most
    // one row per 128 tokens), each region rounded to 16 bytes
    // (the q|k|v bias partials from the attention backward: one row per 32
    // rows of each sequence's 128-row blocks, at most 4 (Mx / 128 + Bmax))
    const size_t ln = (size_t)444 * 3 * C + 4, cs = (size_t)(Mx + 127) / 128, cq = 4 * (cs + m->Bmax);
    m->partials_n = ln + NL * (2 * ln + cs * F + 4 + cq * 3 * C + 4);
  }
  cv.add((void**)&m->partials, m->partials_n * 4);
  cv.add((void**)&m->normpart, m->normblk * 8);
  cv.add((void**)&m->sc, sizeof(DevScalars));
  size_t Bx = m->Bmax;
  size_t kvn = NL * Bx * m->H * (size_t)m->Tmax * m->d;
  cv.add(&m->kc, kvn * es);
  cv.add(&m->vc, kvn * es);
  cv.add(&m->dx, Bx * C * es);
  cv.add(&m->dh, Bx * C * es);
  cv.add(&m->dq, Bx * 3 * C * es);
  cv.add(&m->datt, Bx * C * es);
  cv.add(&m->du, Bx * (size_t)m->UW * es);
  cv.add(&m->da, Bx * F * es);
  cv.add(&m->dxf, Bx * C * es);
  cv.add((void**)&m->dlogits, Bx * m->Vp * 4);
  cv.add((void**)&m->dmu, Bx * 4);
  cv.add((void**)&m->drs, Bx * 4);
  cv.add((void**)&m->dtok, Bx * 4);
  cv.add((void**)&m->dpart, dec_attn_part_floats((int)Bx, m->H, m->d) * 4);
  cv.add((void**)&m->dacnt, Bx * m->H * 4);
  cv.add((void**)&m->dxst, (C / 16 + 1) * Bx * 8);
  cv.add((void**)&m->dsrc, Bx * (size_t)m->Tmax * 4);
  cv.add((void**)&m->dbcs, Bx * BEAM_MAX_WIDTH * 4);
  cv.add((void**)&m->dbct, Bx * BEAM_MAX_WIDTH * 4);
  m->arena_bytes = cv.off + 256;
  cudaError_t e = cudaMalloc((void**)&m->arena, m->arena_bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    m->arena = nullptr;
    m->err = std::string("cudaMalloc of the arena (") + std::to_string(m->arena_bytes) +
             " bytes) failed: " + cudaGetErrorString(e);
    return GPT_ERR_NOMEM;
  }
  for (auto& it : cv.items) *it.first = m->arena + it.second;
  e = cudaMemset(m->dacnt, 0, Bx * m->H * 4);
  // the attention backward adds into dq_acc, and its finishing kernel clears it after each use
  if (e == cudaSuccess) e = cudaMemset(m->dq_acc, 0, m->dq_acc_n * 4);
  if (e != cudaSuccess) { m->err = std::string("cudaMemset: ") + cudaGetErrorString(e); return GPT_ERR_CUDA; }
  if (!m->lp) m->pw = m->p32;
  return GPT_OK;
}

// ---------------------------------------------------------------------------
// GEMM and attention dispatch
// ---------------------------------------------------------------------------
template <typename T>
static EpiParams<T> epi_none() {
  EpiParams<T> e;
  memset(&e, 0, sizeof(e));
  return e;
}
template <typename T>
static EpiParams<T> epi_store(T* out, long ld, const float* bias, const T* resid, long ldr) {
  EpiParams<T> e = epi_none<T>();
  e.kind = EPI_STORE; e.out = out; e.ld_out = ld; e.bias = bias; e.resid = resid; e.ld_resid = ldr;
  return e;
}
template <typename T>
static EpiParams<T> epi_gelu(T* u, T* a, long ld, const float* bias) {
  EpiParams<T> e = epi_none<T>();
  e.kind = EPI_GELU; e.out = u; e.ld_out = ld; e.out2 = a; e.ld_out2 = ld; e.bias = bias;
  return e;
}
template <typename T>
static EpiParams<T> epi_dgelu(T* out, long ld, const T* u) {
  EpiParams<T> e = epi_none<T>();
  e.kind = EPI_DGELU; e.out = out; e.ld_out = ld; e.aux = u; e.ld_aux = ld;
  return e;
}
template <typename T>
static EpiParams<T> epi_f32(float* out, long ld) {
  EpiParams<T> e = epi_none<T>();
  e.kind = EPI_F32; e.outf = out; e.ld_outf = ld;
  return e;
}

static int g_num_sms = 148;

// C[M,N] = A(M x K) . B(N x K)^T; see launch.h for the operand conventions.
static int gemm_cls(bool a_t, bool b_t) { return a_t ? PC_GEMM_DW : (b_t ? PC_GEMM_DX : PC_GEMM_FWD); }

static int gemm(gpt_model* m, int M, int N, int K, const float* A, long lda, bool a_t, const float* B,
                long ldb, bool b_t, EpiParams<float> epi) {
  ProfScope ps(m, gemm_cls(a_t, b_t), 2.0 * M * N * K, 0.0);
  if (epi.kind == EPI_F32 && m->accum_now) epi.kind = EPI_F32_ADD;   // gradient accumulation
  CK(launch_gemm_simt<float>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, 1, m->stream));
  return GPT_OK;
}

// The tensor-core GEMM for either 16-bit type (fp16 is flagged in the
// epilogue record; the operand and output layouts are the same).
template <typename T16>
static cudaError_t tc_gemm(int M, int N, int K, const T16* A, long lda, bool a_t, const T16* B, long ldb, bool b_t,
                           const EpiParams<T16>& epi, int splits, unsigned* err, cudaStream_t s) {
  static_assert(sizeof(EpiParams<T16>) == sizeof(EpiParams<bf16>), "one layout for both 16-bit types");
  EpiParams<bf16> e;
  memcpy(&e, &epi, sizeof(e));
  e.f16 = std::is_same<T16, f16>::value ? 1 : 0;
  return launch_gemm_tc(M, N, K, reinterpret_cast<const bf16*>(A), lda, a_t, reinterpret_cast<const bf16*>(B), ldb,
                        b_t, e, splits, err, s);
}

template <typename T16>
static int gemm16(gpt_model* m, int M, int N, int K, const T16* A, long lda, bool a_t, const T16* B,
                  long ldb, bool b_t, EpiParams<T16> epi) {
  ProfScope ps(m, gemm_cls(a_t, b_t), 2.0 * M * N * K, 0.0);
  // gradient accumulation: weight gradients are added onto the stored ones
  const bool add_f32 = epi.kind == EPI_F32 && m->accum_now;
  if (!gemm_tc_supported(M, N, K, lda, a_t, ldb, b_t)) {
    if (epi.rowdot) FAIL(GPT_ERR_ARG, "row-dot epilogue needs the tensor-core GEMM");
    if (add_f32) epi.kind = EPI_F32_ADD;
    CK(launch_gemm_simt<T16>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, 1, m->stream));
    return GPT_OK;
  }
  int splits = 1;
  if (epi.kind == EPI_F32) {
    // weight gradients: short output, long contraction -> split K so the
    // 256 x 256 CTA-pair tiles fill the machine's pairs in whole waves
    const long tiles = (long)((M + 255) / 256) * ((N + 255) / 256), slots = g_num_sms / 2;
    double best = 0.0;
    for (int sp = 1; sp <= 8; sp *= 2) {
      if (sp > 1 && K / sp < 512) break;
      const long u = tiles * sp, waves = (u + slots - 1) / slots;
      const double eff = (double)u / ((double)waves * slots);
      if (eff > best * 1.05) { best = eff; splits = sp; }
    }
    int kb_total = (K + 63) / 64, kbs = (kb_total + splits - 1) / splits;
    splits = (kb_total + kbs - 1) / kbs;   // no empty split
    if (splits > 1 && epi.ld_outf != N && !m->accum_now) splits = 1;   // the zeroing below wants a dense output
  }
  if (splits > 1 || add_f32) {
    // K slices add their products onto the zeroed weight gradient (TMA bulk
    // reduce-add): no partial slabs, no separate summation pass; when
    // accumulating, onto the stored gradient instead
    EpiParams<T16> e2 = epi;
    e2.kind = EPI_F32_ADD;
    if (!add_f32) CK(launch_zero(epi.outf, (size_t)M * N * 4, m->stream));
    CK(tc_gemm<T16>(M, N, K, A, lda, a_t, B, ldb, b_t, e2, splits, &m->sc->err, m->stream));
  } else {
    CK(tc_gemm<T16>(M, N, K, A, lda, a_t, B, ldb, b_t, epi, 1, &m->sc->err, m->stream));
  }
  return GPT_OK;
}

static int gemm(gpt_model* m, int M, int N, int K, const bf16* A, long lda, bool a_t, const bf16* B, long ldb,
                bool b_t, EpiParams<bf16> epi) {
  return gemm16<bf16>(m, M, N, K, A, lda, a_t, B, ldb, b_t, epi);
}
static int gemm(gpt_model* m, int M, int N, int K, const f16* A, long lda, bool a_t, const f16* B, long ldb,
                bool b_t, EpiParams<f16> epi) {
  return gemm16<f16>(m, M, N, K, A, lda, a_t, B, ldb, b_t, epi);
}

// Allowed (query, key) pairs of a causal pass, all heads; a packed pass has
// fewer, counted on the device by the input preparation (see ProfRec)
static double attn_pairs(int B, int T, int H, bool seg) { return seg ? 0.0 : (double)B * H * T * (T + 1) / 2.0; }
static double attn_pair_mult(const gpt_model* m, double per_pair) { return m->seg_used ? per_pair * m->H : 0.0; }

static int attn_fwd(gpt_model* m, const float* qkv, float* out, float* lse, int B, int T,
                    const AttnLayout* = nullptr, int = 0) {
  ProfScope ps(m, PC_ATTN_FWD, 4.0 * m->d * attn_pairs(B, T, m->H, m->seg_used), 0.0, attn_pair_mult(m, 4.0 * m->d));
  CK(launch_attn_fwd_simt<float>(qkv, out, lse, m->dstart, B, T, m->H, m->d, m->stream));
  return GPT_OK;
}
template <typename T16>
static int attn_fwd(gpt_model* m, const T16* qkv, T16* out, float* lse, int B, int T, const AttnLayout* lay = nullptr,
                    int layer = 0) {
  ProfScope ps(m, PC_ATTN_FWD, 4.0 * m->d * attn_pairs(B, T, m->H, m->seg_used), 0.0, attn_pair_mult(m, 4.0 * m->d));
  constexpr bool F16 = std::is_same<T16, f16>::value;
  if (lay && !attn_tc_supported(m->d)) FAIL(GPT_ERR_ARG, "grouped key/value heads need the tensor-core attention");
  if (!lay && m->apad) {
    // heads of d < 64: the d = 64 tensor-core kernel on zero-padded copies
    // (the layer's padded q|k|v stays for its backward)
    const long rows = (long)B * T;
    bf16 *qp = (bf16*)m->apad + (size_t)layer * m->Mmax * 3 * m->H * 64, *op = (bf16*)m->opad;
    CK(launch_attn_pad(reinterpret_cast<const bf16*>(qkv), qp, rows, 3 * m->H, m->d, true, m->stream));
    CK(launch_attn_fwd_tc(qp, op, lse, m->dstart, B, T, m->H, &m->sc->err, m->stream, F16, nullptr, m->d));
    CK(launch_attn_pad(op, reinterpret_cast<bf16*>(out), rows, m->H, m->d, false, m->stream));
  } else if (attn_tc_supported(m->d))
    CK(launch_attn_fwd_tc(reinterpret_cast<const bf16*>(qkv), reinterpret_cast<bf16*>(out), lse, m->dstart, B, T,
                          m->H, &m->sc->err, m->stream, F16, lay));
  else if (!F16 && attn_mma_supported(m->d))
    CK(launch_attn_fwd_mma(reinterpret_cast<const bf16*>(qkv), reinterpret_cast<bf16*>(out), lse, m->dstart, B, T,
                           m->H, m->d, m->stream));
  else CK(launch_attn_fwd_simt<T16>(qkv, out, lse, m->dstart, B, T, m->H, m->d, m->stream));
  return GPT_OK;
}
static int attn_bwd(gpt_model* m, const float* qkv, const float* out, const float* dout, const float* lse,
                    float* dqkv, int B, int T, bool, const AttnLayout* = nullptr, int = 0, float* = nullptr) {
  ProfScope ps(m, PC_ATTN_BWD, 8.0 * m->d * attn_pairs(B, T, m->H, m->seg_used), 0.0, attn_pair_mult(m, 8.0 * m->d));
  CK(launch_attn_bwd_simt<float>(qkv, out, dout, lse, m->attD, m->dstart, dqkv, B, T, m->H, m->d, m->stream));
  return GPT_OK;
}
// d_ready: m->attD already holds D = rowsum(dO o O) (tensor-core path only)
template <typename T16>
static int attn_bwd(gpt_model* m, const T16* qkv, const T16* out, const T16* dout, const float* lse,
                    T16* dqkv, int B, int T, bool d_ready, const AttnLayout* lay = nullptr, int layer = 0,
                    float* bias_part = nullptr) {
  ProfScope ps(m, PC_ATTN_BWD, 8.0 * m->d * attn_pairs(B, T, m->H, m->seg_used), 0.0, attn_pair_mult(m, 8.0 * m->d));
  constexpr bool F16 = std::is_same<T16, f16>::value;
  auto cb = [](const T16* p) { return reinterpret_cast<const bf16*>(p); };
  if (lay && !attn_tc_supported(m->d)) FAIL(GPT_ERR_ARG, "grouped key/value heads need the tensor-core attention");
  if (!lay && m->apad) {
    // heads of d < 64 on the zero-padded copies (the forward took the same
    // path: its base-2 logsumexp is in this scale); D = rowsum(dO o O) is the
    // same over the padded columns, which add nothing
    const long rows = (long)B * T;
    // the layer's q|k|v as its forward padded them
    const bf16* qp = (const bf16*)m->apad + (size_t)layer * m->Mmax * 3 * m->H * 64;
    bf16 *dop = (bf16*)m->opad, *gp = (bf16*)m->dqkvpad;
    if (!d_ready) CK(launch_attn_rowdot(cb(out), cb(dout), m->attD, B, T, m->H, m->d, F16, m->stream));
    CK(launch_attn_pad(cb(dout), dop, rows, m->H, m->d, true, m->stream));
    CK(launch_attn_bwd_tc(qp, nullptr, dop, lse, m->attD, true, m->dq_acc, m->dstart, gp, B, T, m->H, &m->sc->err,
                          m->stream, F16, nullptr, m->d));
    CK(launch_attn_pad(gp, reinterpret_cast<bf16*>(dqkv), rows, 3 * m->H, m->d, false, m->stream));
  } else if (attn_tc_supported(m->d))
    CK(launch_attn_bwd_tc(cb(qkv), cb(out), cb(dout), lse, m->attD, d_ready, m->dq_acc, m->dstart,
                          reinterpret_cast<bf16*>(dqkv), B, T, m->H, &m->sc->err, m->stream, F16, lay, 64, bias_part));
  else if (!F16 && attn_mma_supported(m->d))
    CK(launch_attn_bwd_mma(cb(qkv), cb(out), cb(dout), lse, m->attD, m->dstart, reinterpret_cast<bf16*>(dqkv), B, T,
                           m->H, m->d, m->stream));
  else
    CK(launch_attn_bwd_simt<T16>(qkv, out, dout, lse, m->attD, m->dstart, dqkv, B, T, m->H, m->d, m->stream));
  return GPT_OK;
}

// ---------------------------------------------------------------------------
// Forward, loss, backward
// ---------------------------------------------------------------------------
template <typename T>
struct Acts {
  gpt_model* m;
  size_t MC, M3C, MF, MU, Mx;
  explicit Acts(gpt_model* mm) : m(mm) {
    Mx = m->Mmax; MC = Mx * m->C; M3C = 3 * MC; MF = Mx * m->F; MU = Mx * m->UW;
  }
  T* x(int l) const { return (T*)m->xs + l * MC; }
  T* xmid(int l) const { return (T*)m->xmid + l * MC; }
  T* h1(int l) const { return (T*)m->h1 + l * MC; }
  T* h2(int l) const { return (T*)m->h2 + l * MC; }
  T* qkv(int l) const { return (T*)m->qkv + l * M3C; }
  T* att(int l) const { return (T*)m->att + l * MC; }
  T* u(int l) const { return (T*)m->u + l * MU; }
  T* a(int l) const { return (T*)m->a + l * MF; }
  float* mu1(int l) const { return m->mu1 + l * Mx; }
  float* rs1(int l) const { return m->rs1 + l * Mx; }
  float* mu2(int l) const { return m->mu2 + l * Mx; }
  float* rs2(int l) const { return m->rs2 + l * Mx; }
  float* lse(int l) const { return m->lse + l * Mx * m->H; }
  const T* W(size_t off) const { return (const T*)m->pw + off; }
  const float* P(size_t off) const { return m->p32 + off; }
  float* G(size_t off) const { return m->g32 + off; }
};

template <typename T>
static int forward_llama(gpt_model* m, const int32_t* tokens, const int32_t* targets, const int32_t* seg, int B,
                         int T_, float* loss_dev);
template <typename T>
static int backward_llama(gpt_model* m);

template <typename T>
static int forward_impl(gpt_model* m, const int32_t* tokens, const int32_t* targets, const int32_t* seg, int B,
                        int T_, float* loss_dev) {
  if constexpr (sizeof(T) == 2) {
    if (m->llama) return forward_llama<T>(m, tokens, targets, seg, B, T_, loss_dev);
  }
  cudaStream_t s = m->stream;
  Acts<T> A(m);
  const int M = B * T_, C = m->C, F = m->F;
  const float eps = m->cfg.ln_eps;
  const double es = sizeof(T), lnb = (double)M * C * 2 * es + 8.0 * M;
  m->seg_used = seg != nullptr;
  { ProfScope ps(m, PC_EMBED, 0, (double)M * C * (8 + es) + 16.0 * M);
    CK(launch_prep(tokens, targets, seg, B, T_, m->V, m->tok, m->tgt, m->pos, m->dstart, m->sc, s));
    CK(launch_embed_fwd<T>(m->tok, m->pos, A.P(m->o_wte), A.P(m->o_wpe), A.x(0), M, C, s)); }
  for (int l = 0; l < m->NL; ++l) {
    const LayerOff& lo = m->L[l];
    { ProfScope ps(m, PC_LN_FWD, 0, lnb);
      CK(launch_ln_fwd<T>(A.x(l), A.P(lo.ln1_g), A.P(lo.ln1_b), A.h1(l), A.mu1(l), A.rs1(l), M, C, eps, s)); }
    CKI(gemm(m, M, 3 * C, C, A.h1(l), C, false, A.W(lo.w_qkv), C, false,
             epi_store<T>(A.qkv(l), 3 * C, A.P(lo.b_qkv), nullptr, 0)));
    CKI(attn_fwd(m, A.qkv(l), A.att(l), A.lse(l), B, T_, nullptr, l));
    CKI(gemm(m, M, C, C, A.att(l), C, false, A.W(lo.w_o), C, false,
             epi_store<T>(A.xmid(l), C, A.P(lo.b_o), A.x(l), C)));
    { ProfScope ps(m, PC_LN_FWD, 0, lnb);
      CK(launch_ln_fwd<T>(A.xmid(l), A.P(lo.ln2_g), A.P(lo.ln2_b), A.h2(l), A.mu2(l), A.rs2(l), M, C, eps, s)); }
    CKI(gemm(m, M, F, C, A.h2(l), C, false, A.W(lo.w_fc), C, false,
             epi_gelu<T>(A.u(l), A.a(l), F, A.P(lo.b_fc))));
    CKI(gemm(m, M, C, F, A.a(l), F, false, A.W(lo.w_fc2), F, false,
             epi_store<T>(A.x(l + 1), C, A.P(lo.b_fc2), A.xmid(l), C)));
  }
  { ProfScope ps(m, PC_LN_FWD, 0, lnb);
    CK(launch_ln_fwd<T>(A.x(m->NL), A.P(m->o_lnf_g), A.P(m->o_lnf_b), (T*)m->xf, m->muf, m->rsf, M, C, eps, s)); }
  CKI(gemm(m, M, m->Vp, C, (const T*)m->xf, C, false, A.W(m->o_head), C, false,
           epi_store<T>((T*)m->logits, m->ldl, nullptr, nullptr, 0)));
  if (targets) {
    ProfScope ps(m, PC_XENT, 0, 2.0 * es * M * m->Vp);
    CK(launch_xent<T>((T*)m->logits, m->ldl, m->tgt, M, m->V, m->Vp, m->rowloss, m->sc, s));
    CK(launch_loss_finalize(m->rowloss, M, m->sc, loss_dev, s));
  }
  m->fwd_B = B;
  m->fwd_T = T_;
  m->have_targets = targets != nullptr;
  m->logits_valid = targets == nullptr;
  return GPT_OK;
}

template <typename T>
static int backward_impl(gpt_model* m) {
  if constexpr (sizeof(T) == 2) {
    if (m->llama) return backward_llama<T>(m);
  }
  cudaStream_t s = m->stream;
  Acts<T> A(m);
  const int B = m->fwd_B, T_ = m->fwd_T, M = B * T_, C = m->C, F = m->F, Vp = m->Vp;
  T* dC = (T*)m->dC;
  T* dF = (T*)m->dF;
  T* dq = (T*)m->dqkv;
  T* drt = (T*)m->dres_t;
  const T* dz = (const T*)m->logits;
  const T* xf = (const T*)m->xf;
  int nblk = 0;
  const double es = sizeof(T), lnbb = (double)M * C * (3 * es + 8) + 8.0 * M;
  // Partial rows (LayerNorm dg/db, bias column sums) take consecutive regions
  // of the partials arena; one deferred launch reduces them all at the end.
  std::vector<RedSeg>& segs = m->redsegs;
  segs.clear();
  float* pp = m->partials;
  float* const pend = m->partials + m->partials_n;
  auto take = [&](size_t n) -> float* {
    float* p = pp;
    pp += (n + 3) & ~(size_t)3;
    return pp <= pend ? p : nullptr;
  };
  auto seg = [&](const float* src, float* dst, int rows, int cols, int ld) {
    segs.push_back({src, dst, rows, cols, ld, 0});
  };
  // LayerNorm backward; its partial rows are [dg | db | column sums of the
  // outgoing residual gradient] (the latter = the bias gradient `bias_dst`)
  auto ln_bwd = [&](const T* x, const float* mu, const float* rs, const float* g, const float* din, float* gdst,
                    float* bias_dst) -> int {
    float* part = take((size_t)444 * 3 * C);
    if (!part) FAIL(GPT_ERR_NOMEM, "partials arena too small");
    ProfScope ps(m, PC_LN_BWD, 0, lnbb);
    CK(launch_ln_bwd<T>(dC, x, mu, rs, g, din, m->dres32, drt, part, M, C, &nblk, s, false, &m->sc->err));
    seg(part, gdst, nblk, 2 * C, 3 * C);
    if (bias_dst) seg(part + 2 * C, bias_dst, nblk, C, 3 * C);
    return GPT_OK;
  };
  // LM head: dxf = dz . W_head;  dW_head = dz^T . xf  (into dwte when tied)
  CKI(gemm(m, M, C, Vp, dz, m->ldl, false, A.W(m->o_head), C, true, epi_store<T>(dC, C, nullptr, nullptr, 0)));
  CKI(gemm(m, Vp, C, M, dz, m->ldl, true, xf, C, true, epi_f32<T>(A.G(m->o_head), C)));
  // column sums of the gradient entering the last block = its fc2 bias gradient
  CKI(ln_bwd(A.x(m->NL), m->muf, m->rsf, A.P(m->o_lnf_g), nullptr, A.G(m->o_lnf_g), A.G(m->L[m->NL - 1].b_fc2)));
  for (int l = m->NL - 1; l >= 0; --l) {
    const LayerOff& lo = m->L[l];
    // MLP: x_out = x_mid + gelu(h2 W_fc^T + b_fc) W_fc2^T + b_fc2  (b_fc2 gradient already taken)
    CKI(gemm(m, C, F, M, drt, C, true, A.a(l), F, true, epi_f32<T>(A.G(lo.w_fc2), F)));
    // on the tensor-core path the GELU' epilogue also sums dF per column over
    // each 128-row tile (the fc bias gradient's partial rows)
    const bool fused_bfc = sizeof(T) == 2 && gemm_tc_supported(M, F, C, C, false, F, true);
    float* bpart = take((size_t)((M + 127) / 128) * F);
    if (!bpart) FAIL(GPT_ERR_NOMEM, "partials arena too small");
    {
      EpiParams<T> e = epi_dgelu<T>(dF, F, A.u(l));
      if (fused_bfc) e.colsum = bpart;
      CKI(gemm(m, M, F, C, drt, C, false, A.W(lo.w_fc2), F, true, e));
    }
    if (fused_bfc) {
      seg(bpart, A.G(lo.b_fc), (M + 127) / 128, F, F);
    } else {
      ProfScope ps(m, PC_BIAS, 0, (double)M * F * es);
      int rows = 0;
      CK(launch_colsum<T>(dF, F, M, F, bpart, &rows, s));
      seg(bpart, A.G(lo.b_fc), rows, F, F);
    }
    CKI(gemm(m, F, C, M, dF, F, true, A.h2(l), C, true, epi_f32<T>(A.G(lo.w_fc), C)));
    CKI(gemm(m, M, C, F, dF, F, false, A.W(lo.w_fc), C, true, epi_store<T>(dC, C, nullptr, nullptr, 0)));
    CKI(ln_bwd(A.xmid(l), A.mu2(l), A.rs2(l), A.P(lo.ln2_g), m->dres32, A.G(lo.ln2_g), A.G(lo.b_o)));
    // attention: x_mid = x + attn(h1 W_qkv^T + b_qkv) W_o^T + b_o  (b_o gradient already taken)
    CKI(gemm(m, C, C, M, drt, C, true, A.att(l), C, true, epi_f32<T>(A.G(lo.w_o), C)));
    // dO = d(attention output); on the tensor-core path its GEMM epilogue also
    // takes D = rowsum(dO o O) per row and head for the attention backward
    // (the row-dot epilogue sums 64-column heads: d = 64 only)
    const bool fuse_d = sizeof(T) == 2 && attn_tc_supported(m->d) && gemm_tc_supported(M, C, C, C, false, C, true);
    {
      EpiParams<T> e = epi_store<T>(dC, C, nullptr, nullptr, 0);
      if (fuse_d) { e.aux = A.att(l); e.ld_aux = C; e.rowdot = m->attD; e.rd_T = T_; }
      CKI(gemm(m, M, C, C, drt, C, false, A.W(lo.w_o), C, true, e));
    }
    // the q|k|v bias gradient: on the tensor-core attention of 64-column heads
    // its column sums come out of the backward kernels (one partial row per 32
    // rows), otherwise from a column-sum pass over dq
    const bool fuse_bq = sizeof(T) == 2 && attn_tc_supported(m->d) && !m->apad;
    if (fuse_bq) {
      const int crows = B * ((T_ + 127) / 128) * 4;
      float* qpart = take((size_t)crows * 3 * C);
      if (!qpart) FAIL(GPT_ERR_NOMEM, "partials arena too small");
      CKI(attn_bwd(m, A.qkv(l), A.att(l), dC, A.lse(l), dq, B, T_, fuse_d, nullptr, l, qpart));
      seg(qpart, A.G(lo.b_qkv), crows, 3 * C, 3 * C);
    } else {
      CKI(attn_bwd(m, A.qkv(l), A.att(l), dC, A.lse(l), dq, B, T_, fuse_d, nullptr, l));
      float* qpart = take((size_t)((M + 127) / 128) * 3 * C);
      if (!qpart) FAIL(GPT_ERR_NOMEM, "partials arena too small");
      ProfScope ps(m, PC_BIAS, 0, (double)M * 3 * C * es);
      int rows = 0;
      CK(launch_colsum<T>(dq, 3 * C, M, 3 * C, qpart, &rows, s));
      seg(qpart, A.G(lo.b_qkv), rows, 3 * C, 3 * C);
    }
    CKI(gemm(m, 3 * C, C, M, dq, 3 * C, true, A.h1(l), C, true, epi_f32<T>(A.G(lo.w_qkv), C)));
    CKI(gemm(m, M, C, 3 * C, dq, 3 * C, false, A.W(lo.w_qkv), C, true, epi_store<T>(dC, C, nullptr, nullptr, 0)));
    CKI(ln_bwd(A.x(l), A.mu1(l), A.rs1(l), A.P(lo.ln1_g), m->dres32, A.G(lo.ln1_g),
               l > 0 ? A.G(m->L[l - 1].b_fc2) : nullptr));
  }
  // all LayerNorm and bias gradients from their partial rows, one launch
  {
    double pb = 0;
    for (const RedSeg& g : segs) pb += (double)g.rows * g.cols * 4;
    ProfScope ps(m, PC_BIAS, 0, pb);
    CK(launch_reduce_segs(segs.data(), (int)segs.size(), m->accum_now, s));
  }
  // embeddings: scatter-add by token and by position
  ProfScope ps_emb(m, PC_EMBED, 0, (double)M * C * 12);
  if (!m->accum_now) {
    if (!m->cfg.tied) CK(launch_zero(A.G(m->o_wte), (size_t)Vp * C * 4, s));
    CK(launch_zero(A.G(m->o_wpe), (size_t)m->Tmax * C * 4, s));
  }
  CK(launch_embed_bwd<T>(m->dres32, m->tok, m->pos, A.G(m->o_wte), A.G(m->o_wpe), M, C, s));
  m->have_targets = false;
  return GPT_OK;
}

// ---------------------------------------------------------------------------
// Llama-style block ("NTransformer" page, key features: RoPE, GQA, SwiGLU):
// RMSNorm (the LayerNorm kernels without mean and shift), rotary positions
// applied in place to the q and k heads after the qkv GEMM (and their inverse
// to dq, dk), grouped key/value heads read by the tensor-core attention
// through its column layout, SwiGLU between the up and down GEMMs; no biases.
// ---------------------------------------------------------------------------
// q|k|v column layout of the grouped heads; dkv: where the attention backward
// writes the per-query-head key/value gradients
static AttnLayout llama_layout(const gpt_model* m, void* dqkv) {
  AttnLayout a;
  a.qw = m->QW;
  a.kcol = m->C;
  a.vcol = m->C + m->Hkv * m->d;
  a.G = m->H / m->Hkv;
  if (a.G == 1) {
    a.dkv = dqkv ? (bf16*)dqkv + m->C : nullptr;   // dK, dV straight into dqkv (same columns)
    a.ld_kv = m->QW;
    a.v_off = m->C;
  } else {
    a.dkv = (bf16*)m->dkvq;                       // per query head; summed by launch_gqa_reduce
    a.ld_kv = 2L * m->C;
    a.v_off = m->C;
  }
  return a;
}

template <typename T>
static int forward_llama(gpt_model* m, const int32_t* tokens, const int32_t* targets, const int32_t* seg, int B,
                         int T_, float* loss_dev) {
  cudaStream_t s = m->stream;
  Acts<T> A(m);
  const int M = B * T_, C = m->C, F = m->F, QW = m->QW;
  const float eps = m->cfg.ln_eps;
  const double es = sizeof(T), lnb = (double)M * C * 2 * es + 8.0 * M;
  m->seg_used = seg != nullptr;
  const AttnLayout lay = llama_layout(m, nullptr);
  { ProfScope ps(m, PC_EMBED, 0, (double)M * C * (4 + es) + 16.0 * M);
    CK(launch_prep(tokens, targets, seg, B, T_, m->V, m->tok, m->tgt, m->pos, m->dstart, m->sc, s));
    CK(launch_embed_fwd<T>(m->tok, m->pos, A.P(m->o_wte), nullptr, A.x(0), M, C, s)); }
  for (int l = 0; l < m->NL; ++l) {
    const LayerOff& lo = m->L[l];
    { ProfScope ps(m, PC_LN_FWD, 0, lnb);
      CK(launch_ln_fwd<T>(A.x(l), A.P(lo.ln1_g), nullptr, A.h1(l), A.mu1(l), A.rs1(l), M, C, eps, s)); }
    CKI(gemm(m, M, QW, C, A.h1(l), C, false, A.W(lo.w_qkv), C, false, epi_store<T>(A.qkv(l), QW, nullptr, nullptr, 0)));
    CK(launch_rope<T>(A.qkv(l), QW, M, m->H, C, m->Hkv, m->d, m->pos, 0, nullptr, m->rope_tab, m->Tmax, false, s));
    CKI(attn_fwd(m, A.qkv(l), A.att(l), A.lse(l), B, T_, &lay));
    CKI(gemm(m, M, C, C, A.att(l), C, false, A.W(lo.w_o), C, false, epi_store<T>(A.xmid(l), C, nullptr, A.x(l), C)));
    { ProfScope ps(m, PC_LN_FWD, 0, lnb);
      CK(launch_ln_fwd<T>(A.xmid(l), A.P(lo.ln2_g), nullptr, A.h2(l), A.mu2(l), A.rs2(l), M, C, eps, s)); }
    CKI(gemm(m, M, 2 * F, C, A.h2(l), C, false, A.W(lo.w_fc), C, false,
             epi_store<T>(A.u(l), 2 * F, nullptr, nullptr, 0)));
    CK(launch_swiglu<T>(A.u(l), A.a(l), M, F, s));
    CKI(gemm(m, M, C, F, A.a(l), F, false, A.W(lo.w_fc2), F, false,
             epi_store<T>(A.x(l + 1), C, nullptr, A.xmid(l), C)));
  }
  { ProfScope ps(m, PC_LN_FWD, 0, lnb);
    CK(launch_ln_fwd<T>(A.x(m->NL), A.P(m->o_lnf_g), nullptr, (T*)m->xf, m->muf, m->rsf, M, C, eps, s)); }
  CKI(gemm(m, M, m->Vp, C, (const T*)m->xf, C, false, A.W(m->o_head), C, false,
           epi_store<T>((T*)m->logits, m->ldl, nullptr, nullptr, 0)));
  if (targets) {
    ProfScope ps(m, PC_XENT, 0, 2.0 * es * M * m->Vp);
    CK(launch_xent<T>((T*)m->logits, m->ldl, m->tgt, M, m->V, m->Vp, m->rowloss, m->sc, s));
    CK(launch_loss_finalize(m->rowloss, M, m->sc, loss_dev, s));
  }
  m->fwd_B = B;
  m->fwd_T = T_;
  m->have_targets = targets != nullptr;
  m->logits_valid = targets == nullptr;
  return GPT_OK;
}

template <typename T>
static int backward_llama(gpt_model* m) {
  cudaStream_t s = m->stream;
  Acts<T> A(m);
  const int B = m->fwd_B, T_ = m->fwd_T, M = B * T_, C = m->C, F = m->F, Vp = m->Vp, QW = m->QW;
  T* dC = (T*)m->dC;
  T* dgu = (T*)m->dF;                       // [M, 2F]
  T* da = (T*)m->dF + (size_t)m->Mmax * 2 * F;   // [M, F]
  T* dq = (T*)m->dqkv;                      // [M, QW]
  T* drt = (T*)m->dres_t;
  const T* dz = (const T*)m->logits;
  const T* xf = (const T*)m->xf;
  int nblk = 0;
  const double es = sizeof(T), lnbb = (double)M * C * (3 * es + 8) + 8.0 * M;
  const AttnLayout lay = llama_layout(m, m->dqkv);
  std::vector<RedSeg>& segs = m->redsegs;
  segs.clear();
  float* pp = m->partials;
  float* const pend = m->partials + m->partials_n;
  auto take = [&](size_t n) -> float* {
    float* p = pp;
    pp += (n + 3) & ~(size_t)3;
    return pp <= pend ? p : nullptr;
  };
  // RMSNorm backward; its partial rows are [dg | (unused) | column sums]
  auto rms_bwd = [&](const T* x, const float* mu, const float* rs, const float* g, const float* din,
                     float* gdst) -> int {
    float* part = take((size_t)444 * 3 * C);
    if (!part) FAIL(GPT_ERR_NOMEM, "partials arena too small");
    ProfScope ps(m, PC_LN_BWD, 0, lnbb);
    CK(launch_ln_bwd<T>(dC, x, mu, rs, g, din, m->dres32, drt, part, M, C, &nblk, s, true, &m->sc->err));
    segs.push_back({part, gdst, nblk, C, 3 * C, 0});
    return GPT_OK;
  };
  CKI(gemm(m, M, C, Vp, dz, m->ldl, false, A.W(m->o_head), C, true, epi_store<T>(dC, C, nullptr, nullptr, 0)));
  CKI(gemm(m, Vp, C, M, dz, m->ldl, true, xf, C, true, epi_f32<T>(A.G(m->o_head), C)));
  CKI(rms_bwd(A.x(m->NL), m->muf, m->rsf, A.P(m->o_lnf_g), nullptr, A.G(m->o_lnf_g)));
  for (int l = m->NL - 1; l >= 0; --l) {
    const LayerOff& lo = m->L[l];
    // MLP: x_out = x_mid + swiglu(h2 W_gu^T) W_down^T
    CKI(gemm(m, C, F, M, drt, C, true, A.a(l), F, true, epi_f32<T>(A.G(lo.w_fc2), F)));
    CKI(gemm(m, M, F, C, drt, C, false, A.W(lo.w_fc2), F, true, epi_store<T>(da, F, nullptr, nullptr, 0)));
    CK(launch_swiglu_bwd<T>(da, A.u(l), dgu, M, F, s));
    CKI(gemm(m, 2 * F, C, M, dgu, 2 * F, true, A.h2(l), C, true, epi_f32<T>(A.G(lo.w_fc), C)));
    CKI(gemm(m, M, C, 2 * F, dgu, 2 * F, false, A.W(lo.w_fc), C, true, epi_store<T>(dC, C, nullptr, nullptr, 0)));
    CKI(rms_bwd(A.xmid(l), A.mu2(l), A.rs2(l), A.P(lo.ln2_g), m->dres32, A.G(lo.ln2_g)));
    // attention: x_mid = x + attn(rope(h1 W_qkv^T)) W_o^T
    CKI(gemm(m, C, C, M, drt, C, true, A.att(l), C, true, epi_f32<T>(A.G(lo.w_o), C)));
    {
      EpiParams<T> e = epi_store<T>(dC, C, nullptr, nullptr, 0);
      e.aux = A.att(l); e.ld_aux = C; e.rowdot = m->attD; e.rd_T = T_;
      CKI(gemm(m, M, C, C, drt, C, false, A.W(lo.w_o), C, true, e));
    }
    CKI(attn_bwd(m, A.qkv(l), A.att(l), dC, A.lse(l), dq, B, T_, true, &lay));
    if (lay.G > 1)
      CK(launch_gqa_reduce<T>((const T*)m->dkvq, dq, QW, lay.kcol, lay.vcol, M, m->Hkv, lay.G, m->d, s));
    CK(launch_rope<T>(dq, QW, M, m->H, C, m->Hkv, m->d, m->pos, 0, nullptr, m->rope_tab, m->Tmax, true, s));
    CKI(gemm(m, QW, C, M, dq, QW, true, A.h1(l), C, true, epi_f32<T>(A.G(lo.w_qkv), C)));
    CKI(gemm(m, M, C, QW, dq, QW, false, A.W(lo.w_qkv), C, true, epi_store<T>(dC, C, nullptr, nullptr, 0)));
    CKI(rms_bwd(A.x(l), A.mu1(l), A.rs1(l), A.P(lo.ln1_g), m->dres32, A.G(lo.ln1_g)));
  }
  {
    double pb = 0;
    for (const RedSeg& g : segs) pb += (double)g.rows * g.cols * 4;
    ProfScope ps(m, PC_BIAS, 0, pb);
    CK(launch_reduce_segs(segs.data(), (int)segs.size(), m->accum_now, s));
  }
  ProfScope ps_emb(m, PC_EMBED, 0, (double)M * C * 8);
  if (!m->cfg.tied && !m->accum_now) CK(launch_zero(A.G(m->o_wte), (size_t)Vp * C * 4, s));
  CK(launch_embed_bwd<T>(m->dres32, m->tok, m->pos, A.G(m->o_wte), nullptr, M, C, s));
  m->have_targets = false;
  return GPT_OK;
}

// ---------------------------------------------------------------------------
// Greedy decoding
// ---------------------------------------------------------------------------
// One projection of a decode step: y = x W^T with the gemv epilogue `mode`
// (0: + bias + residual, 1: u = + bias and gelu(u), 2: fp32 logits).  Up to
// 32 rows of a 16-bit model run on the mma.sync kernel that spreads 16-row
// weight slices over every SM; fp32 models on the GEMV that streams each
// weight row once.
// With st (the projections that write the residual rows) the kernel also
// leaves their LayerNorm statistics there for the next dec_ln_proj; st is
// dropped (and the next LayerNorm takes its own) where the kernel cannot.
template <typename T>
static cudaError_t dec_proj(gpt_model* m, const T* X, int B, int K, const T* W, int N, const float* bias,
                            const T* resid, int mode, T* out, T* out2, float* outf, cudaStream_t s,
                            float2* st = nullptr) {
  if constexpr (sizeof(T) == 2) {
    if (dec_mma_supported(B, K, N))
      return launch_dec_mma<T>(X, B, K, W, N, bias, resid, mode, out, out2, outf, &m->sc->err, s, nullptr, nullptr,
                               0.f, mode == 0 && N % 16 == 0 ? st : nullptr);
  }
  return launch_gemv<T>(X, B, K, W, N, bias, resid, mode, out, out2, outf, s);
}
// LayerNorm of the residual rows x (gains g, shift b; Llama: RMSNorm, b
// null) followed by a projection of the normalised rows: one kernel where the
// mma.sync projection can normalise its own input, else the LayerNorm kernel
// into h and the projection.
template <typename T>
static cudaError_t dec_ln_proj(gpt_model* m, const T* x, const float* g, const float* b, T* h, int B, int K,
                               const T* W, int N, const float* bias, const T* resid, int mode, T* out, T* out2,
                               float* outf, cudaStream_t s, const float2* st = nullptr) {
  if constexpr (sizeof(T) == 2) {
    if (dec_mma_supported(B, K, N, true))
      return launch_dec_mma<T>(x, B, K, W, N, bias, resid, mode, out, out2, outf, &m->sc->err, s, g, b,
                               m->cfg.ln_eps, nullptr, K % 16 == 0 ? st : nullptr);
  }
  cudaError_t e = launch_ln_fwd<T>(x, g, b, h, m->dmu, m->drs, B, K, m->cfg.ln_eps, s);
  if (e != cudaSuccess) return e;
  return dec_proj<T>(m, h, B, K, W, N, bias, resid, mode, out, out2, outf, s);
}

// The Llama-style kernels exist for the 16-bit types only (the block needs
// 16-bit precision; create() refuses it in fp32 mode).
template <typename T>
static cudaError_t rope16(T* x, long ld, int rows, int nq, int kcol, int nk, int d, const int* pos, int pos0,
                          const int* step, const float2* tab, int max_seq, bool inverse, cudaStream_t s) {
  if constexpr (sizeof(T) == 2) return launch_rope<T>(x, ld, rows, nq, kcol, nk, d, pos, pos0, step, tab, max_seq, inverse, s);
  else return cudaErrorNotSupported;
}
template <typename T>
static cudaError_t swiglu16(const T* gu, T* a, int rows, int F, cudaStream_t s) {
  if constexpr (sizeof(T) == 2) return launch_swiglu<T>(gu, a, rows, F, s);
  else return cudaErrorNotSupported;
}

static DecLayout dec_layout(const gpt_model* m) {
  DecLayout L;
  L.qw = m->QW;
  L.kcol = m->C;
  L.vcol = m->C + m->Hkv * m->d;
  L.Hkv = m->Hkv;
  L.src = m->beam_w ? m->dsrc : nullptr;
  return L;
}

template <typename T>
static int decode_step(gpt_model* m, int B, int Tp, int n_new, int32_t* out, cudaStream_t s) {
  Acts<T> A(m);
  const int C = m->C, F = m->F, H = m->H, d = m->d, QW = m->QW;
  const bool ll = m->llama;
  const DecLayout DL = dec_layout(m);
  size_t kvl = (size_t)m->Bmax * m->Hkv * m->Tmax * d;
  T* kc = (T*)m->kc;
  T* vc = (T*)m->vc;
  T *x = (T*)m->dx, *h = (T*)m->dh, *q = (T*)m->dq, *att = (T*)m->datt, *u = (T*)m->du, *a = (T*)m->da,
    *xf = (T*)m->dxf;
  int* stepc = &m->sc->dec_step;
  // LayerNorm parameters (Llama: RMSNorm, gains only) and biases (Llama: none)
  auto P0 = [&](size_t off) -> const float* { return ll ? nullptr : A.P(off); };
  // LayerNorm statistics of the residual rows travel from the kernel that
  // writes the rows (embedding, output projection, fc2) to the next
  // LayerNorm-fused projection where both run the 16-bit decode kernels
  float2* st = C % 16 == 0 ? m->dxst : nullptr;
  const bool mma = sizeof(T) == 2;
  const float2* st_o = mma && dec_mma_supported(B, C, C) ? st : nullptr;    // after the output projection
  const float2* st_f2 = mma && dec_mma_supported(B, F, C) ? st : nullptr;   // after fc2
  // the token fed at step st sits at position Tp - 1 + st; a greedy step's
  // input row was embedded by the previous step's argmax (the first one by
  // decode_impl)
  const bool greedy = !m->beam_w && !m->smp_on;
  if (!greedy)
    CK(launch_dec_embed<T>(m->dtok, A.P(m->o_wte), ll ? nullptr : A.P(m->o_wpe), x, B, C, Tp - 1, stepc, m->Tmax,
                           &m->sc->err, s, st));
  for (int l = 0; l < m->NL; ++l) {
    const LayerOff& lo = m->L[l];
    CK(dec_ln_proj<T>(m, x, A.P(lo.ln1_g), P0(lo.ln1_b), h, B, C, A.W(lo.w_qkv), QW, P0(lo.b_qkv), nullptr, 0, q,
                      nullptr, nullptr, s, l == 0 ? st : st_f2));
    if (ll) CK(rope16<T>(q, QW, B, H, C, m->Hkv, d, nullptr, Tp - 1, stepc, m->rope_tab, m->Tmax, false, s));
    CK(launch_dec_attn<T>(q, kc + l * kvl, vc + l * kvl, att, m->dpart, m->dacnt, B, H, d, m->Tmax, Tp - 1, stepc, DL,
                          s));
    CK(dec_proj<T>(m, att, B, C, A.W(lo.w_o), C, P0(lo.b_o), x, 0, x, nullptr, nullptr, s, st));
    if (ll) {
      CK(dec_ln_proj<T>(m, x, A.P(lo.ln2_g), nullptr, h, B, C, A.W(lo.w_fc), 2 * F, nullptr, nullptr, 0, u, nullptr,
                        nullptr, s, st_o));
      CK(swiglu16<T>(u, a, B, F, s));
    } else {
      CK(dec_ln_proj<T>(m, x, A.P(lo.ln2_g), A.P(lo.ln2_b), h, B, C, A.W(lo.w_fc), F, A.P(lo.b_fc), nullptr, 1, u, a,
                        nullptr, s, st_o));
    }
    CK(dec_proj<T>(m, a, B, F, A.W(lo.w_fc2), C, P0(lo.b_fc2), x, 0, x, nullptr, nullptr, s, st));
  }
  CK(dec_ln_proj<T>(m, x, A.P(m->o_lnf_g), P0(m->o_lnf_b), xf, B, C, A.W(m->o_head), m->Vp, nullptr, nullptr, 2,
                    nullptr, nullptr, m->dlogits, s, m->NL > 0 ? st_f2 : st));
  if (m->beam_w) {
    const int W = m->beam_w;
    CK(launch_beam_topk(m->dlogits, m->Vp, m->V, B / W, W, false, m->beam_scores, m->dbcs, m->dbct, s));
    CK(launch_beam_merge(m->dbcs, m->dbct, B / W, W, m->V, Tp, m->dsrc, m->Tmax, m->beam_scores, m->dtok, out, n_new,
                         stepc, s));
  } else if (m->smp_on)
    CK(launch_sample(m->dlogits, B, m->V, m->Vp, m->smp_temp, m->smp_topk, m->smp_topp, m->smp_u, n_new, m->dtok, out,
                     n_new, stepc, s));
  else {
    // the choice, the next input row and the step advance in one kernel
    GreedyNext<T> nx;
    nx.wte = A.P(m->o_wte);
    nx.wpe = ll ? nullptr : A.P(m->o_wpe);
    nx.x = x;
    nx.C = C;
    nx.pos0 = Tp - 1;
    nx.max_seq = m->Tmax;
    nx.st = st;
    nx.cnt = &m->sc->dec_cnt;
    nx.step = stepc;
    CK(launch_argmax<T>(m->dlogits, B, m->V, m->Vp, m->dtok, out, n_new, stepc, s, &nx));
  }
  if (!greedy) CK(launch_step_advance(stepc, s));
  return GPT_OK;
}

template <typename T>
static int decode_impl(gpt_model* m, const int32_t* prompt, int B, int Tp, int n_new, int32_t* out) {
  cudaStream_t s = m->stream;
  Acts<T> A(m);
  const int C = m->C, H = m->H, d = m->d;
  CKI(forward_impl<T>(m, prompt, nullptr, nullptr, B, Tp, nullptr));
  m->logits_valid = false;
  size_t kvl = (size_t)m->Bmax * m->Hkv * m->Tmax * d;
  const DecLayout DL = dec_layout(m);
  for (int l = 0; l < m->NL; ++l)
    CK(launch_kv_fill<T>(A.qkv(l), (T*)m->kc + l * kvl, (T*)m->vc + l * kvl, B, Tp, d, m->Tmax, DL, s));
  // first new token: from the prefill's last position
  CK(launch_gather_last<T>((const T*)m->xf, B, Tp, C, (T*)m->dxf, s));
  CK(dec_proj<T>(m, (const T*)m->dxf, B, C, A.W(m->o_head), m->Vp, nullptr, nullptr, 2, nullptr, nullptr,
                 m->dlogits, s));
  if (m->beam_w) {
    // every beam of a prompt starts from the prompt's prefill row
    const int W = m->beam_w;
    CK(launch_beam_init(m->dsrc, m->Tmax, m->beam_scores, B, W, Tp, s));
    CK(launch_beam_topk(m->dlogits, m->Vp, m->V, B, W, true, m->beam_scores, m->dbcs, m->dbct, s));
    CK(launch_beam_merge(m->dbcs, m->dbct, B, W, m->V, Tp, m->dsrc, m->Tmax, m->beam_scores, m->dtok, out, n_new,
                         nullptr, s));
  } else if (m->smp_on)
    CK(launch_sample(m->dlogits, B, m->V, m->Vp, m->smp_temp, m->smp_topk, m->smp_topp, m->smp_u, n_new, m->dtok, out,
                     n_new, nullptr, s));
  else
    CK(launch_argmax(m->dlogits, B, m->V, m->Vp, m->dtok, out, n_new, nullptr, s));
  if (n_new == 1) return GPT_OK;
  const int Bd = m->beam_w ? B * m->beam_w : B;   // decode rows
  const int one = 1;
  CK(cudaMemcpyAsync(&m->sc->dec_step, &one, sizeof(int), cudaMemcpyHostToDevice, s));
  if (!m->beam_w && !m->smp_on) {
    // the first replayed step's input row (later ones come from the step's argmax)
    CK(launch_dec_embed<T>(m->dtok, A.P(m->o_wte), m->llama ? nullptr : A.P(m->o_wpe), (T*)m->dx, B, C, Tp - 1,
                           &m->sc->dec_step, m->Tmax, &m->sc->err, s, C % 16 == 0 ? m->dxst : nullptr));
  }
  // later tokens: one captured step (about 7 L + 5 kernels), replayed n_new - 1 times
  if (!m->cap_stream) CK(cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking));
  if (!m->ev_a) {
    CK(cudaEventCreateWithFlags(&m->ev_a, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&m->ev_b, cudaEventDisableTiming));
  }
  const bool same_smp = m->dec_smp_on == m->smp_on && m->dec_smp_temp == m->smp_temp &&
                        m->dec_smp_topk == m->smp_topk && m->dec_smp_topp == m->smp_topp && m->dec_smp_u == m->smp_u &&
                        m->dec_beam_w == m->beam_w && m->dec_beam_scores == m->beam_scores;
  if (!m->dec_graph || m->dec_B != Bd || m->dec_Tp != Tp || m->dec_nnew != n_new || m->dec_out != out || !same_smp) {
    if (m->dec_graph) { cudaGraphExecDestroy(m->dec_graph); m->dec_graph = nullptr; }
    cudaGraph_t g = nullptr;
    unsigned long long n0 = g_kernel_launches;
    CK(cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal));
    int r = decode_step<T>(m, Bd, Tp, n_new, out, m->cap_stream);
    cudaError_t ec = cudaStreamEndCapture(m->cap_stream, &g);
    if (r != GPT_OK) { if (g) cudaGraphDestroy(g); return r; }
    CK(ec);
    cudaError_t ei = cudaGraphInstantiate(&m->dec_graph, g, 0);
    cudaGraphDestroy(g);
    CK(ei);
    m->dec_kernels = (int)(g_kernel_launches - n0);   // the kernels one replay launches
    g_kernel_launches = n0;
    m->dec_B = Bd; m->dec_Tp = Tp; m->dec_nnew = n_new; m->dec_out = out;
    m->dec_smp_on = m->smp_on; m->dec_smp_temp = m->smp_temp; m->dec_smp_topk = m->smp_topk;
    m->dec_smp_topp = m->smp_topp; m->dec_smp_u = m->smp_u;
    m->dec_beam_w = m->beam_w; m->dec_beam_scores = m->beam_scores;
  }
  CK(cudaEventRecord(m->ev_a, s));
  CK(cudaStreamWaitEvent(m->cap_stream, m->ev_a, 0));
  for (int st = 1; st < n_new; ++st) CK(cudaGraphLaunch(m->dec_graph, m->cap_stream));
  g_kernel_launches += (unsigned long long)m->dec_kernels * (n_new - 1);
  CK(cudaEventRecord(m->ev_b, m->cap_stream));
  CK(cudaStreamWaitEvent(s, m->ev_b, 0));
  return GPT_OK;
}

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
static int validate_cfg(const gpt_config* c, std::string& why) {
  if (c->vocab < 1 || c->vocab_padded < c->vocab) { why = "vocab / vocab_padded"; return 0; }
  if (c->d_model < 8 || c->d_model % 8 || c->d_model > 1024) { why = "d_model must be a multiple of 8 in [8, 1024]"; return 0; }
  if (c->n_heads < 1 || c->d_model % c->n_heads) { why = "d_model must be a multiple of n_heads"; return 0; }
  int d = c->d_model / c->n_heads;
  if (d != 16 && d != 32 && d != 64 && d != 128) { why = "head size must be 16, 32, 64 or 128"; return 0; }
  if (c->d_mlp < 8 || c->d_mlp % 8) { why = "d_mlp must be a positive multiple of 8"; return 0; }
  if (c->n_layers < 1 || c->max_seq < 1 || c->max_batch < 1) { why = "n_layers, max_seq, max_batch >= 1"; return 0; }
  if (c->precision != GPT_PRECISION_FP32 && c->precision != GPT_PRECISION_BF16 && c->precision != GPT_PRECISION_FP16) {
    why = "precision";
    return 0;
  }
  if (!(c->ln_eps > 0.f) || !(c->init_std >= 0.f)) { why = "ln_eps > 0, init_std >= 0"; return 0; }
  if (c->loss_scaling && !(c->init_loss_scale > 0.f)) { why = "init_loss_scale > 0"; return 0; }
  if (c->arch != GPT_ARCH_GPT2 && c->arch != GPT_ARCH_LLAMA) { why = "arch"; return 0; }
  if (c->arch == GPT_ARCH_LLAMA) {
    if (c->precision == GPT_PRECISION_FP32) { why = "the Llama-style block needs 16-bit precision"; return 0; }
    if (d != 64) { why = "the Llama-style block needs head size 64"; return 0; }
    const int hkv = c->n_kv_heads ? c->n_kv_heads : c->n_heads;
    if (hkv < 1 || c->n_heads % hkv) { why = "n_kv_heads must divide n_heads"; return 0; }
    if (c->d_mlp % 16) { why = "d_mlp must be a multiple of 16 for the Llama-style block"; return 0; }
    if (!(c->rope_base >= 0.f)) { why = "rope_base >= 0"; return 0; }
  }
  return 1;
}

static thread_local std::string g_create_err;

// Error text for calls without a model handle (reported by gpt_last_error(NULL)).
void set_global_error(const char* msg) { g_create_err = msg ? msg : ""; }

extern "C" {

int gpt_create(const gpt_config* cfg, uint64_t seed, gpt_model** out) {
  if (!cfg || !out) return GPT_ERR_ARG;
  *out = nullptr;
  std::string why;
  if (!validate_cfg(cfg, why)) { g_create_err = why; return GPT_ERR_ARG; }
  gpt_model* m = new gpt_model();
  m->cfg = *cfg;
  if (cudaGetDevice(&m->device) != cudaSuccess) { delete m; cudaGetLastError(); return GPT_ERR_CUDA; }
  int nsm = 0;
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, m->device) == cudaSuccess && nsm > 0)
    g_num_sms = nsm;
  m->lp = cfg->precision == GPT_PRECISION_BF16 || cfg->precision == GPT_PRECISION_FP16;
  m->fp16 = cfg->precision == GPT_PRECISION_FP16;
  m->V = cfg->vocab; m->Vp = cfg->vocab_padded; m->C = cfg->d_model; m->H = cfg->n_heads;
  m->d = m->C / m->H; m->F = cfg->d_mlp; m->NL = cfg->n_layers; m->Tmax = cfg->max_seq;
  m->Bmax = cfg->max_batch; m->Mmax = (long)m->Bmax * m->Tmax;
  m->ldl = (m->Vp + 7) / 8 * 8;
  m->llama = cfg->arch == GPT_ARCH_LLAMA;
  m->Hkv = m->llama && cfg->n_kv_heads ? cfg->n_kv_heads : m->H;
  m->QW = m->llama ? m->C + 2 * m->Hkv * m->d : 3 * m->C;
  m->UW = m->llama ? 2 * m->F : m->F;
  layout_params(m);
  int r = build_arena(m);
  if (r != GPT_OK) { g_create_err = m->err; delete m; return r; }
  std::vector<float> h;
  init_host_params(m, seed, h);
  cudaError_t e = cudaMemcpy(m->p32, h.data(), m->N * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && m->llama) {
    // rotary table: (cos, sin) of p * base^(-2i/d), evaluated in double precision
    const double base = cfg->rope_base > 0.f ? (double)cfg->rope_base : 10000.0;
    const int hd = m->d / 2;
    std::vector<float2> tab((size_t)m->Tmax * hd);
    for (int p = 0; p < m->Tmax; ++p)
      for (int i = 0; i < hd; ++i) {
        const double a = (double)p * pow(base, -2.0 * i / m->d);
        tab[(size_t)p * hd + i] = make_float2((float)cos(a), (float)sin(a));
      }
    e = cudaMemcpy(m->rope_tab, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess) e = cudaMemset(m->g32, 0, m->N * 4);
  if (e == cudaSuccess) e = cudaMemset(m->m32, 0, m->N * 4);
  if (e == cudaSuccess) e = cudaMemset(m->v32, 0, m->N * 4);
  if (e == cudaSuccess && m->fp16) e = launch_cast<f16>(m->p32, (f16*)m->pw, m->N, 0);
  else if (e == cudaSuccess && m->lp) e = launch_cast<bf16>(m->p32, (bf16*)m->pw, m->N, 0);
  DevScalars sc;
  memset(&sc, 0, sizeof(sc));
  sc.loss_scale = cfg->loss_scaling ? cfg->init_loss_scale : 1.0f;
  sc.loss_scaling = cfg->loss_scaling ? 1 : 0;
  sc.coef = 1.f; sc.bc1 = 1.f; sc.bc2 = 1.f;
  sc.loss_weight = 1.f;
  if (e == cudaSuccess) e = cudaMemcpy(m->sc, &sc, sizeof(sc), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    g_create_err = std::string("initialisation: ") + cudaGetErrorString(e);
    cudaFree(m->arena);
    delete m;
    return GPT_ERR_CUDA;
  }
  *out = m;
  return GPT_OK;
}

void gpt_destroy(gpt_model* m) {
  if (!m) return;
  cudaDeviceSynchronize();
  for (auto e : m->evpool) cudaEventDestroy(e);
  if (m->dec_graph) cudaGraphExecDestroy(m->dec_graph);
  if (m->train_graph) cudaGraphExecDestroy(m->train_graph);
  if (m->ev_a) cudaEventDestroy(m->ev_a);
  if (m->ev_b) cudaEventDestroy(m->ev_b);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  if (m->arena) cudaFree(m->arena);
  delete m;
}

int gpt_set_stream(gpt_model* m, void* stream) {
  if (!m) return GPT_ERR_ARG;
  m->stream = (cudaStream_t)stream;
  return GPT_OK;
}

int gpt_forward_loss(gpt_model* m, const int32_t* tokens, const int32_t* targets, const int32_t* seg_ids, int B,
                     int T, float* loss_dev) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!tokens) FAIL(GPT_ERR_ARG, "tokens is NULL");
  if (B < 1 || B > m->Bmax) FAIL(GPT_ERR_ARG, "B out of range [1, max_batch]");
  if (T < 1 || T > m->Tmax) FAIL(GPT_ERR_ARG, "T out of range [1, max_seq]");
  if (m->fp16) return forward_impl<f16>(m, tokens, targets, seg_ids, B, T, loss_dev);
  if (m->lp) return forward_impl<bf16>(m, tokens, targets, seg_ids, B, T, loss_dev);
  return forward_impl<float>(m, tokens, targets, seg_ids, B, T, loss_dev);
}

int gpt_backward(gpt_model* m) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!m->have_targets) FAIL(GPT_ERR_STATE, "gpt_backward needs a preceding gpt_forward_loss with targets");
  m->accum_now = false;
  if (m->fp16) return backward_impl<f16>(m);
  if (m->lp) return backward_impl<bf16>(m);
  return backward_impl<float>(m);
}

int gpt_backward_accumulate(gpt_model* m) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!m->have_targets) FAIL(GPT_ERR_STATE, "gpt_backward_accumulate needs a preceding gpt_forward_loss with targets");
  m->accum_now = true;
  const int r = m->fp16 ? backward_impl<f16>(m) : m->lp ? backward_impl<bf16>(m) : backward_impl<float>(m);
  m->accum_now = false;
  return r;
}

int gpt_set_loss_weight(gpt_model* m, float w) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!(w > 0.f) || !(w < 1e30f)) FAIL(GPT_ERR_ARG, "loss weight must be positive and finite");
  CK(cudaMemcpyAsync(&m->sc->loss_weight, &w, sizeof(float), cudaMemcpyHostToDevice, m->stream));
  CK(cudaStreamSynchronize(m->stream));
  return GPT_OK;
}

int gpt_clip_adamw_step(gpt_model* m, const gpt_adamw* hp, float* grad_norm_dev, int32_t* skipped_dev) {
  if (!m || !hp) return GPT_ERR_ARG;
  m->err.clear();
  if (!(hp->clip_norm > 0.f)) FAIL(GPT_ERR_ARG, "clip_norm must be > 0");
  cudaStream_t s = m->stream;
  ProfScope ps(m, PC_OPT, 0, (double)m->N * (m->lp ? 34.0 : 32.0));
  {
    // one cooperative launch; the three-launch form below if it cannot run
    cudaError_t e;
    if (m->fp16)
      e = launch_clip_adamw_fused<f16>(m->p32, m->g32, m->m32, m->v32, (f16*)m->pw, m->N, m->normpart, m->normblk,
                                       hp->clip_norm, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, hp->lr, m->sc,
                                       grad_norm_dev, skipped_dev, s);
    else if (m->lp)
      e = launch_clip_adamw_fused<bf16>(m->p32, m->g32, m->m32, m->v32, (bf16*)m->pw, m->N, m->normpart, m->normblk,
                                        hp->clip_norm, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, hp->lr, m->sc,
                                        grad_norm_dev, skipped_dev, s);
    else
      e = launch_clip_adamw_fused<float>(m->p32, m->g32, m->m32, m->v32, nullptr, m->N, m->normpart, m->normblk,
                                         hp->clip_norm, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, hp->lr,
                                         m->sc, grad_norm_dev, skipped_dev, s);
    if (e == cudaSuccess) return GPT_OK;
    cudaGetLastError();
  }
  CK(launch_sumsq(m->g32, m->N, m->normpart, m->normblk, s));
  CK(launch_opt_finalize(m->normpart, m->normblk, hp->clip_norm, hp->beta1, hp->beta2, hp->lr, m->sc,
                         grad_norm_dev, skipped_dev, s));
  if (m->fp16)
    CK(launch_adamw<f16>(m->p32, m->g32, m->m32, m->v32, (f16*)m->pw, m->N, hp->beta1, hp->beta2,
                         hp->eps, hp->weight_decay, m->sc, s));
  else if (m->lp)
    CK(launch_adamw<bf16>(m->p32, m->g32, m->m32, m->v32, (bf16*)m->pw, m->N, hp->beta1, hp->beta2,
                          hp->eps, hp->weight_decay, m->sc, s));
  else
    CK(launch_adamw<float>(m->p32, m->g32, m->m32, m->v32, nullptr, m->N, hp->beta1, hp->beta2,
                           hp->eps, hp->weight_decay, m->sc, s));
  return GPT_OK;
}

int gpt_set_lr_schedule(gpt_model* m, const gpt_lr_schedule* sched) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  gpt_lr_schedule z;
  memset(&z, 0, sizeof(z));
  const gpt_lr_schedule& q = sched ? *sched : z;
  if (q.kind != GPT_LR_CONSTANT && q.kind != GPT_LR_COSINE) FAIL(GPT_ERR_ARG, "unknown schedule kind");
  if (q.kind == GPT_LR_COSINE) {
    if (q.warmup_steps < 0 || q.total_steps <= q.warmup_steps) FAIL(GPT_ERR_ARG, "need 0 <= warmup_steps < total_steps");
    if (!(q.min_lr >= 0.f) || !(q.max_lr >= q.min_lr)) FAIL(GPT_ERR_ARG, "need 0 <= min_lr <= max_lr");
  }
  DevScalars sc;
  CK(cudaStreamSynchronize(m->stream));
  CK(cudaMemcpy(&sc, m->sc, sizeof(sc), cudaMemcpyDeviceToHost));
  sc.sched_kind = q.kind;
  sc.sched_warmup = q.warmup_steps;
  sc.sched_total = q.total_steps;
  sc.sched_max_lr = q.max_lr;
  sc.sched_min_lr = q.min_lr;
  CK(cudaMemcpy(m->sc, &sc, sizeof(sc), cudaMemcpyHostToDevice));
  return GPT_OK;
}

int gpt_train_step(gpt_model* m, const int32_t* tokens, const int32_t* targets, const int32_t* seg_ids, int B, int T,
                   const gpt_adamw* hp, float* loss_dev, float* grad_norm_dev, int32_t* skipped_dev) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!tokens || !targets || !hp) FAIL(GPT_ERR_ARG, "tokens, targets and hp must be non-NULL");
  if (B < 1 || B > m->Bmax) FAIL(GPT_ERR_ARG, "B out of range [1, max_batch]");
  if (T < 1 || T > m->Tmax) FAIL(GPT_ERR_ARG, "T out of range [1, max_seq]");
  if (!(hp->clip_norm > 0.f)) FAIL(GPT_ERR_ARG, "clip_norm must be > 0");
  auto plain = [&]() -> int {
    int r = gpt_forward_loss(m, tokens, targets, seg_ids, B, T, loss_dev);
    if (r == GPT_OK) r = gpt_backward(m);
    if (r == GPT_OK) r = gpt_clip_adamw_step(m, hp, grad_norm_dev, skipped_dev);
    return r;
  };
  // profiling records host-side events per kernel class: no graph then
  if (m->prof || !m->train_graph_ok) return plain();
  gpt_model::TrainKey key;
  memset(&key, 0, sizeof(key));
  key.tok = tokens; key.tgt = targets; key.seg = seg_ids; key.loss = loss_dev; key.gn = grad_norm_dev;
  key.skip = skipped_dev; key.B = B; key.T = T; key.lr = hp->lr; key.beta1 = hp->beta1; key.beta2 = hp->beta2;
  key.eps = hp->eps; key.wd = hp->weight_decay; key.clip = hp->clip_norm;
  if (!m->train_graph || !(key == m->train_key)) {
    if (m->train_graph) { cudaGraphExecDestroy(m->train_graph); m->train_graph = nullptr; }
    if (!m->cap_stream) CK(cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking));
    // capture on the library's own stream (the caller's may be the legacy
    // default stream, which cannot be captured); nothing runs during capture
    cudaStream_t s0 = m->stream;
    m->stream = m->cap_stream;
    const unsigned long long n0 = g_kernel_launches;
    cudaGraph_t g = nullptr;
    cudaError_t eb = cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal);
    int r = GPT_ERR_CUDA;
    unsigned long long n1 = n0;
    if (eb == cudaSuccess) {
      r = plain();
      n1 = g_kernel_launches;
      cudaError_t ec = cudaStreamEndCapture(m->cap_stream, &g);
      if (r == GPT_OK && ec != cudaSuccess) r = GPT_ERR_CUDA;
    }
    m->stream = s0;
    g_kernel_launches = n0;   // counted per replay below
    cudaError_t ei = cudaErrorUnknown;
    if (r == GPT_OK && g) ei = cudaGraphInstantiate(&m->train_graph, g, 0);
    if (g) cudaGraphDestroy(g);
    if (r != GPT_OK || ei != cudaSuccess) {
      // an argument or state error is the caller's; a capture the runtime
      // refused falls back to plain launches for good
      cudaGetLastError();
      m->train_graph = nullptr;
      if (r == GPT_ERR_ARG || r == GPT_ERR_STATE) return r;
      m->train_graph_ok = false;
      m->err.clear();
      return plain();
    }
    m->train_kernels = (int)(n1 - n0);
    m->train_key = key;
  }
  CK(cudaGraphLaunch(m->train_graph, m->stream));
  g_kernel_launches += (unsigned long long)m->train_kernels;
  // the host-side state a plain step leaves
  m->seg_used = seg_ids != nullptr;
  m->fwd_B = B;
  m->fwd_T = T;
  m->have_targets = false;
  m->logits_valid = false;
  m->accum_now = false;
  return GPT_OK;
}

int gpt_train_steps(gpt_model* m, const int32_t* tokens, const int32_t* targets, const int32_t* seg_ids, int K,
                    int B, int T, const gpt_adamw* hp, float* losses_dev, float* grad_norms_dev,
                    int32_t* skipped_dev) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!tokens || !targets || !hp) FAIL(GPT_ERR_ARG, "tokens, targets and hp must be non-NULL");
  if (K < 1) FAIL(GPT_ERR_ARG, "K must be >= 1");
  const size_t bt = (size_t)B * T;
  for (int k = 0; k < K; ++k) {
    CKI(gpt_forward_loss(m, tokens + k * bt, targets + k * bt, seg_ids ? seg_ids + k * bt : nullptr, B, T,
                         losses_dev ? losses_dev + k : nullptr));
    CKI(gpt_backward(m));
    CKI(gpt_clip_adamw_step(m, hp, grad_norms_dev ? grad_norms_dev + k : nullptr,
                            skipped_dev ? skipped_dev + k : nullptr));
  }
  return GPT_OK;
}

int gpt_greedy_decode(gpt_model* m, const int32_t* prompt, int B, int Tp, int n_new, int32_t* out) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!prompt || !out) FAIL(GPT_ERR_ARG, "prompt / out is NULL");
  if (B < 1 || B > m->Bmax || B > 32) FAIL(GPT_ERR_ARG, "B out of range [1, min(max_batch, 32)]");
  if (Tp < 1 || n_new < 1) FAIL(GPT_ERR_ARG, "Tp and n_new must be >= 1");
  if ((long)Tp + n_new - 1 > m->Tmax) FAIL(GPT_ERR_STATE, "Tp + n_new - 1 exceeds max_seq");
  m->have_targets = false;
  if (m->fp16) return decode_impl<f16>(m, prompt, B, Tp, n_new, out);
  if (m->lp) return decode_impl<bf16>(m, prompt, B, Tp, n_new, out);
  return decode_impl<float>(m, prompt, B, Tp, n_new, out);
}

int gpt_sample_decode(gpt_model* m, const int32_t* prompt, int B, int Tp, int n_new, const gpt_sampling* sp,
                      const float* uniforms, int32_t* out) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!prompt || !out || !sp || !uniforms) FAIL(GPT_ERR_ARG, "prompt / out / sampling / uniforms is NULL");
  if (!(sp->temperature >= 0.f) || sp->top_k < 0 || !(sp->top_p > 0.f && sp->top_p <= 1.f))
    FAIL(GPT_ERR_ARG, "need temperature >= 0, top_k >= 0, 0 < top_p <= 1");
  if (m->V > SMP_MAX_VOCAB) FAIL(GPT_ERR_ARG, "vocabulary too large for the sampling kernel");
  if (B < 1 || B > m->Bmax || B > 32) FAIL(GPT_ERR_ARG, "B out of range [1, min(max_batch, 32)]");
  if (Tp < 1 || n_new < 1) FAIL(GPT_ERR_ARG, "Tp and n_new must be >= 1");
  if ((long)Tp + n_new - 1 > m->Tmax) FAIL(GPT_ERR_STATE, "Tp + n_new - 1 exceeds max_seq");
  m->have_targets = false;
  m->smp_on = true;
  m->smp_temp = sp->temperature;
  m->smp_topk = sp->top_k;
  m->smp_topp = sp->top_p;
  m->smp_u = uniforms;
  const int r = m->fp16 ? decode_impl<f16>(m, prompt, B, Tp, n_new, out)
                : m->lp ? decode_impl<bf16>(m, prompt, B, Tp, n_new, out) : decode_impl<float>(m, prompt, B, Tp, n_new, out);
  m->smp_on = false;
  return r;
}

int gpt_beam_decode(gpt_model* m, const int32_t* prompt, int B, int Tp, int n_new, int width, int32_t* out,
                    float* scores) {
  if (!m) return GPT_ERR_ARG;
  m->err.clear();
  if (!prompt || !out || !scores) FAIL(GPT_ERR_ARG, "prompt / out / scores is NULL");
  if (width < 1 || width > BEAM_MAX_WIDTH) FAIL(GPT_ERR_ARG, "width out of range [1, 8]");
  if (m->V < width) FAIL(GPT_ERR_ARG, "width exceeds the vocabulary");
  if (m->V > SMP_MAX_VOCAB) FAIL(GPT_ERR_ARG, "vocabulary too large for the beam kernel");
  if (B < 1 || (long)B * width > m->Bmax || (long)B * width > 32)
    FAIL(GPT_ERR_ARG, "B * width out of range [1, min(max_batch, 32)]");
  if (Tp < 1 || n_new < 1) FAIL(GPT_ERR_ARG, "Tp and n_new must be >= 1");
  if ((long)Tp + n_new - 1 > m->Tmax) FAIL(GPT_ERR_STATE, "Tp + n_new - 1 exceeds max_seq");
  if ((uintptr_t)scores & 3) FAIL(GPT_ERR_ARG, "scores must be 4-byte aligned");
  m->have_targets = false;
  m->beam_w = width;
  m->beam_scores = scores;
  const int r = m->fp16 ? decode_impl<f16>(m, prompt, B, Tp, n_new, out)
                : m->lp ? decode_impl<bf16>(m, prompt, B, Tp, n_new, out) : decode_impl<float>(m, prompt, B, Tp, n_new, out);
  m->beam_w = 0;
  m->beam_scores = nullptr;
  return r;
}

int gpt_num_params(const gpt_model* m, size_t* n) {
  if (!m || !n) return GPT_ERR_ARG;
  *n = m->N;
  return GPT_OK;
}

static int copy_state(gpt_model* m, void* dst, const void* src, size_t n) {
  if (!dst || !src) FAIL(GPT_ERR_ARG, "NULL pointer");
  if (n != m->N) FAIL(GPT_ERR_ARG, "n must equal gpt_num_params");
  CK(cudaStreamSynchronize(m->stream));
  CK(cudaMemcpy(dst, src, n * 4, cudaMemcpyDefault));
  return GPT_OK;
}

int gpt_get_params(gpt_model* m, float* dst, size_t n) { return m ? copy_state(m, dst, m->p32, n) : GPT_ERR_ARG; }
int gpt_get_grads(gpt_model* m, float* dst, size_t n) { return m ? copy_state(m, dst, m->g32, n) : GPT_ERR_ARG; }
int gpt_get_adam_m(gpt_model* m, float* dst, size_t n) { return m ? copy_state(m, dst, m->m32, n) : GPT_ERR_ARG; }
int gpt_get_adam_v(gpt_model* m, float* dst, size_t n) { return m ? copy_state(m, dst, m->v32, n) : GPT_ERR_ARG; }
int gpt_set_grads(gpt_model* m, const float* src, size_t n) { return m ? copy_state(m, m->g32, src, n) : GPT_ERR_ARG; }
int gpt_set_adam_m(gpt_model* m, const float* src, size_t n) { return m ? copy_state(m, m->m32, src, n) : GPT_ERR_ARG; }
int gpt_set_adam_v(gpt_model* m, const float* src, size_t n) { return m ? copy_state(m, m->v32, src, n) : GPT_ERR_ARG; }

int gpt_set_params(gpt_model* m, const float* src, size_t n) {
  if (!m) return GPT_ERR_ARG;
  CKI(copy_state(m, m->p32, src, n));
  if (m->fp16) {
    CK(launch_cast<f16>(m->p32, (f16*)m->pw, m->N, m->stream));
    CK(cudaStreamSynchronize(m->stream));
  } else if (m->lp) {
    CK(launch_cast<bf16>(m->p32, (bf16*)m->pw, m->N, m->stream));
    CK(cudaStreamSynchronize(m->stream));
  }
  return GPT_OK;
}

int gpt_get_logits(gpt_model* m, float* dst, size_t n) {
  if (!m || !dst) return GPT_ERR_ARG;
  m->err.clear();
  if (!m->logits_valid) FAIL(GPT_ERR_STATE, "no logits: run gpt_forward_loss with targets = NULL first");
  int M = m->fwd_B * m->fwd_T;
  if (n != (size_t)M * m->Vp) FAIL(GPT_ERR_ARG, "n must be B*T*vocab_padded");
  cudaPointerAttributes at;
  bool dev = cudaPointerGetAttributes(&at, dst) == cudaSuccess && at.type == cudaMemoryTypeDevice;
  cudaGetLastError();
  float* tmp = dst;
  if (!dev) CK(cudaMalloc((void**)&tmp, n * 4));
  cudaError_t e;
  if (m->fp16) e = launch_to_f32<f16>((const f16*)m->logits, m->ldl, M, m->Vp, tmp, m->stream);
  else if (m->lp) e = launch_to_f32<bf16>((const bf16*)m->logits, m->ldl, M, m->Vp, tmp, m->stream);
  else e = launch_to_f32<float>((const float*)m->logits, m->ldl, M, m->Vp, tmp, m->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(m->stream);
  if (e == cudaSuccess && !dev) e = cudaMemcpy(dst, tmp, n * 4, cudaMemcpyDeviceToHost);
  if (!dev) cudaFree(tmp);
  CK(e);
  return GPT_OK;
}

int gpt_get_residual(gpt_model* m, int layer, float* dst, size_t n) {
  if (!m || !dst) return GPT_ERR_ARG;
  m->err.clear();
  if (m->fwd_B == 0) FAIL(GPT_ERR_STATE, "no forward pass yet");
  if (layer < 0 || layer > m->NL) FAIL(GPT_ERR_ARG, "layer out of range [0, n_layers]");
  int M = m->fwd_B * m->fwd_T;
  if (n != (size_t)M * m->C) FAIL(GPT_ERR_ARG, "n must be B*T*d_model");
  size_t off = (size_t)layer * m->Mmax * m->C;
  cudaPointerAttributes at;
  bool dev = cudaPointerGetAttributes(&at, dst) == cudaSuccess && at.type == cudaMemoryTypeDevice;
  cudaGetLastError();
  float* tmp = dst;
  if (!dev) CK(cudaMalloc((void**)&tmp, n * 4));
  cudaError_t e;
  if (m->fp16) e = launch_to_f32<f16>((const f16*)m->xs + off, m->C, M, m->C, tmp, m->stream);
  else if (m->lp) e = launch_to_f32<bf16>((const bf16*)m->xs + off, m->C, M, m->C, tmp, m->stream);
  else e = launch_to_f32<float>((const float*)m->xs + off, m->C, M, m->C, tmp, m->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(m->stream);
  if (e == cudaSuccess && !dev) e = cudaMemcpy(dst, tmp, n * 4, cudaMemcpyDeviceToHost);
  if (!dev) cudaFree(tmp);
  CK(e);
  return GPT_OK;
}

int gpt_get_scalars(gpt_model* m, gpt_scalars* out) {
  if (!m || !out) return GPT_ERR_ARG;
  DevScalars sc;
  CK(cudaStreamSynchronize(m->stream));
  CK(cudaMemcpy(&sc, m->sc, sizeof(sc), cudaMemcpyDeviceToHost));
  out->loss_scale = sc.loss_scale;
  out->good_steps = sc.good_steps;
  out->step = sc.step;
  out->last_loss = sc.loss;
  out->last_grad_norm = sc.grad_norm;
  out->last_skipped = sc.skipped;
  out->last_lr = sc.lr;
  return GPT_OK;
}

int gpt_set_scalars(gpt_model* m, const gpt_scalars* in) {
  if (!m || !in) return GPT_ERR_ARG;
  DevScalars sc;
  CK(cudaStreamSynchronize(m->stream));
  CK(cudaMemcpy(&sc, m->sc, sizeof(sc), cudaMemcpyDeviceToHost));
  sc.loss_scale = in->loss_scale;
  sc.good_steps = in->good_steps;
  sc.step = in->step;
  CK(cudaMemcpy(m->sc, &sc, sizeof(sc), cudaMemcpyHostToDevice));
  return GPT_OK;
}

int gpt_status(gpt_model* m) {
  if (!m) return GPT_ERR_ARG;
  cudaError_t e = cudaStreamSynchronize(m->stream);
  if (e != cudaSuccess) {
    m->err = std::string("stream: ") + cudaGetErrorString(e);
    return GPT_ERR_CUDA;
  }
  unsigned bits = 0;
  CK(cudaMemcpy(&bits, &m->sc->err, 4, cudaMemcpyDeviceToHost));
  if (!bits) return GPT_OK;
  CK(cudaMemset(&m->sc->err, 0, 4));
  m->err = "device error word 0x" + std::to_string(bits);
  return (bits & GPT_DEVERR_TIMEOUT) ? GPT_ERR_TIMEOUT : GPT_ERR_DEVICE;
}

int gpt_device_error(gpt_model* m, uint32_t* bits) {
  if (!m || !bits) return GPT_ERR_ARG;
  CK(cudaStreamSynchronize(m->stream));
  CK(cudaMemcpy(bits, &m->sc->err, 4, cudaMemcpyDeviceToHost));
  return GPT_OK;
}

const char* gpt_last_error(const gpt_model* m) {
  if (!m) return g_create_err.c_str();
  return m->err.c_str();
}

int gpt_gemm_bf16(int M, int N, int K, const void* A, long lda, int a_t, const void* B, long ldb, int b_t,
                  float* C, long ldc, void* stream) {
  if (!A || !B || !C || M < 1 || N < 1 || K < 1 || ldc < N) return GPT_ERR_ARG;
  if (!gemm_tc_supported(M, N, K, lda, a_t != 0, ldb, b_t != 0)) return GPT_ERR_ARG;
  EpiParams<bf16> e = epi_f32<bf16>(C, ldc);
  static unsigned* err = nullptr;
  if (!err && cudaMalloc((void**)&err, 4) != cudaSuccess) return GPT_ERR_CUDA;
  cudaError_t r = launch_gemm_tc(M, N, K, (const bf16*)A, lda, a_t != 0, (const bf16*)B, ldb, b_t != 0, e, 1, err,
                                 (cudaStream_t)stream);
  return r == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

int gpt_kernel_launches(uint64_t* out) {
  if (!out) return GPT_ERR_ARG;
  *out = g_kernel_launches;
  return GPT_OK;
}

int gpt_profile_enable(gpt_model* m, int on) {
  if (!m) return GPT_ERR_ARG;
  if (on) {
    CK(cudaStreamSynchronize(m->stream));
    m->recs.clear();
    m->evused = 0;
  }
  m->prof = on != 0;
  return GPT_OK;
}

int gpt_profile_read(gpt_model* m, gpt_prof_entry* out, int max_entries, int* n_out) {
  if (!m || !out || !n_out || max_entries < 0) return GPT_ERR_ARG;
  CK(cudaStreamSynchronize(m->stream));
  gpt_prof_entry acc[PC_COUNT];
  memset(acc, 0, sizeof(acc));
  unsigned long long pairs = 0;
  CK(cudaMemcpy(&pairs, &m->sc->attn_pairs, sizeof(pairs), cudaMemcpyDeviceToHost));
  for (auto& r : m->recs) {
    if (!r.b) continue;
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, r.a, r.b));
    acc[r.cls].launches += 1;
    acc[r.cls].ms += ms;
    acc[r.cls].flops += r.flops + r.pair_mult * (double)pairs;
    acc[r.cls].bytes += r.bytes;
  }
  int n = 0;
  for (int c = 0; c < PC_COUNT && n < max_entries; ++c) {
    if (!acc[c].launches) continue;
    out[n] = acc[c];
    strncpy(out[n].name, kProfNames[c], sizeof(out[n].name) - 1);
    ++n;
  }
  *n_out = n;
  return GPT_OK;
}

int gpt_debug_poison_grad(gpt_model* m, size_t index, float value) {
  if (!m) return GPT_ERR_ARG;
  if (index >= m->N) FAIL(GPT_ERR_ARG, "index out of range");
  CK(cudaStreamSynchronize(m->stream));
  CK(cudaMemcpy(m->g32 + index, &value, 4, cudaMemcpyHostToDevice));
  return GPT_OK;
}

int gpt_debug_wait_timeout(gpt_model* m, int timeout_us) {
  if (!m || timeout_us < 1 || timeout_us > 10000000) return GPT_ERR_ARG;
  int khz = 0;
  CK(cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, m->device));
  long long cycles = (long long)khz * timeout_us / 1000;
  CK(launch_wait_timeout_probe(&m->sc->err, cycles, m->stream));
  return gpt_status(m);
}

}  // extern "C"
