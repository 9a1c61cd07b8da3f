// Flash attention on tcgen05 tensor cores (sm_100a), head size 64, causal
// with the block-diagonal mask of packed documents (query i sees keys j with
// dstart[i] <= j <= i).  Same layouts as the other attention kernels: qkv
// [B*T, 3C] (or any column layout with the query, key and value heads at
// given column offsets: grouped key/value heads), out / dout [B*T, C],
// lse / D [B, H, T].
//
// Both kernels are warp-specialised, one CTA per SM (all 512 TMEM columns):
//   warp 0     TMA producer (tiles of Q, K, V, dO with a 128-byte swizzle)
//   warp 1     MMA issuer (one thread; tcgen05.mma kind::f16, M = 128)
//   the rest   elementwise warps: thread t owns accumulator row t (TMEM lane
//              t); they read scores from TMEM and write P (TMEM) or dS
//              (shared memory) as the next MMA's operand.
//
//   forward   CTA = two 128-query tiles, 128-key blocks: S = Q K^T in one of
//             three rotating TMEM buffers, P = exp2(S log2e / 8 - m) written
//             back over S as 16-bit pairs, O += P V in TMEM (A from TMEM).
//   backward  CTA = 128 keys, 128-query blocks: S^T = K Q^T, dP^T = V dO^T
//             (TMEM); P^T (TMEM) and dS^T = P^T (dP^T - D) (smem); dV += P^T
//             dO and dK += dS^T Q accumulate in TMEM across query blocks;
//             dQ = dS K per block, added in fp32 to a global accumulator by
//             TMA bulk reduce-add.
// A 64-wide 16-bit row is one 128-byte swizzle atom, so one shared-memory
// tile serves as a K-major operand and as an MN-major one.  Blocks outside
// the document ranges are skipped, not masked.
#include "tc_common.cuh"

#define AT_D 64
#define AT_BLK 128
#define AT_TILE_BYTES (AT_BLK * AT_D * 2)   // 16 KB: 128 rows x 128 B
#define LOG2E_F 1.4426950408889634f

__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return smem_desc(addr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, uint32_t lbo) { return smem_desc(addr, lbo, 1024); }

__device__ __forceinline__ uint32_t pk_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Bounded barrier among the 128 softmax threads (an mbarrier with count 128):
// every thread arrives, then waits for the phase to complete.
__device__ __forceinline__ bool group_sync(uint32_t bar, uint32_t& phase, volatile int* abort_flag) {
  mbar_arrive(bar);
  bool ok = mbar_wait(bar, phase, abort_flag);
  phase ^= 1;
  return ok;
}

__device__ __forceinline__ void trap_timeout(volatile int* abort_flag, unsigned* err) {
  *abort_flag = 1;
  atomicOr(err, GPT_DEVERR_TIMEOUT);
}

#define AT_BK 64                             // iterated block (keys in fwd / dQ, queries in dK dV)
#define AT_HALF (AT_BK * AT_D * 2)           // 8 KB: 64 rows x 128 B

__device__ __forceinline__ void tc_alloc(uint32_t slot, int cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(cols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tc_dealloc(uint32_t tmem, int cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(cols));
}

__device__ __forceinline__ int ld_once(const int* p) {
  int v;
  asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// D[tmem] (+)= A[tmem] * B[smem]: A is read from tensor memory (128 lanes x 16 bf16).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Packed fp32 pairs (sm_100): (d0, d1) = (a0, a1) * b + c and (a0, a1) + (b0, b1).
__device__ __forceinline__ void fma_x2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n.reg .b64 ra, rb, rc, rd;\nmov.b64 ra, {%2, %3};\nmov.b64 rb, {%4, %4};\nmov.b64 rc, {%5, %5};\n"
      "fma.rn.f32x2 rd, ra, rb, rc;\nmov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
__device__ __forceinline__ void add_x2(float& a0, float& a1, float b0, float b1) {
  asm("{\n.reg .b64 ra, rb;\nmov.b64 ra, {%0, %1};\nmov.b64 rb, {%2, %3};\n"
      "add.rn.f32x2 ra, ra, rb;\nmov.b64 {%0, %1}, ra;\n}\n"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}

__device__ __forceinline__ void fma_x2v(float& d0, float& d1, float a0, float a1, float b0, float b1, float c) {
  asm("{\n.reg .b64 ra, rb, rc, rd;\nmov.b64 ra, {%2, %3};\nmov.b64 rb, {%4, %5};\nmov.b64 rc, {%6, %6};\n"
      "fma.rn.f32x2 rd, ra, rb, rc;\nmov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c));
}

// 2^x for a pair of arguments on the FMA pipe instead of the MUFU unit:
// x = n + f with n = round(x) (the 1.5 * 2^23 rounding trick) and f in
// [-1/2, 1/2]; 2^f by a cubic fitted here as a near-minimax relative
// approximation on that interval (max relative error 7.7e-5, about 2^-13.7,
// far below the 2^-9 of the bf16 P it feeds); 2^n is added to the exponent
// field.  Arguments below -126 are clamped (their P is 0 in bf16 anyway).
#define EXP2_C0 0.99992877245f
#define EXP2_C1 0.69326078892f
#define EXP2_C2 0.24260069430f
#define EXP2_C3 0.05516735464f
__device__ __forceinline__ void exp2_poly_x2(float x0, float x1, float& y0, float& y1) {
  const float RND = 12582912.0f;   // 1.5 * 2^23
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  float t0 = x0, t1 = x1;
  add_x2(t0, t1, RND, RND);
  float n0 = t0, n1 = t1;
  add_x2(n0, n1, -RND, -RND);
  float f0 = x0, f1 = x1;
  add_x2(f0, f1, -n0, -n1);
  float p0, p1;
  fma_x2v(p0, p1, f0, f1, EXP2_C3, EXP2_C3, EXP2_C2);
  fma_x2v(p0, p1, p0, p1, f0, f1, EXP2_C1);
  fma_x2v(p0, p1, p0, p1, f0, f1, EXP2_C0);
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Pairs k of a 32-score chunk (k = 0..15) with (k & 7) < FW_POLY_PAIRS take
// the polynomial, the others the MUFU ex2: the two units run side by side.
#ifndef FW_POLY_PAIRS
#define FW_POLY_PAIRS 0
#endif

// Optional: exponentials two at a time with ex2.approx.f16x2 on fp16 pairs of
// arguments (at most 2^8 under the lazy running max; the row sums stay fp32).
// Off by default: measured slower than two fp32 ex2 (the pair costs the MUFU
// the same, and the conversions cost issue slots) and less accurate.
#ifndef FW_EXP16
#define FW_EXP16 0
#endif
__device__ __forceinline__ uint32_t ex2_f16x2(uint32_t a) {
  uint32_t d;
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// One 32-score chunk of a row: fold the (masked) raw scores into mx
// (three-input max), put P = exp2(s sl2 - mb) as 16 packed 16-bit pairs into
// pw and add their sum to sum.  Masked chunks keep key e (0..31) when
// lo <= e <= hi (relative to the chunk), branch-free: ((e - lo) | (hi - e))
// >= 0.  The exponent arguments and the sums run as packed fp32 pairs.
template <bool MASK, bool F16>
__device__ __forceinline__ void fwd_chunk(const uint32_t* sr, int lo, int hi, float sl2, float mb, uint32_t* pw,
                                          float& mx, float& sum) {
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float s0 = __uint_as_float(sr[e]), s1 = __uint_as_float(sr[e + 1]);
    if (MASK) {
      s0 = ((e - lo) | (hi - e)) >= 0 ? s0 : -INFINITY;
      s1 = ((e + 1 - lo) | (hi - e - 1)) >= 0 ? s1 : -INFINITY;
    }
    mx = fmax3f(mx, s0, s1);
    float x0, x1;
    fma_x2(x0, x1, s0, s1, sl2, -mb);
    float p0, p1;
    if constexpr (FW_EXP16) {
      const uint32_t e2 = ex2_f16x2(pack16x2<true>(x0, x1));
      const float2 pf = __half22float2(*reinterpret_cast<const __half2*>(&e2));
      p0 = pf.x;
      p1 = pf.y;
      add_x2(l0, l1, p0, p1);
      pw[e / 2] = F16 ? e2 : pack16x2<false>(p0, p1);
      continue;
    }
    if (((e >> 1) & 7) < FW_POLY_PAIRS) {
      exp2_poly_x2(x0, x1, p0, p1);
      if (MASK) {   // the polynomial maps -inf to a tiny value, not 0
        p0 = s0 == -INFINITY ? 0.f : p0;
        p1 = s1 == -INFINITY ? 0.f : p1;
      }
    } else {
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    add_x2(l0, l1, p0, p1);
    pw[e / 2] = pack16x2<F16>(p0, p1);
  }
  sum += l0 + l1;
}

// One pass over a row's 128 scores at tS with the running max mb: four
// chunks of 32, each chunk's TMEM load issued before the previous chunk's
// arithmetic (tcgen05.wait::ld waits for every load in flight, so each wait
// covers a load that had a chunk of arithmetic to land).  P of chunk c goes
// over columns 16c..16c+15 of S, whose scores (chunk c/2) are already in
// registers.  A chunk whose max exceeds thr (the running max + 2^8 in the
// exp2 domain, voted warp-wide) stops the pass before its P is stored:
// the return value is that chunk (4: none), and S of it and of every later
// chunk is still intact.  sum collects the stored chunks' P.
template <bool MASK, bool F16>
__device__ __forceinline__ int fwd_pass(uint32_t tS, int lo, int hi, float sl2, float mb, float thr, float& mx,
                                        float& sum) {
  uint32_t ra[32], rb[32], pw[16];
  tmem_ld32(tS, ra);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t* cur = (c & 1) ? rb : ra;
    uint32_t* nxt = (c & 1) ? ra : rb;
    if (c + 1 < 4) tmem_ld32(tS + 32 * (c + 1), nxt);
    float csum = 0.f;
    fwd_chunk<MASK, F16>(cur, lo - 32 * c, hi - 32 * c, sl2, mb, pw, mx, csum);
    if (c + 1 < 4) tmem_wait_ld();
    if (__any_sync(0xffffffffu, mx * sl2 > thr)) return c;
    sum += csum;
    tmem_st16(tS + 16 * c, pw);
  }
  return 4;
}

// The rare continuation of a pass stopped at chunk ct (the block raised the
// max past the threshold): the block max over the remaining chunks gives the
// new running max m_new; the P already stored (chunks < ct, each <= 2^8) is
// scaled by 2^(mb - m_new) in place (a power of two: exact unless it
// underflows), and chunks ct..3 are exponentiated with m_new.  mb is the
// max the stored P was computed with (0 where m_use is still -inf).
template <bool MASK, bool F16>
__device__ __noinline__ void fwd_raise(uint32_t tS, int lo, int hi, float sl2, float m_use, float mb, int ct,
                                       float mx_before, float& m_new, float& sum) {
  tmem_wait_st();   // the P of chunks < ct is read back below
  float mx = mx_before;
  for (int c = ct; c < 4; ++c) {
    uint32_t ra[32];
    tmem_ld32(tS + 32 * c, ra);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float s0 = __uint_as_float(ra[e]);
      if (MASK) s0 = ((e - (lo - 32 * c)) | ((hi - 32 * c) - e)) >= 0 ? s0 : -INFINITY;
      mx = fmaxf(mx, s0);
    }
  }
  m_new = fmaxf(m_use, mx * sl2);
  // a row with no allowed key yet keeps m_new = -inf (all its P are 0)
  const float mb_new = m_new == -INFINITY ? 0.f : m_new;
  // no running max yet: the chunks already stored held no allowed key (any
  // finite score stops the pass), so their P and sum are exactly 0
  const float sc = m_use == -INFINITY ? 0.f : exp2f(mb - mb_new);
  sum *= sc;
  for (int c = 0; c < ct; ++c) {
    uint32_t pw[16];
    tmem_ld16(tS + 16 * c, pw);
    tmem_wait_ld();
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f[8];
      unpack16x8<F16>(make_uint4(pw[4 * u], pw[4 * u + 1], pw[4 * u + 2], pw[4 * u + 3]), f);
#pragma unroll
      for (int e = 0; e < 4; ++e) pw[4 * u + e] = pack16x2<F16>(f[2 * e] * sc, f[2 * e + 1] * sc);
    }
    tmem_st16(tS + 16 * c, pw);
  }
  for (int c = ct; c < 4; ++c) {
    uint32_t ra[32], pw[16];
    tmem_ld32(tS + 32 * c, ra);
    tmem_wait_ld();
    float dummy = -INFINITY;
    fwd_chunk<MASK, F16>(ra, lo - 32 * c, hi - 32 * c, sl2, mb_new, pw, dummy, sum);
    tmem_st16(tS + 16 * c, pw);
  }
}

// The row's (masked) maximum score over a block, without exponentials: the
// first block of a row sets the running max from it.
template <bool MASK>
__device__ __forceinline__ float fwd_max(uint32_t tS, int lo, int hi) {
  uint32_t ra[32];
  float mx = -INFINITY;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    tmem_ld32(tS + 32 * c, ra);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      float s0 = __uint_as_float(ra[e]), s1 = __uint_as_float(ra[e + 1]);
      if (MASK) {
        s0 = ((e - (lo - 32 * c)) | ((hi - 32 * c) - e)) >= 0 ? s0 : -INFINITY;
        s1 = ((e + 1 - (lo - 32 * c)) | ((hi - 32 * c) - e - 1)) >= 0 ? s1 : -INFINITY;
      }
      mx = fmax3f(mx, s0, s1);
    }
  }
  return mx;
}

// ============================================================== forward
// CTA = two 128-query tiles (256 queries) sharing each 128-key block of K
// and V.  Per tile g and key block j:
//   S = Q_g K_j^T                (TMEM, 128 x 128 fp32)
//   P = exp2(S log2e / 8 - m)    (16-bit pairs, written over S's first 64 columns)
//   O_g += P V_j                 (TMEM, 128 x 64 fp32, A operand from TMEM)
// The (tile, key block) items run in the order (j, g); their score tiles
// rotate through three TMEM buffers, so the MMA warp computes the next
// items' S while the softmax warps work on the current ones and a tile's
// softmax warps go from one block to the next without waiting for an MMA.
// A buffer is reused three items later: its S MMA is issued after the P V
// MMA that read its P (tcgen05.mma ops of one thread run in issue order).
// The running max m is set by a row's first block (a max-only pass) and later
// raised (O and l rescaled) only when a block's max exceeds it by more than
// 2^8; otherwise the stale max is kept, which bounds every P by 256.  P is
// held in registers until that check, so a block that does raise the max is
// exponentiated again from S.
// 320 threads: warp 0 loads, warp 1 issues MMAs, warps 2-5 (tile 0) and 6-9
// (tile 1) run the softmax, thread t of a group owning query row t.
#define FW_THREADS 320
#define FW_QT 256                                    // queries per CTA
#define FW_ST 3                                      // K / V stages
#define FW_NB 3                                      // score buffers
#define FW_RESCALE 8.0f                              // log2 of the largest tolerated P
struct FwdSmem {
  static constexpr int Q = 0;                        // 2 tiles x 16 KB
  static constexpr int KV = Q + 2 * AT_TILE_BYTES;   // FW_ST stages x (K 16 KB, V 16 KB)
  static constexpr int BAR = KV + FW_ST * 2 * AT_TILE_BYTES;
  static constexpr int TOTAL = BAR + 256;
  static constexpr int TMEM_COLS = 512;              // O_g at 64 g; score buffer k at 128 + 128 k
};

template <bool F16>
__global__ void __launch_bounds__(FW_THREADS, 1)
attn_fwd_tc(const __grid_constant__ CUtensorMap tmQKV, bf16* __restrict__ out, float* __restrict__ lse,
            const int* __restrict__ dstart, int T, int H, int kcol0, int vcol0, int G, unsigned* err, float sl2) {
  // sl2 = log2(e) / sqrt(d): the score scale in the exp2 domain (d = 64, or
  // the true head size of heads zero-padded to 64 columns)
  extern __shared__ __align__(1024) uint8_t at_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)at_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + FwdSmem::BAR);
  // Parity waits need the waiter within one phase of the barrier, so
  // S_FULL + 2 k + g: S of tile g's items in buffer k (a barrier per tile:
  // a tile's first item can sit several items into the sequence, behind
  // the other tile's uses of the same buffer);
  // O_DONE + 2 g + (m & 1): P V of tile g's m-th block complete (two barriers
  // per tile, alternating, so that a waiter is never two phases behind)
  enum { Q_FULL = 0, KV_FULL = 1, KV_EMPTY = 1 + FW_ST, S_FULL = 1 + 2 * FW_ST, P_FULL = S_FULL + 2 * FW_NB,
         O_DONE = P_FULL + FW_NB, DRAIN = O_DONE + 4, NBARS = DRAIN + 1 };
  uint32_t* tmem_slot = (uint32_t*)(bars + NBARS);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  int* s_info = (int*)(tmem_slot + 2);
  const uint32_t b0 = smem_u32(bars);
  auto bar = [&](int i) { return b0 + 8u * i; };
  const uint32_t sQ = smem_u32(sm + FwdSmem::Q), sKV = smem_u32(sm + FwdSmem::KV);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqt = (T + FW_QT - 1) / FW_QT;
  const int qt = nqt - 1 - blockIdx.y;   // heaviest query tiles first (y is the slow grid index)
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const int C = H * AT_D;
  const int q0 = qt * FW_QT;
  const long rowbase = (long)b * T;
  const int* dsr = dstart + rowbase;
  griddep_wait();
  griddep_release();

  if (threadIdx.x == 0) {
    mbar_init(bar(Q_FULL), 1);
    for (int i = 0; i < FW_ST; ++i) {
      mbar_init(bar(KV_FULL + i), 1);
      mbar_init(bar(KV_EMPTY + i), 1);
    }
    for (int k = 0; k < FW_NB; ++k) {
      mbar_init(bar(S_FULL + 2 * k), 1);
      mbar_init(bar(S_FULL + 2 * k + 1), 1);
      mbar_init(bar(P_FULL + k), 4);
    }
    for (int k = 0; k < 4; ++k) mbar_init(bar(O_DONE + k), 1);
    mbar_init(bar(DRAIN), 1);
    *abort_flag = 0;
    // key blocks of each tile: from its first query's document start to its last query
    for (int g = 0; g < 2; ++g) {
      const int qa = min(q0 + 128 * g, T - 1), qz = min(q0 + 128 * g + 127, T - 1);
      s_info[2 * g] = dsr[qa] / AT_BLK;
      s_info[2 * g + 1] = qz / AT_BLK;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) tc_alloc(smem_u32(tmem_slot), FwdSmem::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int lo0 = s_info[0], hi0 = s_info[1], lo1 = s_info[2], hi1 = s_info[3];
  const bool two = q0 + 128 < T;          // the second tile has queries
  const int jlo = lo0, jhi = two ? hi1 : hi0;   // document starts and last queries never decrease
  auto in_tile = [&](int g, int j) { return g == 0 ? (j >= lo0 && j <= hi0) : (two && j >= lo1 && j <= hi1); };
  // items (tile g, block j) in (j, g) order: the index of (g, j) and the total
  auto blocks_before = [&](int g, int j) {
    if (g == 1 && !two) return 0;
    const int lo_ = g ? lo1 : lo0, e = min(j, (g ? hi1 : hi0) + 1);
    return e > lo_ ? e - lo_ : 0;
  };
  auto item_of = [&](int g, int j) {
    return blocks_before(0, j) + blocks_before(1, j) + ((g == 1 && in_tile(0, j)) ? 1 : 0);
  };
  const int n_items = blocks_before(0, jhi + 1) + blocks_before(1, jhi + 1);

  if (warp == 0 && lane == 0) {
    // ---------------- producer
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQKV)) : "memory");
    mbar_expect_tx(bar(Q_FULL), 2 * AT_TILE_BYTES);
    tma_load_2d(sQ, &tmQKV, bar(Q_FULL), h * AT_D, (int)(rowbase + q0));
    tma_load_2d(sQ + AT_TILE_BYTES, &tmQKV, bar(Q_FULL), h * AT_D, (int)(rowbase + q0 + 128));
    bool ok = true;
    for (int j = jlo; j <= jhi && ok; ++j) {
      const int n = j - jlo, st = n % FW_ST;
      if (!mbar_wait(bar(KV_EMPTY + st), ((n / FW_ST) & 1) ^ 1, abort_flag)) { ok = false; break; }
      mbar_expect_tx(bar(KV_FULL + st), 2 * AT_TILE_BYTES);
      const uint32_t dst = sKV + st * 2 * AT_TILE_BYTES;
      tma_load_2d(dst, &tmQKV, bar(KV_FULL + st), kcol0 + (h / G) * AT_D, (int)(rowbase + j * AT_BLK));
      tma_load_2d(dst + AT_TILE_BYTES, &tmQKV, bar(KV_FULL + st), vcol0 + (h / G) * AT_D, (int)(rowbase + j * AT_BLK));
    }
    if (!ok) trap_timeout(abort_flag, err);
    volatile int never = 0;
    mbar_wait(bar(Q_FULL), 0, &never, 1ll << 28);
    const int nj = jhi - jlo + 1;
    for (int n = max(0, nj - FW_ST); n < nj; ++n) mbar_wait(bar(KV_FULL + n % FW_ST), (n / FW_ST) & 1, &never, 1ll << 28);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: S of item i + FW_NB is issued right after P V of item i
    constexpr uint32_t ID_S = instr_desc_t(F16, 128, false, false);   // S = Q K^T: 128 x 128, K = 64
    constexpr uint32_t ID_O = instr_desc_t(F16, 64, false, true);     // O = P V: 128 x 64, K = 128 keys (V MN-major)
    bool ok = mbar_wait(bar(Q_FULL), 0, abort_flag);
    int np0 = 0, np1 = 0;   // P V products issued per tile
    // item iterators: (g, j) of the next S and the next P V
    auto advance = [&](int& g, int& j) {
      do {
        if (g == 0) g = 1;
        else { g = 0; ++j; }
      } while (j <= jhi && !in_tile(g, j));
    };
    int sg = 0, sj = jlo, pg = 0, pj = jlo;
    if (!in_tile(0, jlo)) { advance(sg, sj); advance(pg, pj); }
    auto issue_s = [&](int i, int g, int j) -> bool {
      const int n = j - jlo;
      if (!mbar_wait(bar(KV_FULL + n % FW_ST), (n / FW_ST) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t sK = sKV + (n % FW_ST) * 2 * AT_TILE_BYTES, q = sQ + g * AT_TILE_BYTES;
      const uint32_t d = tmem + 128 + 128 * (i % FW_NB);
#pragma unroll
      for (int k = 0; k < AT_D / 16; ++k) umma_bf16(d, kdesc(q + k * 32), kdesc(sK + k * 32), ID_S, k > 0);
      umma_commit(bar(S_FULL + 2 * (i % FW_NB) + g));
      return true;
    };
    int is = 0;
    for (; is < FW_NB && is < n_items && ok; ++is) {
      ok = issue_s(is, sg, sj);
      advance(sg, sj);
    }
    for (int i = 0; i < n_items && ok; ++i) {
      // P V of item i, once its softmax has written P
      if (!mbar_wait(bar(P_FULL + i % FW_NB), (i / FW_NB) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const int n = pj - jlo;
      const uint32_t sV = sKV + (n % FW_ST) * 2 * AT_TILE_BYTES + AT_TILE_BYTES;
      const uint32_t pbuf = tmem + 128 + 128 * (i % FW_NB);
#pragma unroll
      for (int kk = 0; kk < AT_BLK / 16; ++kk)
        umma_bf16_ts(tmem + 64 * pg, pbuf + 8 * kk, mndesc(sV + kk * 2048, 8192), ID_O,
                     ((pg ? np1 : np0) > 0 || kk > 0));
      umma_commit(bar(O_DONE + 2 * pg + ((pg ? np1 : np0) & 1)));
      if (pg) ++np1;
      else ++np0;
      const int pj_done = pj;
      advance(pg, pj);
      if (pj != pj_done) umma_commit(bar(KV_EMPTY + n % FW_ST));   // K / V of block pj_done no longer read
      if (is < n_items) {
        if (!issue_s(is, sg, sj)) { ok = false; break; }
        advance(sg, sj);
        ++is;
      }
    }
    if (!ok) trap_timeout(abort_flag, err);
    umma_commit(bar(DRAIN));
    volatile int never = 0;
    mbar_wait(bar(DRAIN), 0, &never, 1ll << 28);
  } else if (warp >= 2) {
    // ---------------- softmax warps: thread owns query row r of tile g
    const int quarter = warp & 3;
    const int g = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int q = q0 + 128 * g + r;
    const bool qv = q < T;
    // document starts are read once into registers (a volatile load: the
    // compiler must not re-issue it inside the per-element mask)
    const int ds_q = qv ? ld_once(dsr + q) : 0x7fffffff;
    const int lo = g == 0 ? lo0 : lo1, hi = g == 0 ? hi0 : hi1;
    const int qlast = min(q0 + 128 * g + 127, T - 1);
    const int ds_last = ld_once(dsr + qlast);
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off + 64 * g;
    auto wait_w = [&](uint32_t bb, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bb, parity, abort_flag)); };
    // wait until P V of this tile's m-th block has completed.  Called for m
    // in increasing order, each m at a point where P V of block m - 2 has been
    // waited for and P V of block m + 2 cannot have been issued, so the
    // barrier is within one phase of the one asked for.
    auto wait_pv = [&](int m) { return wait_w(bar(O_DONE + 2 * g + (m & 1)), (m >> 1) & 1); };
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    int n = 0;
    uint32_t su = 0;   // bit k: parity of this tile's next use of score buffer k
    if (g == 0 || two) {
      for (int j = lo; j <= hi; ++j, ++n) {
        if (n >= 2 && !wait_pv(n - 2)) { ok = false; break; }
        const int it = item_of(g, j), kb = it % FW_NB;
        const uint32_t tS = tmem + lane_off + 128 + 128 * kb;
        if (!wait_w(bar(S_FULL + 2 * kb + g), (su >> kb) & 1)) { ok = false; break; }
        su ^= 1u << kb;
        tc_fence_after();
        const int kb0 = j * AT_BLK;
        // masked blocks: a key may be later than a query or before its document
        // (voted warp-wide so the warp runs one code path)
        const bool need_mask = __any_sync(0xffffffffu, kb0 + AT_BLK - 1 > q0 + 128 * g || ds_last > kb0 || !qv);
        const int lo_h = ds_q - kb0, hi_h = q - kb0;   // allowed keys relative to the block
        if (n == 0) {
          // the row's first block sets the running max (no O or l to rescale yet)
          const float m0 = (need_mask ? fwd_max<true>(tS, lo_h, hi_h) : fwd_max<false>(tS, lo_h, hi_h)) * sl2;
          m_use = m0;
        }
        float bsum = 0.f, mx = -INFINITY;
        const float mb = m_use == -INFINITY ? 0.f : m_use;
        const float thr = m_use + FW_RESCALE;
        const int ct = need_mask ? fwd_pass<true, F16>(tS, lo_h, hi_h, sl2, mb, thr, mx, bsum)
                                 : fwd_pass<false, F16>(tS, lo_h, hi_h, sl2, mb, thr, mx, bsum);
        if (ct < 4) {
          // this block raised the max past the threshold (never the first
          // block): finish it with the new max, then scale O (P V of the
          // earlier blocks: wait for the last one) and l
          float m_new;
          if (need_mask) fwd_raise<true, F16>(tS, lo_h, hi_h, sl2, m_use, mb, ct, mx, m_new, bsum);
          else fwd_raise<false, F16>(tS, lo_h, hi_h, sl2, m_use, mb, ct, mx, m_new, bsum);
          const float sc = m_use == -INFINITY ? 0.f : exp2f(m_use - m_new);
          if (!wait_pv(n - 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t orr[32];
            tmem_ld32(tO + 32 * c, orr);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * sc);
            tmem_st32(tO + 32 * c, orr);
          }
          l *= sc;
          m_use = m_new;
        }
        l += bsum;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(P_FULL + it % FW_NB));
      }
    }
    if (!ok) trap_timeout(abort_flag, err);
    // O / l for the row, after the last P V (and the one before it, in order)
    if (ok && n >= 2) ok = wait_pv(n - 2);
    if (ok && n > 0 && wait_pv(n - 1)) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16* orow = out + (rowbase + q) * C + h * AT_D;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t orr[32];
        tmem_ld32(tO + 32 * c, orr);
        tmem_wait_ld();
        if (qv) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            w.x = pack16x2<F16>(__uint_as_float(orr[8 * u]) * inv, __uint_as_float(orr[8 * u + 1]) * inv);
            w.y = pack16x2<F16>(__uint_as_float(orr[8 * u + 2]) * inv, __uint_as_float(orr[8 * u + 3]) * inv);
            w.z = pack16x2<F16>(__uint_as_float(orr[8 * u + 4]) * inv, __uint_as_float(orr[8 * u + 5]) * inv);
            w.w = pack16x2<F16>(__uint_as_float(orr[8 * u + 6]) * inv, __uint_as_float(orr[8 * u + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + 32 * c + 8 * u) = w;
          }
        }
      }
      if (qv) lse[(long)bh * T + q] = m_use + log2f(l);   // base-2 log-sum-exp of the scaled scores
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tc_dealloc(tmem, FwdSmem::TMEM_COLS);
}

// ============================================================== backward
// Work items are (head, 128-key block) pairs; the grid is persistent (one CTA
// per SM) and a CTA takes items blockIdx.x, blockIdx.x + gridDim.x, ... in
// key-block-major order (the first key blocks see the most queries, so the
// heaviest items go first).  For its item the CTA walks the 128-query blocks
// that can see the keys and, per block,
//   S^T = K Q^T, dP^T = V dO^T                  (TMEM, 128 x 128 each)
//   P^T = exp2(S^T log2e / 8 - lse2)            (bf16, back into TMEM; lse2 is
//                                                 the forward's base-2 log-sum-exp)
//   dS^T = P^T (dP^T - D)                       (bf16, shared memory)
//   dV += P^T dO,  dK += dS^T Q                  (TMEM, across query blocks)
//   dQ_blk = dS K                                (TMEM; added in fp32 to a
//                                                 global accumulator by a TMA
//                                                 bulk reduce, scaled by 1/8
//                                                 and rounded by a final pass)
// K and V are double-buffered across items, so the next item's keys (and its
// first query blocks) load while the current item finishes; the per-block
// barriers run on a block counter that continues across items.
// 352 threads: warp 0 loads, warp 1 issues MMAs, warps 2-9 are two groups of
// four elementwise warps (group g handles query columns 64g..64g+63 of the
// score tiles and d columns 32g..32g+31 of the dQ, dK, dV accumulators) and
// warp 10 issues the dQ bulk reduces.
#define BW_THREADS 352
#define BW_QB 128                                    // queries per iterated block
#ifndef BW_ST
#define BW_ST 2                                      // Q / dO pipeline stages
#endif
#ifndef BW_KVB
#define BW_KVB 2                                     // K / V buffers (items in flight)
#endif
// The MMA warp issues the next item's first S^T before this item's last dV / dK
// / dQ (whose completion frees this item's K / V buffer): one buffer would
// deadlock that look-ahead.
static_assert(BW_KVB >= 2, "the MMA look-ahead across items needs two K / V buffers");
#define BW_MAX_ITEMS 128                             // items per CTA (at most)
struct BwdSmem {
  static constexpr int K = 0;                        // BW_KVB buffers x 16 KB: 128 keys x 64
  static constexpr int V = K + BW_KVB * AT_TILE_BYTES;
  static constexpr int Q = V + BW_KVB * AT_TILE_BYTES;   // BW_ST stages x 16 KB
  static constexpr int DO = Q + BW_ST * AT_TILE_BYTES;
  static constexpr int DST = DO + BW_ST * AT_TILE_BYTES;   // 32 KB: [128 keys][128 queries] as two 64-query blocks
  static constexpr int DQS = DST + 2 * AT_TILE_BYTES;      // 2 groups x 16 KB: [128 queries][32 fp32]
  static constexpr int AUX = DQS + 2 * AT_TILE_BYTES;      // BW_ST stages x (lse2, D, dstart) x 128
  static constexpr int NIT = AUX + BW_ST * 3 * BW_QB * 4;  // query blocks of each of the CTA's items
  static constexpr int BAR = NIT + BW_MAX_ITEMS * 4;
  static constexpr int TOTAL = BAR + 256;
  // TMEM columns: S^T 0, dP^T 128, dV 256, dK 320, dQ 384, P^T (bf16 pairs) 448
  static constexpr int TMEM_COLS = 512;
};

// NC columns of P^T and dS^T for one key row: p = exp2(s sl2 - lse2), ds = p (dp - D),
// packed into 16-bit pairs.  MASK applies causality and document starts.
template <bool MASK, bool F16, int NC>
__device__ __forceinline__ void bwd_elementwise(const uint32_t* sr, const uint32_t* dr, const float* L2,
                                                const float* Dq, const int* DSq, int q_first, int k, float sl2,
                                                uint32_t* pw, uint32_t* dw) {
#pragma unroll
  for (int c8 = 0; c8 < NC; c8 += 8) {
    const float4 la = *reinterpret_cast<const float4*>(L2 + c8), lb = *reinterpret_cast<const float4*>(L2 + c8 + 4);
    const float4 da = *reinterpret_cast<const float4*>(Dq + c8), db = *reinterpret_cast<const float4*>(Dq + c8 + 4);
    const float lv[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
    const float dv[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
    int dsq[8];
    if (MASK) {
      const int4 sa = *reinterpret_cast<const int4*>(DSq + c8), sb = *reinterpret_cast<const int4*>(DSq + c8 + 4);
      dsq[0] = sa.x; dsq[1] = sa.y; dsq[2] = sa.z; dsq[3] = sa.w;
      dsq[4] = sb.x; dsq[5] = sb.y; dsq[6] = sb.z; dsq[7] = sb.w;
    }
    float pv[8], gv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float x = ex2_approx(fmaf(__uint_as_float(sr[c8 + e]), sl2, -lv[e]));
      if (MASK) x = ((q_first + c8 + e - k) | (k - dsq[e])) >= 0 ? x : 0.f;   // q >= k and dstart[q] <= k
      pv[e] = x;
      gv[e] = x * (__uint_as_float(dr[c8 + e]) - dv[e]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      pw[c8 / 2 + e] = pack16x2<F16>(pv[2 * e], pv[2 * e + 1]);
      dw[c8 / 2 + e] = pack16x2<F16>(gv[2 * e], gv[2 * e + 1]);
    }
  }
}

// Bulk copy of `bytes` (a multiple of 16, 16-byte aligned ends) from global to
// shared memory, completing on mbarrier `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// Query blocks qb_lo .. nqb - 1 that can see a key block ending at last_key:
// a prefix (document starts never decrease), counted from 8 loads at a time.
__device__ __forceinline__ int bwd_niter(const int* dsr, int qb_lo, int nqb, int last_key) {
  int n = 0;
  for (int base = qb_lo; base < nqb; base += 8) {
    int v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = base + u < nqb ? ld_once(dsr + (base + u) * BW_QB) : 0x7fffffff;
    int c = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) c += v[u] <= last_key;
    n += c;
    if (c < 8) break;
  }
  return n;
}

// Column sums of a warp's 32 x 32 block (lane = row, a[j] = column j): five
// exchange rounds, each keeping half of the columns, leave lane l with the sum
// of column l over the 32 rows.
__device__ __forceinline__ float warp_colsum32(float (&a)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < o; ++j) {
      const float send = up ? a[j] : a[j + o];
      const float keep = up ? a[j + o] : a[j];
      a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return a[0];
}

template <bool F16>
__global__ void __launch_bounds__(BW_THREADS, 1)
attn_bwd_tc(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
            const __grid_constant__ CUtensorMap tmDQ, const float* __restrict__ lse, const float* __restrict__ Dbuf,
            const int* __restrict__ dstart, int T, int H, int BH, int kcol0, int vcol0, int G, bf16* __restrict__ dkv,
            long ld_kv, int v_off, unsigned* err, float sl2, float* __restrict__ cpart, long cp_ld) {
  // sl2 = log2(e) / sqrt(d) as in the forward; dK carries the 1 / sqrt(d) factor
  // cpart (optional): column sums of dK and dV per 32 keys, row ((b nkb + key
  // block) 4 + quarter) at cpart + row cp_ld, dK columns from 0, dV from v_off
  const float dk_scale = sl2 * (1.0f / LOG2E_F);
  extern __shared__ __align__(1024) uint8_t at_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)at_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + BwdSmem::BAR);
  // bars: kv_full[2], kv_empty[2] (per item, by K/V buffer), q_full[BW_ST] (TMA tiles + per-query
  //       values), q_empty[BW_ST], s_full, s_free, p_full, mma_done (P^T / dS^T read, dQ_blk
  //       complete), dq_free, dkv_free (dK / dV read out), drain, staging written (per group,
  //       128 arrivals), staging free (per group)
  enum { KV_FULL = 0, KV_EMPTY = 2, Q_FULL = 4, Q_EMPTY = Q_FULL + BW_ST, S_FULL = Q_EMPTY + BW_ST,
         S_FREE = S_FULL + 1, P_FULL = S_FREE + 1, MMA_DONE = P_FULL + 1, DQ_FREE = MMA_DONE + 1,
         DKV_FREE = DQ_FREE + 1, DRAIN = DKV_FREE + 1, ST_FULL = DRAIN + 1, ST_FREE = ST_FULL + 2,
         NBARS = ST_FREE + 2 };
  uint32_t* tmem_slot = (uint32_t*)(bars + NBARS);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const uint32_t b0 = smem_u32(bars);
  auto bar = [&](int i) { return b0 + 8u * i; };
  const uint32_t sK0 = smem_u32(sm + BwdSmem::K), sV0 = smem_u32(sm + BwdSmem::V);
  const uint32_t sQ = smem_u32(sm + BwdSmem::Q), sDO = smem_u32(sm + BwdSmem::DO);
  const uint32_t sDST = smem_u32(sm + BwdSmem::DST);
  const uint32_t sDQ = smem_u32(sm + BwdSmem::DQS);
  float* aux = (float*)(sm + BwdSmem::AUX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + BW_QB - 1) / BW_QB, nkb = (T + AT_BLK - 1) / AT_BLK;
  const int n_items = nkb * BH;
  int* s_nit = (int*)(sm + BwdSmem::NIT);
  // item it (the ic-th of this CTA): key block it / BH, head-row bh = it % BH
  struct Item { int bh, b, h, k0, qb_lo, niter; long rowbase; const int* dsr; };
  auto item_at = [&](int it, int ic) {
    Item I;
    const int kb = it / BH;
    I.bh = it % BH;
    I.b = I.bh / H;
    I.h = I.bh % H;
    I.k0 = kb * AT_BLK;
    I.rowbase = (long)I.b * T;
    I.dsr = dstart + I.rowbase;
    I.qb_lo = I.k0 / BW_QB;
    I.niter = s_nit[ic];
    return I;
  };
  griddep_wait();
  griddep_release();
  if (warp == 0) {
    // the query-block count of every item of this CTA, one lane per item
    for (int j = lane, it = blockIdx.x + lane * gridDim.x; it < n_items; j += 32, it += 32 * gridDim.x) {
      const int k0 = (it / BH) * AT_BLK;
      const int* dsr = dstart + (long)((it % BH) / H) * T;
      s_nit[j] = bwd_niter(dsr, k0 / BW_QB, nqb, min(k0 + AT_BLK - 1, T - 1));
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(KV_FULL + i), 1);
      mbar_init(bar(KV_EMPTY + i), 1);
    }
    for (int i = 0; i < BW_ST; ++i) {
      mbar_init(bar(Q_FULL + i), 1);   // lane 0's arrival with the byte count
      mbar_init(bar(Q_EMPTY + i), 1);
    }
    mbar_init(bar(S_FULL), 1);
    mbar_init(bar(S_FREE), 8);
    mbar_init(bar(P_FULL), 8);
    mbar_init(bar(MMA_DONE), 1);
    mbar_init(bar(DQ_FREE), 8);
    mbar_init(bar(DKV_FREE), 8);
    mbar_init(bar(DRAIN), 1);
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(ST_FULL + g), 128);
      mbar_init(bar(ST_FREE + g), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) tc_alloc(smem_u32(tmem_slot), BwdSmem::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer (lane 0: TMA; all lanes: per-query lse2, D, dstart)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQKV)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmDO)) : "memory");
    }
    bool ok = true;
    int gb = 0, ic = 0, ic_loaded = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ic) {
      const Item I = item_at(it, ic);
      const int kvb = ic % BW_KVB;
      // the K / V buffer of item ic - BW_KVB has been read by its last MMA
      if (!mbar_wait(bar(KV_EMPTY + kvb), ((ic / BW_KVB) & 1) ^ 1, abort_flag)) { ok = false; break; }
      if (lane == 0) {
        mbar_expect_tx(bar(KV_FULL + kvb), 2 * AT_TILE_BYTES);
        tma_load_2d(sK0 + kvb * AT_TILE_BYTES, &tmQKV, bar(KV_FULL + kvb), kcol0 + (I.h / G) * AT_D,
                    (int)(I.rowbase + I.k0));
        tma_load_2d(sV0 + kvb * AT_TILE_BYTES, &tmQKV, bar(KV_FULL + kvb), vcol0 + (I.h / G) * AT_D,
                    (int)(I.rowbase + I.k0));
      }
      ic_loaded = ic + 1;
      for (int i = 0; i < I.niter; ++i, ++gb) {
        const int st = gb % BW_ST;
        const uint32_t ph = (gb / BW_ST) & 1;
        const int q0 = (I.qb_lo + i) * BW_QB;
        // per-query values (base-2 lse, D, document start): a full block with
        // 16-byte aligned rows moves by bulk copy with the Q / dO tiles; a
        // ragged one by lane loads (queries past T get INT_MAX starts)
        const long lo_ = (long)I.bh * T + q0, ds_ = I.rowbase + q0;
        const bool bulk = q0 + BW_QB <= T && ((lo_ | ds_) & 3) == 0;
        float l2v[4], dv[4];
        int dsv[4];
        if (!bulk) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int qq = q0 + lane + 32 * e;
            const bool v = qq < T;
            l2v[e] = v ? lse[(long)I.bh * T + qq] : 0.f;
            dv[e] = v ? Dbuf[(long)I.bh * T + qq] : 0.f;
            dsv[e] = v ? I.dsr[qq] : 0x7fffffff;
          }
        }
        if (!mbar_wait(bar(Q_EMPTY + st), ph ^ 1, abort_flag)) { ok = false; break; }
        float* L2 = aux + st * 3 * BW_QB;
        float* Dq = L2 + BW_QB;
        int* DSq = reinterpret_cast<int*>(Dq + BW_QB);
        if (!bulk) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            L2[lane + 32 * e] = l2v[e];
            Dq[lane + 32 * e] = dv[e];
            DSq[lane + 32 * e] = dsv[e];
          }
          __syncwarp();   // the lanes' values precede lane 0's arrival (release)
        }
        if (lane == 0) {
          mbar_expect_tx(bar(Q_FULL + st), 2 * AT_TILE_BYTES + (bulk ? 3 * BW_QB * 4 : 0));
          tma_load_2d(sQ + st * AT_TILE_BYTES, &tmQKV, bar(Q_FULL + st), I.h * AT_D, (int)(I.rowbase + q0));
          tma_load_2d(sDO + st * AT_TILE_BYTES, &tmDO, bar(Q_FULL + st), I.h * AT_D, (int)(I.rowbase + q0));
          if (bulk) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            bulk_g2s(smem_u32(L2), lse + lo_, BW_QB * 4, bar(Q_FULL + st));
            bulk_g2s(smem_u32(Dq), Dbuf + lo_, BW_QB * 4, bar(Q_FULL + st));
            bulk_g2s(smem_u32(DSq), dstart + ds_, BW_QB * 4, bar(Q_FULL + st));
          }
        }
      }
    }
    if (!ok && lane == 0) trap_timeout(abort_flag, err);
    if (lane == 0) {
      // every copy issued has landed before the CTA leaves
      volatile int never = 0;
      for (int i = max(0, ic_loaded - BW_KVB); i < ic_loaded; ++i)
        mbar_wait(bar(KV_FULL + i % BW_KVB), (i / BW_KVB) & 1, &never, 1ll << 28);
      for (int i = max(0, gb - BW_ST); i < gb; ++i)
        mbar_wait(bar(Q_FULL + i % BW_ST), (i / BW_ST) & 1, &never, 1ll << 28);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: the S^T / dP^T of the next block (next item
    // included) go out before this block's dV, dK and dQ
    constexpr uint32_t ID_SS = instr_desc_t(F16, 128, false, false);   // S^T, dP^T: 128 keys x 128 queries, K = d
    constexpr uint32_t ID_KV = instr_desc_t(F16, 64, false, true);     // dV, dK: 128 keys x 64, K = 128 queries
    constexpr uint32_t ID_DQ = instr_desc_t(F16, 64, true, true);      // dQ: 128 queries x 64, K = 128 keys
    bool ok = true;
    // S issue cursor: item it_s (ic_s-th of this CTA, niter_s blocks), block i_s, global block gs
    int it_s = blockIdx.x, ic_s = 0, i_s = 0, gs = 0, niter_s = 0;
    if (it_s < n_items) niter_s = s_nit[0];
    auto issue_s = [&]() -> bool {   // S^T and dP^T of the block at the cursor, then advance it
      const int st = gs % BW_ST, kvb = ic_s % BW_KVB;
      if (i_s == 0 && !mbar_wait(bar(KV_FULL + kvb), (ic_s / BW_KVB) & 1, abort_flag)) return false;
      if (!mbar_wait(bar(Q_FULL + st), (gs / BW_ST) & 1, abort_flag)) return false;
      if (!mbar_wait(bar(S_FREE), (gs & 1) ^ 1, abort_flag)) return false;   // previous S^T / dP^T read
      tc_fence_after();
      const uint32_t q = sQ + st * AT_TILE_BYTES, o = sDO + st * AT_TILE_BYTES;
      const uint32_t sK = sK0 + kvb * AT_TILE_BYTES, sV = sV0 + kvb * AT_TILE_BYTES;
#pragma unroll
      for (int k = 0; k < AT_D / 16; ++k) {
        umma_bf16(tmem + 0, kdesc(sK + k * 32), kdesc(q + k * 32), ID_SS, k > 0);
        umma_bf16(tmem + 128, kdesc(sV + k * 32), kdesc(o + k * 32), ID_SS, k > 0);
      }
      umma_commit(bar(S_FULL));
      ++gs;
      if (++i_s == niter_s) {
        i_s = 0;
        ++ic_s;
        it_s += gridDim.x;
        niter_s = it_s < n_items ? s_nit[ic_s] : 0;
      }
      return true;
    };
    int g_total = 0;   // blocks of all of this CTA's items
    for (int it = blockIdx.x, j = 0; it < n_items; it += gridDim.x, ++j) g_total += s_nit[j];
    if (g_total > 0) ok = issue_s();
    int gb = 0, ic = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ic) {
      const int niter = s_nit[ic], kvb = ic % BW_KVB;
      const uint32_t sK = sK0 + kvb * AT_TILE_BYTES;
      for (int i = 0; i < niter; ++i, ++gb) {
        const int st = gb % BW_ST;
        if (gb + 1 < g_total && !issue_s()) { ok = false; break; }
        if (!mbar_wait(bar(P_FULL), gb & 1, abort_flag)) { ok = false; break; }   // P^T, dS^T written
        // the previous item's dK / dV have been read out of TMEM before they are overwritten
        if (i == 0 && ic > 0 && !mbar_wait(bar(DKV_FREE), (ic - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q = sQ + st * AT_TILE_BYTES, o = sDO + st * AT_TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < BW_QB / 16; ++kk) {
          const uint32_t off = (kk >> 2) * AT_TILE_BYTES + (kk & 3) * 32;
          umma_bf16_ts(tmem + 256, tmem + 448 + 8 * kk, mndesc(o + kk * 2048, 8192), ID_KV, (i > 0 || kk > 0));
          umma_bf16(tmem + 320, kdesc(sDST + off), mndesc(q + kk * 2048, 8192), ID_KV, (i > 0 || kk > 0));
        }
        umma_commit(bar(Q_EMPTY + st));   // Q / dO stage free
        // dQ_blk = dS K once the previous block's dQ has been read out
        if (gb > 0 && !mbar_wait(bar(DQ_FREE), (gb - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < AT_BLK / 16; ++kk)
          umma_bf16(tmem + 384, mndesc(sDST + kk * 2048, AT_TILE_BYTES), mndesc(sK + kk * 2048, 8192), ID_DQ,
                    kk > 0);
        umma_commit(bar(MMA_DONE));
        if (i + 1 == niter) umma_commit(bar(KV_EMPTY + kvb));   // this item's K / V no longer read
      }
    }
    if (!ok) trap_timeout(abort_flag, err);
    umma_commit(bar(DRAIN));
    volatile int never = 0;
    mbar_wait(bar(DRAIN), 0, &never, 1ll << 28);
  } else if (warp >= 2 && warp < 10) {
    // ---------------- elementwise warps: thread owns key row r (and query row r of dQ)
    const int quarter = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t st_full = bar(ST_FULL + grp), st_free = bar(ST_FREE + grp);
    const uint32_t sDQg = sDQ + grp * AT_TILE_BYTES;
    bool ok = true;
    // waits are voted warp-wide so that the .sync.aligned TMEM accesses after
    // them are never reached by part of a warp
    auto wait_w = [&](uint32_t bb, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bb, parity, abort_flag)); };
    // dQ of global block j: TMEM -> fp32 staging (128-byte swizzle); warp 10
    // issues the bulk reduce-add once all 128 rows of the group are written
    auto flush_dq = [&](int j) -> bool {
      uint32_t rr[32];
      tmem_ld32(tmem + lane_off + 384 + 32 * grp, rr);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(DQ_FREE));   // the dQ accumulator may be overwritten
      // the reduce of block j-1 has read the staging
      if (j > 0 && !wait_w(st_free, (j - 1) & 1)) return false;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t a = sDQg + r * 128 + ((u ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(rr[4 * u]), "r"(rr[4 * u + 1]),
                     "r"(rr[4 * u + 2]), "r"(rr[4 * u + 3])
                     : "memory");
      }
      fence_async_smem();
      mbar_arrive(st_full);
      return true;
    };
    int gb = 0, ic = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ic) {
      const Item I = item_at(it, ic);
      const int k = I.k0 + r;
      for (int i = 0; i < I.niter; ++i, ++gb) {
        const int q0 = (I.qb_lo + i) * BW_QB;
        const int st = gb % BW_ST;
        const float* L2 = aux + st * 3 * BW_QB + 64 * grp;
        const float* Dq = L2 + BW_QB;
        const int* DSq = reinterpret_cast<const int*>(L2 + 2 * BW_QB);
        if (!wait_w(bar(Q_FULL + st), (gb / BW_ST) & 1)) { ok = false; break; }   // per-query values
        if (!wait_w(bar(S_FULL), gb & 1)) { ok = false; break; }
        tc_fence_after();
        // masking only where a key can be later than a query or before its document
        // (document starts never decrease, queries past T carry INT_MAX)
        const bool need_mask = q0 < I.k0 + AT_BLK || DSq[BW_QB - 1 - 64 * grp] > I.k0;
        // two 32-column halves of the group's 64 query columns (a variant that
        // pipelined 16-column quarters, each quarter's loads issued before the
        // previous quarter's arithmetic, measured 4 % slower)
        uint32_t pw[32], dw[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tmem + lane_off + 64 * grp + 32 * half, sr);
          tmem_ld32(tmem + lane_off + 128 + 64 * grp + 32 * half, dr);
          tmem_wait_ld();
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(S_FREE));   // S^T / dP^T may be overwritten
          }
          const int qf = q0 + 64 * grp + 32 * half;
          if (need_mask)
            bwd_elementwise<true, F16, 32>(sr, dr, L2 + 32 * half, Dq + 32 * half, DSq + 32 * half, qf, k, sl2,
                                           pw + 16 * half, dw + 16 * half);
          else
            bwd_elementwise<false, F16, 32>(sr, dr, L2 + 32 * half, Dq + 32 * half, DSq + 32 * half, qf, k, sl2,
                                            pw + 16 * half, dw + 16 * half);
        }
        // the previous block's P^T / dS^T have been consumed and its dQ is complete
        if (gb > 0 && !wait_w(bar(MMA_DONE), (gb - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        tmem_st32(tmem + lane_off + 448 + 32 * grp, pw);
        {
          const uint32_t db = sDST + grp * AT_TILE_BYTES + r * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t sw = (u ^ (r & 7)) << 4;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(db + sw), "r"(dw[4 * u]),
                         "r"(dw[4 * u + 1]), "r"(dw[4 * u + 2]), "r"(dw[4 * u + 3])
                         : "memory");
          }
        }
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(P_FULL));
        if (i > 0) {
          tc_fence_after();
          if (!flush_dq(gb - 1)) { ok = false; break; }
        }
      }
      if (!ok) break;
      // the item's last dQ, then dK and dV
      if (!wait_w(bar(MMA_DONE), (gb - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      if (!flush_dq(gb - 1)) { ok = false; break; }
      bf16* row = dkv + (I.rowbase + k) * ld_kv;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const float sc = part == 0 ? dk_scale : 1.f;
        uint32_t rr[32];
        tmem_ld32(tmem + lane_off + (part == 0 ? 320 : 256) + 32 * grp, rr);
        tmem_wait_ld();
        if (part == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(DKV_FREE));   // the next item's dV / dK may overwrite TMEM
        }
        if (cpart) {
          // the warp's 32 keys summed per column (keys past T add nothing): lane l
          // ends with column 32 grp + l of the head
          float a[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) a[j] = k < T ? __uint_as_float(rr[j]) * sc : 0.f;
          const float cs = warp_colsum32(a, lane);
          const long crow = ((long)I.b * nkb + I.k0 / AT_BLK) * 4 + quarter;
          cpart[crow * cp_ld + (part == 0 ? 0 : v_off) + I.h * AT_D + 32 * grp + lane] = cs;
        }
        if (k >= T) continue;
        bf16* dst = row + (part == 0 ? 0 : v_off) + I.h * AT_D + 32 * grp;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack16x2<F16>(__uint_as_float(rr[8 * u]) * sc, __uint_as_float(rr[8 * u + 1]) * sc);
          w.y = pack16x2<F16>(__uint_as_float(rr[8 * u + 2]) * sc, __uint_as_float(rr[8 * u + 3]) * sc);
          w.z = pack16x2<F16>(__uint_as_float(rr[8 * u + 4]) * sc, __uint_as_float(rr[8 * u + 5]) * sc);
          w.w = pack16x2<F16>(__uint_as_float(rr[8 * u + 6]) * sc, __uint_as_float(rr[8 * u + 7]) * sc);
          *reinterpret_cast<uint4*>(dst + 8 * u) = w;
        }
      }
    }
    if (!ok) trap_timeout(abort_flag, err);
  } else if (warp == 10 && lane == 0) {
    // ---------------- dQ reducer: per block, both groups' staging -> global fp32 accumulator
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmDQ)) : "memory");
    bool ok = true;
    int gb = 0, ic = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ic) {
      const Item I = item_at(it, ic);
      for (int j = 0; j < I.niter && ok; ++j, ++gb) {
        for (int gg = 0; gg < 2; ++gg) {
          if (!mbar_wait(bar(ST_FULL + gg), gb & 1, abort_flag)) { ok = false; break; }
          tma_reduce_add_2d(&tmDQ, sDQ + gg * AT_TILE_BYTES, I.h * AT_D + 32 * gg,
                            (int)(I.rowbase + (I.qb_lo + j) * BW_QB));
          bulk_commit();
        }
        if (!ok) break;
        bulk_wait_read<0>();   // both stagings read: the groups may overwrite them
        mbar_arrive(bar(ST_FREE + 0));
        mbar_arrive(bar(ST_FREE + 1));
      }
    }
    if (!ok) trap_timeout(abort_flag, err);
    bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tc_dealloc(tmem, BwdSmem::TMEM_COLS);
}

// dq[row, head h] = bf16 or fp16 (F16) of dQacc / sqrt(d); the accumulator is cleared for the next use.
template <bool F16>
__global__ void attn_dq_finish_kernel(float* __restrict__ dq_acc, bf16* __restrict__ dqkv, long rows, int C, long ld_q,
                                      float scale) {
  griddep_wait();
  griddep_release();
  const long n8 = rows * C / 8;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n8; i += (long)gridDim.x * blockDim.x) {
    const long e = i * 8, row = e / C;
    const int c = (int)(e % C);
    float4* src = reinterpret_cast<float4*>(dq_acc + e);
    const float4 a = src[0], bq = src[1];
    uint4 w;
    w.x = pack16x2<F16>(a.x * scale, a.y * scale);
    w.y = pack16x2<F16>(a.z * scale, a.w * scale);
    w.z = pack16x2<F16>(bq.x * scale, bq.y * scale);
    w.w = pack16x2<F16>(bq.z * scale, bq.w * scale);
    *reinterpret_cast<uint4*>(dqkv + row * ld_q + c) = w;
    src[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    src[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// The same finish over one 32-row slab per block (rows b T + 128 kb + 32 q + [0, 32)
// below T, slab (b nkb + kb) 4 + q), also writing the slab's column sums of dq to
// cpart + slab cp_ld (the bias gradient's partial rows; zeros for an empty slab).
// Thread (lane rl, chunk ch) takes 8 columns of rows rl, rl + RL, ...; the RL row
// lanes' sums are added in a fixed order through shared memory.
#define DQF_THREADS 384
template <bool F16>
__global__ void __launch_bounds__(DQF_THREADS) attn_dq_finish_cs_kernel(float* __restrict__ dq_acc,
                                                                        bf16* __restrict__ dqkv, int T, int C,
                                                                        long ld_q, float scale, int nkb,
                                                                        float* __restrict__ cpart, long cp_ld) {
  extern __shared__ float dqf_red[];   // [RL][C]
  griddep_wait();
  griddep_release();
  const int slab = blockIdx.x, qq = slab & 3, bk = slab >> 2;
  const int b = bk / nkb, t0 = (bk % nkb) * AT_BLK + 32 * qq;
  const int nr = min(32, T - t0);
  const long row0 = (long)b * T + t0;
  const int nch = C / 8;
  const int RL = nch >= DQF_THREADS ? 1 : DQF_THREADS / nch;
  const int rl = threadIdx.x / nch;
  for (int ch = threadIdx.x % nch; ch < nch && rl < RL; ch += DQF_THREADS) {
    float cs[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) cs[j] = 0.f;
#pragma unroll 4
    for (int r = rl; r < nr; r += RL) {
      float4* src = reinterpret_cast<float4*>(dq_acc + (row0 + r) * C + ch * 8);
      const float4 a = src[0], bq = src[1];
      const float v[8] = {a.x * scale, a.y * scale, a.z * scale, a.w * scale,
                          bq.x * scale, bq.y * scale, bq.z * scale, bq.w * scale};
      uint4 w;
      w.x = pack16x2<F16>(v[0], v[1]);
      w.y = pack16x2<F16>(v[2], v[3]);
      w.z = pack16x2<F16>(v[4], v[5]);
      w.w = pack16x2<F16>(v[6], v[7]);
      *reinterpret_cast<uint4*>(dqkv + (row0 + r) * ld_q + ch * 8) = w;
      src[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      src[1] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j) cs[j] += v[j];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) dqf_red[rl * C + ch * 8 + j] = cs[j];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += DQF_THREADS) {
    float acc = 0.f;
    for (int i = 0; i < RL; ++i) acc += dqf_red[i * C + c];
    cpart[(long)slab * cp_ld + c] = acc;
  }
}

// D[b, h, t] = dO[b*T+t, head h] . O[b*T+t, head h]   (one thread per (row, head))
template <bool F16>
__global__ void attn_rowdot_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout, float* __restrict__ Dbuf,
                                   int B, int T, int H, int d) {
  griddep_wait();
  griddep_release();
  long i = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (i >= (long)B * T * H) return;
  const int h = i % H;
  const long row = i / H;
  const int t = row % T, b = row / T;
  const long off = row * H * d + h * d;
  float acc = 0.f;
  for (int c = 0; c < d; c += 8) {
    float x[8], y[8];
    unpack16x8<F16>(*reinterpret_cast<const uint4*>(dout + off + c), x);
    unpack16x8<F16>(*reinterpret_cast<const uint4*>(out + off + c), y);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc += x[k] * y[k];
  }
  Dbuf[((long)b * H + h) * T + t] = acc;
}

// ============================================================== launchers
bool attn_tc_supported(int d) { return d == AT_D && get_encode() != nullptr; }

template <typename K>
static cudaError_t tc_smem_attr(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

AttnLayout attn_layout_mha(bf16* dqkv, int C) {
  AttnLayout a;
  a.qw = 3 * C; a.kcol = C; a.vcol = 2 * C; a.G = 1;
  a.dkv = dqkv ? dqkv + C : nullptr; a.ld_kv = 3L * C; a.v_off = C;
  return a;
}

template <bool F16>
static cudaError_t attn_fwd_tc_t(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T, int H,
                                 unsigned* err, cudaStream_t s, const AttnLayout& L, int d_real) {
  const long rows = (long)B * T;
  CUtensorMap tqkv;
  if (!make_map_ex(&tqkv, MapKey{qkv, rows, (long)L.qw, (long)L.qw, 1, 0, AT_D, AT_BLK, 0, 128}))
    return cudaErrorInvalidValue;
  const int smem = FwdSmem::TOTAL + 1024;
  static bool attr = false;
  if (!attr) { cudaError_t e = tc_smem_attr(attn_fwd_tc<F16>, smem); if (e) return e; attr = true; }
  dim3 grid(B * H, (T + FW_QT - 1) / FW_QT);
  ++g_kernel_launches;
  return launch_k(attn_fwd_tc<F16>, grid, dim3(FW_THREADS), smem, s, tqkv, out, lse, dstart, T, H, L.kcol, L.vcol, L.G,
                  err, LOG2E_F / sqrtf((float)d_real));
}

static bool layout_ok(const AttnLayout& L, int H) {
  // 16-byte aligned TMA columns and row strides; whole key / value groups
  return L.G >= 1 && H % L.G == 0 && L.qw % 8 == 0 && L.kcol % 8 == 0 && L.vcol % 8 == 0 && L.ld_kv % 8 == 0 &&
         L.v_off % 8 == 0;
}

cudaError_t launch_attn_fwd_tc(const bf16* qkv, bf16* out, float* lse, const int* dstart, int B, int T, int H,
                               unsigned* err, cudaStream_t s, bool f16, const AttnLayout* lay, int d_real) {
  const AttnLayout L = lay ? *lay : attn_layout_mha(nullptr, H * AT_D);
  if (!layout_ok(L, H) || d_real < 1 || d_real > AT_D) return cudaErrorInvalidValue;
  return f16 ? attn_fwd_tc_t<true>(qkv, out, lse, dstart, B, T, H, err, s, L, d_real)
             : attn_fwd_tc_t<false>(qkv, out, lse, dstart, B, T, H, err, s, L, d_real);
}

template <bool F16>
static cudaError_t attn_bwd_tc_t(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dbuf,
                                 bool d_ready, float* dq_acc, const int* dstart, bf16* dqkv, int B, int T, int H,
                                 unsigned* err, cudaStream_t s, const AttnLayout& L, int d_real, float* cpart) {
  const int C = H * AT_D;
  const float scale = 1.0f / sqrtf((float)d_real);
  const long rows = (long)B * T;
  CUtensorMap tqkv, tdo, tdq;
  if (!make_map_ex(&tqkv, MapKey{qkv, rows, (long)L.qw, (long)L.qw, 1, 0, AT_D, AT_BLK, 0, 128}) ||
      !make_map_ex(&tdo, MapKey{dout, rows, (long)C, (long)C, 1, 0, AT_D, BW_QB, 0, 128}) ||
      !make_map_ex(&tdq, MapKey{dq_acc, rows, (long)C, (long)C, 1, 0, 32, BW_QB, 1, 128}))
    return cudaErrorInvalidValue;
  const int smem = BwdSmem::TOTAL + 1024;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = tc_smem_attr(attn_bwd_tc<F16>, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaError_t e;
  if (!d_ready) {   // D = rowsum(dO o O), unless the producer of dO already wrote it
    long n = rows * H;
    ++g_kernel_launches;
    attn_rowdot_kernel<F16><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(out, dout, Dbuf, B, T, H, AT_D);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // persistent: one CTA per SM (or fewer, for fewer items)
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
  }
  const int n_items = B * H * ((T + AT_BLK - 1) / AT_BLK);
  const int grid = n_items < sms ? n_items : sms;
  if (n_items > (long)grid * BW_MAX_ITEMS) return cudaErrorInvalidValue;
  ++g_kernel_launches;
  const long cp_ld = 3L * C;   // partial rows of the q|k|v bias gradient
  e = launch_k(attn_bwd_tc<F16>, dim3(grid), dim3(BW_THREADS), smem, s, tqkv, tdo, tdq, lse, Dbuf, dstart, T, H, B * H,
               L.kcol, L.vcol, L.G, L.dkv, L.ld_kv, L.v_off, err, scale * LOG2E_F, cpart ? cpart + C : nullptr, cp_ld);
  if (e != cudaSuccess) return e;
  ++g_kernel_launches;
  if (cpart) {
    const int nkb = (T + AT_BLK - 1) / AT_BLK;
    const int nch = C / 8, rl = nch >= DQF_THREADS ? 1 : DQF_THREADS / nch;
    const size_t red = (size_t)rl * C * sizeof(float);
    if (red > 48 * 1024) return cudaErrorInvalidValue;
    return launch_k(attn_dq_finish_cs_kernel<F16>, dim3((unsigned)(B * nkb * 4)), dim3(DQF_THREADS), red, s, dq_acc,
                    dqkv, T, C, (long)L.qw, scale, nkb, cpart, cp_ld);
  }
  return launch_k(attn_dq_finish_kernel<F16>, dim3(148 * 8), dim3(256), 0, s, dq_acc, dqkv, rows, C, (long)L.qw, scale);
}

cudaError_t launch_attn_bwd_tc(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dbuf,
                               bool d_ready, float* dq_acc, const int* dstart, bf16* dqkv, int B, int T, int H,
                               unsigned* err, cudaStream_t s, bool f16, const AttnLayout* lay, int d_real,
                               float* bias_part) {
  const AttnLayout L = lay ? *lay : attn_layout_mha(dqkv, H * AT_D);
  if (!layout_ok(L, H) || !L.dkv || d_real < 1 || d_real > AT_D) return cudaErrorInvalidValue;
  // the bias column sums index q|k|v columns of one fused row: plain heads only
  if (bias_part && (lay || d_real != AT_D)) return cudaErrorInvalidValue;
  return f16 ? attn_bwd_tc_t<true>(qkv, out, dout, lse, Dbuf, d_ready, dq_acc, dstart, dqkv, B, T, H, err, s, L, d_real,
                                   bias_part)
             : attn_bwd_tc_t<false>(qkv, out, dout, lse, Dbuf, d_ready, dq_acc, dstart, dqkv, B, T, H, err, s, L, d_real,
                                    bias_part);
}

// ------------------------------------------------------------ zero-padded heads
// Heads of d < 64 columns (64 % d == 0) run the d = 64 kernels on copies whose
// heads are widened to 64 columns with zeros: a zero column adds nothing to a
// score, a zero value column gives a zero output column, and the padded
// gradient columns are dropped.  attn_pad: dst [rows][groups][64] <- src
// [rows][groups][d] (zeros beyond d); attn_unpad: the reverse copy.
template <bool PAD>
__global__ void attn_pad_kernel(const bf16* __restrict__ src, bf16* __restrict__ dst, long rows, int groups, int d) {
  griddep_wait();
  griddep_release();
  const int cpg = AT_D / 8;   // 16-byte chunks per padded group
  const long n = rows * groups * cpg;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const long rg = i / cpg;
    const int c = (int)(i % cpg) * 8;
    const long row = rg / groups;
    const int g = (int)(rg % groups);
    const long p = (row * groups + g) * AT_D + c, u = (row * groups + g) * d + c;
    if (PAD) {
      *reinterpret_cast<uint4*>(dst + p) = c < d ? *reinterpret_cast<const uint4*>(src + u) : make_uint4(0u, 0u, 0u, 0u);
    } else if (c < d) {
      *reinterpret_cast<uint4*>(dst + u) = *reinterpret_cast<const uint4*>(src + p);
    }
  }
}

cudaError_t launch_attn_rowdot(const bf16* out, const bf16* dout, float* Dbuf, int B, int T, int H, int d, bool f16,
                               cudaStream_t s) {
  if (d % 8) return cudaErrorInvalidValue;
  const long n = (long)B * T * H;
  ++g_kernel_launches;
  return f16 ? launch_k(attn_rowdot_kernel<true>, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, out, dout, Dbuf, B,
                        T, H, d)
             : launch_k(attn_rowdot_kernel<false>, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, out, dout, Dbuf,
                        B, T, H, d);
}

bool attn_tc_pad_supported(int d) { return d >= 8 && d < AT_D && AT_D % d == 0 && get_encode() != nullptr; }

cudaError_t launch_attn_pad(const bf16* src, bf16* dst, long rows, int groups, int d, bool pad, cudaStream_t s) {
  if (!attn_tc_pad_supported(d)) return cudaErrorInvalidValue;
  const long n = rows * groups * (AT_D / 8);
  const int blocks = (int)std::min<long>((n + 255) / 256, 148L * 8);
  ++g_kernel_launches;
  return pad ? launch_k(attn_pad_kernel<true>, dim3(blocks), dim3(256), 0, s, src, dst, rows, groups, d)
             : launch_k(attn_pad_kernel<false>, dim3(blocks), dim3(256), 0, s, src, dst, rows, groups, d);
}
