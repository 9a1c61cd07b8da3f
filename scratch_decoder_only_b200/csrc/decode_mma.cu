// Decode projections of 1 to 32 rows on the tensor cores ("RustGPT",
// "Technical implementation": greedy decoding; "NTransformer" page, "No
// PyTorch, no cuBLAS": per-token projections over a KV-cached step):
// y[b, n] = sum_k x[b, k] W[n, k] with the epilogues of the decode GEMV
// (bias + residual, bias + GELU, fp32 logits).
//
// A decode step reads every weight once and multiplies it by a handful of
// rows, so the work is a weight stream.  The weights are cut into 16-row
// slices spread over every SM, two CTAs per SM.  A CTA owns one k range of
// the input (all of K up to DM_KC columns, else a 1/nkc share) and a list of
// slices:
//   - each slice's k range moves into a ring of nbuf shared-memory slots by
//     bulk copy (one copy for a whole-K slice, whose 16 rows are contiguous;
//     one per row for a share of K), several slices in flight;
//   - the eight warps split the k range in 32-column blocks and multiply
//     with mma.sync m16n8k16, each warp keeping its blocks of x in registers
//     as A fragments for the whole launch (loaded once from global memory);
//   - the k order inside a 32-column block is permuted, the same way for x
//     and W (a sum over k does not depend on its order): lane (g, t) takes
//     columns 8t .. 8t + 7 of row g with one 16-byte load, columns 8t + 0..3
//     serving the block's first MMA and 8t + 4..7 its second.  One 16-byte
//     shared-memory load per lane and n tile then yields the B fragments of
//     two MMAs, with at most two lanes of a quarter-warp on the same banks
//     (ldmatrix of rows K * 2 bytes apart would put all eight on them);
//   - the warps' partial tiles are summed in a fixed order in shared memory.
// A LayerNorm (or RMSNorm) of x can run in the kernel (K <= DM_KC): the CTA
// holds all of x's columns, so the row statistics come from the registers
// (two passes, quad shuffles and a fixed-order sum over the warps) and the
// normalised values, rounded to 16 bits as the LayerNorm kernel stores them,
// replace the fragments.
// With a split k range the nkc CTAs of a slice group form a thread-block
// cluster: each stores its partial tile into the first CTA's shared memory
// (distributed shared memory), one cluster barrier per slice, and the first
// CTA adds the nkc partials in k order and runs the epilogue (two partial
// areas alternate, so the next slice's stores never meet this one's reads).  Weight copies are issued before
// the programmatic-dependent-launch wait: the stream starts while the
// previous kernel drains.
#include "launch.h"
#include "tc_common.cuh"

#define DM_THREADS 256
#define DM_WARPS (DM_THREADS / 32)
#define DM_ROWS 16                 // weight rows per slice
#define DM_KC 768                  // k columns of one CTA's range (at most)
#define DM_KB (DM_KC / 32 / DM_WARPS)   // 32-column blocks per warp (at most)
#define DM_MAXBUF 6                // slice slots (at most)
#define DM_SMEM_BUDGET (110 * 1024)     // two CTAs per SM
#define DM_MAX_SPLIT 8              // cluster size (portable limit)
#ifndef DM_CTAS
#define DM_CTAS 2                  // CTAs per SM in the grid
#endif

template <bool F16>
__device__ __forceinline__ void dm_mma(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  if constexpr (F16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 dm_lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Output (bb, n) from the dot product y, the bias value pb and the residual
// value pr (both loaded ahead, zero where absent).
template <typename T>
__device__ __forceinline__ float dm_epilogue(float y, float pb, float pr, int bb, int n, int N, int mode, T* out,
                                             T* out2, float* outf) {
  const long oi = (long)bb * N + n;
  if (mode == 2) {
    outf[oi] = y;
    return y;
  } else if (mode == 1) {
    const T uq = from_f<T>(y + pb);
    out[oi] = uq;
    out2[oi] = from_f<T>(gelu_f(to_f(uq)));
    return to_f(uq);
  }
  const T v = from_f<T>(y + pb + pr);
  out[oi] = v;
  return to_f(v);
}
// LayerNorm statistics of a row's 16-column group (the slice's outputs of
// row bb, held by 16 consecutive lanes): mean and sum of squared deviations
// into st[slice][bb] (an LN-fused projection merges the groups).  Every lane
// of the warp calls it; ok: this lane holds a stored value v.
__device__ __forceinline__ void dm_group_stats(float v, bool ok, float2* st, int slice, int B, int bb, int lane) {
  float sm = ok ? v : 0.f;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
  const float mean = sm * (1.f / 16.f), d = ok ? v - mean : 0.f;
  float q = d * d;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  if (ok && (lane & 15) == 0) st[(long)slice * B + bb] = make_float2(mean, q);
}
#define DM_OPT (16 * 32 / DM_THREADS)   // outputs per thread and slice (at most)

__device__ __forceinline__ void dm_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Store v at this CTA's shared address addr mapped into cluster CTA rank.
__device__ __forceinline__ void dm_st_cluster(uint32_t addr, uint32_t rank, float v) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(addr), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

// MT = 16-row tiles of x (B <= 16 MT).  Grid = ngrp groups x nkc k ranges;
// CTA (grp, kc) takes columns [kc kcl, min(K, (kc + 1) kcl)) of every slice
// grp + j ngrp; with nkc > 1 the CTAs of a group form one cluster (rank kc).
// Shared memory: nbuf slots of [16 rows][kcl] 16-bit values, the warps'
// partial tiles [DM_WARPS][16 MT][16] fp32, then the LayerNorm's gains and
// shifts [2][K] fp32 (nkc == 1) or the cluster's partial areas [2][nkc][B
// 16] fp32 (nkc > 1).
template <typename T, int MT>
__global__ void __launch_bounds__(DM_THREADS, 2)
dec_mma_kernel(const T* __restrict__ X, int B, int K, const T* __restrict__ W, int N, int nkc, int kcl,
               const float* __restrict__ bias, const T* resid, int mode, T* out, T* out2, float* outf, int nbuf,
               unsigned* err, const float* __restrict__ lng, const float* __restrict__ lnb, float eps,
               float2* st_out, const float2* __restrict__ st_in) {
  constexpr bool F16 = std::is_same<T, f16>::value;
  extern __shared__ __align__(128) uint8_t dm_smem[];
  __shared__ __align__(8) uint64_t bars[DM_MAXBUF];
  __shared__ __align__(8) uint64_t lnbar;
  __shared__ int s_abort;
  const int kc = blockIdx.x % nkc, grp = blockIdx.x / nkc, ngrp = gridDim.x / nkc;
  const int k0 = kc * kcl, kn = min(kcl, K - k0);   // this CTA's columns [k0, k0 + kn), kn % 32 == 0
  const int nslices = (N + DM_ROWS - 1) / DM_ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  int nmine = 0;
  for (int sl = grp; sl < nslices; sl += ngrp) ++nmine;
  const uint32_t slot0 = smem_u32(dm_smem), slot_bytes = (uint32_t)DM_ROWS * kcl * 2;
  float* red = reinterpret_cast<float*>(dm_smem + nbuf * slot_bytes);
  if (threadIdx.x == 0) {
    for (int i = 0; i < nbuf; ++i) mbar_init(smem_u32(&bars[i]), 1);
    mbar_init(smem_u32(&lnbar), 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // thread 0: this CTA's k range of slice j (rows past N are not copied)
  // into slot j % nbuf, rows kcl values apart
  auto issue = [&](int j) {
    const int r0 = (grp + j * ngrp) * DM_ROWS, rr = min(DM_ROWS, N - r0);
    const uint32_t dst = slot0 + (j % nbuf) * slot_bytes, bar = smem_u32(&bars[j % nbuf]);
    mbar_expect_tx(bar, (uint32_t)rr * kn * 2);
    if (nkc == 1) {
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(dst), "l"(reinterpret_cast<uint64_t>(W + (long)r0 * K)), "r"((uint32_t)rr * K * 2),
                   "r"(bar) : "memory");
    } else {
      for (int r = 0; r < rr; ++r)
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     ::"r"(dst + (uint32_t)r * kcl * 2), "l"(reinterpret_cast<uint64_t>(W + (long)(r0 + r) * K + k0)),
                     "r"((uint32_t)kn * 2), "r"(bar) : "memory");
    }
  };
  int issued = 0;
  if (threadIdx.x == 0)
    for (; issued < nbuf && issued < nmine; ++issued) issue(issued);
  // the LayerNorm parameters (constant) move before the wait: by bulk copy
  // when 16-byte aligned (waited for after the statistics), else by loads
  float* lns = red + DM_WARPS * 16 * MT * 16;
  float* cred = lns;   // nkc > 1: [2][nkc][B 16] partial areas of the cluster's first CTA
  // every CTA of the cluster has started before any partial crosses to rank 0
  if (nkc > 1) dm_cluster_sync();
  const bool ln_bulk = lng && !((reinterpret_cast<uintptr_t>(lng) | reinterpret_cast<uintptr_t>(lnb)) & 15);
  if (ln_bulk) {
    if (threadIdx.x == 0) {
      const uint32_t bar = smem_u32(&lnbar);
      mbar_expect_tx(bar, (uint32_t)K * 4 * (lnb ? 2 : 1));
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(smem_u32(lns)), "l"(reinterpret_cast<uint64_t>(lng)), "r"((uint32_t)K * 4), "r"(bar)
                   : "memory");
      if (lnb)
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     ::"r"(smem_u32(lns + K)), "l"(reinterpret_cast<uint64_t>(lnb)), "r"((uint32_t)K * 4), "r"(bar)
                     : "memory");
    }
    if (!lnb)
      for (int i = threadIdx.x; i < K; i += DM_THREADS) lns[K + i] = 0.f;
  } else if (lng) {
    for (int i = threadIdx.x; i < K; i += DM_THREADS) {
      lns[i] = lng[i];
      lns[K + i] = lnb ? lnb[i] : 0.f;
    }
  }
  // x, the residual, the outputs and the workspace belong to the previous kernel until here
  griddep_wait();
  griddep_release();
  // A fragments: this warp's 32-column blocks kb = warp + 8 j of the range;
  // lane (g, t) holds columns 8t .. 8t + 7 of x rows g and g + 8 of each tile
  uint4 xa[DM_KB][MT][2];
#pragma unroll
  for (int j = 0; j < DM_KB; ++j) {
    const int col = 32 * (warp + DM_WARPS * j) + 8 * tig;
#pragma unroll
    for (int bt = 0; bt < MT; ++bt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = bt * 16 + h * 8 + g;
        xa[j][bt][h] = (col < kn && r < B) ? *reinterpret_cast<const uint4*>(X + (long)r * K + k0 + col)
                                           : make_uint4(0u, 0u, 0u, 0u);
      }
  }
  bool lnwait = false;   // a timed-out wait for the LayerNorm parameters
  if (lng) {
    // x <- LayerNorm(x) (RMSNorm without lnb), nkc == 1: columns [0, K).
    // Statistics with one barrier: each lane takes the mean and the sum of
    // squared deviations (M2) of its values of a row (registers only); the
    // quad's four equal-count parts merge pairwise by shuffles (mean' = (ma +
    // mb) / 2, M2' = M2a + M2b + d^2 n / 2 for n values each, d = mb - ma:
    // the pairwise update of Chan, Golub and LeVeque); the warps' parts merge
    // in warp order as mean = sum_w n_w mean_w / K and M2 = sum_w (M2_w +
    // n_w (mean_w - mean)^2).  RMSNorm keeps every mean 0 and sums squares.
    float mu[MT][2], rs[MT][2];
    const float inK = 1.f / K;
    if (st_in) {
      // statistics from the producer's 16-column groups: thread (r, p) takes
      // groups p, p + TPR, ... of row r; the row's TPR lanes merge by shuffles
      // as mean = 16 sum_g mean_g / K, M2 = sum_g (M2_g + 16 (mean_g - mean)^2)
      constexpr int R = 16 * MT, TPR = DM_THREADS / R, GPL = (DM_KC / 16 + TPR - 1) / TPR;
      float2* srow = reinterpret_cast<float2*>(red);   // [16 MT] (mean, rstd)
      const int r = threadIdx.x / TPR, p = threadIdx.x % TPR, NG = K / 16;
      float2 gv[GPL];
      float sm = 0.f;
#pragma unroll
      for (int i = 0; i < GPL; ++i) {
        const int gi = p + TPR * i;
        gv[i] = gi < NG && r < B ? st_in[(long)gi * B + r] : make_float2(0.f, 0.f);
        sm += gv[i].x;
      }
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
      const float m = lnb ? 16.f * sm * inK : 0.f;
      float q = 0.f;
#pragma unroll
      for (int i = 0; i < GPL; ++i)
        if (p + TPR * i < NG) q += gv[i].y + 16.f * (gv[i].x - m) * (gv[i].x - m);
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      if (p == 0) srow[r] = make_float2(m, 1.0f / sqrtf(q * inK + eps));
      __syncthreads();
#pragma unroll
      for (int bt = 0; bt < MT; ++bt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 t = srow[bt * 16 + h * 8 + g];
          mu[bt][h] = t.x;
          rs[bt][h] = t.y;
        }
    } else {
      float2* sred = reinterpret_cast<float2*>(red);   // [DM_WARPS][16 MT] (mean, M2) of the warp's columns
      const int nw = min(DM_KB, (kn / 32 - warp + DM_WARPS - 1) / DM_WARPS);   // this warp's blocks in range
      const float nl = 8.f * nw;                                             // values per lane
      const float inl = nw > 0 ? 1.f / nl : 0.f;
#pragma unroll
      for (int bt = 0; bt < MT; ++bt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float m = 0.f, q = 0.f;
          if (nw > 0 && bt * 16 + h * 8 + g < B) {
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < DM_KB; ++j)
              if (j < nw) {
                float v[8];
                unpack16x8<F16>(xa[j][bt][h], v);
#pragma unroll
                for (int i = 0; i < 8; ++i) sum += v[i];
              }
            m = lnb ? sum * inl : 0.f;
#pragma unroll
            for (int j = 0; j < DM_KB; ++j)
              if (j < nw) {
                float v[8];
                unpack16x8<F16>(xa[j][bt][h], v);
#pragma unroll
                for (int i = 0; i < 8; ++i) q = fmaf(v[i] - m, v[i] - m, q);
              }
          }
          // quad merge: four lanes with equal counts
          float n = nl;
#pragma unroll
          for (int o = 1; o <= 2; o <<= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o), q2 = __shfl_xor_sync(0xffffffffu, q, o);
            const float d = m2 - m;
            q = q + q2 + d * d * (0.5f * n);   // na = nb = n: d^2 na nb / (2n) = d^2 n / 2
            m = m + 0.5f * d;
            n *= 2.f;
          }
          if (tig == 0) sred[warp * 16 * MT + bt * 16 + h * 8 + g] = make_float2(m, q);
        }
      __syncthreads();
#pragma unroll
      for (int bt = 0; bt < MT; ++bt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float sm = 0.f, q = 0.f;
#pragma unroll
          for (int w = 0; w < DM_WARPS; ++w) {
            const float nb = 32.f * min(DM_KB, (kn / 32 - w + DM_WARPS - 1) / DM_WARPS);
            sm = fmaf(nb, sred[w * 16 * MT + bt * 16 + h * 8 + g].x, sm);
          }
          const float m = lnb ? sm * inK : 0.f;
#pragma unroll
          for (int w = 0; w < DM_WARPS; ++w) {
            const float nb = 32.f * min(DM_KB, (kn / 32 - w + DM_WARPS - 1) / DM_WARPS);
            const float2 t = sred[w * 16 * MT + bt * 16 + h * 8 + g];
            const float d = t.x - m;
            q += t.y + nb * d * d;
          }
          mu[bt][h] = m;
          // RMSNorm: q is the sum of squares (every mean stayed 0)
          rs[bt][h] = 1.0f / sqrtf(q * inK + eps);
        }
    }
    if (ln_bulk) lnwait = !mbar_wait(smem_u32(&lnbar), 0, &s_abort);
#pragma unroll
    for (int j = 0; j < DM_KB; ++j) {
      const int col = 32 * (warp + DM_WARPS * j) + 8 * tig;
      if (col < kn) {
        float gv[8], bv[8];
        *reinterpret_cast<float4*>(gv) = *reinterpret_cast<const float4*>(lns + col);
        *reinterpret_cast<float4*>(gv + 4) = *reinterpret_cast<const float4*>(lns + col + 4);
        *reinterpret_cast<float4*>(bv) = *reinterpret_cast<const float4*>(lns + K + col);
        *reinterpret_cast<float4*>(bv + 4) = *reinterpret_cast<const float4*>(lns + K + col + 4);
#pragma unroll
        for (int bt = 0; bt < MT; ++bt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (bt * 16 + h * 8 + g >= B) continue;   // rows past B stay zero
            float v[8];
            unpack16x8<F16>(xa[j][bt][h], v);
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[i] = pack16x2<F16>((v[2 * i] - mu[bt][h]) * rs[bt][h] * gv[2 * i] + bv[2 * i],
                                   (v[2 * i + 1] - mu[bt][h]) * rs[bt][h] * gv[2 * i + 1] + bv[2 * i + 1]);
            xa[j][bt][h] = make_uint4(w[0], w[1], w[2], w[3]);
          }
      }
    }
  }
  // A timed-out wait is voted block-wide; the CTA then runs its remaining
  // slices without data so that every slice counter still receives its nkc
  // arrivals (and returns to zero), and drains its copies before leaving.
  bool dead = __syncthreads_or(lnwait);
  int landed = 0;   // slices whose copies completed
  for (int j = 0; j < nmine; ++j) {
    const int s = grp + j * ngrp, r0 = s * DM_ROWS;
    // the vote is also the barrier after the previous slice's reads of red
    if (!dead) dead = __syncthreads_or(!mbar_wait(smem_u32(&bars[j % nbuf]), (j / nbuf) & 1, &s_abort));
    else __syncthreads();
    if (!dead) landed = j + 1;
    // this thread's outputs o = threadIdx.x + DM_THREADS t: bias and residual
    // values load while the tensor cores run
    float pb[DM_OPT], pr[DM_OPT];
#pragma unroll
    for (int t = 0; t < DM_OPT; ++t) {
      const int o = threadIdx.x + DM_THREADS * t, bb = o / DM_ROWS, n = r0 + o % DM_ROWS;
      const bool ok = o < B * DM_ROWS && n < N;
      pb[t] = ok && bias && mode != 2 ? bias[n] : 0.f;
      pr[t] = ok && resid && mode == 0 ? to_f(resid[(long)bb * N + n]) : 0.f;
    }
    float acc[MT][2][4];
#pragma unroll
    for (int bt = 0; bt < MT; ++bt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[bt][nt][e] = 0.f;
    if (!dead) {
      const uint32_t slot = slot0 + (j % nbuf) * slot_bytes;
#pragma unroll
      for (int jj = 0; jj < DM_KB; ++jj) {
        const int col = 32 * (warp + DM_WARPS * jj) + 8 * tig;
        if (32 * (warp + DM_WARPS * jj) < kn) {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const uint4 w = dm_lds128(slot + (uint32_t)((nt * 8 + g) * kcl + col) * 2);
#pragma unroll
            for (int bt = 0; bt < MT; ++bt) {
              const uint4 p = xa[jj][bt][0], q = xa[jj][bt][1];
              dm_mma<F16>(acc[bt][nt], p.x, q.x, p.y, q.y, w.x, w.y);
              dm_mma<F16>(acc[bt][nt], p.z, q.z, p.w, q.w, w.z, w.w);
            }
          }
        }
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
    // every read of this slot is done: refill it
    if (threadIdx.x == 0 && !dead && issued < nmine) issue(issued++);
#pragma unroll
    for (int t = 0; t < DM_OPT; ++t) {
      const int o = threadIdx.x + DM_THREADS * t, bb = o / DM_ROWS, nn = o % DM_ROWS, n = r0 + nn;
      const bool ok = o < B * DM_ROWS && n < N;
      float y = 0.f, v = 0.f;
      if (ok) {
#pragma unroll
        for (int w = 0; w < DM_WARPS; ++w) y += red[((w * 16 * MT) + bb) * 16 + nn];
        if (nkc == 1) v = dm_epilogue<T>(y, pb[t], pr[t], bb, n, N, mode, out, out2, outf);
        else dm_st_cluster(smem_u32(cred + ((j & 1) * nkc + kc) * (B * DM_ROWS) + o), 0u, y);
      }
      if (nkc == 1 && st_out) dm_group_stats(v, ok, st_out, s, B, bb, lane);
    }
    if (nkc > 1) {
      // every CTA arrives here once per slice, a timed-out one included
      dm_cluster_sync();
      if (kc == 0) {
#pragma unroll
        for (int t = 0; t < DM_OPT; ++t) {
          const int o = threadIdx.x + DM_THREADS * t, bb = o / DM_ROWS, n = r0 + o % DM_ROWS;
          const bool ok = o < B * DM_ROWS && n < N;
          float v = 0.f;
          if (ok) {
            float y = 0.f;
            for (int q = 0; q < nkc; ++q) y += cred[((j & 1) * nkc + q) * (B * DM_ROWS) + o];
            v = dm_epilogue<T>(y, pb[t], pr[t], bb, n, N, mode, out, out2, outf);
          }
          if (st_out) dm_group_stats(v, ok, st_out, s, B, bb, lane);
        }
      }
    }
  }
  // no CTA leaves while another may still store into its shared memory
  if (nkc > 1) dm_cluster_sync();
  if (dead && threadIdx.x == 0) {
    set_dev_err(err, GPT_DEVERR_TIMEOUT);
    // let the copies still in flight land before leaving
    volatile int never = 0;
    if (ln_bulk) mbar_wait(smem_u32(&lnbar), 0, &never, 1ll << 28);
    for (int q = landed; q < issued; ++q) mbar_wait(smem_u32(&bars[q % nbuf]), (q / nbuf) & 1, &never, 1ll << 28);
  }
}

static int g_dm_sms = 0;

bool dec_mma_supported(int B, int K, int N, bool ln) {
  return B >= 1 && B <= 32 && K >= 32 && K % 32 == 0 && N >= 1 && K <= (ln ? DM_KC : DM_KC * DM_MAX_SPLIT);
}

template <typename T>
cudaError_t launch_dec_mma(const T* X, int B, int K, const T* W, int N, const float* bias, const T* resid, int mode,
                           T* out, T* out2, float* outf, unsigned* err, cudaStream_t s, const float* lng,
                           const float* lnb, float eps, float2* st_out, const float2* st_in) {
  if (!dec_mma_supported(B, K, N, lng != nullptr)) return cudaErrorInvalidValue;
  if ((st_out && (mode != 0 || N % 16)) || (st_in && (!lng || K % 16))) return cudaErrorInvalidValue;
  if (((uintptr_t)X & 15) || ((uintptr_t)W & 15)) return cudaErrorInvalidValue;
  if (!g_dm_sms) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_dm_sms = n > 0 ? n : 148;
  }
  const int MT = B <= 16 ? 1 : 2;
  const int nslices = (N + DM_ROWS - 1) / DM_ROWS;
  // k ranges of at most DM_KC columns, multiples of 32
  const int nkc = (K + DM_KC - 1) / DM_KC, kcl = ((K + nkc - 1) / nkc + 31) / 32 * 32;
  if ((nkc - 1) * kcl >= K || nkc > DM_MAX_SPLIT) return cudaErrorInvalidValue;   // no empty last range
  const size_t slot = (size_t)DM_ROWS * kcl * 2;
  const size_t red = (size_t)DM_WARPS * 16 * MT * 16 * 4 + (lng ? (size_t)2 * K * 4 : 0) +
                     (nkc > 1 ? (size_t)2 * nkc * B * DM_ROWS * 4 : 0);
  int nbuf = (int)((DM_SMEM_BUDGET - (long)red) / (long)slot);
  if (nbuf > DM_MAXBUF) nbuf = DM_MAXBUF;
  if (nbuf < 2) nbuf = 2;
  const size_t smem = nbuf * slot + red;
  void (*kern)(const T*, int, int, const T*, int, int, int, const float*, const T*, int, T*, T*, float*, int,
               unsigned*, const float*, const float*, float, float2*, const float2*) =
      MT == 1 ? dec_mma_kernel<T, 1> : dec_mma_kernel<T, 2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, DM_THREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidValue;
  const int ngrp = std::min(g_dm_sms * std::min(per_sm, DM_CTAS) / nkc, nslices);
  if (ngrp < 1) return cudaErrorInvalidValue;
  ++g_kernel_launches;
  if (nkc == 1)
    return launch_k(kern, dim3(ngrp), dim3(DM_THREADS), smem, s, X, B, K, W, N, nkc, kcl, bias, resid, mode, out, out2,
                    outf, nbuf, err, lng, lnb, eps, st_out, st_in);
  // clusters of nkc CTAs (and the programmatic dependent launch of launch_k)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ngrp * nkc);
  cfg.blockDim = dim3(DM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = nkc;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, X, B, K, W, N, nkc, kcl, bias, resid, mode, out, out2, outf, nbuf, err, lng,
                            lnb, eps, st_out, st_in);
}

template cudaError_t launch_dec_mma<bf16>(const bf16*, int, int, const bf16*, int, const float*, const bf16*, int,
                                          bf16*, bf16*, float*, unsigned*, cudaStream_t, const float*, const float*,
                                          float, float2*, const float2*);
template cudaError_t launch_dec_mma<f16>(const f16*, int, int, const f16*, int, const float*, const f16*, int, f16*,
                                         f16*, float*, unsigned*, cudaStream_t, const float*, const float*, float,
                                         float2*, const float2*);
