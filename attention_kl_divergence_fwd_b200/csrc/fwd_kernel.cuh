// fwd_kernel.cuh - StreamKL forward on sm_100a (tcgen05 + TMEM + TMA).
//
// The one-pass forward of "StreamKL: Fast and Memory-Efficient KL Divergence for
// Boosting Attention Distillation" (abstract: an online formulation of the coupled
// two-distribution KL reduction, streaming query-key tiles through on-chip memory).
//
// CTA = two 128-row query tiles of one (batch, head). Key tiles of 64 rows stream
// through a TMA ring. Per key tile and query tile the tensor core computes the teacher
// and student score tiles into TMEM (two buffers per query tile). Each query tile has
// two warpgroups, one thread per query row, taking the even and the odd key tiles; each
// folds its tiles into its own online state
//     m_T, m_S   running maxima of t = s * log2(e)
//     l_T, l_S   running sums of 2^(t - m)
//     A          running sum of 2^(t_T - m_T) * (t_T - t_S)
// and the two states of a row are merged at the end (the state is associative), so
// KL = ln2 * A / l_T - LSE_T + LSE_S. Nothing of size N_Q x N_K ever leaves the SM.
//
// Warp roles (576 threads): warps 0-15 statistics (warpgroup w: query tile w>>1, key
// tiles of parity w&1), warp 16 TMA producer, warp 17 TMEM allocator + MMA issuer.
#pragma once

#include "ptx.cuh"

namespace skl {

struct FwdArgs {
  int BH, N_Q, N_K;
  int causal;
  int off;            // N_K - N_Q (bottom-right causal alignment)
  float cT, cS;       // |scale| * log2(e); the MMA negates A when the scale is negative
  int n_ctas_per_bh;  // ceil(N_Q / 256)
  float* kl;
  float* lse_t;
  float* lse_s;
};

template <int DT, int DS>
struct FwdCfg {
  static constexpr int BM = 128;  // query rows per tile = TMEM lanes
  static constexpr int NQ = 2;    // query tiles per CTA
  static constexpr int BN = 64;   // keys per tile
  static constexpr int QT_TILE = BM * DT * 2;
  static constexpr int QS_TILE = BM * DS * 2;
  static constexpr int KT_TILE = BN * DT * 2;
  static constexpr int KS_TILE = BN * DS * 2;
  static constexpr int STAGE = KT_TILE + KS_TILE;
  static constexpr int QBYTES = NQ * (QT_TILE + QS_TILE);
  static constexpr int SMEM_MAX = 232448;
  static constexpr int BAR_BYTES = 256;
  static constexpr int NST_FIT = (SMEM_MAX - BAR_BYTES - QBYTES) / STAGE;
  static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;
  static constexpr int SMEM = QBYTES + NST * STAGE + BAR_BYTES;  // base is 1024-aligned
  static constexpr int THREADS = 576;
  static_assert(NST >= 2, "key ring needs two stages");
  static_assert(SMEM <= SMEM_MAX, "shared memory budget");
};

struct FwdBars {
  uint64_t q_full;
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t s_full[2][2];
  uint64_t s_free[2][2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void skl_fail(volatile int* abort_flag) {
  atomicOr(&g_skl_error, 1u);
  *abort_flag = 1;
}

// Online state of one query row over the keys one warpgroup has seen (base-2 units).
struct RowState {
  float mT, mS, lT, lS, A;
};

// Folds 32 keys (v[0..31] teacher scores, v[32..63] student scores, raw dot products)
// into the row state. Columns c > lim are masked. Every fourth exponential (c % 4 == 3)
// runs on the FMA pipe (exp2_fma) so the MUFU is not the only unit doing them.
template <bool MASK>
__device__ __forceinline__ void fold_chunk(RowState& st, const uint32_t (&v)[64], float cT,
                                           float cS, int lim) {
  float mxT, mxS;
  {
    float a[32], b[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      a[c] = (!MASK || c <= lim) ? __uint_as_float(v[c]) : -INFINITY;
      b[c] = (!MASK || c <= lim) ? __uint_as_float(v[32 + c]) : -INFINITY;
    }
    mxT = max_tree32(a);
    mxS = max_tree32(b);
  }
  const float mT_new = fmaxf(st.mT, cT * mxT);  // NaN (cT=0, all masked) keeps the old max
  const float mS_new = fmaxf(st.mS, cS * mxS);
  const float mT_use = (mT_new == -INFINITY) ? 0.f : mT_new;
  const float mS_use = (mS_new == -INFINITY) ? 0.f : mS_new;
  // Rescale the running sums only when some row of the warp raised its maximum.
  if (__any_sync(0xffffffffu, (mT_new > st.mT) || (mS_new > st.mS))) {
    const float aT = ex2_approx(st.mT - mT_use);  // -inf - x -> 0
    const float aS = ex2_approx(st.mS - mS_use);
    st.lT *= aT;
    st.A *= aT;
    st.lS *= aS;
  }
  float sT0 = 0.f, sT1 = 0.f, sS0 = 0.f, sS1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    const float xT0 = fmaf(__uint_as_float(v[c]), cT, -mT_use);
    const float xT1 = fmaf(__uint_as_float(v[c + 1]), cT, -mT_use);
    const float xS0 = fmaf(__uint_as_float(v[32 + c]), cS, -mS_use);
    const float xS1 = fmaf(__uint_as_float(v[32 + c + 1]), cS, -mS_use);
    float eT0 = ex2_approx(xT0);
    float eS0 = ex2_approx(xS0);
    float eT1, eS1;
    if ((c & 3) == 2) {
      eT1 = exp2_fma(xT1);
      eS1 = exp2_fma(xS1);
    } else {
      eT1 = ex2_approx(xT1);
      eS1 = ex2_approx(xS1);
    }
    if (MASK) {
      eT0 = c <= lim ? eT0 : 0.f;
      eS0 = c <= lim ? eS0 : 0.f;
      eT1 = c + 1 <= lim ? eT1 : 0.f;
      eS1 = c + 1 <= lim ? eS1 : 0.f;
    }
    sT0 += eT0;
    sT1 += eT1;
    sS0 += eS0;
    sS1 += eS1;
    b0 = fmaf(eT0, xT0 - xS0, b0);
    b1 = fmaf(eT1, xT1 - xS1, b1);
  }
  const float sumT = sT0 + sT1;
  st.lT += sumT;
  st.lS += sS0 + sS1;
  st.A += (b0 + b1) + (mT_use - mS_use) * sumT;
  st.mT = mT_new;
  st.mS = mS_new;
}

template <int DT, int DS>
__global__ void __launch_bounds__(576, 1)
streamkl_fwd_kernel(const __grid_constant__ CUtensorMap map_qt,
                    const __grid_constant__ CUtensorMap map_kt,
                    const __grid_constant__ CUtensorMap map_qs,
                    const __grid_constant__ CUtensorMap map_ks,
                    const FwdArgs args, const uint32_t idesc_t, const uint32_t idesc_s) {
  using C = FwdCfg<DT, DS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t s_base = smem_u32(smem);
  if (s_base & 1023u) {  // the swizzled tiles need 1024-byte alignment; never expected to fire
    if (threadIdx.x == 0) atomicOr(&g_skl_error, 4u);
    return;
  }
  const uint32_t s_qt = s_base;                               // [NQ][DT/64][128][64]
  const uint32_t s_qs = s_base + C::NQ * C::QT_TILE;          // [NQ][DS/64][128][64]
  const uint32_t s_k = s_base + C::QBYTES;                    // [NST]{K_T, K_S}
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::QBYTES + C::NST * C::STAGE);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Heaviest (last) query tiles first for causal load balance, all heads interleaved.
  const int t = blockIdx.x;
  const int bh = t % args.BH;
  const int qpair = args.n_ctas_per_bh - 1 - t / args.BH;
  const int q0 = qpair * (C::NQ * C::BM);
  const int n_ktiles_all = (args.N_K + C::BN - 1) / C::BN;

  // Key tiles needed by each query tile.
  int nk[C::NQ];
#pragma unroll
  for (int q = 0; q < C::NQ; ++q) {
    const int first = q0 + q * C::BM;
    if (first >= args.N_Q) {
      nk[q] = 0;
    } else if (!args.causal) {
      nk[q] = n_ktiles_all;
    } else {
      const int last_row = min(first + C::BM, args.N_Q) - 1;
      const int last_key = last_row + args.off;
      nk[q] = last_key < 0 ? 0 : min(n_ktiles_all, last_key / C::BN + 1);
    }
  }
  const int nk_max = max(nk[0], nk[1]);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int q = 0; q < 2; ++q)
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&bars->s_full[q][b]), 1);
        mbar_init(smem_u32(&bars->s_free[q][b]), 4);
      }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 17) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 16) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&map_qt);
      tma_prefetch_desc(&map_kt);
      tma_prefetch_desc(&map_qs);
      tma_prefetch_desc(&map_ks);
      const uint64_t keep = l2_policy_evict_last();
      const uint64_t once = l2_policy_evict_first();
      const uint32_t qb = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qb, C::QBYTES);
      for (int q = 0; q < C::NQ; ++q) {
        for (int blk = 0; blk < DT / 64; ++blk)
          tma_load_3d(s_qt + q * C::QT_TILE + blk * (C::BM * 128), &map_qt, qb, blk * 64,
                      q0 + q * C::BM, bh, once);
        for (int blk = 0; blk < DS / 64; ++blk)
          tma_load_3d(s_qs + q * C::QS_TILE + blk * (C::BM * 128), &map_qs, qb, blk * 64,
                      q0 + q * C::BM, bh, once);
      }
      int issued = 0;
      for (int j = 0; j < nk_max; ++j) {
        const int s = j % C::NST;
        if (!mbar_wait(smem_u32(&bars->empty[s]), ((j / C::NST) & 1) ^ 1)) {
          skl_fail(abort_flag);
          break;
        }
        const uint32_t fb = smem_u32(&bars->full[s]);
        mbar_arrive_expect_tx(fb, C::STAGE);
        const uint32_t st = s_k + s * C::STAGE;
        for (int blk = 0; blk < DT / 64; ++blk)
          tma_load_3d(st + blk * (C::BN * 128), &map_kt, fb, blk * 64, j * C::BN, bh, keep);
        for (int blk = 0; blk < DS / 64; ++blk)
          tma_load_3d(st + C::KT_TILE + blk * (C::BN * 128), &map_ks, fb, blk * 64, j * C::BN,
                      bh, keep);
        issued = j + 1;
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA can exit.
        mbar_wait(qb, 0);
        for (int j = max(0, issued - C::NST); j < issued; ++j)
          mbar_wait(smem_u32(&bars->full[j % C::NST]), (j / C::NST) & 1);
      }
    }
  } else if (warp == 17) {
    // ------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0);
      if (!ok) skl_fail(abort_flag);
      for (int j = 0; ok && j < nk_max; ++j) {
        const int s = j % C::NST;
        if (!mbar_wait(smem_u32(&bars->full[s]), (j / C::NST) & 1)) {
          skl_fail(abort_flag);
          break;
        }
        tc_fence_after();
        const uint32_t st = s_k + s * C::STAGE;
#pragma unroll
        for (int q = 0; q < C::NQ; ++q) {
          if (j >= nk[q]) continue;
          const int b = j & 1;
          if (!mbar_wait(smem_u32(&bars->s_free[q][b]), ((j >> 1) & 1) ^ 1)) {
            skl_fail(abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_t = tmem + q * 256 + b * 128;
          const uint32_t d_s = d_t + 64;
#pragma unroll
          for (int kk = 0; kk < DT / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t a = sdesc_sw128(s_qt + q * C::QT_TILE + (kk >> 2) * (C::BM * 128) + off,
                                           16, 1024);
            const uint64_t bd = sdesc_sw128(st + (kk >> 2) * (C::BN * 128) + off, 16, 1024);
            umma_bf16_ss(d_t, a, bd, idesc_t, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < DS / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t a = sdesc_sw128(s_qs + q * C::QS_TILE + (kk >> 2) * (C::BM * 128) + off,
                                           16, 1024);
            const uint64_t bd =
                sdesc_sw128(st + C::KT_TILE + (kk >> 2) * (C::BN * 128) + off, 16, 1024);
            umma_bf16_ss(d_s, a, bd, idesc_s, kk > 0);
          }
          umma_commit(smem_u32(&bars->s_full[q][b]));
        }
        umma_commit(smem_u32(&bars->empty[s]));
      }
      // Every MMA this thread issued must be complete before TMEM is released.
      umma_commit(smem_u32(&bars->drain));
      if (!mbar_wait(smem_u32(&bars->drain), 0)) skl_fail(abort_flag);
    }
  } else {
    // --------------------------------------------------- statistics warpgroups
    const int wg = warp >> 2;
    const int q = wg >> 1;            // query tile
    const int par = wg & 1;           // key tiles j with j & 1 == par (TMEM buffer par)
    const int quarter = warp & 3;     // TMEM lane quarter of this warp
    const int rloc = quarter * 32 + lane;
    const int row = q0 + q * C::BM + rloc;
    const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + q * 256 + par * 128;
    const float cT = args.cT, cS = args.cS;
    const int first_row = q0 + q * C::BM;
    const int nkq = nk[q];

    RowState st{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
    bool ok = true;
    for (int j = par; j < nkq; j += 2) {
      if (!mbar_wait(smem_u32(&bars->s_full[q][par]), (j >> 1) & 1)) {
        skl_fail(abort_flag);
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = j * C::BN;
      const bool need_mask =
          (k0 + C::BN > args.N_K) || (args.causal && k0 + C::BN - 1 > first_row + args.off);
      int lim = C::BN - 1;  // last allowed column of this tile for this row
      if (need_mask) {
        int last = args.N_K - 1;
        if (args.causal) last = min(last, row + args.off);
        lim = last - k0;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[64];  // keys 64j+32h .. +31: v[0..31] teacher, v[32..63] student
        tmem_ld_2x32_wait(ta + 32 * h, ta + 64 + 32 * h, v);
        if (h == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[q][par]));
        }
        if (need_mask)
          fold_chunk<true>(st, v, cT, cS, lim - 32 * h);
        else
          fold_chunk<false>(st, v, cT, cS, 0);
      }
    }

    // Merge the odd-tile state into the even-tile warpgroup. The merge area is this
    // query tile's Q_T buffer, free once every MMA of the tile has completed.
    float* merge = reinterpret_cast<float*>(smem + q * C::QT_TILE);
    bool ready = ok && mbar_wait(smem_u32(&bars->q_full), 0);
    if (ready && nkq > 0) {
      const int jl = nkq - 1;
      ready = mbar_wait(smem_u32(&bars->s_full[q][jl & 1]), (jl >> 1) & 1);
    }
    if (!ready && ok) skl_fail(abort_flag);
    fence_async_smem();
    if (par == 1 && ready) {
      merge[0 * C::BM + rloc] = st.mT;
      merge[1 * C::BM + rloc] = st.mS;
      merge[2 * C::BM + rloc] = st.lT;
      merge[3 * C::BM + rloc] = st.lS;
      merge[4 * C::BM + rloc] = st.A;
    }
    named_bar_sync(1 + q, 256);
    if (par == 0 && ready && row < args.N_Q) {
      const float mT1 = merge[0 * C::BM + rloc], mS1 = merge[1 * C::BM + rloc];
      const float mT = fmaxf(st.mT, mT1), mS = fmaxf(st.mS, mS1);
      const float mT_use = (mT == -INFINITY) ? 0.f : mT;
      const float mS_use = (mS == -INFINITY) ? 0.f : mS;
      const float a0T = ex2_approx(st.mT - mT_use), a1T = ex2_approx(mT1 - mT_use);
      const float a0S = ex2_approx(st.mS - mS_use), a1S = ex2_approx(mS1 - mS_use);
      const float lT = a0T * st.lT + a1T * merge[2 * C::BM + rloc];
      const float lS = a0S * st.lS + a1S * merge[3 * C::BM + rloc];
      const float A = a0T * st.A + a1T * merge[4 * C::BM + rloc];
      const float LN2 = 0.69314718055994530942f;
      float kl, lse_t, lse_s;
      if (lT > 0.f) {
        const float l2T = log2f(lT), l2S = log2f(lS);
        lse_t = LN2 * (mT + l2T);
        lse_s = LN2 * (mS + l2S);
        // Grouped so that identical teacher and student statistics give exactly 0.
        kl = LN2 * ((A / lT) + ((mS - mT) + (l2S - l2T)));
      } else {
        kl = 0.f;
        lse_t = -INFINITY;
        lse_s = -INFINITY;
      }
      const size_t o = (size_t)bh * args.N_Q + row;
      args.kl[o] = kl;
      args.lse_t[o] = lse_t;
      args.lse_s[o] = lse_s;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 17) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace skl
