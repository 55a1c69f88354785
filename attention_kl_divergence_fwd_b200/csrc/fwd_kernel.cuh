// fwd_kernel.cuh - StreamKL forward on sm_100a (tcgen05 + TMEM + TMA).
//
// The one-pass forward of "StreamKL: Fast and Memory-Efficient KL Divergence for
// Boosting Attention Distillation" (abstract: an online formulation of the coupled
// two-distribution KL reduction, streaming query-key tiles through on-chip memory).
//
// CTA = two 128-row query tiles of one (batch, head). Key tiles of 64 rows stream
// through a TMA ring. Per key tile and query tile the tensor core computes the
// teacher and student score tiles into TMEM (double-buffered per query tile), and
// one warpgroup per query tile (one thread per query row) folds them into the
// online state
//     m_T, m_S   running maxima of t = s * log2(e)
//     l_T, l_S   running sums of 2^(t - m)
//     A          running sum of 2^(t_T - m_T) * (t_T - t_S)
// so that KL = ln2 * A / l_T - LSE_T + LSE_S at the end. Nothing of size N_Q x N_K
// ever leaves the SM.
//
// Warp roles (320 threads): warps 0-3 query tile 0, warps 4-7 query tile 1,
// warp 8 TMA producer, warp 9 TMEM allocator + MMA issuer.
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
  static constexpr int NST_FIT = (SMEM_MAX - 1024 - BAR_BYTES - QBYTES) / STAGE;
  static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;
  static constexpr int SMEM = 1024 + QBYTES + NST * STAGE + BAR_BYTES;
  static constexpr int THREADS = 320;
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

template <int DT, int DS>
__global__ void __launch_bounds__(320, 1)
streamkl_fwd_kernel(const __grid_constant__ CUtensorMap map_qt,
                    const __grid_constant__ CUtensorMap map_kt,
                    const __grid_constant__ CUtensorMap map_qs,
                    const __grid_constant__ CUtensorMap map_ks,
                    const FwdArgs args, const uint32_t idesc_t, const uint32_t idesc_s) {
  using C = FwdCfg<DT, DS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
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
  if (warp == 9) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
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
  } else if (warp == 9) {
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
    const int q = warp >> 2;          // query tile of this warpgroup
    const int quarter = warp & 3;     // TMEM lane quarter of this warp
    const int row = q0 + q * C::BM + quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float cT = args.cT, cS = args.cS;
    const int first_row = q0 + q * C::BM;

    float mT = -INFINITY, mS = -INFINITY, lT = 0.f, lS = 0.f, A = 0.f;
    bool ok = true;
    for (int j = 0; j < nk[q]; ++j) {
      const int b = j & 1;
      if (!mbar_wait(smem_u32(&bars->s_full[q][b]), (j >> 1) & 1)) {
        skl_fail(abort_flag);
        ok = false;
        break;
      }
      tc_fence_after();
      // Raw teacher / student scores of keys 64j..64j+63 for this thread's row.
      const uint32_t ta = tmem + lane_off + q * 256 + b * 128;
      uint32_t vt_u[64], vs_u[64];
      tmem_ld_2x32_wait(ta, ta + 32, vt_u);
      tmem_ld_2x32_wait(ta + 64, ta + 96, vs_u);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[q][b]));

      const int k0 = j * C::BN;
      const bool need_mask =
          (k0 + C::BN > args.N_K) || (args.causal && k0 + C::BN - 1 > first_row + args.off);
      int lim = C::BN - 1;  // last allowed column of this tile for this row
      if (need_mask) {
        int last = args.N_K - 1;
        if (args.causal) last = min(last, row + args.off);
        lim = last - k0;
      }

      float mxT = -INFINITY, mxS = -INFINITY;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < C::BN; ++c) {
          const bool ok_c = c <= lim;
          mxT = fmaxf(mxT, ok_c ? __uint_as_float(vt_u[c]) : -INFINITY);
          mxS = fmaxf(mxS, ok_c ? __uint_as_float(vs_u[c]) : -INFINITY);
        }
      } else {
#pragma unroll
        for (int c = 0; c < C::BN; ++c) {
          mxT = fmaxf(mxT, __uint_as_float(vt_u[c]));
          mxS = fmaxf(mxS, __uint_as_float(vs_u[c]));
        }
      }
      const float mT_new = fmaxf(mT, cT * mxT);
      const float mS_new = fmaxf(mS, cS * mxS);
      const float mT_use = (mT_new == -INFINITY) ? 0.f : mT_new;
      const float mS_use = (mS_new == -INFINITY) ? 0.f : mS_new;
      const float aT = ex2_approx(mT - mT_use);
      const float aS = ex2_approx(mS - mS_use);

      float sT0 = 0.f, sT1 = 0.f, sS0 = 0.f, sS1 = 0.f, b0 = 0.f, b1 = 0.f;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < C::BN; c += 2) {
          const float xT0 = fmaf(__uint_as_float(vt_u[c]), cT, -mT_use);
          const float xT1 = fmaf(__uint_as_float(vt_u[c + 1]), cT, -mT_use);
          const float xS0 = fmaf(__uint_as_float(vs_u[c]), cS, -mS_use);
          const float xS1 = fmaf(__uint_as_float(vs_u[c + 1]), cS, -mS_use);
          const float eT0 = c <= lim ? ex2_approx(xT0) : 0.f;
          const float eT1 = c + 1 <= lim ? ex2_approx(xT1) : 0.f;
          const float eS0 = c <= lim ? ex2_approx(xS0) : 0.f;
          const float eS1 = c + 1 <= lim ? ex2_approx(xS1) : 0.f;
          sT0 += eT0; sT1 += eT1; sS0 += eS0; sS1 += eS1;
          b0 = fmaf(eT0, xT0 - xS0, b0);
          b1 = fmaf(eT1, xT1 - xS1, b1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < C::BN; c += 2) {
          const float xT0 = fmaf(__uint_as_float(vt_u[c]), cT, -mT_use);
          const float xT1 = fmaf(__uint_as_float(vt_u[c + 1]), cT, -mT_use);
          const float xS0 = fmaf(__uint_as_float(vs_u[c]), cS, -mS_use);
          const float xS1 = fmaf(__uint_as_float(vs_u[c + 1]), cS, -mS_use);
          const float eT0 = ex2_approx(xT0), eT1 = ex2_approx(xT1);
          const float eS0 = ex2_approx(xS0), eS1 = ex2_approx(xS1);
          sT0 += eT0; sT1 += eT1; sS0 += eS0; sS1 += eS1;
          b0 = fmaf(eT0, xT0 - xS0, b0);
          b1 = fmaf(eT1, xT1 - xS1, b1);
        }
      }
      const float sumT = sT0 + sT1;
      lT = fmaf(aT, lT, sumT);
      lS = fmaf(aS, lS, sS0 + sS1);
      A = fmaf(aT, A, (b0 + b1) + (mT_use - mS_use) * sumT);
      mT = mT_new;
      mS = mS_new;
    }

    if (ok && row < args.N_Q) {
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace skl
