// fwd_persistent.cuh - persistent form of the StreamKL forward (dense layout).
//
// The same one-pass forward as fwd_kernel.cuh ("StreamKL: Fast and Memory-Efficient KL
// Divergence for Boosting Attention Distillation", abstract: one forward pass reduces both
// distributions together with a running per-row state while query and key tiles pass
// through on-chip memory), run by one CTA per SM that walks a list of work units instead of
// one CTA per unit. A unit is a pair of 128-row query tiles of one (batch, head), as in the
// non-persistent kernel.
//
// Schedule (longest processing time first): the units are ordered heaviest first over all
// heads (under causal masking the last query tiles see the most keys), and CTA c of G takes
// units c, 2G-1-c, 2G+c, 4G-1-c, ... (a snake over rounds of G units), so that a CTA that
// drew one of the heaviest units of a round draws one of the lightest of the next. The list
// is a closed form of (blockIdx.x, gridDim.x): no work counter, no device memory beyond the
// caller's buffers.
//
// What persistence removes is the per-unit prologue of a fresh CTA (barrier setup, TMEM
// allocation, the query tiles' load from memory) and the tail of a one-CTA-per-unit grid:
// * barriers keep counting phases across units (per query tile, a running key-tile count);
// * TMEM is allocated once;
// * the two half-row states of a unit are exchanged through 8 columns of the query tile's
//   TMEM score buffer instead of the query tiles' shared memory, so that shared memory is
//   free as soon as the query rows have been copied into TMEM; the producer loads the next
//   unit's query tiles there once it has issued the current unit's last key tile.
// Warp roles, register split, MMA shapes and the fold are those of the non-persistent
// kernel (SKL_FWD_SPLIT and SKL_FWD_QTMEM are required).
#pragma once

#include "fwd_kernel.cuh"

namespace skl {

static_assert(SKL_FWD_SPLIT && SKL_FWD_QTMEM, "the persistent forward assumes the split warps "
                                             "and the query tiles in TMEM");

// Unit of the k-th round of CTA c (grid of G CTAs): snake order over rounds.
__device__ __forceinline__ int persist_unit(int k, int c, int G) {
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

// Work unit t (heaviest first over all heads) of a dense problem: head bh, first query row
// q0 of the pair of query tiles, key tiles nk[q] needed by each query tile.
template <int BM, int BN>
__device__ __forceinline__ void persist_decode(const FwdArgs& a, int t, int& bh, int& q0,
                                               int (&nk)[2], SeqView& seq) {
  const int rank = t / a.BH;  // 0 = the heaviest unit of every head
  bh = t - rank * a.BH;
  const int qpair = a.n_ctas_per_bh - 1 - rank;
  seq_view(nullptr, nullptr, bh, a.H, a.gT, a.gS, a.N_Q, a.N_K, 0, 0, a.off_adj, seq);
  q0 = qpair * (2 * BM);
  const int n_ktiles_all = (seq.nk + BN - 1) / BN;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int first = q0 + q * BM;
    if (first >= seq.nq) {
      nk[q] = 0;
    } else if (!a.causal) {
      nk[q] = n_ktiles_all;
    } else {
      const int last_row = min(first + BM, seq.nq) - 1;
      const int last_key = last_row + seq.off;
      nk[q] = last_key < 0 ? 0 : min(n_ktiles_all, last_key / BN + 1);
    }
  }
}

template <int DT, int DS>
__global__ void __launch_bounds__(kFwdThreads, 1)
streamkl_fwd_persistent_kernel(const __grid_constant__ CUtensorMap map_qt,
                               const __grid_constant__ CUtensorMap map_kt,
                               const __grid_constant__ CUtensorMap map_qs,
                               const __grid_constant__ CUtensorMap map_ks,
                               const FwdArgs args, const uint32_t idesc_t,
                               const uint32_t idesc_s) {
  using C = FwdCfg<DT, DS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t s_base = smem_u32(smem);
  if (s_base & 1023u) {  // the swizzled tiles need 1024-byte alignment; never expected to fire
    if (threadIdx.x == 0) atomicOr(&g_skl_error, 4u);
    return;
  }
  const uint32_t s_qt = s_base;                       // [NQ][DT/64][128][64]
  const uint32_t s_qs = s_base + C::NQ * C::QT_TILE;  // [NQ][DS/64][128][64]
  const uint32_t s_k = s_base + C::QBYTES;            // [NST]{K_T, K_S}
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::QBYTES + C::NST * C::STAGE);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int T = args.BH * args.n_ctas_per_bh;  // work units

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int q = 0; q < 2; ++q)
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&bars->s_full[q][b]), 1);
        mbar_init(smem_u32(&bars->s_free[q][b]), 4 * kFwdHalves);
      }
    mbar_init(smem_u32(&bars->q_tmem), kFwdStatWarps);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kFwdMmaWarp) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < kFwdStatWarps) {
    regs_inc<kFwdRegsStat>();
    // --------------------------------------------------- statistics warpgroups
    const int q = warp / (4 * kFwdHalves);   // query tile of this warp
    const int half = (warp >> 2) & 1;        // key half of every tile
    const int quarter = warp & 3;            // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;       // row within the query tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float cT = args.cT, cS = args.cS;
    uint32_t J = 0;  // key tiles of this query tile folded so far (all units): barrier phases
    bool ok = true;
    // Every warp of a query tile passes the tile's named barrier exactly once per unit, and
    // all of them leave the loop together (the barrier returns one decision to all), so no
    // warp can be left waiting at it.
    for (int k = 0;; ++k) {
      const int t = persist_unit(k, cta, G);
      if (t >= T) break;
      int bh, q0, nk[2];
      SeqView seq;
      persist_decode<C::BM, C::BN>(args, t, bh, q0, nk, seq);
      const int row = q0 + q * C::BM + r;
      const int first_row = q0 + q * C::BM;
      // This unit's query rows into TMEM: half 0 the row of Q_T, half 1 the row of Q_S. The
      // previous unit's MMAs on this query tile have completed (this warp waited for their
      // last score tile).
      if (ok && mbar_wait(smem_u32(&bars->q_full), k & 1)) {
        if (half == 0)
          row_to_tmem<DT>(s_qt + q * C::QT_TILE + r * 128, tmem + lane_off + C::tm_qt(q), r);
        else
          row_to_tmem<DS>(s_qs + q * C::QS_TILE + r * 128, tmem + lane_off + C::tm_qs(q), r);
      } else if (ok) {
        skl_fail(abort_flag);
        ok = false;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->q_tmem));

      RowState st{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
      for (int j = 0; ok && j < nk[q]; ++j, ++J) {
        const int b = J & 1;
        if (!mbar_wait(smem_u32(&bars->s_full[q][b]), (J >> 1) & 1)) {
          skl_fail(abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        const int k0 = j * C::BN;
        const bool need_mask =
            (k0 + C::BN > seq.nk) || (args.causal && k0 + C::BN - 1 > first_row + seq.off);
        const uint32_t ta = tmem + lane_off + C::tm_s(q, b);
        const uint32_t fr = smem_u32(&bars->s_free[q][b]);
        if (need_mask) {
          int last = seq.nk - 1;
          if (args.causal) last = min(last, row + seq.off);
          fold_half<true>(st, ta + 32 * half, ta + 64 + 32 * half, cT, cS,
                          last - k0 - 32 * half, fr, lane);
        } else {
          fold_half<false>(st, ta + 32 * half, ta + 64 + 32 * half, cT, cS, 31, fr, lane);
        }
      }

      // Half 1 hands its row state to half 0 through 8 columns of this query tile's score
      // buffer: the first 8 of its own teacher columns (32 .. 39), which it has already read
      // and half 0 never reads (half 0 may still be loading its columns of the last tile
      // when half 1 gets here). No MMA writes that buffer between this unit's last score
      // MMA on the tile (completed: its scores were read) and the next unit's first, which
      // the MMA thread issues only after every statistics warp has copied the next unit's
      // query rows, i.e. after half 0 has read the state below.
      const uint32_t tx = tmem + lane_off + C::tm_s(q, 0) + 32;
      if (half == 1) {
        const uint32_t xs[8] = {__float_as_uint(st.mT), __float_as_uint(st.mS),
                                __float_as_uint(st.lT), __float_as_uint(st.lS),
                                __float_as_uint(st.A),  ok ? 1u : 0u, 0u, 0u};
        tmem_st_8(tx, xs);
        tmem_st_wait();
      }
      tc_fence_before();
      const bool stop = named_bar_any(1 + q, 8 * 32, !ok || *abort_flag != 0);
      tc_fence_after();
      if (half == 0) {
        uint32_t xv[8];
        tmem_ld_8_wait(tx, xv);
        const RowState other{__uint_as_float(xv[0]), __uint_as_float(xv[1]),
                             __uint_as_float(xv[2]), __uint_as_float(xv[3]),
                             __uint_as_float(xv[4])};
        merge_state(st, other);
        if (ok && xv[5] != 0u && row < seq.nq) {
          const size_t o = (size_t)(seq.ob + row);
          if (args.state) {
            float* p = args.state + o;
            p[0] = st.mT;
            p[args.plane] = st.mS;
            p[2 * args.plane] = st.lT;
            p[3 * args.plane] = st.lS;
            p[4 * args.plane] = st.A;
          } else {
            float kl, lse_t, lse_s;
            finalize_row(st.mT, st.mS, st.lT, st.lS, st.A, kl, lse_t, lse_s);
            args.kl[o] = kl;
            args.lse_t[o] = lse_t;
            args.lse_s[o] = lse_s;
          }
        }
      }
      if (stop) break;
    }
  } else {
    regs_dec<kFwdRegsCtrl>();
    if (warp == kFwdTmaWarp) {
      // ------------------------------------------------------------ TMA producer
      if (elect_one()) {
        tma_prefetch_desc(&map_qt);
        tma_prefetch_desc(&map_kt);
        tma_prefetch_desc(&map_qs);
        tma_prefetch_desc(&map_ks);
        const uint64_t keep = l2_policy_evict_last();
        const uint64_t once = l2_policy_evict_first();
        const uint32_t qb = smem_u32(&bars->q_full);
        auto load_q = [&](int t) {
          int bh, q0, nk[2];
          SeqView seq;
          persist_decode<C::BM, C::BN>(args, t, bh, q0, nk, seq);
          mbar_arrive_expect_tx(qb, C::QBYTES);
          for (int q = 0; q < C::NQ; ++q) {
            for (int blk = 0; blk < DT / 64; ++blk)
              tma_load_3d(s_qt + q * C::QT_TILE + blk * (C::BM * 128), &map_qt, qb, blk * 64,
                          seq.qr + q0 + q * C::BM, seq.zq, once);
            for (int blk = 0; blk < DS / 64; ++blk)
              tma_load_3d(s_qs + q * C::QS_TILE + blk * (C::BM * 128), &map_qs, qb, blk * 64,
                          seq.qr + q0 + q * C::BM, seq.zq, once);
          }
        };
        int q_loads = 0;   // query-tile loads issued (one per unit)
        uint32_t kt = 0;   // key tiles issued (all units): ring stage and phase
        bool ok = true;
        if (persist_unit(0, cta, G) < T) {
          load_q(persist_unit(0, cta, G));
          q_loads = 1;
        }
        for (int k = 0; ok; ++k) {
          const int t = persist_unit(k, cta, G);
          if (t >= T || *abort_flag) break;
          int bh, q0, nk[2];
          SeqView seq;
          persist_decode<C::BM, C::BN>(args, t, bh, q0, nk, seq);
          const int nk_max = max(nk[0], nk[1]);
          for (int j = 0; j < nk_max; ++j, ++kt) {
            const int s = kt % C::NST;
            if (!mbar_wait(smem_u32(&bars->empty[s]), ((kt / C::NST) & 1) ^ 1)) {
              skl_fail(abort_flag);
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&bars->full[s]);
            mbar_arrive_expect_tx(fb, C::STAGE);
            const uint32_t stg = s_k + s * C::STAGE;
            for (int blk = 0; blk < DT / 64; ++blk)
              tma_load_3d(stg + blk * (C::BN * 128), &map_kt, fb, blk * 64, seq.kr + j * C::BN,
                          seq.zkt, keep);
            for (int blk = 0; blk < DS / 64; ++blk)
              tma_load_3d(stg + C::KT_TILE + blk * (C::BN * 128), &map_ks, fb, blk * 64,
                          seq.kr + j * C::BN, seq.zks, keep);
          }
          if (!ok) break;
          // The next unit's query tiles, once every statistics warp has copied this unit's
          // rows into TMEM (the tiles' shared memory is then no longer read).
          const int tn = persist_unit(k + 1, cta, G);
          if (tn < T) {
            if (!mbar_wait(smem_u32(&bars->q_tmem), k & 1)) {
              skl_fail(abort_flag);
              break;
            }
            load_q(tn);
            ++q_loads;
          }
        }
        if (*abort_flag) {
          // Let every copy this thread started land before the CTA can exit.
          if (q_loads > 0) mbar_wait(qb, (q_loads - 1) & 1);
          const uint32_t first = kt > (uint32_t)C::NST ? kt - C::NST : 0u;
          for (uint32_t i = first; i < kt; ++i)
            mbar_wait(smem_u32(&bars->full[i % C::NST]), (i / C::NST) & 1);
        }
      }
    } else if (warp == kFwdMmaWarp) {
      // ------------------------------------------------------------- MMA issuer
      if (elect_one()) {
        uint32_t kt = 0;            // key tiles consumed (all units)
        uint32_t J[2] = {0u, 0u};   // score tiles issued per query tile (all units)
        bool ok = true;
        for (int k = 0; ok; ++k) {
          const int t = persist_unit(k, cta, G);
          if (t >= T || *abort_flag) break;
          int bh, q0, nk[2];
          SeqView seq;
          persist_decode<C::BM, C::BN>(args, t, bh, q0, nk, seq);
          const int nk_max = max(nk[0], nk[1]);
          if (!mbar_wait(smem_u32(&bars->q_tmem), k & 1)) {
            skl_fail(abort_flag);
            break;
          }
          for (int j = 0; ok && j < nk_max; ++j, ++kt) {
            const int s = kt % C::NST;
            if (!mbar_wait(smem_u32(&bars->full[s]), (kt / C::NST) & 1)) {
              skl_fail(abort_flag);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t stg = s_k + s * C::STAGE;
#pragma unroll
            for (int q = 0; q < C::NQ; ++q) {
              if (j >= nk[q]) continue;
              const uint32_t Jq = J[q];
              // Single score buffer per query tile: free once the previous score tile of
              // this query tile (possibly of the previous unit) has been read.
              if (Jq > 0 && !mbar_wait(smem_u32(&bars->s_free[q][(Jq - 1) & 1]),
                                       ((Jq - 1) >> 1) & 1)) {
                skl_fail(abort_flag);
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t d_t = tmem + C::tm_s(q, Jq & 1);
              const uint32_t d_s = d_t + 64;
#pragma unroll
              for (int kk = 0; kk < DT / 16; ++kk) {
                const uint64_t bd =
                    sdesc_sw128(stg + (kk >> 2) * (C::BN * 128) + (kk & 3) * 32, 16, 1024);
                umma_bf16_ts(d_t, tmem + C::tm_qt(q) + kk * 8, bd, idesc_t, kk > 0);
              }
#pragma unroll
              for (int kk = 0; kk < DS / 16; ++kk) {
                const uint64_t bd = sdesc_sw128(
                    stg + C::KT_TILE + (kk >> 2) * (C::BN * 128) + (kk & 3) * 32, 16, 1024);
                umma_bf16_ts(d_s, tmem + C::tm_qs(q) + kk * 8, bd, idesc_s, kk > 0);
              }
              umma_commit(smem_u32(&bars->s_full[q][Jq & 1]));
              J[q] = Jq + 1;
            }
            umma_commit(smem_u32(&bars->empty[s]));
          }
        }
        // Every MMA this thread issued must be complete before TMEM is released.
        umma_commit(smem_u32(&bars->drain));
        if (!mbar_wait(smem_u32(&bars->drain), 0)) skl_fail(abort_flag);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kFwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace skl
