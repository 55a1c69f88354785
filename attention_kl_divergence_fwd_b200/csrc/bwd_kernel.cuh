// bwd_kernel.cuh - StreamKL backward on sm_100a (tcgen05 + TMEM + TMA).
//
// The recompute backward of "StreamKL: Fast and Memory-Efficient KL Divergence for
// Boosting Attention Distillation" (abstract: the backward recomputes attention
// probabilities tile by tile instead of storing quadratic intermediates).
//
// With the teacher frozen and g[i] = dLoss/dKL[i]:
//     dS[i,j] = g[i] * scale_S * (P_S[i,j] - P_T[i,j]),   P_X = 2^(t_X - LSE_X*log2 e)
//     dQ_S = dS K_S,   dK_S = dS^T Q_S.
//
// CTA = one tile of 128 keys of one (batch, head), resident in shared memory. It
// walks the 128-row query tiles that can see those keys. Per query tile:
//   1. tensor core: S_T^T = K_T Q_T^T and S_S^T = K_S Q_S^T into TMEM (keys on lanes);
//   2. two warpgroups (one thread per key, 64 query columns each) recompute P_T, P_S,
//      form dS^T in registers and store it to shared memory as bf16;
//   3. tensor core: dK_S += dS^T Q_S (TMEM accumulator over all query tiles) and
//      dQ_part = dS K_S (TMEM);
//   4. the same warpgroups add dQ_part into dq_s with fp32 vector reductions.
// The score tiles of step s+1 are computed while the warpgroups work on step s.
//
// Warp roles (320 threads): warps 0-3 and 4-7 statistics/dS (query columns 0-63 and
// 64-127), warp 8 TMA producer + row-statistics loader, warp 9 TMEM allocator + MMA.
#pragma once

#include "ptx.cuh"

namespace skl {

struct BwdArgs {
  int BH, N_Q, N_K;
  int causal;
  int off;          // N_K - N_Q
  float cT, cS;     // |scale| * log2(e)
  float scale_S;    // signed student scale (folded into G = g * scale_S)
  int n_ktiles;     // ceil(N_K / 128)
  int n_qtiles;     // ceil(N_Q / 128)
  const float* lse_t;
  const float* lse_s;
  const float* g;
  float* dq_s;
  float* dk_s;
};

template <int DT, int DS>
struct BwdCfg {
  static constexpr int BN = 128;  // keys per CTA (TMEM lanes)
  static constexpr int BM = 128;  // queries per step
  static constexpr int KT_TILE = BN * DT * 2;
  static constexpr int KS_TILE = BN * DS * 2;
  static constexpr int QT_TILE = BM * DT * 2;
  static constexpr int QS_TILE = BM * DS * 2;
  static constexpr int DS_TILE = BN * BM * 2;
  static constexpr int STATS = 3 * BM * 4;  // -LSE_T*log2e, -LSE_S*log2e, g*scale_S
  static constexpr int OFF_KT = 0;
  static constexpr int OFF_KS = OFF_KT + KT_TILE;
  static constexpr int OFF_QT = OFF_KS + KS_TILE;
  static constexpr int OFF_QS = OFF_QT + QT_TILE;        // two slots
  static constexpr int OFF_DS = OFF_QS + 2 * QS_TILE;
  static constexpr int OFF_ST = OFF_DS + DS_TILE;         // two slots
  static constexpr int OFF_BAR = OFF_ST + 2 * STATS;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = 1024 + OFF_BAR + BAR_BYTES;
  static constexpr int THREADS = 320;
  // TMEM columns
  static constexpr int TM_ST = 0, TM_SS = 128, TM_DK = 256, TM_DQ = 384;
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct BwdBars {
  uint64_t k_full;
  uint64_t qt_full, qt_empty;
  uint64_t qs_full[2], qs_empty[2];
  uint64_t st_full[2], st_empty[2];
  uint64_t s_full, s_free;
  uint64_t ds_full, ds_empty;
  uint64_t dq_full, dq_free;
  uint64_t dk_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void skl_fail_b(volatile int* abort_flag) {
  atomicOr(&g_skl_error, 2u);
  *abort_flag = 1;
}

template <int DT, int DS>
__global__ void __launch_bounds__(320, 1)
streamkl_bwd_kernel(const __grid_constant__ CUtensorMap map_qt,
                    const __grid_constant__ CUtensorMap map_kt,
                    const __grid_constant__ CUtensorMap map_qs,
                    const __grid_constant__ CUtensorMap map_ks, const BwdArgs args,
                    const uint32_t idesc_st, const uint32_t idesc_ss, const uint32_t idesc_dk,
                    const uint32_t idesc_dq) {
  using C = BwdCfg<DT, DS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::OFF_BAR);
  float* stats = reinterpret_cast<float*>(smem + C::OFF_ST);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int bh = t % args.BH;
  const int kt = t / args.BH;  // causal: key tile 0 sees the most query tiles
  const int k0 = kt * C::BN;

  int jq_begin = 0;
  if (args.causal) {
    const int first_q = k0 - args.off;  // first query row that sees key k0
    jq_begin = first_q <= 0 ? 0 : first_q / C::BM;
  }
  const int n_steps = max(0, args.n_qtiles - jq_begin);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->k_full), 1);
    mbar_init(smem_u32(&bars->qt_full), 1);
    mbar_init(smem_u32(&bars->qt_empty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->qs_full[i]), 1);
      mbar_init(smem_u32(&bars->qs_empty[i]), 1);
      mbar_init(smem_u32(&bars->st_full[i]), 32);
      mbar_init(smem_u32(&bars->st_empty[i]), 8);
    }
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->s_free), 8);
    mbar_init(smem_u32(&bars->ds_full), 8);
    mbar_init(smem_u32(&bars->ds_empty), 1);
    mbar_init(smem_u32(&bars->dq_full), 1);
    mbar_init(smem_u32(&bars->dq_free), 8);
    mbar_init(smem_u32(&bars->dk_full), 1);
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
    // --------------------------------------- TMA producer + row-statistics loader
    const uint64_t keep = l2_policy_evict_last();
    int qt_issued = 0, qs_issued = 0;
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&map_qt);
      tma_prefetch_desc(&map_kt);
      tma_prefetch_desc(&map_qs);
      tma_prefetch_desc(&map_ks);
      const uint32_t kb = smem_u32(&bars->k_full);
      mbar_arrive_expect_tx(kb, C::KT_TILE + C::KS_TILE);
      for (int blk = 0; blk < DT / 64; ++blk)
        tma_load_3d(sb + C::OFF_KT + blk * (C::BN * 128), &map_kt, kb, blk * 64, k0, bh, keep);
      for (int blk = 0; blk < DS / 64; ++blk)
        tma_load_3d(sb + C::OFF_KS + blk * (C::BN * 128), &map_ks, kb, blk * 64, k0, bh, keep);
    }
    const float LOG2E = 1.4426950408889634f;
    for (int s = 0; s < n_steps && ok; ++s) {
      const int i0 = (jq_begin + s) * C::BM;
      // Lane 0 does every wait of this warp and issues the copies; the verdict is
      // then shared so the whole warp leaves the loop together.
      if (lane == 0) {
        if (!mbar_wait(smem_u32(&bars->qt_empty), (s & 1) ^ 1)) {
          ok = false;
        } else {
          const uint32_t fb = smem_u32(&bars->qt_full);
          mbar_arrive_expect_tx(fb, C::QT_TILE);
          for (int blk = 0; blk < DT / 64; ++blk)
            tma_load_3d(sb + C::OFF_QT + blk * (C::BM * 128), &map_qt, fb, blk * 64, i0, bh, keep);
          qt_issued = s + 1;
        }
        if (ok && !mbar_wait(smem_u32(&bars->qs_empty[s & 1]), ((s >> 1) & 1) ^ 1)) {
          ok = false;
        } else if (ok) {
          const uint32_t fb = smem_u32(&bars->qs_full[s & 1]);
          mbar_arrive_expect_tx(fb, C::QS_TILE);
          for (int blk = 0; blk < DS / 64; ++blk)
            tma_load_3d(sb + C::OFF_QS + (s & 1) * C::QS_TILE + blk * (C::BM * 128), &map_qs, fb,
                        blk * 64, i0, bh, keep);
          qs_issued = s + 1;
        }
        if (ok && !mbar_wait(smem_u32(&bars->st_empty[s & 1]), ((s >> 1) & 1) ^ 1)) ok = false;
        if (!ok) skl_fail_b(abort_flag);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      // Row statistics of this query tile: -LSE_T*log2e, -LSE_S*log2e, g*scale_S.
      float* st = stats + (s & 1) * (3 * C::BM);
#pragma unroll
      for (int r = 0; r < C::BM / 32; ++r) {
        const int qi = r * 32 + lane;
        const int row = i0 + qi;
        float nlt = -INFINITY, nls = -INFINITY, gs = 0.f;
        if (row < args.N_Q) {
          const size_t o = (size_t)bh * args.N_Q + row;
          const float lt = args.lse_t[o];
          const float ls = args.lse_s[o];
          if (lt != -INFINITY && ls != -INFINITY) {
            nlt = -lt * LOG2E;
            nls = -ls * LOG2E;
            gs = args.g[o] * args.scale_S;
          }
        }
        st[qi] = nlt;
        st[C::BM + qi] = nls;
        st[2 * C::BM + qi] = gs;
      }
      mbar_arrive(smem_u32(&bars->st_full[s & 1]));
    }
    if (lane == 0 && *abort_flag) {
      mbar_wait(smem_u32(&bars->k_full), 0);
      if (qt_issued > 0) mbar_wait(smem_u32(&bars->qt_full), (qt_issued - 1) & 1);
      for (int s = max(0, qs_issued - 2); s < qs_issued; ++s)
        mbar_wait(smem_u32(&bars->qs_full[s & 1]), (s >> 1) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      const uint32_t t_st = tmem + C::TM_ST, t_ss = tmem + C::TM_SS;
      const uint32_t t_dk = tmem + C::TM_DK, t_dq = tmem + C::TM_DQ;
      const uint32_t s_kt = sb + C::OFF_KT, s_ks = sb + C::OFF_KS, s_qt = sb + C::OFF_QT;
      const uint32_t s_ds = sb + C::OFF_DS;
      bool ok = mbar_wait(smem_u32(&bars->k_full), 0);
      // Score tiles of step s: S_T^T = K_T Q_T^T, S_S^T = K_S Q_S^T (keys on lanes).
      auto issue_scores = [&](int s) -> bool {
        if (!mbar_wait(smem_u32(&bars->qt_full), s & 1)) return false;
        if (!mbar_wait(smem_u32(&bars->qs_full[s & 1]), (s >> 1) & 1)) return false;
        if (!mbar_wait(smem_u32(&bars->s_free), (s & 1) ^ 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DT / 16; ++kk) {
          const uint32_t o = (kk >> 2) * (C::BN * 128) + (kk & 3) * 32;
          umma_bf16_ss(t_st, sdesc_sw128(s_kt + o, 16, 1024), sdesc_sw128(s_qt + o, 16, 1024),
                       idesc_st, kk > 0);
        }
        umma_commit(smem_u32(&bars->qt_empty));
        const uint32_t s_qs = sb + C::OFF_QS + (s & 1) * C::QS_TILE;
#pragma unroll
        for (int kk = 0; kk < DS / 16; ++kk) {
          const uint32_t o = (kk >> 2) * (C::BN * 128) + (kk & 3) * 32;
          umma_bf16_ss(t_ss, sdesc_sw128(s_ks + o, 16, 1024), sdesc_sw128(s_qs + o, 16, 1024),
                       idesc_ss, kk > 0);
        }
        umma_commit(smem_u32(&bars->s_full));
        return true;
      };
      if (ok && n_steps > 0) ok = issue_scores(0);
      for (int s = 0; ok && s < n_steps; ++s) {
        if (s + 1 < n_steps && !issue_scores(s + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait(smem_u32(&bars->ds_full), s & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t s_qs = sb + C::OFF_QS + (s & 1) * C::QS_TILE;
        // dK_S += dS^T Q_S : A = dS^T (keys x queries, K-major), B = Q_S (d x queries, MN-major)
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk) {
          const uint64_t a = sdesc_sw128(s_ds + (kk >> 2) * (C::BN * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(s_qs + kk * 2048, C::BM * 128, 1024);
          umma_bf16_ss(t_dk, a, b, idesc_dk, (s > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&bars->qs_empty[s & 1]));
        if (!mbar_wait(smem_u32(&bars->dq_free), (s & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // dQ_part = dS K_S : A = dS (queries x keys, MN-major), B = K_S (d x keys, MN-major)
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t a = sdesc_sw128(s_ds + kk * 2048, C::BN * 128, 1024);
          const uint64_t b = sdesc_sw128(s_ks + kk * 2048, C::BN * 128, 1024);
          umma_bf16_ss(t_dq, a, b, idesc_dq, kk > 0 ? 1u : 0u);
        }
        umma_commit(smem_u32(&bars->ds_empty));
        umma_commit(smem_u32(&bars->dq_full));
      }
      if (!ok) skl_fail_b(abort_flag);
      umma_commit(smem_u32(&bars->dk_full));
      umma_commit(smem_u32(&bars->drain));
      if (!mbar_wait(smem_u32(&bars->drain), 0)) skl_fail_b(abort_flag);
    }
  } else {
    // ------------------------------------------------- dS / reduction warpgroups
    const int half = warp >> 2;       // query columns [64*half, 64*half + 64) of each step
    const int quarter = warp & 3;
    const int kl = quarter * 32 + lane;  // key row within the tile = TMEM lane
    const int key = k0 + kl;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float cT = args.cT, cS = args.cS;
    const uint32_t s_ds = sb + C::OFF_DS + half * (C::BN * 128) + (kl >> 3) * 1024 + (kl & 7) * 128;
    constexpr int DQH = DS / 2;  // dQ / dK columns handled by this warpgroup

    auto drain_dq = [&](int s) -> bool {
      if (!mbar_wait(smem_u32(&bars->dq_full), s & 1)) return false;
      tc_fence_after();
      uint32_t v[DQH];
      if constexpr (DQH == 64) {
        tmem_ld_2x32_wait(tmem + lane_off + C::TM_DQ + half * DQH,
                          tmem + lane_off + C::TM_DQ + half * DQH + 32, v);
      } else {
        tmem_ld_32_wait(tmem + lane_off + C::TM_DQ + half * DQH, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->dq_free));
      const int row = (jq_begin + s) * C::BM + kl;  // dQ lanes are query rows
      if (row < args.N_Q) {
        float* dst = args.dq_s + ((size_t)bh * args.N_Q + row) * DS + half * DQH;
#pragma unroll
        for (int c = 0; c < DQH; c += 4)
          red_add_v4(dst + c, __uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                     __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
      }
      return true;
    };

    bool ok = true;
    for (int s = 0; s < n_steps; ++s) {
      const int i0 = (jq_begin + s) * C::BM + half * 64;  // first query column of this thread
      if (!mbar_wait(smem_u32(&bars->s_full), s & 1)) { ok = false; break; }
      tc_fence_after();
      uint32_t vt[64], vs[64];
      tmem_ld_2x32_wait(tmem + lane_off + C::TM_ST + half * 64,
                        tmem + lane_off + C::TM_ST + half * 64 + 32, vt);
      tmem_ld_2x32_wait(tmem + lane_off + C::TM_SS + half * 64,
                        tmem + lane_off + C::TM_SS + half * 64 + 32, vs);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->s_free));

      if (!mbar_wait(smem_u32(&bars->st_full[s & 1]), (s >> 1) & 1)) { ok = false; break; }
      const float* st = stats + (s & 1) * (3 * C::BM) + half * 64;

      // Query column c is allowed for this key iff i0 + c >= key - off.
      const bool need_mask = args.causal && (i0 + args.off < k0 + C::BN - 1);
      const int cmin = need_mask ? (key - args.off - i0) : -1;
      uint32_t packed[32];  // dS^T row of this key, 64 bf16 values
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // 8 query columns = one 16-byte chunk per iteration
        const float4 nlt0 = *reinterpret_cast<const float4*>(st + u * 8);
        const float4 nlt1 = *reinterpret_cast<const float4*>(st + u * 8 + 4);
        const float4 nls0 = *reinterpret_cast<const float4*>(st + C::BM + u * 8);
        const float4 nls1 = *reinterpret_cast<const float4*>(st + C::BM + u * 8 + 4);
        const float4 g0 = *reinterpret_cast<const float4*>(st + 2 * C::BM + u * 8);
        const float4 g1 = *reinterpret_cast<const float4*>(st + 2 * C::BM + u * 8 + 4);
        const float nlt[8] = {nlt0.x, nlt0.y, nlt0.z, nlt0.w, nlt1.x, nlt1.y, nlt1.z, nlt1.w};
        const float nls[8] = {nls0.x, nls0.y, nls0.z, nls0.w, nls1.x, nls1.y, nls1.z, nls1.w};
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        float d[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = u * 8 + e;
          const float pT = ex2_approx(fmaf(__uint_as_float(vt[c]), cT, nlt[e]));
          const float pS = ex2_approx(fmaf(__uint_as_float(vs[c]), cS, nls[e]));
          float ds = gg[e] * (pS - pT);
          if (need_mask && c < cmin) ds = 0.f;
          d[e] = ds;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) packed[u * 4 + e] = pack_bf16x2(d[2 * e], d[2 * e + 1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->st_empty[s & 1]));
      // The dS buffer is free once the previous step's dK/dQ MMAs have read it.
      if (!mbar_wait(smem_u32(&bars->ds_empty), (s & 1) ^ 1)) { ok = false; break; }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        st_shared_v4(s_ds + ((u ^ (kl & 7)) << 4), packed[4 * u], packed[4 * u + 1],
                     packed[4 * u + 2], packed[4 * u + 3]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->ds_full));
      if (s > 0 && !drain_dq(s - 1)) { ok = false; break; }
    }
    if (ok && n_steps > 0 && !drain_dq(n_steps - 1)) ok = false;

    // dK_S rows of this key tile (TMEM lanes = keys); zero when no query sees them.
    if (ok) {
      uint32_t v[DQH];
      if (n_steps > 0) {
        if (!mbar_wait(smem_u32(&bars->dk_full), 0)) {
          ok = false;
        } else {
          tc_fence_after();
          if constexpr (DQH == 64) {
            tmem_ld_2x32_wait(tmem + lane_off + C::TM_DK + half * DQH,
                              tmem + lane_off + C::TM_DK + half * DQH + 32, v);
          } else {
            tmem_ld_32_wait(tmem + lane_off + C::TM_DK + half * DQH, v);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < DQH; ++c) v[c] = 0u;
      }
      if (ok && key < args.N_K) {
        float4* dst = reinterpret_cast<float4*>(args.dk_s + ((size_t)bh * args.N_K + key) * DS +
                                                half * DQH);
#pragma unroll
        for (int c = 0; c < DQH; c += 4)
          dst[c / 4] = make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                   __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
      }
    }
    if (!ok) skl_fail_b(abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace skl
