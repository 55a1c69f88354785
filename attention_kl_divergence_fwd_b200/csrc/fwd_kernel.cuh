// fwd_kernel.cuh - StreamKL forward on sm_100a (tcgen05 + TMEM + TMA).
//
// The one-pass forward of "StreamKL: Fast and Memory-Efficient KL Divergence for
// Boosting Attention Distillation" (abstract: an online formulation of the coupled
// two-distribution KL reduction, streaming query-key tiles through on-chip memory).
//
// CTA = two 128-row query tiles of one (batch, head). Key tiles of 64 rows stream
// through a TMA ring. Per key tile and query tile the tensor core computes the teacher
// and student score tiles into TMEM (two buffers per query tile, so the next tile is
// computed while the current one is folded). One warpgroup per query tile, one thread
// per query row, folds each tile into the row's online state
//     m_T, m_S   running maxima of t = s * log2(e)
//     l_T, l_S   running sums of 2^(t - m)
//     A          running sum of 2^(t_T - m_T) * (t_T - t_S)
// so that KL = ln2 * A / l_T - LSE_T + LSE_S at the end. Per tile: one pass over TMEM
// for the row maxima, a second pass (two 32-key halves) for the exponentials, with the
// fp32 work issued as packed pairs and a share of the exponentials on the FMA pipe.
// Nothing of size N_Q x N_K ever leaves the SM.
//
// Warp roles (384 threads): warps 0-3 query tile 0, warps 4-7 query tile 1 (224 registers
// each), warp 8 TMA producer, warp 9 TMEM allocator + MMA issuer, warps 10-11 idle (the
// control warpgroup runs with 56 registers).
#pragma once

#include "ptx.cuh"

namespace skl {

struct FwdArgs {
  int BH, N_Q, N_K;   // B*H; queries / keys per sequence (packed: the longest sequence)
  int causal;
  float cT, cS;       // |scale| * log2(e); the MMA negates A when the scale is negative
  int n_ctas_per_bh;  // ceil(N_Q / 256)
  int group;          // heads per scheduling group (grouped_order)
  int H;              // query heads per batch entry
  int gT, gS;         // query heads per teacher / student K head (GQA; 1 = one K head each)
  const int* cu_q;    // packed layout: [B+1] sequence offsets (null: dense [B, H, N, d])
  const int* cu_k;
  int total_q, total_k;  // packed layout: rows of the packed Q / K tensors
  int off_adj;           // causal shift of a key shard (context parallelism), else 0
  float* state;          // non-null: write the raw row state (5 planes of plane floats)
  long long plane;       //   instead of KL / LSE (context parallelism)
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
  static constexpr int THREADS = 384;
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

// Which column pairs (c, c+1) of a 32-key chunk send their second exponential of both
// distributions to the FMA pipe: pairs 1, 3, 5, 7 of every 8 (25 % of the exponentials),
// plus pair 6 when kPolyHeavy (37.5 %).
constexpr bool kPolyHeavy = true;
__host__ __device__ constexpr bool poly_pair(int pair) {
  return (pair & 1) || (kPolyHeavy && (pair & 7) == 6);
}

// New running maxima from a tile's raw maxima; rescales the sums when any row of the
// warp raised its maximum. Returns the reference maxima (0 while still -inf).
__device__ __forceinline__ void update_max(RowState& st, float mxT, float mxS, float cT, float cS,
                                           float& mT_use, float& mS_use) {
  const float mT_new = fmaxf(st.mT, cT * mxT);  // NaN (cT=0, all masked) keeps the old max
  const float mS_new = fmaxf(st.mS, cS * mxS);
  mT_use = (mT_new == -INFINITY) ? 0.f : mT_new;
  mS_use = (mS_new == -INFINITY) ? 0.f : mS_new;
  if (__any_sync(0xffffffffu, (mT_new > st.mT) || (mS_new > st.mS))) {
    const float aT = ex2_approx(st.mT - mT_use);  // -inf - x -> 0
    const float aS = ex2_approx(st.mS - mS_use);
    st.lT *= aT;
    st.A *= aT;
    st.lS *= aS;
  }
  st.mT = mT_new;
  st.mS = mS_new;
}

// Accumulates 16 keys (v[0..15] teacher scores, v[16..31] student scores, raw dot
// products) into the packed partial sums. Columns c > lim are masked (MASK).
template <bool MASK>
__device__ __forceinline__ void fold_part(const uint32_t (&v)[32], uint64_t cT2, uint64_t cS2,
                                          uint64_t nmT2, uint64_t nmS2, int lim, int pair0,
                                          uint64_t& sT2, uint64_t& sS2, uint64_t& b2) {
#pragma unroll
  for (int c = 0; c < 16; c += 2) {
    const uint64_t xT = f2_fma(f2_pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), cT2, nmT2);
    const uint64_t xS =
        f2_fma(f2_pack(__uint_as_float(v[16 + c]), __uint_as_float(v[16 + c + 1])), cS2, nmS2);
    float xT0, xT1, xS0, xS1;
    f2_unpack(xT, xT0, xT1);
    f2_unpack(xS, xS0, xS1);
    float eT0 = ex2_approx(xT0), eS0 = ex2_approx(xS0), eT1, eS1;
    if (poly_pair(pair0 + (c >> 1))) {
      f2_unpack(exp2_fma2(f2_pack(xT1, xS1)), eT1, eS1);
    } else {
      eT1 = ex2_approx(xT1);
      eS1 = ex2_approx(xS1);
    }
    uint64_t d = f2_sub(xT, xS);
    if (MASK) {
      const bool k0 = c <= lim, k1 = c + 1 <= lim;
      eT0 = k0 ? eT0 : 0.f;
      eS0 = k0 ? eS0 : 0.f;
      eT1 = k1 ? eT1 : 0.f;
      eS1 = k1 ? eS1 : 0.f;
      float d0, d1;
      f2_unpack(d, d0, d1);
      d = f2_pack(k0 ? d0 : 0.f, k1 ? d1 : 0.f);
    }
    const uint64_t eT = f2_pack(eT0, eT1);
    sT2 = f2_add(sT2, eT);
    sS2 = f2_add(sS2, f2_pack(eS0, eS1));
    b2 = f2_fma(eT, d, b2);
  }
}

// Folds one 64-key tile (TMEM columns: ta .. ta+63 teacher, ta+64 .. ta+127 student)
// into the row state; releases the TMEM buffer (s_free) once it has been read.
template <bool MASK>
__device__ __forceinline__ void fold_tile(RowState& st, uint32_t ta, float cT, float cS, int lim,
                                          uint32_t s_free, int lane) {
  float mxT, mxS;
  {
    uint32_t v[64];
    tmem_ld_2x32_wait(ta, ta + 32, v);
    mxT = fmaxf(max_tree32<MASK>(v, 0, lim), max_tree32<MASK>(v, 32, lim - 32));
    tmem_ld_2x32_wait(ta + 64, ta + 96, v);
    mxS = fmaxf(max_tree32<MASK>(v, 0, lim), max_tree32<MASK>(v, 32, lim - 32));
  }
  float mT_use, mS_use;
  update_max(st, mxT, mxS, cT, cS, mT_use, mS_use);
  const uint64_t cT2 = f2_pack(cT, cT), cS2 = f2_pack(cS, cS);
  const uint64_t nmT2 = f2_pack(-mT_use, -mT_use), nmS2 = f2_pack(-mS_use, -mS_use);
  uint64_t sT2 = f2_pack(0.f, 0.f), sS2 = sT2, b2 = sT2;
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    uint32_t v[32];  // keys 16h .. 16h+15: v[0..15] teacher, v[16..31] student
    tmem_ld_2x16_wait(ta + 16 * h, ta + 64 + 16 * h, v);
    if (h == 3) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
    }
    fold_part<MASK>(v, cT2, cS2, nmT2, nmS2, lim - 16 * h, 8 * h, sT2, sS2, b2);
  }
  float s0, s1, u0, u1, w0, w1;
  f2_unpack(sT2, s0, s1);
  f2_unpack(sS2, u0, u1);
  f2_unpack(b2, w0, w1);
  const float sumT = s0 + s1;
  st.lT += sumT;
  st.lS += u0 + u1;
  st.A += (w0 + w1) + (mT_use - mS_use) * sumT;
}

template <int DT, int DS>
__global__ void __launch_bounds__(384, 1)
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

  // Heaviest (last) query tiles first for causal load balance, heads in groups.
  int bh, unit;
  grouped_order(blockIdx.x, args.BH, args.n_ctas_per_bh, args.group, bh, unit);
  const int qpair = args.n_ctas_per_bh - 1 - unit;
  SeqView seq;
  if (!seq_view(args.cu_q, args.cu_k, bh, args.H, args.gT, args.gS, args.N_Q, args.N_K,
                args.total_q, args.total_k, args.off_adj, seq)) {
    if (threadIdx.x == 0) atomicOr(&g_skl_error, kErrBadOffsets);
    return;
  }
  const int q0 = qpair * (C::NQ * C::BM);
  if (q0 >= seq.nq) return;  // packed layout: this sequence is shorter than the longest
  const int n_ktiles_all = (seq.nk + C::BN - 1) / C::BN;

  // Key tiles needed by each query tile.
  int nk[C::NQ];
#pragma unroll
  for (int q = 0; q < C::NQ; ++q) {
    const int first = q0 + q * C::BM;
    if (first >= seq.nq) {
      nk[q] = 0;
    } else if (!args.causal) {
      nk[q] = n_ktiles_all;
    } else {
      const int last_row = min(first + C::BM, seq.nq) - 1;
      const int last_key = last_row + seq.off;
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

  if (warp < 8) {
    regs_inc<200>();
    // --------------------------------------------------- statistics warpgroups
    const int q = warp >> 2;          // query tile of this warpgroup
    const int quarter = warp & 3;     // TMEM lane quarter of this warp
    const int row = q0 + q * C::BM + quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float cT = args.cT, cS = args.cS;
    const int first_row = q0 + q * C::BM;

    RowState st{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
    bool ok = true;
    for (int j = 0; j < nk[q]; ++j) {
      const int b = j & 1;
      if (!mbar_wait(smem_u32(&bars->s_full[q][b]), (j >> 1) & 1)) {
        skl_fail(abort_flag);
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = j * C::BN;
      const bool need_mask =
          (k0 + C::BN > seq.nk) || (args.causal && k0 + C::BN - 1 > first_row + seq.off);
      const uint32_t ta = tmem + lane_off + q * 256 + b * 128;
      const uint32_t fr = smem_u32(&bars->s_free[q][b]);
      if (need_mask) {
        int last = seq.nk - 1;
        if (args.causal) last = min(last, row + seq.off);
        fold_tile<true>(st, ta, cT, cS, last - k0, fr, lane);
      } else {
        fold_tile<false>(st, ta, cT, cS, C::BN - 1, fr, lane);
      }
    }

    if (ok && row < seq.nq) {
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
  } else {
    regs_dec<104>();
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
                        seq.qr + q0 + q * C::BM, seq.zq, once);
          for (int blk = 0; blk < DS / 64; ++blk)
            tma_load_3d(s_qs + q * C::QS_TILE + blk * (C::BM * 128), &map_qs, qb, blk * 64,
                        seq.qr + q0 + q * C::BM, seq.zq, once);
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
            tma_load_3d(st + blk * (C::BN * 128), &map_kt, fb, blk * 64, seq.kr + j * C::BN,
                        seq.zkt, keep);
          for (int blk = 0; blk < DS / 64; ++blk)
            tma_load_3d(st + C::KT_TILE + blk * (C::BN * 128), &map_ks, fb, blk * 64,
                        seq.kr + j * C::BN, seq.zks, keep);
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
