// bwd_kernel.cuh - StreamKL backward on sm_100a (tcgen05 + TMEM + TMA).
//
// The recompute backward of "StreamKL: Fast and Memory-Efficient KL Divergence for
// Boosting Attention Distillation" (abstract: the backward regenerates the attention
// probabilities one tile at a time and keeps no quadratic intermediate).
//
// With g[i] = dLoss/dKL[i] and P_X = 2^(t_X - LSE_X*log2 e):
//   student (TEACHER = false): dS[i,j] = g[i] * scale_S * (P_S[i,j] - P_T[i,j]),
//                              dQ_S = dS K_S,   dK_S = dS^T Q_S;
//   trainable teacher (TEACHER = true):
//                              dS[i,j] = g[i] * scale_T * P_T[i,j] * ((s_T - s_S)[i,j] - E_i),
//                              E_i = KL_i + LSE_T,i - LSE_S,i,
//                              dQ_T = dS K_T,   dK_T = dS^T Q_T.
// Both recompute both score tiles; the teacher variant needs one exponential per pair.
//
// CTA = one tile of 128 keys of one (batch, head), resident in shared memory (and, by
// default, copied into TMEM). It walks the 64-row query tiles ("steps") that can see those
// keys. Per step s:
//   1. tensor core: S_T^T = K_T Q_T^T and S_S^T = K_S Q_S^T into TMEM (keys on the 128
//      lanes, 64 query columns), K read from TMEM as the A operand;
//   2. the dS warps of step parity s&1 (one thread per key row, each warp 32 of the 64
//      query columns) recompute P_T, P_S, form dS^T in registers and store it as bf16
//      into shared-memory buffer s&1; for the student gradient the teacher score MMAs are
//      committed on their own, so P_T is computed while the student score MMAs still run;
//   3. tensor core: dK += dS^T Q (TMEM accumulator over all steps) and
//      dQ^T_part = K^T dS^T into TMEM buffer s&1 (d on the lanes, queries on columns);
//   4. the same warps copy dQ^T_part from TMEM into the fp32 staging tile of parity s&1,
//      laid out as dQ rows, and one thread adds the tile into dQ with a bulk tensor
//      reduce-add (the fp32 adds happen in L2).
// dS tiles, dQ parts and staging tiles are double-buffered by step parity, so the two
// groups of dS warps work on alternate steps while the tensor core computes the next.
//
// Warp roles (640 threads, the default switches): warps 0-15 dS (warp w: step parity
// (w >> 2) & 1, query columns 32 (w >> 3) .. +31, key rows 32 (w & 3) .. +31), warp 16 TMA
// producer, warp 17 TMEM allocator + MMA issuer, warp 18 row-statistics loader (global
// loads issued several steps ahead so their latency never reaches the pipeline), warp 19
// issues the dQ (and shared-K dK) reduce-adds. The switches below select the measured
// alternatives (8 dS warps, K only in shared memory, one staging tile).
#pragma once

#include "ptx.cuh"

namespace skl {

struct BwdArgs {
  int BH, N_Q, N_K;  // B*H; queries / keys per sequence (packed: the longest sequence)
  int causal;
  float cT, cS;     // |scale| * log2(e)
  float aT, aS;     // |scale| (natural units, teacher gradient only)
  float scale_G;    // signed scale of the side being differentiated (G = g * scale_G)
  int n_ktiles;     // ceil(N_K / 128)
  int group;        // heads per scheduling group (grouped_order)
  int H;            // query heads per batch entry
  int gT, gS;       // query heads per teacher / student K head (GQA; 1 = one K head each)
  int dk_reduce;    // 1: several query heads share the differentiated K head, so dK
                    //    tiles are added into the zeroed dk (bulk reduce) instead of stored
  const int* cu_q;  // packed layout: [B+1] sequence offsets (null: dense [B, H, N, d])
  const int* cu_k;
  int total_q, total_k;    // packed layout: rows of the packed Q / K tensors
  long long dk_hs, dk_rs;  // dk element strides of a K head and of a key row
  int off_adj;             // causal shift of a key shard (context parallelism), else 0
  const float* lse_t;
  const float* lse_s;
  const float* g;
  const float* kl;  // teacher gradient only: E = KL + LSE_T - LSE_S
  float* dq;        // dQ of the differentiated side (fp32, the layout of Q)
  float* dk;        // dK of the differentiated side (fp32, the layout of K)
};

// SKL_BWD_KTMEM: the K tiles are also copied into tensor memory (one key row per lane),
// where the score MMAs read them as their A operand instead of re-reading them from
// shared memory every step; the score tile is then single-buffered to make room.
#ifndef SKL_BWD_KTMEM
#define SKL_BWD_KTMEM 1
#endif

// Warp layout. Default (SKL_BWD_SPLIT): 16 dS warps; warp w takes the steps of parity
// (w >> 2) & 1, query columns 32 (w >> 3) .. +31 of each step and key rows
// 32 (w & 3) .. +31 (its TMEM lane quarter). SKL_BWD_SPLIT = 0: 8 dS warps, all 64 columns.
#ifndef SKL_BWD_SPLIT
#define SKL_BWD_SPLIT 1
#endif
constexpr int kBwdHalves = SKL_BWD_SPLIT ? 2 : 1;      // query-column halves per step
constexpr int kBwdDsWarps = 8 * kBwdHalves;            // warps 0 .. kBwdDsWarps-1
constexpr int kBwdTmaWarp = kBwdDsWarps;               // TMA producer
constexpr int kBwdMmaWarp = kBwdDsWarps + 1;           // TMEM owner + MMA issuer
constexpr int kBwdStatWarp = kBwdDsWarps + 2;          // row-statistics loader
constexpr int kBwdRedWarp = kBwdDsWarps + 3;           // dQ / dK reduce issuer
constexpr int kBwdThreads = 32 * (kBwdDsWarps + 4);
constexpr int kBwdArrive = 4 * kBwdHalves;             // dS warps working on one step
#ifndef SKL_BWD_RS
#define SKL_BWD_RS 96
#endif
#ifndef SKL_BWD_RC
#define SKL_BWD_RC 88
#endif
// The trainable-teacher variant (one exponential per pair, more products) takes 104 / 64:
// its dS warps no longer spill (+4.9 % at N=16K, d=128); the student keeps 96 / 88.
#ifndef SKL_BWD_RS_T
#define SKL_BWD_RS_T 104
#endif
#ifndef SKL_BWD_RC_T
#define SKL_BWD_RC_T 64
#endif
static_assert(!SKL_BWD_SPLIT || kBwdDsWarps * SKL_BWD_RS + 4 * SKL_BWD_RC <=
                                    (kBwdDsWarps + 4) * ((65536 / kBwdThreads) & ~7),
              "register split exceeds the launch's register pool");
static_assert(!SKL_BWD_SPLIT || kBwdDsWarps * SKL_BWD_RS_T + 4 * SKL_BWD_RC_T <=
                                    (kBwdDsWarps + 4) * ((65536 / kBwdThreads) & ~7),
              "register split exceeds the launch's register pool");

// SKL_BWD_TFIRST (student gradient, lean MMA issue): the teacher score MMAs of a step are
// committed to their own barrier, so the dS warps load S_T^T and compute P_T while the
// student score MMAs are still running.
#ifndef SKL_BWD_TFIRST
#define SKL_BWD_TFIRST 1
#endif

// SKL_BWD_LEANMMA (with SKL_BWD_KTMEM): the MMA thread's per-step work reduced to adds of
// compile-time constants to precomputed descriptor halves and addresses.
#ifndef SKL_BWD_LEANMMA
#define SKL_BWD_LEANMMA 1
#endif
static_assert(!SKL_BWD_TFIRST || (SKL_BWD_LEANMMA && SKL_BWD_KTMEM && SKL_BWD_SPLIT),
              "teacher scores first assume the lean MMA issue, K in TMEM and 16 dS warps");

// SKL_BWD_NSTG = 2: two fp32 staging tiles for the dQ reduce-adds, one per step parity (each
// dS warpgroup drains into its own tile while the previous reduce is still reading the
// other). The second tile is the shared K tile of the side that is not differentiated: with
// SKL_BWD_KTMEM it is only read by the copy into tensor memory, which completes before the
// first score MMA and so before any drain. Used where that tile is large enough.
#ifndef SKL_BWD_NSTG
#define SKL_BWD_NSTG 2
#endif

// TEACHER = false: gradients of the student (dQ_S, dK_S), d_G = d_S.
// TEACHER = true: gradients of a trainable teacher (dQ_T, dK_T), d_G = d_T.
template <int DT, int DS, bool TEACHER = false>
struct BwdCfg {
  static constexpr int BN = 128;  // keys per CTA (TMEM lanes)
  static constexpr int BM = 64;   // queries per step
  static constexpr int NQST = 3;  // query-tile stages
  static constexpr int NSTS = 2;  // row-statistics slots
  static constexpr int KT_TILE = BN * DT * 2;
  static constexpr int KS_TILE = BN * DS * 2;
  static constexpr int QT_TILE = BM * DT * 2;
  static constexpr int QS_TILE = BM * DS * 2;
  static constexpr int Q_STAGE = QT_TILE + QS_TILE;
  static constexpr int DS_TILE = BN * BM * 2;  // bf16 dS^T [128 keys][64 queries]
  static constexpr int DG = TEACHER ? DT : DS;  // head dim of the differentiated side
  static constexpr int STATS = 4 * BM * 4;     // -LSE_T*log2e, -LSE_S*log2e, g*scale_G, E
  static constexpr int OFF_KT = 0;
  static constexpr int OFF_KS = OFF_KT + KT_TILE;
  static constexpr int OFF_Q = OFF_KS + KS_TILE;           // NQST stages {Q_T, Q_S}
  static constexpr int OFF_DS = OFF_Q + NQST * Q_STAGE;    // two dS tiles
  static constexpr int STG_TILE = BM * DG * 4;             // fp32 dQ staging tile
  static constexpr int OFF_STG = OFF_DS + 2 * DS_TILE;
  static constexpr int OFF_ST = OFF_STG + STG_TILE;        // NSTS statistics slots
  // K tile of the side that is not differentiated (second staging tile, see SKL_BWD_NSTG).
  static constexpr int OFF_KX = TEACHER ? OFF_KS : OFF_KT;
  static constexpr int KX_TILE = TEACHER ? KS_TILE : KT_TILE;
  static constexpr int NSTG =
      (SKL_BWD_NSTG == 2 && SKL_BWD_KTMEM && KX_TILE >= STG_TILE) ? 2 : 1;  // staging tiles
  // Staging tile of use p (dQ part of step p, or dK round p - n_steps).
  static __device__ __forceinline__ uint32_t stg_off(int p) {
    return (NSTG == 2 && (p & 1)) ? OFF_KX : OFF_STG;
  }
  static constexpr int OFF_BAR = OFF_ST + NSTS * STATS;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM = OFF_BAR + BAR_BYTES;  // the dynamic base is 1024-byte aligned
  static constexpr int THREADS = kBwdThreads;
  // TMEM columns: S_T^T / S_S^T per buffer, dK, dQ^T per buffer.
  static constexpr int NSB = SKL_BWD_KTMEM ? 1 : 2;  // score-tile buffers
  static constexpr int TM_S = 0;          // buffer b: [128b, 128b+64) S_T, [+64, +128) S_S
  static constexpr int TM_DK = 128 * NSB; // d_G columns
  static constexpr int TM_DQ = TM_DK + DG;  // buffer b: + 64 b
  static constexpr int TM_KT = TM_DQ + 2 * BM;  // SKL_BWD_KTMEM: K_T rows, d_T/2 columns
  static constexpr int TM_KS = TM_KT + DT / 2;  //                K_S rows, d_S/2 columns
  static constexpr int DQ_M = DG;         // M of the dQ^T MMA (64 uses half the lanes)
  static_assert((SKL_BWD_KTMEM ? TM_KS + DS / 2 : TM_DQ + 2 * BM) <= 512, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct BwdBars {
  uint64_t k_full;
  uint64_t q_full[3], q_empty[3], st_full[2], st_empty[2];
  uint64_t stg_full[2], stg_free[2];  // indexed by step parity
  uint64_t s_full[2], s_free[2];
  uint64_t t_full[2];  // SKL_BWD_TFIRST: teacher scores of the step (parity) are ready
  uint64_t ds_full[2], ds_empty[2];
  uint64_t dq_full[2], dq_free[2];
  uint64_t dk_full;
  uint64_t k_tmem;  // SKL_BWD_KTMEM: the K rows are in tensor memory (8 warps arrive)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(BwdBars) <= BwdCfg<128, 128, false>::BAR_BYTES,
              "barrier block exceeds its shared-memory reservation");

__device__ __forceinline__ void skl_fail_b(volatile int* abort_flag) {
  atomicOr(&g_skl_error, 2u);
  *abort_flag = 1;
}

template <int DT, int DS, bool TEACHER>
__global__ void __launch_bounds__(kBwdThreads, 1)
streamkl_bwd_kernel(const __grid_constant__ CUtensorMap map_qt,
                    const __grid_constant__ CUtensorMap map_kt,
                    const __grid_constant__ CUtensorMap map_qs,
                    const __grid_constant__ CUtensorMap map_ks,
                    const __grid_constant__ CUtensorMap map_dq,
                    const __grid_constant__ CUtensorMap map_dk, const BwdArgs args,
                    const uint32_t idesc_st, const uint32_t idesc_ss, const uint32_t idesc_dk,
                    const uint32_t idesc_dq) {
  using C = BwdCfg<DT, DS, TEACHER>;
  constexpr int DG = C::DG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sb = smem_u32(smem);
  if (sb & 1023u) {  // the swizzled tiles need 1024-byte alignment; never expected to fire
    if (threadIdx.x == 0) atomicOr(&g_skl_error, 4u);
    return;
  }
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::OFF_BAR);
  float* stats = reinterpret_cast<float*>(smem + C::OFF_ST);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Key tile 0 sees the most query tiles (causal): heaviest first, heads in groups.
  int bh, kt;
  grouped_order(blockIdx.x, args.BH, args.n_ktiles, args.group, bh, kt);
  SeqView seq;
  if (!seq_view(args.cu_q, args.cu_k, bh, args.H, args.gT, args.gS, args.N_Q, args.N_K,
                args.total_q, args.total_k, args.off_adj, seq)) {
    if (threadIdx.x == 0) atomicOr(&g_skl_error, kErrBadOffsets);
    return;
  }
  const int k0 = kt * C::BN;
  if (k0 >= seq.nk) return;  // packed layout: this sequence is shorter than the longest
  const int bkg = TEACHER ? seq.zkt : seq.zks;  // K head that receives this CTA's dK

  int jq_begin = 0;
  if (args.causal) {
    const int first_q = k0 - seq.off;  // first query row that sees key k0
    jq_begin = first_q <= 0 ? 0 : first_q / C::BM;
  }
  const int n_steps = max(0, (seq.nq + C::BM - 1) / C::BM - jq_begin);
  // Staging rounds after the last step that add the dK tile (128 keys = 2 x 64 rows).
  const int dk_rounds = (args.dk_reduce && n_steps > 0) ? 2 : 0;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->k_full), 1);
    for (int i = 0; i < C::NQST; ++i) {
      mbar_init(smem_u32(&bars->q_full[i]), 1);
      mbar_init(smem_u32(&bars->q_empty[i]), 1);
    }
    for (int i = 0; i < C::NSTS; ++i) {
      mbar_init(smem_u32(&bars->st_full[i]), 32);
      mbar_init(smem_u32(&bars->st_empty[i]), kBwdArrive);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->s_full[b]), 1);
      mbar_init(smem_u32(&bars->t_full[b]), 1);
      mbar_init(smem_u32(&bars->s_free[b]), kBwdArrive);
      mbar_init(smem_u32(&bars->ds_full[b]), kBwdArrive);
      mbar_init(smem_u32(&bars->ds_empty[b]), 1);
      mbar_init(smem_u32(&bars->dq_full[b]), 1);
      mbar_init(smem_u32(&bars->dq_free[b]), kBwdArrive);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->stg_full[b]), kBwdArrive);
      mbar_init(smem_u32(&bars->stg_free[b]), 1);
    }
    mbar_init(smem_u32(&bars->dk_full), 1);
    mbar_init(smem_u32(&bars->k_tmem), kBwdDsWarps);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp >= kBwdDsWarps) {
#if SKL_BWD_SPLIT
    regs_dec<TEACHER ? SKL_BWD_RC_T : SKL_BWD_RC>();
#endif
    if (warp == kBwdTmaWarp) {
      // ----------------------------------------------------------- TMA producer
      if (lane == 0) {
        const uint64_t keep = l2_policy_evict_last();
        int issued = 0;
        tma_prefetch_desc(&map_qt);
        tma_prefetch_desc(&map_kt);
        tma_prefetch_desc(&map_qs);
        tma_prefetch_desc(&map_ks);
        const uint32_t kb = smem_u32(&bars->k_full);
        mbar_arrive_expect_tx(kb, C::KT_TILE + C::KS_TILE);
        for (int blk = 0; blk < DT / 64; ++blk)
          tma_load_3d(sb + C::OFF_KT + blk * (C::BN * 128), &map_kt, kb, blk * 64, seq.kr + k0,
                      seq.zkt, keep);
        for (int blk = 0; blk < DS / 64; ++blk)
          tma_load_3d(sb + C::OFF_KS + blk * (C::BN * 128), &map_ks, kb, blk * 64, seq.kr + k0,
                      seq.zks, keep);
        for (int s = 0; s < n_steps; ++s) {
          const int st = s % C::NQST;
          const int i0 = seq.qr + (jq_begin + s) * C::BM;
          if (!mbar_wait(smem_u32(&bars->q_empty[st]), ((s / C::NQST) & 1) ^ 1)) {
            skl_fail_b(abort_flag);
            break;
          }
          const uint32_t fb = smem_u32(&bars->q_full[st]);
          const uint32_t q_base = sb + C::OFF_Q + st * C::Q_STAGE;
          mbar_arrive_expect_tx(fb, C::Q_STAGE);
          for (int blk = 0; blk < DT / 64; ++blk)
            tma_load_3d(q_base + blk * (C::BM * 128), &map_qt, fb, blk * 64, i0, seq.zq, keep);
          for (int blk = 0; blk < DS / 64; ++blk)
            tma_load_3d(q_base + C::QT_TILE + blk * (C::BM * 128), &map_qs, fb, blk * 64, i0,
                        seq.zq, keep);
          issued = s + 1;
        }
        if (*abort_flag) {
          // Let every copy this thread started land before the CTA can exit.
          mbar_wait(smem_u32(&bars->k_full), 0);
          for (int s = max(0, issued - C::NQST); s < issued; ++s)
            mbar_wait(smem_u32(&bars->q_full[s % C::NQST]), (s / C::NQST) & 1);
        }
      }
    } else if (warp == kBwdStatWarp) {
      // ------------------------------------------------ row-statistics loader
      // Each lane owns query rows lane and lane+32 of every step. Raw LSE_T, LSE_S, g (and
      // KL for the teacher gradient) are loaded kStatAhead steps before they are needed and
      // kept in registers.
      constexpr int kStatAhead = 3;
      const float LOG2E = 1.4426950408889634f;
      float r_lt[kStatAhead][2], r_ls[kStatAhead][2], r_g[kStatAhead][2], r_kl[kStatAhead][2];
      auto load_step = [&](int s, float (&lt)[2], float (&ls)[2], float (&gg)[2], float (&kv)[2]) {
    #pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = (jq_begin + s) * C::BM + r * 32 + lane;
          lt[r] = -INFINITY;
          ls[r] = -INFINITY;
          gg[r] = 0.f;
          kv[r] = 0.f;
          if (s < n_steps && row < seq.nq) {
            const size_t o = (size_t)(seq.ob + row);
            lt[r] = __ldg(args.lse_t + o);
            ls[r] = __ldg(args.lse_s + o);
            gg[r] = __ldg(args.g + o);
            if (TEACHER) kv[r] = __ldg(args.kl + o);
          }
        }
      };
    #pragma unroll
      for (int k = 0; k < kStatAhead; ++k) load_step(k, r_lt[k], r_ls[k], r_g[k], r_kl[k]);
      bool ok = true;
      for (int s = 0; s < n_steps; ++s) {
        if (lane == 0 && !mbar_wait(smem_u32(&bars->st_empty[s & 1]), ((s >> 1) & 1) ^ 1)) {
          ok = false;
          skl_fail_b(abort_flag);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        // Slot s&1: -LSE_T*log2e, -LSE_S*log2e, g*scale_G, E = KL + LSE_T - LSE_S
        // (rows without keys: -inf, -inf, 0, 0).
        float* sts = stats + (s & 1) * (4 * C::BM);
    #pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float lt = r_lt[0][r], ls = r_ls[0][r];
          const bool live = lt != -INFINITY && ls != -INFINITY;
          sts[r * 32 + lane] = live ? -lt * LOG2E : -INFINITY;
          sts[C::BM + r * 32 + lane] = live ? -ls * LOG2E : -INFINITY;
          sts[2 * C::BM + r * 32 + lane] = live ? r_g[0][r] * args.scale_G : 0.f;
          sts[3 * C::BM + r * 32 + lane] = live ? r_kl[0][r] + (lt - ls) : 0.f;
        }
        mbar_arrive(smem_u32(&bars->st_full[s & 1]));
    #pragma unroll
        for (int k = 0; k + 1 < kStatAhead; ++k)
    #pragma unroll
          for (int r = 0; r < 2; ++r) {
            r_lt[k][r] = r_lt[k + 1][r];
            r_ls[k][r] = r_ls[k + 1][r];
            r_g[k][r] = r_g[k + 1][r];
            r_kl[k][r] = r_kl[k + 1][r];
          }
        load_step(s + kStatAhead, r_lt[kStatAhead - 1], r_ls[kStatAhead - 1], r_g[kStatAhead - 1],
                  r_kl[kStatAhead - 1]);
      }
    } else if (warp == kBwdRedWarp) {
      // ------------------------------------------- dQ (and shared-K dK) reduce issuer
      if (lane == 0) {
        tma_prefetch_desc(&map_dq);
        if (dk_rounds) tma_prefetch_desc(&map_dk);
        int issued = 0;
        for (int p = 0; p < n_steps + dk_rounds; ++p) {
          if (!mbar_wait(smem_u32(&bars->stg_full[p & 1]), (p >> 1) & 1)) {
            skl_fail_b(abort_flag);
            break;
          }
          const uint32_t src = sb + C::stg_off(p);
          if (p < n_steps) {  // dQ part of step p: 64 query rows
            const int i0 = seq.qr + (jq_begin + p) * C::BM;
    #pragma unroll
            for (int db = 0; db < DG / 32; ++db)
              tma_reduce_add_3d(&map_dq, src + db * (C::BM * 128), db * 32, i0, seq.zq);
          } else {  // dK tile of this CTA, 64 key rows per round
            const int r0 = seq.kr + k0 + (p - n_steps) * 64;
    #pragma unroll
            for (int db = 0; db < DG / 32; ++db)
              tma_reduce_add_3d(&map_dk, src + db * (C::BM * 128), db * 32, r0, bkg);
          }
          bulk_commit_group();
          issued = p + 1;
          if (C::NSTG == 2) {
            // The reduce of use p may still be reading its tile; use p-1's tile is free.
            bulk_wait_group_read1();
            if (p > 0) mbar_arrive(smem_u32(&bars->stg_free[(p - 1) & 1]));
          } else {
            bulk_wait_group_read0();
            mbar_arrive(smem_u32(&bars->stg_free[p & 1]));
          }
        }
        if (C::NSTG == 2 && issued > 0) {
          bulk_wait_group_read0();
          mbar_arrive(smem_u32(&bars->stg_free[(issued - 1) & 1]));
        }
        bulk_wait_group0();
      }
    } else if (warp == kBwdMmaWarp) {
      // ------------------------------------------------------------- MMA issuer
      if (elect_one()) {
        const uint32_t s_kt = sb + C::OFF_KT, s_ks = sb + C::OFF_KS;
        bool ok = mbar_wait(smem_u32(&bars->k_full), 0);
    #if SKL_BWD_KTMEM && SKL_BWD_LEANMMA
        // The dS warps copy the K rows into tensor memory first.
        if (ok) ok = mbar_wait(smem_u32(&bars->k_tmem), 0);
        // This thread's instruction stream is on the step's critical path, so every
        // per-MMA quantity is a precomputed base plus a compile-time constant: descriptor
        // low halves (one shared high half), TMEM column addresses, stage indices and
        // phases tracked incrementally (no divisions).
        const uint32_t hi = sdesc_hi(1024);
        const uint32_t lq0 = sdesc_lo(sb + C::OFF_Q, 16);  // Q_T of stage 0, K-major
        const uint32_t lqg0 =                               // Q of the differentiated side
            sdesc_lo(sb + C::OFF_Q + (TEACHER ? 0 : C::QT_TILE), C::BM * 128);
        const uint32_t lds_k0 = sdesc_lo(sb + C::OFF_DS, 16);           // dS^T buffer 0 as A
        const uint32_t lds_n0 = sdesc_lo(sb + C::OFF_DS, C::BN * 128);  // dS^T buffer 0 as B
        const uint32_t lkg = sdesc_lo(TEACHER ? s_kt : s_ks, C::BN * 128);  // K^T as A
        constexpr uint32_t kQ16 = C::Q_STAGE >> 4, kDs16 = C::DS_TILE >> 4;
        const uint32_t t_st = tmem + C::TM_S, t_ss = t_st + 64, t_dk = tmem + C::TM_DK;
        const uint32_t t_kt = tmem + C::TM_KT, t_ks = tmem + C::TM_KS, t_dq = tmem + C::TM_DQ;
        int s_st = 0;      // query stage of the next score step
        uint32_t s_ph = 0;  // and the phase of its q_full barrier
        auto issue_scores = [&](int s) -> bool {
          if (!mbar_wait(smem_u32(&bars->q_full[s_st]), s_ph)) return false;
          if (s > 0 && !mbar_wait(smem_u32(&bars->s_free[(s - 1) & 1]), ((s - 1) >> 1) & 1))
            return false;
          tc_fence_after();
          const uint32_t lq = lq0 + (uint32_t)s_st * kQ16;
    #pragma unroll
          for (int kk = 0; kk < DT / 16; ++kk) {
            const uint32_t qa = ((kk >> 2) * (C::BM * 128) + (kk & 3) * 32) >> 4;
            umma_bf16_ts_lh(t_st, t_kt + kk * 8, lq + qa, hi, idesc_st, kk > 0);
          }
          if (SKL_BWD_TFIRST && !TEACHER) umma_commit(smem_u32(&bars->t_full[s & 1]));
    #pragma unroll
          for (int kk = 0; kk < DS / 16; ++kk) {
            const uint32_t qa = (C::QT_TILE + (kk >> 2) * (C::BM * 128) + (kk & 3) * 32) >> 4;
            umma_bf16_ts_lh(t_ss, t_ks + kk * 8, lq + qa, hi, idesc_ss, kk > 0);
          }
          umma_commit(smem_u32(&bars->s_full[s & 1]));
          if (++s_st == C::NQST) {
            s_st = 0;
            s_ph ^= 1u;
          }
          return true;
        };
        int pst = 0;  // query stage of step p
        if (ok && n_steps > 0) ok = issue_scores(0);
        for (int p = 0; ok && p < n_steps; ++p) {
          const int pb = p & 1;
          // Scores of step p+1 as soon as the warpgroup of step p has read its scores.
          if (p + 1 < n_steps && !issue_scores(p + 1)) { ok = false; break; }
          if (!mbar_wait(smem_u32(&bars->ds_full[pb]), (p >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          // dK += dS^T Q : A = dS^T [keys][queries] K-major, B = Q [queries][d] MN-major.
          const uint32_t la = lds_k0 + (pb ? kDs16 : 0u), lb = lqg0 + (uint32_t)pst * kQ16;
    #pragma unroll
          for (int kk = 0; kk < C::BM / 16; ++kk)
            umma_bf16_ss_lh(t_dk, la + kk * 2, lb + kk * 128, hi, idesc_dk,
                            (p > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&bars->q_empty[pst]));
          if (!mbar_wait(smem_u32(&bars->dq_free[pb]), ((p >> 1) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          // dQ^T = K^T dS^T : A = K [keys][d] MN-major, B = dS^T [keys][queries] MN-major.
          const uint32_t lbq = lds_n0 + (pb ? kDs16 : 0u), t_dqb = t_dq + (pb ? C::BM : 0);
    #pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk)
            umma_bf16_ss_lh(t_dqb, lkg + kk * 128, lbq + kk * 128, hi, idesc_dq, kk > 0);
          umma_commit(smem_u32(&bars->ds_empty[pb]));
          umma_commit(smem_u32(&bars->dq_full[pb]));
          if (++pst == C::NQST) pst = 0;
        }
    #else
    #if SKL_BWD_KTMEM
        // The dS warps copy the K rows into tensor memory first.
        if (ok) ok = mbar_wait(smem_u32(&bars->k_tmem), 0);
        // S_T^T = K_T Q_T^T and S_S^T = K_S Q_S^T of step s into the single score buffer,
        // A (the K rows) from tensor memory; the buffer is free once step s-1 has been read.
        // Barriers stay per step parity (each warpgroup waits only on its own steps' phases).
        auto issue_scores = [&](int s) -> bool {
          const int st = s % C::NQST;
          if (!mbar_wait(smem_u32(&bars->q_full[st]), (s / C::NQST) & 1)) return false;
          if (s > 0 && !mbar_wait(smem_u32(&bars->s_free[(s - 1) & 1]), ((s - 1) >> 1) & 1))
            return false;
          tc_fence_after();
          const uint32_t q_base = sb + C::OFF_Q + st * C::Q_STAGE;
          const uint32_t d_t = tmem + C::TM_S, d_s = d_t + 64;
    #pragma unroll
          for (int kk = 0; kk < DT / 16; ++kk) {
            const uint32_t qa = (kk >> 2) * (C::BM * 128) + (kk & 3) * 32;
            umma_bf16_ts(d_t, tmem + C::TM_KT + kk * 8, sdesc_sw128(q_base + qa, 16, 1024),
                         idesc_st, kk > 0);
          }
    #pragma unroll
          for (int kk = 0; kk < DS / 16; ++kk) {
            const uint32_t qa = (kk >> 2) * (C::BM * 128) + (kk & 3) * 32;
            umma_bf16_ts(d_s, tmem + C::TM_KS + kk * 8,
                         sdesc_sw128(q_base + C::QT_TILE + qa, 16, 1024), idesc_ss, kk > 0);
          }
          umma_commit(smem_u32(&bars->s_full[s & 1]));
          return true;
        };
        if (ok && n_steps > 0) ok = issue_scores(0);
        for (int p = 0; ok && p < n_steps; ++p) {
          const int pb = p & 1, pst = p % C::NQST;
          // Scores of step p+1 as soon as the warpgroup of step p has read its scores.
          if (p + 1 < n_steps && !issue_scores(p + 1)) { ok = false; break; }
          constexpr bool early = true;
    #else
        // S_T^T = K_T Q_T^T and S_S^T = K_S Q_S^T of step s into TMEM buffer s&1.
        auto issue_scores = [&](int s) -> bool {
          const int st = s % C::NQST, b = s & 1;
          if (!mbar_wait(smem_u32(&bars->q_full[st]), (s / C::NQST) & 1)) return false;
          if (!mbar_wait(smem_u32(&bars->s_free[b]), ((s >> 1) & 1) ^ 1)) return false;
          tc_fence_after();
          const uint32_t q_base = sb + C::OFF_Q + st * C::Q_STAGE;
          const uint32_t d_t = tmem + C::TM_S + b * 128, d_s = d_t + 64;
    #pragma unroll
          for (int kk = 0; kk < DT / 16; ++kk) {
            const uint32_t ka = (kk >> 2) * (C::BN * 128) + (kk & 3) * 32;
            const uint32_t qa = (kk >> 2) * (C::BM * 128) + (kk & 3) * 32;
            umma_bf16_ss(d_t, sdesc_sw128(s_kt + ka, 16, 1024), sdesc_sw128(q_base + qa, 16, 1024),
                         idesc_st, kk > 0);
          }
    #pragma unroll
          for (int kk = 0; kk < DS / 16; ++kk) {
            const uint32_t ka = (kk >> 2) * (C::BN * 128) + (kk & 3) * 32;
            const uint32_t qa = (kk >> 2) * (C::BM * 128) + (kk & 3) * 32;
            umma_bf16_ss(d_s, sdesc_sw128(s_ks + ka, 16, 1024),
                         sdesc_sw128(q_base + C::QT_TILE + qa, 16, 1024), idesc_ss, kk > 0);
          }
          umma_commit(smem_u32(&bars->s_full[b]));
          return true;
        };
        if (ok && n_steps > 0) ok = issue_scores(0);
        if (ok && n_steps > 1) ok = issue_scores(1);
        for (int p = 0; ok && p < n_steps; ++p) {
          const int pb = p & 1, pst = p % C::NQST;
          // The score tiles of step p+2 reuse buffer pb, which the warpgroup frees as soon as
          // it has read step p's scores; issue them ahead of dK/dQ(p) when their query tile
          // has landed, so the warpgroup finds them ready when it finishes step p.
          bool early = false;
          if (p + 2 < n_steps && mbar_try_wait(smem_u32(&bars->q_full[(p + 2) % C::NQST]),
                                               ((p + 2) / C::NQST) & 1)) {
            if (!issue_scores(p + 2)) { ok = false; break; }
            early = true;
          }
    #endif
          if (!mbar_wait(smem_u32(&bars->ds_full[pb]), (p >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t s_ds = sb + C::OFF_DS + pb * C::DS_TILE;
          // Q tile of the differentiated side (student Q_S, or teacher Q_T).
          const uint32_t s_qg = sb + C::OFF_Q + pst * C::Q_STAGE + (TEACHER ? 0 : C::QT_TILE);
          // dK += dS^T Q : A = dS^T [keys][queries] K-major, B = Q [queries][d] MN-major.
    #pragma unroll
          for (int kk = 0; kk < C::BM / 16; ++kk) {
            umma_bf16_ss(tmem + C::TM_DK, sdesc_sw128(s_ds + kk * 32, 16, 1024),
                         sdesc_sw128(s_qg + kk * 2048, C::BM * 128, 1024), idesc_dk,
                         (p > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&bars->q_empty[pst]));
          if (!mbar_wait(smem_u32(&bars->dq_free[pb]), ((p >> 1) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          // dQ^T = K^T dS^T : A = K [keys][d] MN-major, B = dS^T [keys][queries] MN-major.
          const uint32_t s_kg = TEACHER ? s_kt : s_ks;
    #pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            umma_bf16_ss(tmem + C::TM_DQ + pb * C::BM,
                         sdesc_sw128(s_kg + kk * 2048, C::BN * 128, 1024),
                         sdesc_sw128(s_ds + kk * 2048, C::BN * 128, 1024), idesc_dq, kk > 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&bars->ds_empty[pb]));
          umma_commit(smem_u32(&bars->dq_full[pb]));
          if (!early && p + 2 < n_steps && !issue_scores(p + 2)) { ok = false; break; }
        }
    #endif
        if (!ok) skl_fail_b(abort_flag);
        umma_commit(smem_u32(&bars->dk_full));
        umma_commit(smem_u32(&bars->drain));
        if (!mbar_wait(smem_u32(&bars->drain), 0)) skl_fail_b(abort_flag);
      }
    }
  } else {
    // ------------------------------------------------- dS / reduction warpgroups
#if SKL_BWD_SPLIT
    regs_inc<TEACHER ? SKL_BWD_RS_T : SKL_BWD_RS>();
#endif
    const int wg = (warp >> 2) & 1;      // steps s with s&1 == wg
    const int hh = warp >> 3;            // query-column half (split), else 0
    constexpr int NC = C::BM / kBwdHalves;  // query columns of a step handled by this warp
    const int c0 = hh * NC;
    const int quarter = warp & 3;
    const int kl = quarter * 32 + lane;  // key row within the tile = TMEM lane
    const int key = k0 + kl;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float cT = args.cT, cS = args.cS, aT = args.aT, aS = args.aS;
    const uint32_t s_ds_row = sb + C::OFF_DS + wg * C::DS_TILE + kl * 128;
    // dQ^T lanes are d: all 32 lanes of a quarter for d_S = 128; for d_S = 64 the M=64
    // layout puts rows 16w..16w+15 on lanes 32w..32w+15.
    const bool dq_lane_ok = (C::DQ_M == 128) || lane < 16;
    const int dq_d = (C::DQ_M == 128) ? kl : quarter * 16 + lane;

    // The staging tile of use p is free once the reduce of its previous use has read it:
    // use p-2 with a tile per step parity, use p-1 with a single tile. Barriers are split
    // by step parity so no wait is ever more than one phase ahead.
    auto stg_wait = [&](int p) -> bool {
      if (C::NSTG == 2)
        return p < 2 || mbar_wait(smem_u32(&bars->stg_free[p & 1]), ((p - 2) >> 1) & 1);
      return p < 1 || mbar_wait(smem_u32(&bars->stg_free[(p - 1) & 1]), ((p - 1) >> 1) & 1);
    };

    // dQ^T part of step p (TMEM) -> staging tile (dQ row layout: 32-column boxes of
    // 64 rows x 128 bytes, 128-byte swizzle) -> one bulk reduce-add by the reduce warp.
    auto drain_dq = [&](int p) -> bool {
      if (!mbar_wait(smem_u32(&bars->dq_full[wg]), (p >> 1) & 1)) return false;
      tc_fence_after();
      uint32_t v[NC];  // this warp's query columns c0 .. c0+NC-1 of the dQ^T part
      if constexpr (NC == 64) {
        tmem_ld_2x32_wait(tmem + lane_off + C::TM_DQ + wg * C::BM,
                          tmem + lane_off + C::TM_DQ + wg * C::BM + 32, v);
      } else {
        tmem_ld_32_wait(tmem + lane_off + C::TM_DQ + wg * C::BM + c0, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->dq_free[wg]));
      if (!stg_wait(p)) return false;
      if (dq_lane_ok) {
        const uint32_t col = sb + C::stg_off(p) + (dq_d >> 5) * (C::BM * 128) + ((dq_d & 3) << 2);
        const uint32_t chunk = (dq_d & 31) >> 2;
#pragma unroll
        for (int i = 0; i < NC; ++i) {
          const int c = c0 + i;
          st_shared_f32(col + c * 128 + ((chunk ^ (c & 7)) << 4), __uint_as_float(v[i]));
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->stg_full[p & 1]));
      return true;
    };

    bool ok = true;
#if SKL_BWD_KTMEM
    {
      // K rows into tensor memory (A operand of the score MMAs): warpgroup 0 copies K_T,
      // warpgroup 1 copies K_S, one key row per thread.
      if (hh > 0) {
        // the first column half copies
      } else if (mbar_wait(smem_u32(&bars->k_full), 0)) {
        if (wg == 0)
          row_to_tmem<DT>(sb + C::OFF_KT + kl * 128, tmem + lane_off + C::TM_KT, kl);
        else
          row_to_tmem<DS>(sb + C::OFF_KS + kl * 128, tmem + lane_off + C::TM_KS, kl);
      } else {
        ok = false;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->k_tmem));
    }
    constexpr int sbuf = 0;  // TMEM score buffer (single)
#else
    const int sbuf = wg;
#endif
    int last = -1;
    for (int s = wg; ok && s < n_steps; s += 2) {
      const int st = s % C::NQST;
      const int i0 = (jq_begin + s) * C::BM;  // first query column of this step
#if SKL_BWD_TFIRST
      if constexpr (!TEACHER && NC == 32) {
        // Teacher scores first: P_T of this warp's columns while the student score MMAs of
        // the step are still running, then the student scores.
        if (!mbar_wait(smem_u32(&bars->t_full[wg]), (s >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t vt[NC];
        tmem_ld_32_wait(tmem + lane_off + C::TM_S + sbuf * 128 + c0, vt);
        if (!mbar_wait(smem_u32(&bars->st_full[s & 1]), (s >> 1) & 1)) { ok = false; break; }
        const float* sts = stats + (s & 1) * (4 * C::BM);
        float pt[NC];
#pragma unroll
        for (int u4 = 0; u4 < NC / 4; ++u4) {
          const float4 nl = *reinterpret_cast<const float4*>(sts + c0 + 4 * u4);
          pt[4 * u4 + 0] = ex2_approx(fmaf(__uint_as_float(vt[4 * u4 + 0]), cT, nl.x));
          pt[4 * u4 + 1] = ex2_approx(fmaf(__uint_as_float(vt[4 * u4 + 1]), cT, nl.y));
          pt[4 * u4 + 2] = ex2_approx(fmaf(__uint_as_float(vt[4 * u4 + 2]), cT, nl.z));
          pt[4 * u4 + 3] = ex2_approx(fmaf(__uint_as_float(vt[4 * u4 + 3]), cT, nl.w));
        }
        if (!mbar_wait(smem_u32(&bars->s_full[wg]), (s >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t vs[NC];
        tmem_ld_32_wait(tmem + lane_off + C::TM_S + sbuf * 128 + 64 + c0, vs);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[wg]));
        const bool causal_mask = args.causal && (i0 + seq.off < k0 + C::BN - 1);
        const bool need_mask = causal_mask || (k0 + C::BN > seq.nk);
        const int cmin = key >= seq.nk ? C::BM : (causal_mask ? (key - seq.off - i0) : -1);
        uint32_t pk[NC / 8][4];
#pragma unroll
        for (int uu = 0; uu < NC / 8; ++uu) {
          const int u = c0 / 8 + uu;
          const float4 nls0 = *reinterpret_cast<const float4*>(sts + C::BM + u * 8);
          const float4 nls1 = *reinterpret_cast<const float4*>(sts + C::BM + u * 8 + 4);
          const float4 g0 = *reinterpret_cast<const float4*>(sts + 2 * C::BM + u * 8);
          const float4 g1 = *reinterpret_cast<const float4*>(sts + 2 * C::BM + u * 8 + 4);
          const float nls[8] = {nls0.x, nls0.y, nls0.z, nls0.w, nls1.x, nls1.y, nls1.z, nls1.w};
          const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
          float d[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = u * 8 + e;
            const int ci = uu * 8 + e;
            const float pS = ex2_approx(fmaf(__uint_as_float(vs[ci]), cS, nls[e]));
            float ds = gg[e] * (pS - pt[ci]);
            if (need_mask && c < cmin) ds = 0.f;
            d[e] = ds;
          }
          pk[uu][0] = pack_bf16x2(d[0], d[1]);
          pk[uu][1] = pack_bf16x2(d[2], d[3]);
          pk[uu][2] = pack_bf16x2(d[4], d[5]);
          pk[uu][3] = pack_bf16x2(d[6], d[7]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->st_empty[s & 1]));
        if (!mbar_wait(smem_u32(&bars->ds_empty[wg]), ((s >> 1) & 1) ^ 1)) { ok = false; break; }
#pragma unroll
        for (int uu = 0; uu < NC / 8; ++uu) {
          const int u = c0 / 8 + uu;
          st_shared_v4(s_ds_row + ((u ^ (kl & 7)) << 4), pk[uu][0], pk[uu][1], pk[uu][2],
                       pk[uu][3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->ds_full[wg]));
        if (last >= 0 && !drain_dq(last)) { ok = false; break; }
        last = s;
        continue;
      }
#endif
      if (!mbar_wait(smem_u32(&bars->s_full[wg]), (s >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // Raw teacher / student scores of this key for this warp's query columns.
      uint32_t vt[NC], vs[NC];
      if constexpr (NC == 64) {
        tmem_ld_2x32_wait(tmem + lane_off + C::TM_S + sbuf * 128,
                          tmem + lane_off + C::TM_S + sbuf * 128 + 32, vt);
        tmem_ld_2x32_wait(tmem + lane_off + C::TM_S + sbuf * 128 + 64,
                          tmem + lane_off + C::TM_S + sbuf * 128 + 96, vs);
      } else {
        tmem_ld_32_wait(tmem + lane_off + C::TM_S + sbuf * 128 + c0, vt);
        tmem_ld_32_wait(tmem + lane_off + C::TM_S + sbuf * 128 + 64 + c0, vs);
      }
      // The score buffer can take step s+2 as soon as every lane has read it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[wg]));
      if (!mbar_wait(smem_u32(&bars->st_full[s & 1]), (s >> 1) & 1)) { ok = false; break; }
      const float* sts = stats + (s & 1) * (4 * C::BM);

      // Query column c is allowed for this key iff i0 + c >= key - off; keys past the end
      // of the sequence (the next sequence's keys in the packed layout, zero fill in the
      // dense one) get dS = 0 for every column.
      const bool causal_mask = args.causal && (i0 + seq.off < k0 + C::BN - 1);
      const bool need_mask = causal_mask || (k0 + C::BN > seq.nk);
      const int cmin = key >= seq.nk ? C::BM : (causal_mask ? (key - seq.off - i0) : -1);
      // dS of this step into registers (bf16 pairs) first; it is stored once the dK/dQ MMAs
      // of step s-2 have read the dS buffer, so this arithmetic overlaps those MMAs.
      uint32_t pk[NC / 8][4];
#pragma unroll
      for (int uu = 0; uu < NC / 8; ++uu) {  // 8 query columns = one 16-byte chunk of dS^T
        const int u = c0 / 8 + uu;
        const float4 nlt0 = *reinterpret_cast<const float4*>(sts + u * 8);
        const float4 nlt1 = *reinterpret_cast<const float4*>(sts + u * 8 + 4);
        const float4 nls0 = *reinterpret_cast<const float4*>(sts + C::BM + u * 8);
        const float4 nls1 = *reinterpret_cast<const float4*>(sts + C::BM + u * 8 + 4);
        const float4 g0 = *reinterpret_cast<const float4*>(sts + 2 * C::BM + u * 8);
        const float4 g1 = *reinterpret_cast<const float4*>(sts + 2 * C::BM + u * 8 + 4);
        const float nlt[8] = {nlt0.x, nlt0.y, nlt0.z, nlt0.w, nlt1.x, nlt1.y, nlt1.z, nlt1.w};
        const float nls[8] = {nls0.x, nls0.y, nls0.z, nls0.w, nls1.x, nls1.y, nls1.z, nls1.w};
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        float ee[8];
        if (TEACHER) {
          const float4 e0 = *reinterpret_cast<const float4*>(sts + 3 * C::BM + u * 8);
          const float4 e1 = *reinterpret_cast<const float4*>(sts + 3 * C::BM + u * 8 + 4);
          ee[0] = e0.x; ee[1] = e0.y; ee[2] = e0.z; ee[3] = e0.w;
          ee[4] = e1.x; ee[5] = e1.y; ee[6] = e1.z; ee[7] = e1.w;
        }
        float d[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = u * 8 + e;   // query column within the step
          const int ci = uu * 8 + e;  // its register index
          const float pT = ex2_approx(fmaf(__uint_as_float(vt[ci]), cT, nlt[e]));
          float ds;
          if (TEACHER) {
            // g*scale_T * P_T * ((s_T - s_S) - E), scores in natural units; both products
            // rounded alike so that identical teacher and student scores cancel exactly.
            const float w = __fsub_rn(__fmul_rn(__uint_as_float(vt[ci]), aT),
                                      __fmul_rn(__uint_as_float(vs[ci]), aS)) - ee[e];
            ds = gg[e] * pT * w;
          } else {
            const float pS = ex2_approx(fmaf(__uint_as_float(vs[ci]), cS, nls[e]));
            ds = gg[e] * (pS - pT);
          }
          if (need_mask && c < cmin) ds = 0.f;
          d[e] = ds;
        }
        pk[uu][0] = pack_bf16x2(d[0], d[1]);
        pk[uu][1] = pack_bf16x2(d[2], d[3]);
        pk[uu][2] = pack_bf16x2(d[4], d[5]);
        pk[uu][3] = pack_bf16x2(d[6], d[7]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->st_empty[s & 1]));
      // The dS buffer is free once the dK/dQ MMAs of step s-2 have read it.
      if (!mbar_wait(smem_u32(&bars->ds_empty[wg]), ((s >> 1) & 1) ^ 1)) { ok = false; break; }
#pragma unroll
      for (int uu = 0; uu < NC / 8; ++uu) {
        const int u = c0 / 8 + uu;
        st_shared_v4(s_ds_row + ((u ^ (kl & 7)) << 4), pk[uu][0], pk[uu][1], pk[uu][2],
                     pk[uu][3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->ds_full[wg]));
      if (last >= 0 && !drain_dq(last)) { ok = false; break; }
      last = s;
    }
    if (ok && last >= 0 && !drain_dq(last)) ok = false;

    // dK rows of this key tile (TMEM lanes = keys); zero when no query sees them. With a
    // K head shared by several query heads (dk_reduce) the tile is added into the zeroed
    // dk through the staging tile in two 64-row rounds, continuing the staging sequence.
    constexpr int DKH = DG / (2 * kBwdHalves);  // dK columns handled by this warp
    const int col0 = (hh * 2 + wg) * DKH;
    uint32_t v[DKH];
#pragma unroll
    for (int c = 0; c < DKH; ++c) v[c] = 0u;
    if (ok && n_steps > 0) {
      if (!mbar_wait(smem_u32(&bars->dk_full), 0)) {
        ok = false;
      } else {
        tc_fence_after();
        if constexpr (DKH == 64) {
          tmem_ld_2x32_wait(tmem + lane_off + C::TM_DK + col0,
                            tmem + lane_off + C::TM_DK + col0 + 32, v);
        } else if constexpr (DKH == 32) {
          tmem_ld_32_wait(tmem + lane_off + C::TM_DK + col0, v);
        } else {
          tmem_ld_16_wait(tmem + lane_off + C::TM_DK + col0, v);
        }
      }
    }
    if (ok && !dk_rounds && key < seq.nk) {
      float4* dst = reinterpret_cast<float4*>(args.dk + bkg * args.dk_hs +
                                              (long long)(seq.kr + key) * args.dk_rs + col0);
#pragma unroll
      for (int c = 0; c < DKH; c += 4)
        dst[c / 4] = make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                 __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
    }
    if (dk_rounds) {
      // Every dS warp reaches this barrier (dk_rounds is uniform over the CTA), after its
      // last dQ drain, so each staging wait below is at most one phase ahead of its barrier.
      named_bar_sync(1, 32 * kBwdDsWarps);
      ok = __all_sync(0xffffffffu, ok);
      for (int r = 0; ok && r < 2; ++r) {
        const int p = n_steps + r;
        ok = __all_sync(0xffffffffu, stg_wait(p));
        if (!ok) break;
        if ((quarter >> 1) == r) {  // this warp's lanes are rows 64r .. 64r+63 of the tile
          const int row = kl - 64 * r;
#pragma unroll
          for (int c = 0; c < DKH; c += 4) {
            const int dcol = col0 + c;
            const uint32_t addr = sb + C::stg_off(p) + (dcol >> 5) * (C::BM * 128) + row * 128 +
                                  ((((dcol & 31) >> 2) ^ (row & 7)) << 4);
            st_shared_v4(addr, v[c], v[c + 1], v[c + 2], v[c + 3]);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->stg_full[p & 1]));
        }
      }
    }
    if (!ok) skl_fail_b(abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace skl
