// fwd_kernel.cuh - StreamKL forward on sm_100a (tcgen05 + TMEM + TMA).
//
// The one-pass forward of "StreamKL: Fast and Memory-Efficient KL Divergence for
// Boosting Attention Distillation" (abstract: one forward pass reduces both distributions
// together with a running per-row state while query and key tiles pass through on-chip
// memory).
//
// CTA = two 128-row query tiles of one (batch, head). Key tiles of 64 rows stream
// through a TMA ring. Per key tile and query tile the tensor core computes the teacher
// and student score tiles into TMEM, with the query tiles themselves held in TMEM as the
// MMA's A operand (SKL_FWD_QTMEM; one score buffer per query tile, whose next tile is
// computed as soon as the current one has been read, so the fold overlaps those MMAs).
// Each query row is folded by two threads (one per 32-key half of every tile), each
// keeping its own online state
//     m_T, m_S   reference maxima of t = s * log2(e) (at most the running maxima)
//     l_T, l_S   running sums of 2^(t - m)
//     A          running sum of 2^(t_T - m_T) * (t_T - t_S)
// which merge at the end, so that KL = ln2 * A / l_T - LSE_T + LSE_S. Per tile a thread
// reads its 64 scores from TMEM in one round trip and releases the buffer at once; the
// fp32 work is issued as packed pairs, with a share of the exponentials on the FMA pipe.
// Unmasked tiles are folded against the reference maxima as they stand (no per-tile max;
// the state is exact for any reference); masked tiles, a row's first tile and a tile
// whose exponentials would reach 2^64 raise the references to the running maxima first.
// Nothing of size N_Q x N_K ever leaves the SM.
//
// Warp roles (640 threads, SKL_FWD_SPLIT): warps 0-7 query tile 0 and 8-15 query tile 1
// (warps 4k..4k+3 cover the tile's four 32-row quarters for one key half; 104 registers
// each), warp 16 TMA producer, warp 17 TMEM allocator + MMA issuer, warps 18-19 idle (the
// control warpgroup runs with 56 registers). With SKL_FWD_SPLIT = 0: 384 threads, one
// thread per row over whole tiles (200 registers), warps 8 / 9 TMA / MMA.
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

// Warp layout. Default: 8 statistics warps (one thread per query row, whole key tiles).
// SKL_FWD_SPLIT: 16 statistics warps, two per row quarter, each folding one half (32 keys)
// of every tile into its own row state; the two states merge once at the end.
#ifndef SKL_FWD_SPLIT
#define SKL_FWD_SPLIT 1
#endif
constexpr int kFwdHalves = SKL_FWD_SPLIT ? 2 : 1;        // key halves per tile
constexpr int kFwdStatWarps = 8 * kFwdHalves;            // warps 0 .. kFwdStatWarps-1
constexpr int kFwdTmaWarp = kFwdStatWarps;               // TMA producer
constexpr int kFwdMmaWarp = kFwdStatWarps + 1;           // TMEM owner + MMA issuer
constexpr int kFwdThreads = 32 * (kFwdStatWarps + 4);    // + TMA, MMA and two idle warps
// Registers after setmaxnreg: statistics / control warps (sum within the launch's pool).
// SKL_FWD_QTMEM: the query tiles are also copied into tensor memory, where the score MMAs
// read them as their A operand (an N = 64 MMA with both operands in shared memory is
// bound by shared-memory bandwidth); each query tile's score buffer is then single.
#ifndef SKL_FWD_QTMEM
#define SKL_FWD_QTMEM 1
#endif
static_assert(!SKL_FWD_QTMEM || SKL_FWD_SPLIT, "the Q copy into TMEM assumes split warps");

#ifndef SKL_FWD_RS
#define SKL_FWD_RS (SKL_FWD_SPLIT ? 104 : 200)
#endif
#ifndef SKL_FWD_RC
#define SKL_FWD_RC (SKL_FWD_SPLIT ? 56 : 104)
#endif
constexpr int kFwdRegsStat = SKL_FWD_RS;
constexpr int kFwdRegsCtrl = SKL_FWD_RC;
static_assert(kFwdStatWarps * kFwdRegsStat + 4 * kFwdRegsCtrl <=
                  (kFwdStatWarps + 4) * ((65536 / kFwdThreads) & ~7),
              "register split exceeds the launch's register pool");

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
  static constexpr int THREADS = kFwdThreads;
  // TMEM columns: score buffers (query tile q, buffer b), and with SKL_FWD_QTMEM the
  // query rows (Q_T: d_T/2 columns, Q_S: d_S/2 columns per query tile).
  static constexpr int NSB = SKL_FWD_QTMEM ? 1 : 2;
  static __device__ __forceinline__ int tm_s(int q, int b) { return (q * NSB + b % NSB) * 128; }
  static constexpr int TM_Q = NQ * NSB * 128;
  static __device__ __forceinline__ int tm_qt(int q) { return TM_Q + q * (DT + DS) / 2; }
  static __device__ __forceinline__ int tm_qs(int q) { return tm_qt(q) + DT / 2; }
  static_assert(!SKL_FWD_QTMEM || TM_Q + NQ * (DT + DS) / 2 <= 512, "TMEM budget");
  static_assert(NST >= 2, "key ring needs two stages");
  static_assert(SMEM <= SMEM_MAX, "shared memory budget");
};

// SKL_FWD_QORDER (single score buffer per query tile): per key tile the MMA thread serves
// first the query tile whose score buffer is already free, instead of always query tile 0.
#ifndef SKL_FWD_QORDER
#define SKL_FWD_QORDER 1
#endif

struct FwdBars {
  uint64_t q_full;
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t s_full[2][2];
  uint64_t s_free[2][2];
  uint64_t q_tmem;  // SKL_FWD_QTMEM: the query rows are in tensor memory
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(FwdBars) <= FwdCfg<128, 128>::BAR_BYTES,
              "barrier block exceeds its shared-memory reservation");

__device__ __forceinline__ void skl_fail(volatile int* abort_flag) {
  atomicOr(&g_skl_error, 1u);
  *abort_flag = 1;
}

// Online state of one query row over the keys one warpgroup has seen (base-2 units).
struct RowState {
  float mT, mS, lT, lS, A;
};

// Which column pairs (c, c+1) send their second exponential of both distributions to the
// FMA pipe: the first SKL_FWD_POLY entries of the order 1, 5, 3, 7, 6, 2, 4, 0 over every 8
// consecutive pairs, i.e. SKL_FWD_POLY/16 of all exponentials (1: 6.25 %).
#ifndef SKL_FWD_POLY
#define SKL_FWD_POLY 1
#endif
__host__ __device__ constexpr int poly_rank(int p) {
  return p == 1 ? 0 : p == 5 ? 1 : p == 3 ? 2 : p == 7 ? 3 : p == 6 ? 4 : p == 2 ? 5 : p == 4 ? 6 : 7;
}
__host__ __device__ constexpr bool poly_pair(int pair) {
  return poly_rank(pair & 7) < SKL_FWD_POLY;
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

// Accumulates 16 keys (v[tb..tb+15] teacher scores, v[sb..sb+15] student scores, raw dot
// products) into the packed partial sums. Columns c > lim are masked (MASK).
template <bool MASK, int N>
__device__ __forceinline__ void fold_part(const uint32_t (&v)[N], int tb, int sb, uint64_t cT2,
                                          uint64_t cS2, uint64_t nmT2, uint64_t nmS2, int lim,
                                          int pair0, uint64_t& sT2, uint64_t& sS2, uint64_t& b2) {
#pragma unroll
  for (int c = 0; c < 16; c += 2) {
    const uint64_t xT =
        f2_fma(f2_pack(__uint_as_float(v[tb + c]), __uint_as_float(v[tb + c + 1])), cT2, nmT2);
    const uint64_t xS =
        f2_fma(f2_pack(__uint_as_float(v[sb + c]), __uint_as_float(v[sb + c + 1])), cS2, nmS2);
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
  // One TMEM round trip for the whole tile (v[0..63] teacher, v[64..127] student); the
  // buffer is released at once, so the next tile's MMAs overlap all of the arithmetic.
  uint32_t v[128];
  tmem_ld_4x32_wait(ta, ta + 32, ta + 64, ta + 96, v);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(s_free);
  mxT = fmaxf(max_tree32<MASK>(v, 0, lim), max_tree32<MASK>(v, 32, lim - 32));
  mxS = fmaxf(max_tree32<MASK>(v, 64, lim), max_tree32<MASK>(v, 96, lim - 32));
  float mT_use, mS_use;
  update_max(st, mxT, mxS, cT, cS, mT_use, mS_use);
  const uint64_t cT2 = f2_pack(cT, cT), cS2 = f2_pack(cS, cS);
  const uint64_t nmT2 = f2_pack(-mT_use, -mT_use), nmS2 = f2_pack(-mS_use, -mS_use);
  uint64_t sT2 = f2_pack(0.f, 0.f), sS2 = sT2, b2 = sT2;
#pragma unroll
  for (int h = 0; h < 4; ++h)
    fold_part<MASK>(v, 16 * h, 64 + 16 * h, cT2, cS2, nmT2, nmS2, lim - 16 * h, 8 * h, sT2, sS2,
                    b2);
  float s0, s1, u0, u1, w0, w1;
  f2_unpack(sT2, s0, s1);
  f2_unpack(sS2, u0, u1);
  f2_unpack(b2, w0, w1);
  const float sumT = s0 + s1;
  st.lT += sumT;
  st.lS += u0 + u1;
  st.A += (w0 + w1) + (mT_use - mS_use) * sumT;
}

// Sums of one half tile (32 keys) against reference maxima (mT_use, mS_use):
// sumT = sum 2^(t - mT), sumS = sum 2^(s - mS), w = sum 2^(t - mT) * ((t - mT) - (s - mS)).
template <bool MASK>
__device__ __forceinline__ void half_sums(const uint32_t (&v)[64], float cT, float cS,
                                          float mT_use, float mS_use, int lim, float& sumT,
                                          float& sumS, float& w) {
  const uint64_t cT2 = f2_pack(cT, cT), cS2 = f2_pack(cS, cS);
  const uint64_t nmT2 = f2_pack(-mT_use, -mT_use), nmS2 = f2_pack(-mS_use, -mS_use);
  uint64_t sT2 = f2_pack(0.f, 0.f), sS2 = sT2, b2 = sT2;
#pragma unroll
  for (int h = 0; h < 2; ++h)
    fold_part<MASK>(v, 16 * h, 32 + 16 * h, cT2, cS2, nmT2, nmS2, lim - 16 * h, 8 * h, sT2, sS2,
                    b2);
  float s0, s1, u0, u1, w0, w1;
  f2_unpack(sT2, s0, s1);
  f2_unpack(sS2, u0, u1);
  f2_unpack(b2, w0, w1);
  sumT = s0 + s1;
  sumS = u0 + u1;
  w = w0 + w1;
}

// SKL_FWD_LAZY: an unmasked half tile is folded against the row's running maxima as they
// stand, without first taking the tile's maxima (the state is exact for any reference:
// l and A are sums relative to 2^m). The result is kept when every lane's tile sums stay
// below 2^64 (a score at most about 64 above the reference; false for inf and NaN);
// otherwise the tile is folded again the ordinary way. With fewer than 2^26 tiles per row
// the running sums then stay below 2^90, far from fp32 overflow. SKL_FWD_LAZY_RENORM
// additionally raises a reference by a sum's binary exponent k once the sum passes 2^32
// and scales the sums by 2^-k (exact).
#ifndef SKL_FWD_LAZY
#define SKL_FWD_LAZY 1
#endif
#ifndef SKL_FWD_LAZY_RENORM
#define SKL_FWD_LAZY_RENORM 0
#endif

__device__ __forceinline__ void lazy_renorm(float& m, float& l, float* a) {
  if (l >= 0x1p32f) {
    const int k = ((__float_as_int(l) >> 23) & 0xff) - 127;  // 32 .. 127
    const float sc = __int_as_float((127 - k) << 23);        // 2^-k, a normal number
    l *= sc;
    if (a) *a *= sc;
    m += (float)k;
  }
}

// Half a tile (32 keys: TMEM columns tT .. tT+31 teacher, tS .. tS+31 student) folded
// into the row state of one warp of a split pair; lim as in fold_tile, relative to the
// half's first key.
template <bool MASK>
__device__ __forceinline__ void fold_half(RowState& st, uint32_t tT, uint32_t tS, float cT,
                                          float cS, int lim, uint32_t s_free, int lane) {
  uint32_t v[64];
  tmem_ld_2x32_wait(tT, tS, v);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(s_free);
  float sumT, sumS, w;
#if SKL_FWD_LAZY
  if (!MASK && __all_sync(0xffffffffu, st.mT != -INFINITY && st.mS != -INFINITY)) {
    half_sums<false>(v, cT, cS, st.mT, st.mS, 31, sumT, sumS, w);
    if (__all_sync(0xffffffffu, sumT < 0x1p64f && sumS < 0x1p64f)) {
      st.lT += sumT;
      st.lS += sumS;
      st.A += w + (st.mT - st.mS) * sumT;
      if (SKL_FWD_LAZY_RENORM) {
        lazy_renorm(st.mT, st.lT, &st.A);
        lazy_renorm(st.mS, st.lS, nullptr);
      }
      return;
    }
  }
#endif
  const float mxT = max_tree32<MASK>(v, 0, lim), mxS = max_tree32<MASK>(v, 32, lim);
  float mT_use, mS_use;
  update_max(st, mxT, mxS, cT, cS, mT_use, mS_use);
  half_sums<MASK>(v, cT, cS, mT_use, mS_use, lim, sumT, sumS, w);
  st.lT += sumT;
  st.lS += sumS;
  st.A += w + (mT_use - mS_use) * sumT;
}

// Merge of two row states (rescale both to the larger maxima and add).
__device__ __forceinline__ void merge_state(RowState& a, const RowState& b) {
  const float nT = fmaxf(a.mT, b.mT), nS = fmaxf(a.mS, b.mS);
  const float uT = nT == -INFINITY ? 0.f : nT, uS = nS == -INFINITY ? 0.f : nS;
  const float aT = ex2_approx(a.mT - uT), bT = ex2_approx(b.mT - uT);
  const float aS = ex2_approx(a.mS - uS), bS = ex2_approx(b.mS - uS);
  a.lT = a.lT * aT + b.lT * bT;
  a.A = a.A * aT + b.A * bT;
  a.lS = a.lS * aS + b.lS * bS;
  a.mT = nT;
  a.mS = nS;
}

template <int DT, int DS>
__global__ void __launch_bounds__(kFwdThreads, 1)
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
    const int q = warp / (4 * kFwdHalves);           // query tile of this warp
    const int half = (warp >> 2) & (kFwdHalves - 1);  // key half of every tile (split)
    const int quarter = warp & 3;                     // TMEM lane quarter of this warp
    const int row = q0 + q * C::BM + quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float cT = args.cT, cS = args.cS;
    const int first_row = q0 + q * C::BM;

    RowState st{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
    bool ok = true;
#if SKL_FWD_QTMEM
    {
      // Query rows into tensor memory (A operand of the score MMAs): half 0 copies the
      // row of Q_T, half 1 the row of Q_S.
      const int r = quarter * 32 + lane;
      if (mbar_wait(smem_u32(&bars->q_full), 0)) {
        if (half == 0)
          row_to_tmem<DT>(s_qt + q * C::QT_TILE + r * 128, tmem + lane_off + C::tm_qt(q), r);
        else
          row_to_tmem<DS>(s_qs + q * C::QS_TILE + r * 128, tmem + lane_off + C::tm_qs(q), r);
      } else {
        skl_fail(abort_flag);
        ok = false;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->q_tmem));
    }
#endif
    for (int j = 0; ok && j < nk[q]; ++j) {
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
      const uint32_t ta = tmem + lane_off + C::tm_s(q, b);
      const uint32_t fr = smem_u32(&bars->s_free[q][b]);
      if (need_mask) {
        int last = seq.nk - 1;
        if (args.causal) last = min(last, row + seq.off);
#if SKL_FWD_SPLIT
        fold_half<true>(st, ta + 32 * half, ta + 64 + 32 * half, cT, cS, last - k0 - 32 * half,
                        fr, lane);
#else
        fold_tile<true>(st, ta, cT, cS, last - k0, fr, lane);
#endif
      } else {
#if SKL_FWD_SPLIT
        fold_half<false>(st, ta + 32 * half, ta + 64 + 32 * half, cT, cS, 31, fr, lane);
#else
        fold_tile<false>(st, ta, cT, cS, C::BN - 1, fr, lane);
#endif
      }
    }

#if SKL_FWD_SPLIT
    // Half 1 hands its row state to half 0 through this query tile's shared memory: it is
    // no longer read once the tile's MMAs have completed (the last s_full), and its TMA
    // load has landed (q_full; also covers a tile with no keys, never read by an MMA).
    float* xfer = reinterpret_cast<float*>(smem + q * C::QT_TILE);
    const int r = quarter * 32 + lane;
    if (half == 1) {
      if (!mbar_wait(smem_u32(&bars->q_full), 0)) {
        skl_fail(abort_flag);
        ok = false;
      }
      xfer[r] = st.mT;
      xfer[128 + r] = st.mS;
      xfer[256 + r] = st.lT;
      xfer[384 + r] = st.lS;
      xfer[512 + r] = st.A;
      xfer[640 + r] = ok ? 1.f : 0.f;
    }
    named_bar_sync(1 + q, 8 * 32);  // the 8 warps of query tile q
    if (half == 0) {
      const RowState other{xfer[r], xfer[128 + r], xfer[256 + r], xfer[384 + r], xfer[512 + r]};
      ok = ok && xfer[640 + r] != 0.f;
      merge_state(st, other);
    }
#endif

    if (ok && row < seq.nq && half == 0) {
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
    } else if (warp == kFwdMmaWarp) {
      // ------------------------------------------------------------- MMA issuer
      if (elect_one()) {
        bool ok = mbar_wait(smem_u32(&bars->q_full), 0);
#if SKL_FWD_QTMEM
        if (ok) ok = mbar_wait(smem_u32(&bars->q_tmem), 0);
#endif
        if (!ok) skl_fail(abort_flag);
        for (int j = 0; ok && j < nk_max; ++j) {
          const int s = j % C::NST;
          if (!mbar_wait(smem_u32(&bars->full[s]), (j / C::NST) & 1)) {
            skl_fail(abort_flag);
            break;
          }
          tc_fence_after();
          const uint32_t st = s_k + s * C::STAGE;
          int qfirst = 0;
#if SKL_FWD_QTMEM && SKL_FWD_QORDER
          static_assert(C::NQ == 2, "two query tiles per CTA");
          if (j > 0 && j < nk[0] && j < nk[1]) {
            const uint32_t par = ((j - 1) >> 1) & 1;
            if (!mbar_test(smem_u32(&bars->s_free[0][(j - 1) & 1]), par) &&
                mbar_test(smem_u32(&bars->s_free[1][(j - 1) & 1]), par))
              qfirst = 1;
          }
#endif
  #pragma unroll
          for (int qi = 0; qi < C::NQ; ++qi) {
            const int q = qi ^ qfirst;
            if (j >= nk[q]) continue;
            const int b = j & 1;
#if SKL_FWD_QTMEM
            // Single score buffer: free once tile j-1 has been read (per-parity barriers,
            // so every waiter sees each phase of its barrier in order).
            if (j > 0 && !mbar_wait(smem_u32(&bars->s_free[q][(j - 1) & 1]), ((j - 1) >> 1) & 1)) {
#else
            if (!mbar_wait(smem_u32(&bars->s_free[q][b]), ((j >> 1) & 1) ^ 1)) {
#endif
              skl_fail(abort_flag);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_t = tmem + C::tm_s(q, b);
            const uint32_t d_s = d_t + 64;
#if SKL_FWD_QTMEM
  #pragma unroll
            for (int kk = 0; kk < DT / 16; ++kk) {
              const uint64_t bd =
                  sdesc_sw128(st + (kk >> 2) * (C::BN * 128) + (kk & 3) * 32, 16, 1024);
              umma_bf16_ts(d_t, tmem + C::tm_qt(q) + kk * 8, bd, idesc_t, kk > 0);
            }
  #pragma unroll
            for (int kk = 0; kk < DS / 16; ++kk) {
              const uint64_t bd = sdesc_sw128(
                  st + C::KT_TILE + (kk >> 2) * (C::BN * 128) + (kk & 3) * 32, 16, 1024);
              umma_bf16_ts(d_s, tmem + C::tm_qs(q) + kk * 8, bd, idesc_s, kk > 0);
            }
#else
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
#endif
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
  if (warp == kFwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace skl
