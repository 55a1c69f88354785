// streamkl_api.cu - C ABI, argument checks and launch planner of the StreamKL library.
//
// The planner picks the kernel instantiation from (d_T, d_S), encodes the TMA tensor
// maps (dense [B*H, N, d] or packed [total, heads, d] bf16, 128-byte swizzle, zero fill
// out of bounds so ragged N needs no padding), orders the grid so causal work is
// scheduled heaviest-first, and launches on the caller's stream. include/streamkl.h
// states the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "streamkl.h"
#include "fwd_kernel.cuh"
#include "fwd_persistent.cuh"
#include "bwd_kernel.cuh"
#include "merge_kernel.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 map {d, rows, heads}: box of 64 columns (128 bytes) x box_rows x 1 head.
// Dense [BH, N, d]: rows = N with stride d, heads = BH with stride N*d. Packed
// [total, heads, d]: rows = total with stride heads*d, heads with stride d.
bool make_map(CUtensorMap* m, const void* base, int d, long long rows, long long heads,
              long long row_stride, long long head_stride, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)head_stride * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same over an fp32 dQ / dK accumulator: box of 32 columns x 64 rows x 1 head.
bool make_map_f32(CUtensorMap* m, void* base, int d, long long rows, long long heads,
                  long long row_stride, long long head_stride) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)row_stride * 4, (cuuint64_t)head_stride * 4};
  const cuuint32_t box[3] = {32, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One call's problem: dense [B, H, N, d] tensors (cu_q == nullptr) or packed sequences.
struct Problem {
  const int* cu_q = nullptr;  // packed: [B+1] query / key offsets in device memory
  const int* cu_k = nullptr;
  int B = 0, H = 0, H_kv_T = 0, H_kv_S = 0;
  int N_Q = 0, N_K = 0;          // dense sizes; packed: longest query / key sequence
  int total_q = 0, total_k = 0;  // packed: rows of the packed Q / K tensors
  int off_adj = 0;               // dense key shard: N_K_total - N_K - k_offset
  bool packed() const { return cu_q != nullptr; }
  long long q_rows() const { return packed() ? total_q : (long long)B * H * N_Q; }
  long long k_rows(int h_kv) const { return packed() ? total_k : (long long)B * h_kv * N_K; }
};

// Map over a Q (h_kv = 0: H heads) or K tensor of the problem.
bool map_of(CUtensorMap* m, const void* base, const Problem& P, int d, bool is_k, int h_kv,
            int box_rows) {
  const int heads = is_k ? h_kv : P.H;
  if (P.packed()) {
    const long long rows = is_k ? P.total_k : P.total_q;
    // A packed K with no rows is never read (every sequence has no keys); the caller then
    // passes Q's base, and the map covers one row of it (Q has at least as many heads).
    if (rows == 0) return make_map(m, base, d, 1, heads, (long long)P.H * d, d, box_rows);
    return make_map(m, base, d, rows, heads, (long long)heads * d, d, box_rows);
  }
  const int n = is_k ? P.N_K : P.N_Q;
  return make_map(m, base, d, n, (long long)P.B * heads, d, (long long)n * d, box_rows);
}

bool map_of_f32(CUtensorMap* m, void* base, const Problem& P, int d, bool is_k, int h_kv) {
  const int heads = is_k ? h_kv : P.H;
  if (P.packed()) {
    const long long rows = is_k ? P.total_k : P.total_q;
    return make_map_f32(m, base, d, rows < 1 ? 1 : rows, heads, (long long)heads * d, d);
  }
  const int n = is_k ? P.N_K : P.N_Q;
  return make_map_f32(m, base, d, n, (long long)P.B * heads, d, (long long)n * d);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

streamkl_status check_common(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                             const Problem& P, int d_T, int d_S, float scale_T, float scale_S) {
  if (P.B < 1 || P.H < 1) return STREAMKL_ERR_INVALID_ARG;
  if (!std::isfinite(scale_T) || !std::isfinite(scale_S)) return STREAMKL_ERR_INVALID_ARG;
  if ((d_T != 64 && d_T != 128) || (d_S != 64 && d_S != 128)) return STREAMKL_ERR_UNSUPPORTED;
  if (P.H_kv_T < 1 || P.H_kv_S < 1 || P.H % P.H_kv_T != 0 || P.H % P.H_kv_S != 0)
    return STREAMKL_ERR_UNSUPPORTED;
  const long long bh = (long long)P.B * P.H;
  if (bh >= (1ll << 24)) return STREAMKL_ERR_UNSUPPORTED;
  if (P.packed()) {
    if (!P.cu_k || P.N_Q < 0 || P.N_K < 0 || P.total_q < 0 || P.total_k < 0)
      return STREAMKL_ERR_INVALID_ARG;
    if ((long long)P.H * P.total_q >= (1ll << 31) || (long long)P.H * P.total_k >= (1ll << 31))
      return STREAMKL_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(P.cu_q) & 3u) || (reinterpret_cast<uintptr_t>(P.cu_k) & 3u))
      return STREAMKL_ERR_MISALIGNED;
    if (P.total_q > 0 && (!q_t || !q_s)) return STREAMKL_ERR_INVALID_ARG;
    if (P.total_k > 0 && (!k_t || !k_s)) return STREAMKL_ERR_INVALID_ARG;
  } else {
    if (!q_t || !k_t || !q_s || !k_s) return STREAMKL_ERR_INVALID_ARG;
    if (P.N_Q < 1 || P.N_K < 1) return STREAMKL_ERR_INVALID_ARG;
    const long long nmax = P.N_Q > P.N_K ? P.N_Q : P.N_K;
    if (bh * nmax >= (1ll << 31)) return STREAMKL_ERR_UNSUPPORTED;
  }
  if ((q_t && !aligned16(q_t)) || (k_t && !aligned16(k_t)) || (q_s && !aligned16(q_s)) ||
      (k_s && !aligned16(k_s)))
    return STREAMKL_ERR_MISALIGNED;
  return STREAMKL_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

// Streaming multiprocessors of the current device (queried once per device; host threads
// that race on the first query store the same value).
int sm_count() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// A positive integer from the environment, else 0.
int env_positive(const char* name) {
  const char* v = std::getenv(name);
  const int x = v ? std::atoi(v) : 0;
  return x > 0 ? x : 0;
}

// Tuning overrides of the head-group sizes, read once per process (thread-safe static
// initialisation); 0 = no override.
int group_override(bool fwd) {
  static const int f = env_positive("STREAMKL_FWD_GROUP");
  static const int b = env_positive("STREAMKL_BWD_GROUP");
  return fwd ? f : b;
}

// Forward grid form for a dense problem of `units` work units: persistent (one CTA per SM
// walking a heaviest-first snake of units) when there are at most kPersistRounds units per
// SM. There the per-CTA prologue and the tail of a one-CTA-per-unit grid are a visible part
// of the launch, and all of the heads' key tiles are few enough to share L2; with more units
// per SM the head-grouped grid keeps each group's key tiles in L2. STREAMKL_FWD_PERSIST
// (read once) overrides: 0 never, 1 always (dense problems).
constexpr int kPersistRounds = 8;
#ifndef SKL_FWD_PERSIST_MODE
#define SKL_FWD_PERSIST_MODE -1  // -1: by the rule above
#endif
bool fwd_persistent(long long units) {
  static const int mode = [] {
    const char* v = std::getenv("STREAMKL_FWD_PERSIST");
    return v ? std::atoi(v) : SKL_FWD_PERSIST_MODE;
  }();
  if (mode == 0) return false;
  if (mode == 1) return true;
  return units <= (long long)kPersistRounds * sm_count();
}

#ifndef SKL_FWD_GROUP_BASE
#define SKL_FWD_GROUP_BASE 4
#endif
#ifndef SKL_BWD_GROUP_BASE
#define SKL_BWD_GROUP_BASE 2
#endif

// Heads per scheduling group: small enough that a group's tiles stay in the 126 MB L2,
// large enough to fill the SMs with a heaviest-first mix. The base size is raised (up to
// twice) until one group holds at least a wave of CTAs, so that short sequences, with few
// CTAs per head, do not leave a tail of heavy causal tiles (measured at N = 4096:
// +16 % forward, +7 % backward; unchanged for long sequences). Overridable for tuning
// through STREAMKL_FWD_GROUP / STREAMKL_BWD_GROUP (read once, at the first call).
int head_group(bool fwd, int base, int bh, int units_per_head) {
  int g = base;
  if (units_per_head > 0) {
    const int wave = (sm_count() + units_per_head - 1) / units_per_head;
    g = wave > g ? (wave < 2 * base ? wave : 2 * base) : g;
  }
  if (const int x = group_override(fwd)) g = x;
  return g < 1 ? 1 : (g > bh ? bh : g);
}

template <typename Kern>
bool set_smem(Kern k, int bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

template <int DT, int DS>
streamkl_status launch_fwd(const CUtensorMap* maps, const skl::FwdArgs& a, bool negT, bool negS,
                           bool persistent, cudaStream_t stream) {
  using C = skl::FwdCfg<DT, DS>;
  const uint32_t it = skl::idesc_bf16_f32(128, C::BN, false, false, negT);
  const uint32_t is = skl::idesc_bf16_f32(128, C::BN, false, false, negS);
  const long long units = (long long)a.n_ctas_per_bh * a.BH;
  if (persistent) {
    auto kern = skl::streamkl_fwd_persistent_kernel<DT, DS>;
    if (!set_smem(kern, C::SMEM)) return STREAMKL_ERR_LAUNCH;
    const long long grid = units < sm_count() ? units : sm_count();
    kern<<<dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, stream>>>(maps[0], maps[1], maps[2],
                                                                      maps[3], a, it, is);
  } else {
    auto kern = skl::streamkl_fwd_kernel<DT, DS>;
    if (!set_smem(kern, C::SMEM)) return STREAMKL_ERR_LAUNCH;
    kern<<<dim3((unsigned)units), dim3(C::THREADS), C::SMEM, stream>>>(maps[0], maps[1], maps[2],
                                                                       maps[3], a, it, is);
  }
  return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_LAUNCH;
}

template <int DT, int DS, bool TEACHER>
streamkl_status launch_bwd(const CUtensorMap* maps, const skl::BwdArgs& a, bool negT, bool negS,
                           cudaStream_t stream) {
  using C = skl::BwdCfg<DT, DS, TEACHER>;
  auto kern = skl::streamkl_bwd_kernel<DT, DS, TEACHER>;
  if (!set_smem(kern, C::SMEM)) return STREAMKL_ERR_LAUNCH;
  const uint32_t i_st = skl::idesc_bf16_f32(128, C::BM, false, false, negT);
  const uint32_t i_ss = skl::idesc_bf16_f32(128, C::BM, false, false, negS);
  const uint32_t i_dk = skl::idesc_bf16_f32(128, C::DG, false, true);   // dS^T Q
  const uint32_t i_dq = skl::idesc_bf16_f32(C::DG, C::BM, true, true);  // K^T dS^T
  const long long grid = (long long)a.n_ktiles * a.BH;
  kern<<<dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, stream>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], a, i_st, i_ss, i_dk, i_dq);
  return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_LAUNCH;
}

// With state != nullptr the forward writes the raw row state (context parallelism)
// instead of KL / LSE.
streamkl_status fwd_common(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                           const Problem& P, int d_T, int d_S, float scale_T, float scale_S,
                           int causal, float* kl, float* lse_t, float* lse_s,
                           cudaStream_t stream, float* state = nullptr) {
  streamkl_status st = check_common(q_t, k_t, q_s, k_s, P, d_T, d_S, scale_T, scale_S);
  if (st != STREAMKL_OK) return st;
  if (P.q_rows() == 0) return STREAMKL_OK;  // packed, no query rows: nothing to write
  if (state) {
    if (!aligned16(state)) return STREAMKL_ERR_MISALIGNED;
  } else {
    if (!kl || !lse_t || !lse_s) return STREAMKL_ERR_INVALID_ARG;
    if (!aligned16(kl) || !aligned16(lse_t) || !aligned16(lse_s))
      return STREAMKL_ERR_MISALIGNED;
  }
  const bool no_keys = P.packed() && P.total_k == 0;
  CUtensorMap maps[4];
  if (!map_of(&maps[0], q_t, P, d_T, false, 0, 128) ||
      !map_of(&maps[1], no_keys ? q_t : k_t, P, d_T, true, P.H_kv_T, 64) ||
      !map_of(&maps[2], q_s, P, d_S, false, 0, 128) ||
      !map_of(&maps[3], no_keys ? q_s : k_s, P, d_S, true, P.H_kv_S, 64))
    return STREAMKL_ERR_LAUNCH;
  const int bh = P.B * P.H;
  skl::FwdArgs a{};
  a.BH = bh;
  a.N_Q = P.N_Q;
  a.N_K = P.N_K;
  a.causal = causal ? 1 : 0;
  a.cT = std::fabs(scale_T) * kLog2e;
  a.cS = std::fabs(scale_S) * kLog2e;
  a.n_ctas_per_bh = (P.N_Q + 255) / 256;
  a.group = head_group(true, SKL_FWD_GROUP_BASE, bh, a.n_ctas_per_bh);
  a.H = P.H;
  a.gT = P.H / P.H_kv_T;
  a.gS = P.H / P.H_kv_S;
  a.cu_q = P.cu_q;
  a.cu_k = P.cu_k;
  a.total_q = P.total_q;
  a.total_k = P.total_k;
  a.off_adj = P.off_adj;
  a.state = state;
  a.plane = (long long)bh * P.N_Q;
  a.kl = kl;
  a.lse_t = lse_t;
  a.lse_s = lse_s;
  if (a.n_ctas_per_bh == 0) return STREAMKL_OK;  // packed, every sequence empty
  const bool nT = scale_T < 0.f, nS = scale_S < 0.f;
  const bool pers = !P.packed() && fwd_persistent((long long)a.n_ctas_per_bh * bh);
  if (d_T == 128 && d_S == 128) return launch_fwd<128, 128>(maps, a, nT, nS, pers, stream);
  if (d_T == 128 && d_S == 64) return launch_fwd<128, 64>(maps, a, nT, nS, pers, stream);
  if (d_T == 64 && d_S == 128) return launch_fwd<64, 128>(maps, a, nT, nS, pers, stream);
  return launch_fwd<64, 64>(maps, a, nT, nS, pers, stream);
}

// Shared body of the student and trainable-teacher backward entry points.
template <bool TEACHER>
streamkl_status bwd_common(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                           const Problem& P, int d_T, int d_S, float scale_T, float scale_S,
                           int causal, const float* kl, const float* lse_t, const float* lse_s,
                           const float* g, float* dq, float* dk, cudaStream_t stream) {
  streamkl_status st = check_common(q_t, k_t, q_s, k_s, P, d_T, d_S, scale_T, scale_S);
  if (st != STREAMKL_OK) return st;
  const int d_g = TEACHER ? d_T : d_S;
  const int h_kv_g = TEACHER ? P.H_kv_T : P.H_kv_S;  // K heads of the differentiated side
  const long long dq_elems = P.q_rows() * (P.packed() ? (long long)P.H * d_g : d_g);
  const long long dk_elems = P.k_rows(h_kv_g) * (P.packed() ? (long long)h_kv_g * d_g : d_g);
  if ((dq_elems > 0 && !dq) || (dk_elems > 0 && !dk)) return STREAMKL_ERR_INVALID_ARG;
  if ((dq && !aligned16(dq)) || (dk && !aligned16(dk))) return STREAMKL_ERR_MISALIGNED;
  const bool launch = dq_elems > 0 && dk_elems > 0;  // packed: some rows and some keys
  if (launch) {
    if (!lse_t || !lse_s || !g || (TEACHER && !kl)) return STREAMKL_ERR_INVALID_ARG;
    if (!aligned16(lse_t) || !aligned16(lse_s) || !aligned16(g) || (TEACHER && !aligned16(kl)))
      return STREAMKL_ERR_MISALIGNED;
  }
  // dQ is accumulated with reduce-adds; dK too when K heads are shared, and packed dK rows
  // outside every sequence are never written, so those outputs start from zero.
  const bool dk_reduce = P.H / h_kv_g > 1;
  if (dq_elems > 0 && cudaMemsetAsync(dq, 0, dq_elems * sizeof(float), stream) != cudaSuccess)
    return STREAMKL_ERR_LAUNCH;
  if (dk_elems > 0 && (dk_reduce || P.packed() || !launch) &&
      cudaMemsetAsync(dk, 0, dk_elems * sizeof(float), stream) != cudaSuccess)
    return STREAMKL_ERR_LAUNCH;
  if (!launch) return STREAMKL_OK;
  CUtensorMap maps[6];
  if (!map_of(&maps[0], q_t, P, d_T, false, 0, 64) ||
      !map_of(&maps[1], k_t, P, d_T, true, P.H_kv_T, 128) ||
      !map_of(&maps[2], q_s, P, d_S, false, 0, 64) ||
      !map_of(&maps[3], k_s, P, d_S, true, P.H_kv_S, 128) ||
      !map_of_f32(&maps[4], dq, P, d_g, false, 0) ||
      !map_of_f32(&maps[5], dk, P, d_g, true, h_kv_g))
    return STREAMKL_ERR_LAUNCH;
  const int bh = P.B * P.H;
  skl::BwdArgs a{};
  a.BH = bh;
  a.N_Q = P.N_Q;
  a.N_K = P.N_K;
  a.causal = causal ? 1 : 0;
  a.cT = std::fabs(scale_T) * kLog2e;
  a.cS = std::fabs(scale_S) * kLog2e;
  a.aT = std::fabs(scale_T);
  a.aS = std::fabs(scale_S);
  a.scale_G = TEACHER ? scale_T : scale_S;
  a.n_ktiles = (P.N_K + 127) / 128;
  a.group = head_group(false, SKL_BWD_GROUP_BASE, bh, a.n_ktiles);
  a.H = P.H;
  a.gT = P.H / P.H_kv_T;
  a.gS = P.H / P.H_kv_S;
  a.dk_reduce = dk_reduce ? 1 : 0;
  a.cu_q = P.cu_q;
  a.cu_k = P.cu_k;
  a.total_q = P.total_q;
  a.total_k = P.total_k;
  a.dk_hs = P.packed() ? d_g : (long long)P.N_K * d_g;
  a.dk_rs = P.packed() ? (long long)h_kv_g * d_g : d_g;
  a.off_adj = P.off_adj;
  a.lse_t = lse_t;
  a.lse_s = lse_s;
  a.g = g;
  a.kl = kl;
  a.dq = dq;
  a.dk = dk;
  if (a.n_ktiles == 0) return STREAMKL_OK;  // packed, every sequence without keys
  const bool nT = scale_T < 0.f, nS = scale_S < 0.f;
  if (d_T == 128 && d_S == 128) return launch_bwd<128, 128, TEACHER>(maps, a, nT, nS, stream);
  if (d_T == 128 && d_S == 64) return launch_bwd<128, 64, TEACHER>(maps, a, nT, nS, stream);
  if (d_T == 64 && d_S == 128) return launch_bwd<64, 128, TEACHER>(maps, a, nT, nS, stream);
  return launch_bwd<64, 64, TEACHER>(maps, a, nT, nS, stream);
}

Problem dense(int B, int H, int H_kv_T, int H_kv_S, int N_Q, int N_K) {
  Problem P;
  P.B = B;
  P.H = H;
  P.H_kv_T = H_kv_T;
  P.H_kv_S = H_kv_S;
  P.N_Q = N_Q;
  P.N_K = N_K;
  return P;
}

// Dense problem whose keys are one shard [k_offset, k_offset + N_K) of N_K_total keys.
bool shard(Problem& P, int k_offset, int N_K_total) {
  if (k_offset < 0 || N_K_total < 1 || (long long)k_offset + P.N_K > N_K_total) return false;
  P.off_adj = N_K_total - P.N_K - k_offset;
  return true;
}

Problem packed(const int* cu_q, const int* cu_k, int B, int H, int H_kv_T, int H_kv_S,
               int total_q, int total_k, int max_q, int max_k) {
  Problem P = dense(B, H, H_kv_T, H_kv_S, max_q, max_k);
  P.total_q = total_q;
  P.total_k = total_k;
  P.cu_q = cu_q;  // non-null: the entry points reject null offsets before this
  P.cu_k = cu_k;
  return P;
}

}  // namespace

extern "C" {

streamkl_status streamkl_fwd(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                             int B, int H, int N_Q, int N_K, int d_T, int d_S, float scale_T,
                             float scale_S, int causal, float* kl, float* lse_t, float* lse_s,
                             cudaStream_t stream) {
  return fwd_common(q_t, k_t, q_s, k_s, dense(B, H, H, H, N_Q, N_K), d_T, d_S, scale_T, scale_S,
                    causal, kl, lse_t, lse_s, stream);
}

streamkl_status streamkl_fwd_gqa(const void* q_t, const void* k_t, const void* q_s,
                                 const void* k_s, int B, int H, int H_kv_T, int H_kv_S, int N_Q,
                                 int N_K, int d_T, int d_S, float scale_T, float scale_S,
                                 int causal, float* kl, float* lse_t, float* lse_s,
                                 cudaStream_t stream) {
  return fwd_common(q_t, k_t, q_s, k_s, dense(B, H, H_kv_T, H_kv_S, N_Q, N_K), d_T, d_S,
                    scale_T, scale_S, causal, kl, lse_t, lse_s, stream);
}

streamkl_status streamkl_fwd_varlen(const void* q_t, const void* k_t, const void* q_s,
                                    const void* k_s, const int* cu_seqlens_q,
                                    const int* cu_seqlens_k, int B, int H, int H_kv_T,
                                    int H_kv_S, int total_q, int total_k, int max_seqlen_q,
                                    int max_seqlen_k, int d_T, int d_S, float scale_T,
                                    float scale_S, int causal, float* kl, float* lse_t,
                                    float* lse_s, cudaStream_t stream) {
  if (!cu_seqlens_q || !cu_seqlens_k) return STREAMKL_ERR_INVALID_ARG;
  return fwd_common(q_t, k_t, q_s, k_s,
                    packed(cu_seqlens_q, cu_seqlens_k, B, H, H_kv_T, H_kv_S, total_q, total_k,
                           max_seqlen_q, max_seqlen_k),
                    d_T, d_S, scale_T, scale_S, causal, kl, lse_t, lse_s, stream);
}

streamkl_status streamkl_bwd(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                             int B, int H, int N_Q, int N_K, int d_T, int d_S, float scale_T,
                             float scale_S, int causal, const float* lse_t, const float* lse_s,
                             const float* g, float* dq_s, float* dk_s, cudaStream_t stream) {
  return bwd_common<false>(q_t, k_t, q_s, k_s, dense(B, H, H, H, N_Q, N_K), d_T, d_S, scale_T,
                           scale_S, causal, nullptr, lse_t, lse_s, g, dq_s, dk_s, stream);
}

streamkl_status streamkl_bwd_gqa(const void* q_t, const void* k_t, const void* q_s,
                                 const void* k_s, int B, int H, int H_kv_T, int H_kv_S, int N_Q,
                                 int N_K, int d_T, int d_S, float scale_T, float scale_S,
                                 int causal, const float* lse_t, const float* lse_s,
                                 const float* g, float* dq_s, float* dk_s, cudaStream_t stream) {
  return bwd_common<false>(q_t, k_t, q_s, k_s, dense(B, H, H_kv_T, H_kv_S, N_Q, N_K), d_T, d_S,
                           scale_T, scale_S, causal, nullptr, lse_t, lse_s, g, dq_s, dk_s,
                           stream);
}

streamkl_status streamkl_bwd_varlen(const void* q_t, const void* k_t, const void* q_s,
                                    const void* k_s, const int* cu_seqlens_q,
                                    const int* cu_seqlens_k, int B, int H, int H_kv_T,
                                    int H_kv_S, int total_q, int total_k, int max_seqlen_q,
                                    int max_seqlen_k, int d_T, int d_S, float scale_T,
                                    float scale_S, int causal, const float* lse_t,
                                    const float* lse_s, const float* g, float* dq_s,
                                    float* dk_s, cudaStream_t stream) {
  if (!cu_seqlens_q || !cu_seqlens_k) return STREAMKL_ERR_INVALID_ARG;
  return bwd_common<false>(q_t, k_t, q_s, k_s,
                           packed(cu_seqlens_q, cu_seqlens_k, B, H, H_kv_T, H_kv_S, total_q,
                                  total_k, max_seqlen_q, max_seqlen_k),
                           d_T, d_S, scale_T, scale_S, causal, nullptr, lse_t, lse_s, g, dq_s,
                           dk_s, stream);
}

streamkl_status streamkl_bwd_teacher(const void* q_t, const void* k_t, const void* q_s,
                                     const void* k_s, int B, int H, int N_Q, int N_K, int d_T,
                                     int d_S, float scale_T, float scale_S, int causal,
                                     const float* kl, const float* lse_t, const float* lse_s,
                                     const float* g, float* dq_t, float* dk_t,
                                     cudaStream_t stream) {
  return bwd_common<true>(q_t, k_t, q_s, k_s, dense(B, H, H, H, N_Q, N_K), d_T, d_S, scale_T,
                          scale_S, causal, kl, lse_t, lse_s, g, dq_t, dk_t, stream);
}

streamkl_status streamkl_bwd_teacher_gqa(const void* q_t, const void* k_t, const void* q_s,
                                         const void* k_s, int B, int H, int H_kv_T, int H_kv_S,
                                         int N_Q, int N_K, int d_T, int d_S, float scale_T,
                                         float scale_S, int causal, const float* kl,
                                         const float* lse_t, const float* lse_s, const float* g,
                                         float* dq_t, float* dk_t, cudaStream_t stream) {
  return bwd_common<true>(q_t, k_t, q_s, k_s, dense(B, H, H_kv_T, H_kv_S, N_Q, N_K), d_T, d_S,
                          scale_T, scale_S, causal, kl, lse_t, lse_s, g, dq_t, dk_t, stream);
}

streamkl_status streamkl_bwd_teacher_varlen(
    const void* q_t, const void* k_t, const void* q_s, const void* k_s, const int* cu_seqlens_q,
    const int* cu_seqlens_k, int B, int H, int H_kv_T, int H_kv_S, int total_q, int total_k,
    int max_seqlen_q, int max_seqlen_k, int d_T, int d_S, float scale_T, float scale_S,
    int causal, const float* kl, const float* lse_t, const float* lse_s, const float* g,
    float* dq_t, float* dk_t, cudaStream_t stream) {
  if (!cu_seqlens_q || !cu_seqlens_k) return STREAMKL_ERR_INVALID_ARG;
  return bwd_common<true>(q_t, k_t, q_s, k_s,
                          packed(cu_seqlens_q, cu_seqlens_k, B, H, H_kv_T, H_kv_S, total_q,
                                 total_k, max_seqlen_q, max_seqlen_k),
                          d_T, d_S, scale_T, scale_S, causal, kl, lse_t, lse_s, g, dq_t, dk_t,
                          stream);
}

streamkl_status streamkl_fwd_partial(const void* q_t, const void* k_t, const void* q_s,
                                     const void* k_s, int B, int H, int H_kv_T, int H_kv_S,
                                     int N_Q, int N_K_shard, int k_offset, int N_K_total,
                                     int d_T, int d_S, float scale_T, float scale_S, int causal,
                                     float* state, cudaStream_t stream) {
  Problem P = dense(B, H, H_kv_T, H_kv_S, N_Q, N_K_shard);
  if (!state || N_K_shard < 1 || !shard(P, k_offset, N_K_total)) return STREAMKL_ERR_INVALID_ARG;
  return fwd_common(q_t, k_t, q_s, k_s, P, d_T, d_S, scale_T, scale_S, causal, nullptr, nullptr,
                    nullptr, stream, state);
}

streamkl_status streamkl_merge_partial(const float* states, int R, long long rows, float* kl,
                                       float* lse_t, float* lse_s, cudaStream_t stream) {
  if (!states || !kl || !lse_t || !lse_s || R < 1 || rows < 1) return STREAMKL_ERR_INVALID_ARG;
  if ((long long)R * 5 * rows >= (1ll << 40)) return STREAMKL_ERR_UNSUPPORTED;
  if (!aligned16(states) || !aligned16(kl) || !aligned16(lse_t) || !aligned16(lse_s))
    return STREAMKL_ERR_MISALIGNED;
  // Enough 256-thread blocks to cover every row, at most 16 per SM of the 148.
  const long long need = (rows + 255) / 256;
  const unsigned grid = (unsigned)(need < 148 * 16 ? need : 148 * 16);
  skl::streamkl_merge_kernel<<<grid, 256, 0, stream>>>(states, R, rows, kl, lse_t, lse_s);
  return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_LAUNCH;
}

streamkl_status streamkl_bwd_shard(const void* q_t, const void* k_t, const void* q_s,
                                   const void* k_s, int B, int H, int H_kv_T, int H_kv_S,
                                   int N_Q, int N_K_shard, int k_offset, int N_K_total, int d_T,
                                   int d_S, float scale_T, float scale_S, int causal,
                                   const float* lse_t, const float* lse_s, const float* g,
                                   float* dq_s, float* dk_s, cudaStream_t stream) {
  Problem P = dense(B, H, H_kv_T, H_kv_S, N_Q, N_K_shard);
  if (N_K_shard < 1 || !shard(P, k_offset, N_K_total)) return STREAMKL_ERR_INVALID_ARG;
  return bwd_common<false>(q_t, k_t, q_s, k_s, P, d_T, d_S, scale_T, scale_S, causal, nullptr,
                           lse_t, lse_s, g, dq_s, dk_s, stream);
}

streamkl_status streamkl_bwd_teacher_shard(const void* q_t, const void* k_t, const void* q_s,
                                           const void* k_s, int B, int H, int H_kv_T,
                                           int H_kv_S, int N_Q, int N_K_shard, int k_offset,
                                           int N_K_total, int d_T, int d_S, float scale_T,
                                           float scale_S, int causal, const float* kl,
                                           const float* lse_t, const float* lse_s,
                                           const float* g, float* dq_t, float* dk_t,
                                           cudaStream_t stream) {
  Problem P = dense(B, H, H_kv_T, H_kv_S, N_Q, N_K_shard);
  if (N_K_shard < 1 || !shard(P, k_offset, N_K_total)) return STREAMKL_ERR_INVALID_ARG;
  return bwd_common<true>(q_t, k_t, q_s, k_s, P, d_T, d_S, scale_T, scale_S, causal, kl, lse_t,
                          lse_s, g, dq_t, dk_t, stream);
}

streamkl_status streamkl_watchdog_selftest(cudaStream_t stream) {
  skl::streamkl_watchdog_kernel<<<1, 32, 0, stream>>>();
  return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_LAUNCH;
}

streamkl_status streamkl_exp2_eval(const float* x, float* y_scalar, float* y_pair, long long n,
                                   cudaStream_t stream) {
  if (!x || !y_scalar || !y_pair || n < 2 || (n & 1)) return STREAMKL_ERR_INVALID_ARG;
  const long long pairs = n / 2;
  const long long need = (pairs + 255) / 256;
  const unsigned grid = (unsigned)(need < 148 * 16 ? need : 148 * 16);
  skl::streamkl_exp2_kernel<<<grid, 256, 0, stream>>>(x, y_scalar, y_pair, n);
  return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_LAUNCH;
}

streamkl_status streamkl_sm_clock_probe(long long* out, long long ns, cudaStream_t stream) {
  if (!out || ns < 1000 || ns > 10000000) return STREAMKL_ERR_INVALID_ARG;
  skl::streamkl_clock_kernel<<<1, 32, 0, stream>>>(out, ns);
  return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_LAUNCH;
}

const char* streamkl_status_string(streamkl_status s) {
  switch (s) {
    case STREAMKL_OK: return "ok";
    case STREAMKL_ERR_INVALID_ARG: return "invalid argument (null pointer, size out of range, non-finite scale or malformed packed-sequence offsets)";
    case STREAMKL_ERR_UNSUPPORTED: return "unsupported shape (head dims must be 64 or 128; sizes beyond limits)";
    case STREAMKL_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case STREAMKL_ERR_LAUNCH: return "CUDA runtime error during set-up or launch";
    case STREAMKL_ERR_TIMEOUT: return "kernel watchdog fired (pipeline wait exceeded its bound)";
  }
  return "unknown status";
}

streamkl_status streamkl_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return STREAMKL_ERR_LAUNCH;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, skl::g_skl_error, sizeof(v)) != cudaSuccess)
    return STREAMKL_ERR_LAUNCH;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(skl::g_skl_error, &zero, sizeof(zero)) != cudaSuccess)
      return STREAMKL_ERR_LAUNCH;
    // Malformed packed offsets are an argument error found on the device; every other
    // bit is a watchdog (or the never-expected shared-memory alignment check).
    return v == skl::kErrBadOffsets ? STREAMKL_ERR_INVALID_ARG : STREAMKL_ERR_TIMEOUT;
  }
  return STREAMKL_OK;
}

int streamkl_version(void) { return 200; }

}  // extern "C"
