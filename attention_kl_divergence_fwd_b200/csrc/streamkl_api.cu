// streamkl_api.cu - C ABI, argument checks and launch planner of the StreamKL library.
//
// The planner picks the kernel instantiation from (d_T, d_S), encodes the TMA tensor
// maps ([B*H, N, d] bf16, 128-byte swizzle, zero fill out of bounds so ragged N needs
// no padding), orders the grid so causal work is scheduled heaviest-first, and
// launches on the caller's stream. See include/streamkl.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "streamkl.h"
#include "fwd_kernel.cuh"
#include "bwd_kernel.cuh"

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

// 3-D map over a [BH, N, d] bf16 tensor: box of 64 columns (128 bytes) x rows x 1.
bool make_map(CUtensorMap* m, const void* base, int d, int n, int bh, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)bh};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n * d * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the fp32 [BH, N_Q, d] dQ accumulator: box of 32 columns x 64 rows x 1.
bool make_map_f32(CUtensorMap* m, void* base, int d, int n, int bh) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)bh};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)n * d * 4};
  const cuuint32_t box[3] = {32, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

streamkl_status check_common(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                             int B, int H, int N_Q, int N_K, int d_T, int d_S, float scale_T,
                             float scale_S) {
  if (!q_t || !k_t || !q_s || !k_s) return STREAMKL_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N_Q < 1 || N_K < 1) return STREAMKL_ERR_INVALID_ARG;
  if (!std::isfinite(scale_T) || !std::isfinite(scale_S)) return STREAMKL_ERR_INVALID_ARG;
  if ((d_T != 64 && d_T != 128) || (d_S != 64 && d_S != 128)) return STREAMKL_ERR_UNSUPPORTED;
  const long long bh = (long long)B * H;
  const long long nmax = N_Q > N_K ? N_Q : N_K;
  if (bh * nmax >= (1ll << 31) || bh >= (1ll << 24)) return STREAMKL_ERR_UNSUPPORTED;
  if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(q_s) || !aligned16(k_s))
    return STREAMKL_ERR_MISALIGNED;
  return STREAMKL_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

// Heads per scheduling group: small enough that a group's tiles stay in the 126 MB L2,
// large enough to fill the 148 SMs with a heaviest-first mix. Overridable for tuning
// through STREAMKL_FWD_GROUP / STREAMKL_BWD_GROUP.
int head_group(const char* env, int fallback, int bh) {
  int g = fallback;
  if (const char* v = std::getenv(env)) {
    const int x = std::atoi(v);
    if (x > 0) g = x;
  }
  return g < 1 ? 1 : (g > bh ? bh : g);
}

template <typename Kern>
bool set_smem(Kern k, int bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

template <int DT, int DS>
streamkl_status launch_fwd(const CUtensorMap* maps, const skl::FwdArgs& a, bool negT, bool negS,
                           cudaStream_t stream) {
  using C = skl::FwdCfg<DT, DS>;
  auto kern = skl::streamkl_fwd_kernel<DT, DS>;
  if (!set_smem(kern, C::SMEM)) return STREAMKL_ERR_LAUNCH;
  const uint32_t it = skl::idesc_bf16_f32(128, C::BN, false, false, negT);
  const uint32_t is = skl::idesc_bf16_f32(128, C::BN, false, false, negS);
  const long long grid = (long long)a.n_ctas_per_bh * a.BH;
  kern<<<dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, stream>>>(maps[0], maps[1], maps[2],
                                                                    maps[3], a, it, is);
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

// Query heads per K head; UNSUPPORTED unless it divides H.
bool kv_groups(int H, int H_kv_T, int H_kv_S, int& gT, int& gS) {
  if (H_kv_T < 1 || H_kv_S < 1 || H % H_kv_T != 0 || H % H_kv_S != 0) return false;
  gT = H / H_kv_T;
  gS = H / H_kv_S;
  return true;
}

streamkl_status fwd_common(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                           int B, int H, int H_kv_T, int H_kv_S, int N_Q, int N_K, int d_T,
                           int d_S, float scale_T, float scale_S, int causal, float* kl,
                           float* lse_t, float* lse_s, cudaStream_t stream) {
  streamkl_status st = check_common(q_t, k_t, q_s, k_s, B, H, N_Q, N_K, d_T, d_S, scale_T, scale_S);
  if (st != STREAMKL_OK) return st;
  if (!kl || !lse_t || !lse_s) return STREAMKL_ERR_INVALID_ARG;
  int gT, gS;
  if (!kv_groups(H, H_kv_T, H_kv_S, gT, gS)) return STREAMKL_ERR_UNSUPPORTED;
  if (!aligned16(kl) || !aligned16(lse_t) || !aligned16(lse_s)) return STREAMKL_ERR_MISALIGNED;
  const int bh = B * H;
  CUtensorMap maps[4];
  if (!make_map(&maps[0], q_t, d_T, N_Q, bh, 128) ||
      !make_map(&maps[1], k_t, d_T, N_K, B * H_kv_T, 64) ||
      !make_map(&maps[2], q_s, d_S, N_Q, bh, 128) ||
      !make_map(&maps[3], k_s, d_S, N_K, B * H_kv_S, 64))
    return STREAMKL_ERR_LAUNCH;
  skl::FwdArgs a{};
  a.BH = bh;
  a.N_Q = N_Q;
  a.N_K = N_K;
  a.causal = causal ? 1 : 0;
  a.off = N_K - N_Q;
  a.cT = std::fabs(scale_T) * kLog2e;
  a.cS = std::fabs(scale_S) * kLog2e;
  a.n_ctas_per_bh = (N_Q + 255) / 256;
  a.group = head_group("STREAMKL_FWD_GROUP", 4, bh);
  a.H = H;
  a.gT = gT;
  a.gS = gS;
  a.kl = kl;
  a.lse_t = lse_t;
  a.lse_s = lse_s;
  const bool nT = scale_T < 0.f, nS = scale_S < 0.f;
  if (d_T == 128 && d_S == 128) return launch_fwd<128, 128>(maps, a, nT, nS, stream);
  if (d_T == 128 && d_S == 64) return launch_fwd<128, 64>(maps, a, nT, nS, stream);
  if (d_T == 64 && d_S == 128) return launch_fwd<64, 128>(maps, a, nT, nS, stream);
  return launch_fwd<64, 64>(maps, a, nT, nS, stream);
}

// Shared body of the student and trainable-teacher backward entry points.
template <bool TEACHER>
streamkl_status bwd_common(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                           int B, int H, int H_kv_T, int H_kv_S, int N_Q, int N_K, int d_T,
                           int d_S, float scale_T, float scale_S, int causal, const float* kl,
                           const float* lse_t, const float* lse_s, const float* g, float* dq,
                           float* dk, cudaStream_t stream) {
  streamkl_status st = check_common(q_t, k_t, q_s, k_s, B, H, N_Q, N_K, d_T, d_S, scale_T, scale_S);
  if (st != STREAMKL_OK) return st;
  if (!lse_t || !lse_s || !g || !dq || !dk || (TEACHER && !kl)) return STREAMKL_ERR_INVALID_ARG;
  int gT, gS;
  if (!kv_groups(H, H_kv_T, H_kv_S, gT, gS)) return STREAMKL_ERR_UNSUPPORTED;
  if (!aligned16(lse_t) || !aligned16(lse_s) || !aligned16(g) || !aligned16(dq) ||
      !aligned16(dk) || (TEACHER && !aligned16(kl)))
    return STREAMKL_ERR_MISALIGNED;
  const int bh = B * H;
  const int d_g = TEACHER ? d_T : d_S;
  const int g_g = TEACHER ? gT : gS;       // query heads per differentiated K head
  const int bkv_g = B * (H / g_g);         // K heads of the differentiated side
  CUtensorMap maps[6];
  if (!make_map(&maps[0], q_t, d_T, N_Q, bh, 64) ||
      !make_map(&maps[1], k_t, d_T, N_K, B * H_kv_T, 128) ||
      !make_map(&maps[2], q_s, d_S, N_Q, bh, 64) ||
      !make_map(&maps[3], k_s, d_S, N_K, B * H_kv_S, 128) ||
      !make_map_f32(&maps[4], dq, d_g, N_Q, bh) || !make_map_f32(&maps[5], dk, d_g, N_K, bkv_g))
    return STREAMKL_ERR_LAUNCH;
  if (cudaMemsetAsync(dq, 0, (size_t)bh * N_Q * d_g * sizeof(float), stream) != cudaSuccess)
    return STREAMKL_ERR_LAUNCH;
  if (g_g > 1 &&
      cudaMemsetAsync(dk, 0, (size_t)bkv_g * N_K * d_g * sizeof(float), stream) != cudaSuccess)
    return STREAMKL_ERR_LAUNCH;
  skl::BwdArgs a{};
  a.BH = bh;
  a.N_Q = N_Q;
  a.N_K = N_K;
  a.causal = causal ? 1 : 0;
  a.off = N_K - N_Q;
  a.cT = std::fabs(scale_T) * kLog2e;
  a.cS = std::fabs(scale_S) * kLog2e;
  a.aT = std::fabs(scale_T);
  a.aS = std::fabs(scale_S);
  a.scale_G = TEACHER ? scale_T : scale_S;
  a.n_ktiles = (N_K + 127) / 128;
  a.n_qtiles = (N_Q + 63) / 64;
  a.group = head_group("STREAMKL_BWD_GROUP", 2, bh);
  a.H = H;
  a.gT = gT;
  a.gS = gS;
  a.dk_reduce = g_g > 1 ? 1 : 0;
  a.lse_t = lse_t;
  a.lse_s = lse_s;
  a.g = g;
  a.kl = kl;
  a.dq = dq;
  a.dk = dk;
  const bool nT = scale_T < 0.f, nS = scale_S < 0.f;
  if (d_T == 128 && d_S == 128) return launch_bwd<128, 128, TEACHER>(maps, a, nT, nS, stream);
  if (d_T == 128 && d_S == 64) return launch_bwd<128, 64, TEACHER>(maps, a, nT, nS, stream);
  if (d_T == 64 && d_S == 128) return launch_bwd<64, 128, TEACHER>(maps, a, nT, nS, stream);
  return launch_bwd<64, 64, TEACHER>(maps, a, nT, nS, stream);
}

}  // namespace

extern "C" {

streamkl_status streamkl_fwd(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                             int B, int H, int N_Q, int N_K, int d_T, int d_S, float scale_T,
                             float scale_S, int causal, float* kl, float* lse_t, float* lse_s,
                             cudaStream_t stream) {
  return fwd_common(q_t, k_t, q_s, k_s, B, H, H, H, N_Q, N_K, d_T, d_S, scale_T, scale_S, causal,
                    kl, lse_t, lse_s, stream);
}

streamkl_status streamkl_fwd_gqa(const void* q_t, const void* k_t, const void* q_s,
                                 const void* k_s, int B, int H, int H_kv_T, int H_kv_S, int N_Q,
                                 int N_K, int d_T, int d_S, float scale_T, float scale_S,
                                 int causal, float* kl, float* lse_t, float* lse_s,
                                 cudaStream_t stream) {
  return fwd_common(q_t, k_t, q_s, k_s, B, H, H_kv_T, H_kv_S, N_Q, N_K, d_T, d_S, scale_T,
                    scale_S, causal, kl, lse_t, lse_s, stream);
}

streamkl_status streamkl_bwd(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                             int B, int H, int N_Q, int N_K, int d_T, int d_S, float scale_T,
                             float scale_S, int causal, const float* lse_t, const float* lse_s,
                             const float* g, float* dq_s, float* dk_s, cudaStream_t stream) {
  return bwd_common<false>(q_t, k_t, q_s, k_s, B, H, H, H, N_Q, N_K, d_T, d_S, scale_T, scale_S,
                           causal, nullptr, lse_t, lse_s, g, dq_s, dk_s, stream);
}

streamkl_status streamkl_bwd_gqa(const void* q_t, const void* k_t, const void* q_s,
                                 const void* k_s, int B, int H, int H_kv_T, int H_kv_S, int N_Q,
                                 int N_K, int d_T, int d_S, float scale_T, float scale_S,
                                 int causal, const float* lse_t, const float* lse_s,
                                 const float* g, float* dq_s, float* dk_s, cudaStream_t stream) {
  return bwd_common<false>(q_t, k_t, q_s, k_s, B, H, H_kv_T, H_kv_S, N_Q, N_K, d_T, d_S, scale_T,
                           scale_S, causal, nullptr, lse_t, lse_s, g, dq_s, dk_s, stream);
}

streamkl_status streamkl_bwd_teacher(const void* q_t, const void* k_t, const void* q_s,
                                     const void* k_s, int B, int H, int N_Q, int N_K, int d_T,
                                     int d_S, float scale_T, float scale_S, int causal,
                                     const float* kl, const float* lse_t, const float* lse_s,
                                     const float* g, float* dq_t, float* dk_t,
                                     cudaStream_t stream) {
  return bwd_common<true>(q_t, k_t, q_s, k_s, B, H, H, H, N_Q, N_K, d_T, d_S, scale_T, scale_S,
                          causal, kl, lse_t, lse_s, g, dq_t, dk_t, stream);
}

streamkl_status streamkl_bwd_teacher_gqa(const void* q_t, const void* k_t, const void* q_s,
                                         const void* k_s, int B, int H, int H_kv_T, int H_kv_S,
                                         int N_Q, int N_K, int d_T, int d_S, float scale_T,
                                         float scale_S, int causal, const float* kl,
                                         const float* lse_t, const float* lse_s, const float* g,
                                         float* dq_t, float* dk_t, cudaStream_t stream) {
  return bwd_common<true>(q_t, k_t, q_s, k_s, B, H, H_kv_T, H_kv_S, N_Q, N_K, d_T, d_S, scale_T,
                          scale_S, causal, kl, lse_t, lse_s, g, dq_t, dk_t, stream);
}

const char* streamkl_status_string(streamkl_status s) {
  switch (s) {
    case STREAMKL_OK: return "ok";
    case STREAMKL_ERR_INVALID_ARG: return "invalid argument (null pointer, size < 1 or non-finite scale)";
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
    return STREAMKL_ERR_TIMEOUT;
  }
  return STREAMKL_OK;
}

int streamkl_version(void) { return 100; }

}  // extern "C"
