// ptx.cuh - inline-PTX wrappers for sm_100a used by the StreamKL kernels.
//
// mbarriers (with bounded waits), TMA tensor loads (no multicast), tcgen05
// tensor-memory allocation / MMA / loads, shared-memory matrix descriptors and a
// few math helpers. Every wait here is bounded: it gives up after a time limit and
// reports failure to the caller, which records a device error and unwinds.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace skl {

// Device-side error word of this library (one per device, in the library's module):
// bit 0 = a forward watchdog fired, bit 1 = a backward watchdog fired, bit 2 = the
// dynamic shared memory was not 1024-byte aligned, bit 3 = malformed packed-sequence
// offsets, bit 4 = the watchdog self-test's wait expired. Read and cleared by
// streamkl_device_status(). The library is built as one translation unit, so this is the
// only definition.
__device__ unsigned int g_skl_error = 0;

// ----------------------------------------------------------------- misc

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n .reg .pred p;\n elect.sync _|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(pred));
  return pred != 0;
}

// ------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity. A healthy pipeline step takes
// microseconds; the limit only exists so that a broken pipeline cannot hang the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr uint32_t kWaitLimitIters = 1u << 30;

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < kWaitLimitIters; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0u && global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
  return false;
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled bulk tensor load global -> shared, completion on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Make generic-proxy shared-memory writes visible to the async proxy (tensor core).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// -------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulate; one thread issues.
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same two MMA forms with each shared-memory descriptor passed as its two 32-bit
// halves (the low half = start address and leading offset varies per call, the high half
// is the same for every descriptor of a kernel), so that an issuing thread forms each
// descriptor with one add.
__device__ __forceinline__ void umma_bf16_ss_lh(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                                uint32_t hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n .reg .b64 ad, bd;\n mov.b64 ad, {%1, %3};\n mov.b64 bd, {%2, %3};\n"
      " setp.ne.b32 p, %5, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %4, p;\n}\n" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_bf16_ts_lh(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                                uint32_t hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n .reg .b64 bd;\n mov.b64 bd, {%2, %3};\n setp.ne.b32 p, %5, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: A is read from tensor memory (rows on lanes, two bf16
// per 32-bit column, K-major), B through its shared-memory descriptor.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 columns of this warp's 32 lanes: registers -> tensor memory (no wait).
__device__ __forceinline__ void tmem_st_32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 8 columns of this warp's 32 lanes: registers -> tensor memory (no wait).
__device__ __forceinline__ void tmem_st_8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Row r of a [D/64][128 rows][128 B] bf16 tile in shared memory (128-byte swizzle, as TMA
// writes it) into 32-bit TMEM columns dst .. dst+D/2-1 of this thread's lane, two bf16 per
// column in K order: the layout of an MMA A operand read from tensor memory.
__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                             uint32_t& d);
template <int D>
__device__ __forceinline__ void row_to_tmem(uint32_t src_row, uint32_t dst, int r) {
#pragma unroll
  for (int blk = 0; blk < D / 64; ++blk) {
    uint32_t v[32];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      ld_shared_v4(src_row + blk * (128 * 128) + ((c ^ (r & 7)) << 4), v[4 * c], v[4 * c + 1],
                   v[4 * c + 2], v[4 * c + 3]);
    tmem_st_32(dst + blk * 32, v);
  }
  tmem_st_wait();
}

// Arrive once on `bar` when every tcgen05 op issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format (1 = bf16),
//   13 negate A, 15 A major (1 = MN), 16 B major (1 = MN), 17-22 N>>3, 24-28 M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn, bool b_mn,
                                                      bool neg_a = false) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((neg_a ? 1u : 0u) << 13) |
         ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
//   bits 0-13 start>>4, 16-29 leading byte offset>>4, 32-45 stride byte offset>>4,
//   46-47 version (1), 61-63 layout (2 = 128B swizzle).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// The two halves of sdesc_sw128: the low half holds the start address (bits 0-13, the
// address >> 4; shared addresses stay below 2^18, so adding a byte offset >> 4 to the low
// half never carries out of the field) and the leading byte offset (bits 16-29).
__host__ __device__ constexpr uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ constexpr uint32_t sdesc_hi(uint32_t sbo) {
  return ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}

// ------------------------------------------------------- TMEM -> registers

#define SKL_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), \
                  "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])

// Two 32-column loads (lanes = this warp's quarter) followed by the wait, in one
// asm statement so that no use of the outputs can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_2x32_wait(uint32_t ta, uint32_t tb, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : SKL_R8(0), SKL_R8(8), SKL_R8(16), SKL_R8(24), SKL_R8(32), SKL_R8(40), SKL_R8(48),
        SKL_R8(56)
      : "r"(ta), "r"(tb)
      : "memory");
}

// Four 32-column loads followed by one wait (one round trip for 128 columns).
__device__ __forceinline__ void tmem_ld_4x32_wait(uint32_t ta, uint32_t tb, uint32_t tc,
                                                  uint32_t td, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%128];\n"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%129];\n"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95}, [%130];\n"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
      "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%131];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : SKL_R8(0), SKL_R8(8), SKL_R8(16), SKL_R8(24), SKL_R8(32), SKL_R8(40), SKL_R8(48),
        SKL_R8(56), SKL_R8(64), SKL_R8(72), SKL_R8(80), SKL_R8(88), SKL_R8(96), SKL_R8(104),
        SKL_R8(112), SKL_R8(120)
      : "r"(ta), "r"(tb), "r"(tc), "r"(td)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_8_wait(uint32_t ta, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : SKL_R8(0)
      : "r"(ta)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_16_wait(uint32_t ta, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : SKL_R8(0), SKL_R8(8)
      : "r"(ta)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_32_wait(uint32_t ta, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : SKL_R8(0), SKL_R8(8), SKL_R8(16), SKL_R8(24)
      : "r"(ta)
      : "memory");
}

#undef SKL_R8

// ------------------------------------------------------- grid ordering

// Maps a linear CTA index to (head, unit) with heads processed in groups of `group`
// heads: inside a group the units are interleaved across its heads in the order given
// (unit 0 first, the caller puts the heaviest causal unit first), and groups follow one
// another. A group's working set (its heads' K/Q tiles and dQ rows) then stays in L2.
__device__ __forceinline__ void grouped_order(int t, int bh_total, int units, int group,
                                              int& bh, int& unit) {
  const int full = bh_total / group;
  const int per_group = group * units;
  const int g = t / per_group;
  if (g < full) {
    const int r = t - g * per_group;
    unit = r / group;
    bh = g * group + r % group;
  } else {
    const int rest = bh_total - full * group;
    const int r = t - full * per_group;
    unit = r / rest;
    bh = full * group + r % rest;
  }
}

// ------------------------------------------------------------ sequence view
//
// One CTA works on one (sequence, query head) problem. Two tensor layouts:
//  * dense  [B, H, N, d]: every sequence has N_Q queries and N_K keys; the TMA maps are
//    {d, N, B*heads} and the row arrays (KL, LSE, g) are [B*H, N_Q];
//  * packed [total, heads, d] with cu_q / cu_k offsets ([B+1] int32 in device memory):
//    sequence b owns rows cu[b] .. cu[b+1]-1; the TMA maps are {d, total, heads} and the
//    row arrays are [H, total_q]. N_Q / N_K are then the longest sequence lengths.
// Query head h reads teacher K head h/gT and student K head h/gS (grouped-query attention).
struct SeqView {
  int nq, nk;         // queries and keys of this sequence
  int off;            // nk - nq (bottom-right causal alignment within the sequence)
  int qr, kr;         // row of the sequence's first query / key in the tensor maps
  int zq, zkt, zks;   // head coordinate of Q, K_T, K_S in the tensor maps
  long long ob;       // index of the sequence's query row 0 in the row arrays
};

// Returns false when the packed offsets of this sequence are malformed (not
// 0 <= cu[b] <= cu[b+1] <= total, or longer than the longest length given).
// off_adj shifts the causal alignment of a dense problem whose keys are one shard of a
// longer sequence (context parallelism): shard key j is global key k_offset + j and
// off_adj = N_K_total - N_K_shard - k_offset; 0 otherwise.
__device__ __forceinline__ bool seq_view(const int* cu_q, const int* cu_k, int bh, int H,
                                         int gT, int gS, int N_Q, int N_K, int total_q,
                                         int total_k, int off_adj, SeqView& v) {
  const int b = bh / H, h = bh - b * H;
  if (cu_q == nullptr) {
    v.nq = N_Q;
    v.nk = N_K;
    v.qr = 0;
    v.kr = 0;
    v.zq = bh;
    v.zkt = b * (H / gT) + h / gT;
    v.zks = b * (H / gS) + h / gS;
    v.ob = (long long)bh * N_Q;
    v.off = N_K - N_Q + off_adj;
  } else {
    const int q_lo = __ldg(cu_q + b), q_hi = __ldg(cu_q + b + 1);
    const int k_lo = __ldg(cu_k + b), k_hi = __ldg(cu_k + b + 1);
    if (q_lo < 0 || q_hi < q_lo || q_hi > total_q || q_hi - q_lo > N_Q) return false;
    if (k_lo < 0 || k_hi < k_lo || k_hi > total_k || k_hi - k_lo > N_K) return false;
    v.nq = q_hi - q_lo;
    v.nk = k_hi - k_lo;
    v.qr = q_lo;
    v.kr = k_lo;
    v.zq = h;
    v.zkt = h / gT;
    v.zks = h / gS;
    v.ob = (long long)h * total_q + q_lo;
    v.off = v.nk - v.nq;
  }
  return true;
}

// KL and the two natural-log log-sum-exps of one query row from its online state in
// base-2 units: running maxima m_T, m_S, sums l_X = sum 2^(t_X - m_X) and
// A = sum 2^(t_T - m_T) (t_T - t_S). A row with no allowed key (l_T = 0) gets KL = 0 and
// LSE = -inf. Grouped so that identical teacher and student statistics give exactly 0.
__device__ __forceinline__ void finalize_row(float mT, float mS, float lT, float lS, float A,
                                             float& kl, float& lse_t, float& lse_s) {
  const float LN2 = 0.69314718055994530942f;
  if (lT > 0.f) {
    const float l2T = log2f(lT), l2S = log2f(lS);
    lse_t = LN2 * (mT + l2T);
    lse_s = LN2 * (mS + l2S);
    kl = LN2 * ((A / lT) + ((mS - mT) + (l2S - l2T)));
  } else {
    kl = 0.f;
    lse_t = -INFINITY;
    lse_s = -INFINITY;
  }
}

// Error word bit for malformed packed-sequence offsets (found on the device).
constexpr unsigned int kErrBadOffsets = 8u;

// ------------------------------------------------------------------ math

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Maximum of v[base..base+31] (as floats) as a shallow tree of three-input max
// instructions; with MASK, entries past `lim` count as -inf.
template <bool MASK, int N>
__device__ __forceinline__ float max_tree32(const uint32_t (&v)[N], int base, int lim) {
  auto at = [&](int c) -> float {
    return (!MASK || c <= lim) ? __uint_as_float(v[base + c]) : -INFINITY;
  };
  float l1[12];
#pragma unroll
  for (int i = 0; i < 10; ++i) l1[i] = fmax3(at(3 * i), at(3 * i + 1), at(3 * i + 2));
  l1[10] = at(30);
  l1[11] = at(31);
  const float l2a = fmax3(l1[0], l1[1], l1[2]), l2b = fmax3(l1[3], l1[4], l1[5]);
  const float l2c = fmax3(l1[6], l1[7], l1[8]), l2d = fmax3(l1[9], l1[10], l1[11]);
  return fmaxf(fmax3(l2a, l2b, l2c), l2d);
}

// 2^x on the FMA pipe for x in [-125, 64] (arguments are clamped to that range: below, 2^-125,
// which callers only add to sums that are at least 1; above, 2^64, which the forward's
// stale-reference fold reads as too large). Method: Cody-Waite style range reduction
// x = n + f, n = round-to-nearest(x) taken with the 1.5*2^23 shifter, f in [-1/2, 1/2];
// 2^f from a degree-5 polynomial fitted by this project (minimax relative error on
// [-1/2, 1/2] by linear programming, see fit_exp2_poly.py): max relative error 1.9e-7
// in fp32 Horner form; n is added straight into the exponent field.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fminf(fmaxf(x, -125.0f), 64.0f);
  const float kShift = 12582912.0f;
  const float y = __fadd_rn(x, kShift);
  const float f = __fsub_rn(x, __fsub_rn(y, kShift));
  float p = 0.001325405784882605f;
  p = fmaf(p, f, 0.00967527274042368f);
  p = fmaf(p, f, 0.055507827550172806f);
  p = fmaf(p, f, 0.2402212917804718f);
  p = fmaf(p, f, 0.6931469440460205f);
  p = fmaf(p, f, 1.0000001192092896f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(y) << 23));
}

// ---- packed fp32 pairs (one instruction for two lanes of work on sm_100)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// exp2_fma on a packed pair: same steps, the fp32 arithmetic issued as f32x2.
__device__ __forceinline__ uint64_t exp2_fma2(uint64_t x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  x = f2_pack(fminf(fmaxf(x0, -125.0f), 64.0f), fminf(fmaxf(x1, -125.0f), 64.0f));
  const uint64_t kShift = f2_pack(12582912.0f, 12582912.0f);
  const uint64_t y = f2_add(x, kShift);
  const uint64_t f = f2_sub(x, f2_sub(y, kShift));
  uint64_t p = f2_pack(0.001325405784882605f, 0.001325405784882605f);
  p = f2_fma(p, f, f2_pack(0.00967527274042368f, 0.00967527274042368f));
  p = f2_fma(p, f, f2_pack(0.055507827550172806f, 0.055507827550172806f));
  p = f2_fma(p, f, f2_pack(0.2402212917804718f, 0.2402212917804718f));
  p = f2_fma(p, f, f2_pack(0.6931469440460205f, 0.6931469440460205f));
  p = f2_fma(p, f, f2_pack(1.0000001192092896f, 1.0000001192092896f));
  float p0, p1, y0, y1;
  f2_unpack(p, p0, p1);
  f2_unpack(y, y0, y1);
  return f2_pack(__int_as_float(__float_as_int(p0) + (__float_as_int(y0) << 23)),
                 __int_as_float(__float_as_int(p1) + (__float_as_int(y1) << 23)));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                             uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Bulk tensor reduce-add shared -> global (fp32 add performed at L2), tracked by the
// issuing thread's bulk group.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, uint32_t src, int c0,
                                                  int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until every committed bulk group of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Wait until at most one committed bulk group of this thread is still reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Wait until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Per-warpgroup register budget changes (every warp of the warpgroup executes them).
// The kernels using them launch 12 warps at 168 registers and move registers from the
// control warpgroup to the two compute warpgroups, keeping the total: 4*104 + 8*200 = 12*168.
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Named barrier over `count` threads that also returns to every participant whether any of
// them passed pred = true (one uniform decision for all of them).
__device__ __forceinline__ bool named_bar_any(uint32_t id, uint32_t count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %3, 0;\n"
      " barrier.cta.red.or.pred q, %1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(id), "r"(count), "r"(pred ? 1u : 0u)
      : "memory");
  return r != 0;
}

// Named barrier over `count` threads (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace skl
