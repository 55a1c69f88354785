// merge_kernel.cuh - merge of per-row StreamKL states from several key shards.
//
// Context parallelism over N_K splits the keys of a sequence into contiguous shards; the
// forward of each shard leaves, per query row, the online state of the one-pass
// reduction ("StreamKL: Fast and Memory-Efficient KL Divergence for Boosting Attention
// Distillation", abstract: both distributions are reduced together, online, in one
// pass): maxima m_T, m_S and sums l_T, l_S, A in base-2 units. States combine by
// rescaling to the larger maximum and adding, so R shard states merge into the state of
// the whole key range, which is then finalised exactly as the one-pass forward does.
//
// One thread per query row, a grid-stride loop; each state plane is read once, coalesced.
// Bound: HBM (20 R + 12 bytes per row).
#pragma once

#include "ptx.cuh"

namespace skl {

// states: [R][5][rows] fp32 (planes m_T, m_S, l_T, l_S, A); outputs [rows].
__global__ void __launch_bounds__(256)
streamkl_merge_kernel(const float* __restrict__ states, int R, long long rows,
                      float* __restrict__ kl, float* __restrict__ lse_t,
                      float* __restrict__ lse_s) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += stride) {
    float mT = -INFINITY, mS = -INFINITY, lT = 0.f, lS = 0.f, A = 0.f;
    for (int r = 0; r < R; ++r) {
      const float* p = states + (long long)r * 5 * rows + i;
      const float rmT = __ldg(p), rmS = __ldg(p + rows);
      const float rlT = __ldg(p + 2 * rows), rlS = __ldg(p + 3 * rows), rA = __ldg(p + 4 * rows);
      const float nT = fmaxf(mT, rmT), nS = fmaxf(mS, rmS);
      const float uT = nT == -INFINITY ? 0.f : nT;  // reference while every max is -inf
      const float uS = nS == -INFINITY ? 0.f : nS;
      const float wT0 = exp2f(mT - uT), wT1 = exp2f(rmT - uT);  // -inf - x -> 0
      const float wS0 = exp2f(mS - uS), wS1 = exp2f(rmS - uS);
      lT = lT * wT0 + rlT * wT1;
      A = A * wT0 + rA * wT1;
      lS = lS * wS0 + rlS * wS1;
      mT = nT;
      mS = nS;
    }
    float k, a, b;
    finalize_row(mT, mS, lT, lS, A, k, a, b);
    kl[i] = k;
    lse_t[i] = a;
    lse_s[i] = b;
  }
}

// Watchdog self-test: one thread waits, through the same bounded wait as every pipeline
// wait of the library, on an mbarrier that nothing arrives on. The wait gives up after its
// time limit and the error word records it, exactly as a stalled pipeline would.
__global__ void streamkl_watchdog_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    if (!mbar_wait(smem_u32(&bar), 0)) atomicOr(&g_skl_error, 16u);
  }
}

// Evaluates the FMA-pipe exp2 (scalar and packed-pair forms) on n inputs, for checking it
// against the exact 2^x and CUDA's exp2f. n is even; one thread per pair.
__global__ void streamkl_exp2_kernel(const float* __restrict__ x, float* __restrict__ y1,
                                     float* __restrict__ y2, long long n) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; 2 * k < n; k += stride) {
    const float a = x[2 * k], b = x[2 * k + 1];
    y1[2 * k] = exp2_fma(a);
    y1[2 * k + 1] = exp2_fma(b);
    float p, q;
    f2_unpack(exp2_fma2(f2_pack(a, b)), p, q);
    y2[2 * k] = p;
    y2[2 * k + 1] = q;
  }
}

// SM clock probe: one warp spins for about `ns` nanoseconds of the global timer and
// records the SM clock ticks (clock64) that passed meanwhile and the nanoseconds themselves;
// ticks / ns is the clock the SM actually ran at, which NVML's sampled clock can miss.
__global__ void streamkl_clock_kernel(long long* __restrict__ out, long long ns) {
  const uint64_t t0 = global_timer_ns();
  const long long c0 = clock64();
  uint64_t t1 = t0;
  while ((long long)(t1 - t0) < ns) t1 = global_timer_ns();
  const long long c1 = clock64();
  if (threadIdx.x == 0) {
    out[0] = c1 - c0;
    out[1] = (long long)(t1 - t0);
  }
}

}  // namespace skl
