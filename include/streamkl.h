/*
 * streamkl.h - C ABI of the StreamKL attention-KL library for NVIDIA B200 (sm_100a).
 *
 * The operation ("StreamKL: Fast and Memory-Efficient KL Divergence for Boosting
 * Attention Distillation", abstract): for every batch b, head h and query row i,
 *
 *   s_T[i,j] = scale_T * <q_T[i], k_T[j]>,   s_S[i,j] = scale_S * <q_S[i], k_S[j]>
 *   J(i)     = { j < N_K : !causal || j <= i + N_K - N_Q }     (bottom-right causal)
 *   P_X[i,:] = softmax over J(i) of s_X[i,:]                   (X = T teacher, S student)
 *   KL[i]    = sum_{j in J(i)} P_T[i,j] * (log P_T[i,j] - log P_S[i,j])
 *
 * computed without materialising either N_Q x N_K matrix. The forward streams key
 * tiles past a resident query tile and keeps an online state per row (the abstract
 * describes a single forward pass that reduces both distributions together as the tiles
 * go by, with the tiles held on chip). The backward recomputes both probability tiles
 * from the saved log-sum-exps (in the abstract, the backward regenerates the
 * probabilities one tile at a time instead of storing them). streamkl_bwd gives the
 * student's gradients (teacher frozen, the abstract's setting); streamkl_bwd_teacher
 * gives a trainable teacher's.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All pointers are DEVICE pointers on the current CUDA device, owned by the caller.
 *   The library allocates no device memory. Extra device memory beyond the caller's
 *   inputs and outputs is O(1) (one error word per device); the only state passed
 *   from forward to backward is the caller's O(B*H*N_Q) row statistics.
 * - Layout: q_t [B,H,N_Q,d_T], k_t [B,H,N_K,d_T], q_s [B,H,N_Q,d_S], k_s [B,H,N_K,d_S],
 *   contiguous row-major bf16 (d innermost). Row statistics and g are contiguous fp32
 *   [B,H,N_Q]. Gradients are contiguous fp32.
 * - Supported: d_T, d_S in {64, 128}; B, H, N_Q, N_K >= 1; B*H*max(N_Q,N_K) < 2^31, B*H < 2^24;
 *   any finite scale_T, scale_S. N_Q and N_K need not be multiples of any tile size.
 * - Every input/output pointer must be 16-byte aligned.
 * - Calls are asynchronous on `stream`: argument checks happen on the host before any
 *   launch and return a status without touching device memory; launch failures are
 *   reported through cudaGetLastError as STREAMKL_ERR_LAUNCH. A kernel that hits its
 *   internal watchdog (a pipeline wait that exceeds its bound) stops early and records
 *   STREAMKL_ERR_TIMEOUT in a device-side error word, read with
 *   streamkl_device_status(); it never traps.
 * - Rows with an empty J(i) (only causal with N_Q > N_K) get KL = 0, LSE = -inf and a
 *   zero gradient. KL is reported unclamped (rounding can make it slightly negative).
 * - Scheduling: CTAs are ordered in groups of heads (L2 locality, heaviest causal tiles
 *   first). The environment variables STREAMKL_FWD_GROUP and STREAMKL_BWD_GROUP (positive
 *   integers, read once per process at the first call) override the group sizes, which otherwise follow a rule
 *   (4 heads forward, 2 backward, raised up to twice that until a group holds one wave of
 *   CTAs). They change only the speed: results are the same for any group size, except
 *   that dQ is summed in a different order (fp32 reduce-adds across CTAs).
 * - The dense forward runs as a persistent grid (one CTA per SM walking a heaviest-first
 *   snake of work units) when it has at most 8 units (pairs of 128-row query tiles) per SM,
 *   and as one CTA per unit otherwise; STREAMKL_FWD_PERSIST=0 / 1 (read once per process)
 *   forces the per-unit / persistent form. Both give bit-identical results.
 */
#ifndef STREAMKL_H
#define STREAMKL_H

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  STREAMKL_OK = 0,
  STREAMKL_ERR_INVALID_ARG = 1, /* null pointer, size out of range, non-finite scale,
                                   malformed packed-sequence offsets (device-detected) */
  STREAMKL_ERR_UNSUPPORTED = 2, /* head dim outside {64,128} or sizes beyond the limits */
  STREAMKL_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned */
  STREAMKL_ERR_LAUNCH = 4,      /* the CUDA runtime rejected a launch or a set-up call */
  STREAMKL_ERR_TIMEOUT = 5      /* a kernel watchdog fired (see streamkl_device_status) */
} streamkl_status;

/*
 * Forward. Online coupled statistics per query row (running maxima m_T, m_S, sums
 * l_T, l_S and A = sum_j 2^(t_T - m_T) (t_T - t_S) in base-2 units), finalised as
 *   LSE_X = ln2 * (m_X + log2 l_X),   KL = ln2 * A / l_T - LSE_T + LSE_S,
 * i.e. KL = E_{P_T}[s_T - s_S] - LSE_T + LSE_S.
 *
 * Outputs (caller-allocated fp32 [B,H,N_Q], fully overwritten):
 *   kl     per-row KL(P_T || P_S) in nats;
 *   lse_t  per-row natural-log log-sum-exp of s_T over J(i);
 *   lse_s  per-row natural-log log-sum-exp of s_S over J(i).
 * lse_t / lse_s are the only state streamkl_bwd needs.
 */
streamkl_status streamkl_fwd(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                             int B, int H, int N_Q, int N_K, int d_T, int d_S,
                             float scale_T, float scale_S, int causal,
                             float* kl, float* lse_t, float* lse_s, cudaStream_t stream);

/*
 * Backward (teacher frozen). With g[i] = dLoss/dKL[i] (fp32 [B,H,N_Q]) and the forward's
 * lse_t / lse_s, recomputes P_T = exp(s_T - LSE_T) and P_S = exp(s_S - LSE_S) tile by
 * tile and forms
 *   dS[i,j] = g[i] * scale_S * (P_S[i,j] - P_T[i,j])   on J(i), 0 elsewhere,
 *   dq_s = dS K_S   (fp32 [B,H,N_Q,d_S], fully overwritten: zeroed on `stream` first),
 *   dk_s = dS^T Q_S (fp32 [B,H,N_K,d_S], fully overwritten).
 * dq_s is accumulated with fp32 reductions in L2 (one partial per key tile), so its low
 * bits can differ between runs; dk_s is deterministic.
 */
streamkl_status streamkl_bwd(const void* q_t, const void* k_t, const void* q_s, const void* k_s,
                             int B, int H, int N_Q, int N_K, int d_T, int d_S,
                             float scale_T, float scale_S, int causal,
                             const float* lse_t, const float* lse_s, const float* g,
                             float* dq_s, float* dk_s, cudaStream_t stream);

/*
 * Backward for a trainable teacher (the abstract's use of the primitive is one-sided,
 * teacher frozen; this is the same recompute scheme for the other side). With the
 * student fixed, dKL_i/ds_T[i,j] = P_T[i,j] * ((s_T - s_S)[i,j] - E_i) where
 * E_i = sum_j P_T[i,j] (s_T - s_S)[i,j] = KL_i + LSE_T,i - LSE_S,i, so with g[i] = dLoss/dKL[i]:
 *   dS_T[i,j] = g[i] * scale_T * P_T[i,j] * ((s_T - s_S)[i,j] - E_i)   on J(i), else 0,
 *   dq_t = dS_T K_T (fp32 [B,H,N_Q,d_T], fully overwritten: zeroed on `stream` first),
 *   dk_t = dS_T^T Q_T (fp32 [B,H,N_K,d_T], fully overwritten).
 * kl, lse_t and lse_s are the forward's outputs (fp32 [B,H,N_Q]); everything else as in
 * streamkl_bwd. Call both backward entry points to train teacher and student together.
 */
streamkl_status streamkl_bwd_teacher(const void* q_t, const void* k_t, const void* q_s,
                                     const void* k_s, int B, int H, int N_Q, int N_K, int d_T,
                                     int d_S, float scale_T, float scale_S, int causal,
                                     const float* kl, const float* lse_t, const float* lse_s,
                                     const float* g, float* dq_t, float* dk_t,
                                     cudaStream_t stream);

/*
 * Grouped-query attention variants (several query heads share one K head; teacher and
 * student may group differently). Same operations and conventions as above, with
 *   k_t [B,H_kv_T,N_K,d_T], k_s [B,H_kv_S,N_K,d_S]; query head h reads teacher K head
 *   h / (H / H_kv_T) and student K head h / (H / H_kv_S); H_kv_T and H_kv_S must divide H
 *   (else STREAMKL_ERR_UNSUPPORTED).
 * Gradients of a shared K head are summed over the query heads of its group:
 *   dk_s [B,H_kv_S,N_K,d_S] (streamkl_bwd_gqa), dk_t [B,H_kv_T,N_K,d_T]
 *   (streamkl_bwd_teacher_gqa); when a group has more than one query head, dk is zeroed on
 *   `stream` and accumulated with fp32 reductions in L2 (low bits can vary between runs).
 * The entry points without the suffix are these with H_kv_T = H_kv_S = H.
 */
streamkl_status streamkl_fwd_gqa(const void* q_t, const void* k_t, const void* q_s,
                                 const void* k_s, int B, int H, int H_kv_T, int H_kv_S, int N_Q,
                                 int N_K, int d_T, int d_S, float scale_T, float scale_S,
                                 int causal, float* kl, float* lse_t, float* lse_s,
                                 cudaStream_t stream);

streamkl_status streamkl_bwd_gqa(const void* q_t, const void* k_t, const void* q_s,
                                 const void* k_s, int B, int H, int H_kv_T, int H_kv_S, int N_Q,
                                 int N_K, int d_T, int d_S, float scale_T, float scale_S,
                                 int causal, const float* lse_t, const float* lse_s,
                                 const float* g, float* dq_s, float* dk_s, cudaStream_t stream);

streamkl_status streamkl_bwd_teacher_gqa(const void* q_t, const void* k_t, const void* q_s,
                                         const void* k_s, int B, int H, int H_kv_T, int H_kv_S,
                                         int N_Q, int N_K, int d_T, int d_S, float scale_T,
                                         float scale_S, int causal, const float* kl,
                                         const float* lse_t, const float* lse_s, const float* g,
                                         float* dq_t, float* dk_t, cudaStream_t stream);

/*
 * Packed variable-length sequences (the "varlen" layout). B sequences of different
 * lengths are packed token-major into one tensor each:
 *   q_t [total_q,H,d_T], q_s [total_q,H,d_S], k_t [total_k,H_kv_T,d_T], k_s [total_k,H_kv_S,d_S]
 * (contiguous bf16; H_kv_* as in the GQA variants, H_kv = H for one K head per query head).
 * cu_seqlens_q / cu_seqlens_k are DEVICE int32 arrays of B+1 offsets (4-byte aligned):
 * sequence b owns query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and key rows
 * cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1. max_seqlen_q / max_seqlen_k bound every
 * sequence's length (they size the grid). Each sequence is its own problem: its queries
 * see only its keys, and causal alignment is bottom-right within the sequence
 * (j <= i + n_k(b) - n_q(b), with i, j counted from the sequence's first row).
 * Row statistics, kl and g are fp32 [H, total_q] (head-major); gradients are fp32 in the
 * packed shapes of Q and K of the differentiated side.
 * - Sequences may be empty; a sequence with queries but no keys gets KL = 0, LSE = -inf.
 * - total_q, total_k >= 0; H*total_q, H*total_k < 2^31. With total_q = 0 the forward
 *   writes nothing; the backward zeroes its outputs and launches nothing when total_q or
 *   total_k is 0.
 * - kl / lse_* rows that belong to no sequence are not written; dq / dk are zeroed on
 *   `stream` first, so their rows outside every sequence are 0. dk is accumulated with
 *   fp32 reductions in L2 when K heads are shared, as in the GQA variants.
 * - The offsets are read on the device. Offsets that are not 0 <= cu[b] <= cu[b+1] <= total
 *   or describe a sequence longer than max_seqlen_* make the kernels skip that sequence
 *   and record STREAMKL_ERR_INVALID_ARG in the device error word (streamkl_device_status).
 */
streamkl_status streamkl_fwd_varlen(const void* q_t, const void* k_t, const void* q_s,
                                    const void* k_s, const int* cu_seqlens_q,
                                    const int* cu_seqlens_k, int B, int H, int H_kv_T,
                                    int H_kv_S, int total_q, int total_k, int max_seqlen_q,
                                    int max_seqlen_k, int d_T, int d_S, float scale_T,
                                    float scale_S, int causal, float* kl, float* lse_t,
                                    float* lse_s, cudaStream_t stream);

streamkl_status streamkl_bwd_varlen(const void* q_t, const void* k_t, const void* q_s,
                                    const void* k_s, const int* cu_seqlens_q,
                                    const int* cu_seqlens_k, int B, int H, int H_kv_T,
                                    int H_kv_S, int total_q, int total_k, int max_seqlen_q,
                                    int max_seqlen_k, int d_T, int d_S, float scale_T,
                                    float scale_S, int causal, const float* lse_t,
                                    const float* lse_s, const float* g, float* dq_s,
                                    float* dk_s, cudaStream_t stream);

streamkl_status streamkl_bwd_teacher_varlen(
    const void* q_t, const void* k_t, const void* q_s, const void* k_s, const int* cu_seqlens_q,
    const int* cu_seqlens_k, int B, int H, int H_kv_T, int H_kv_S, int total_q, int total_k,
    int max_seqlen_q, int max_seqlen_k, int d_T, int d_S, float scale_T, float scale_S,
    int causal, const float* kl, const float* lse_t, const float* lse_s, const float* g,
    float* dq_t, float* dk_t, cudaStream_t stream);

/*
 * Context parallelism over N_K (keys of one sequence split across GPUs or passes). The
 * abstract's forward keeps an online per-row state; states of disjoint key ranges merge
 * associatively, so each shard runs the forward on its keys and a merge finalises.
 * Dense layout, grouped K heads allowed (H_kv_* as above); k_t / k_s hold only the shard's
 * keys: k_t [B,H_kv_T,N_K_shard,d_T], k_s [B,H_kv_S,N_K_shard,d_S]. Shard key j is global key
 * k_offset + j; causal alignment uses the global indices (j_global <= i + N_K_total - N_Q);
 * 0 <= k_offset, k_offset + N_K_shard <= N_K_total, N_K_shard >= 1 (else INVALID_ARG).
 *
 * streamkl_fwd_partial writes the row state of its shard, fp32 [5,B,H,N_Q], planes in
 * base-2 units (t_X = s_X * log2 e): m_T, m_S (maxima over the shard's allowed keys),
 * l_T, l_S (sum 2^(t_X - m_X)), A (sum 2^(t_T - m_T) (t_T - t_S)); a row that sees no key
 * of the shard gets m = -inf, l = 0, A = 0 (the identity of the merge).
 *
 * streamkl_merge_partial merges R such states, laid out [R,5,rows] (rows = B*H*N_Q, the
 * gathered states of all shards in any order), and writes kl, lse_t, lse_s [rows] exactly
 * as streamkl_fwd would for the whole key range (R = 1 reproduces it bit for bit).
 *
 * streamkl_bwd_shard / streamkl_bwd_teacher_shard take the merged (global) lse_t, lse_s
 * (and kl for the teacher) and g, and write the gradients of the shard's keys (dk, final)
 * and the shard's part of dq (fp32 [B,H,N_Q,d], zeroed first): the full dq is the sum of
 * the parts over all shards (an all-reduce across the shards' ranks).
 */
streamkl_status streamkl_fwd_partial(const void* q_t, const void* k_t, const void* q_s,
                                     const void* k_s, int B, int H, int H_kv_T, int H_kv_S,
                                     int N_Q, int N_K_shard, int k_offset, int N_K_total,
                                     int d_T, int d_S, float scale_T, float scale_S, int causal,
                                     float* state, cudaStream_t stream);

streamkl_status streamkl_merge_partial(const float* states, int R, long long rows, float* kl,
                                       float* lse_t, float* lse_s, cudaStream_t stream);

streamkl_status streamkl_bwd_shard(const void* q_t, const void* k_t, const void* q_s,
                                   const void* k_s, int B, int H, int H_kv_T, int H_kv_S,
                                   int N_Q, int N_K_shard, int k_offset, int N_K_total, int d_T,
                                   int d_S, float scale_T, float scale_S, int causal,
                                   const float* lse_t, const float* lse_s, const float* g,
                                   float* dq_s, float* dk_s, cudaStream_t stream);

streamkl_status streamkl_bwd_teacher_shard(const void* q_t, const void* k_t, const void* q_s,
                                           const void* k_s, int B, int H, int H_kv_T,
                                           int H_kv_S, int N_Q, int N_K_shard, int k_offset,
                                           int N_K_total, int d_T, int d_S, float scale_T,
                                           float scale_S, int causal, const float* kl,
                                           const float* lse_t, const float* lse_s,
                                           const float* g, float* dq_t, float* dk_t,
                                           cudaStream_t stream);

/*
 * Diagnostic: launches one thread that waits, with the library's bounded pipeline wait
 * (2 s), on a barrier nothing arrives on. After it gives up, streamkl_device_status(stream)
 * returns STREAMKL_ERR_TIMEOUT, exactly as for a kernel whose pipeline stalled, and the
 * context stays usable. Returns STREAMKL_OK when the launch succeeded.
 */
streamkl_status streamkl_watchdog_selftest(cudaStream_t stream);

/*
 * Diagnostic: the forward's FMA-pipe 2^x (range reduction with the 1.5*2^23 shifter, a
 * degree-5 minimax polynomial fitted for this library, the integer part added into the
 * exponent field) evaluated on n device floats x (n even), scalar form into y_scalar and
 * packed-pair form into y_pair. Arguments are clamped to [-125, 64]: inputs below give
 * 2^-125, inputs above give 2^64. INVALID_ARG for null pointers or odd n.
 */
streamkl_status streamkl_exp2_eval(const float* x, float* y_scalar, float* y_pair, long long n,
                                   cudaStream_t stream);

/*
 * Diagnostic: one warp spins for about `ns` nanoseconds (1e3 .. 1e7) of the GPU's global
 * timer and writes, to the device array out[2] (caller-owned int64), the SM clock ticks
 * that passed (clock64) and the nanoseconds measured; out[0] / out[1] is the SM clock in
 * GHz at that moment. Asynchronous on `stream`. INVALID_ARG for a null pointer or `ns`
 * outside its range.
 */
streamkl_status streamkl_sm_clock_probe(long long* out, long long ns, cudaStream_t stream);

/* Static description of a status code (never NULL). */
const char* streamkl_status_string(streamkl_status status);

/*
 * Synchronises `stream`, then reads and clears the current device's error word.
 * Returns STREAMKL_OK, STREAMKL_ERR_INVALID_ARG if a varlen kernel found malformed
 * sequence offsets, STREAMKL_ERR_TIMEOUT if a kernel watchdog fired since the last call,
 * or STREAMKL_ERR_LAUNCH if the stream reports a CUDA error.
 */
streamkl_status streamkl_device_status(cudaStream_t stream);

/* Library version as major*10000 + minor*100 + patch. */
int streamkl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STREAMKL_H */
