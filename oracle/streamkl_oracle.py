"""fp64 CPU oracle for the StreamKL attention-KL primitive.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import or call this
module; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` do. It shares no code with the CUDA library.

What it computes ("StreamKL: Fast and Memory-Efficient KL Divergence for
Boosting Attention Distillation", abstract): attention distillation minimises
the row-wise KL divergence between a teacher attention distribution and a
student attention distribution. Written out for one (batch, head):

    s_T[i, j] = scale_T * <q_T[i], k_T[j]>        s_S[i, j] = scale_S * <q_S[i], k_S[j]>
    J(i)      = { j < N_K : not causal  or  j <= i + N_K - N_Q }   (bottom-right causal)
    P_X[i, :] = softmax over J(i) of s_X[i, :]                      (X = T, S)
    KL[i]     = sum_{j in J(i)} P_T[i, j] * (log P_T[i, j] - log P_S[i, j])
    LSE_X[i]  = log sum_{j in J(i)} exp(s_X[i, j])

The method's claim is that it is exact (it removes the materialisation, not the
arithmetic), so the oracle *does* materialise both distributions - the baseline
the abstract describes - one block of query rows at a time, in float64, from the
bf16 inputs converted exactly to float64. The KL is taken in the materialised
form above, not through the online identity, so that tests check the identity
instead of assuming it.

Backward (teacher frozen; g[i] = dLoss/dKL[i]):

    dKL[i]/ds_S[i, j] = P_S[i, j] - P_T[i, j]          (on J(i), else 0)
    dS[i, j]  = g[i] * scale_S * (P_S[i, j] - P_T[i, j])   (gradient w.r.t. <q_S[i], k_S[j]>)
    dQ_S      = dS @ K_S            dK_S = dS^T @ Q_S

Readings where the pages are silent (the plainest reading the rest supports):
* causal alignment for N_Q != N_K is bottom-right (j <= i + N_K - N_Q);
* a row with an empty J(i) has KL = 0, LSE = -inf and zero gradient;
* KL is reported raw (no clamp at 0); LSE is the natural-log value.

Every function below is pinned by tests/test_oracle_pins.py against brute force,
a library routine (torch log_softmax/kl_div + autograd), closed forms,
invariances and finite differences.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Sequence, Tuple

import torch

F64 = torch.float64
NEG_INF = float("-inf")


def _f64(x: torch.Tensor) -> torch.Tensor:
    return x.detach().to("cpu").to(F64)


def allowed(i: torch.Tensor, n_q: int, n_k: int, causal: bool) -> torch.Tensor:
    """Boolean [len(i), N_K] mask of J(i) for the query indices ``i``."""
    j = torch.arange(n_k)
    if not causal:
        return torch.ones(len(i), n_k, dtype=torch.bool)
    return j[None, :] <= (i[:, None] + (n_k - n_q))


def _row_block_stats(qt, kt, qs, ks, rows, scale_t, scale_s, causal, n_q):
    """Scores, mask, LSEs and log-probabilities for a block of query rows.

    qt/qs: [R, d] fp64 query rows; kt/ks: [N_K, d] fp64 keys; rows: [R] indices.
    """
    n_k = kt.shape[0]
    mask = allowed(rows, n_q, n_k, causal)
    s_t = scale_t * (qt @ kt.T)
    s_s = scale_s * (qs @ ks.T)
    s_t = torch.where(mask, s_t, torch.full_like(s_t, NEG_INF))
    s_s = torch.where(mask, s_s, torch.full_like(s_s, NEG_INF))
    lse_t = _logsumexp(s_t)
    lse_s = _logsumexp(s_s)
    return s_t, s_s, mask, lse_t, lse_s


def _logsumexp(s: torch.Tensor) -> torch.Tensor:
    """log sum_j exp(s[:, j]) written as max + log(sum(exp(s - max))); -inf for empty rows."""
    m = s.max(dim=1).values
    empty = torch.isinf(m) & (m < 0)
    m_safe = torch.where(empty, torch.zeros_like(m), m)
    tot = torch.exp(s - m_safe[:, None]).sum(dim=1)
    out = m_safe + torch.log(tot)
    return torch.where(empty, torch.full_like(out, NEG_INF), out)


def _probs(s: torch.Tensor, lse: torch.Tensor, mask: torch.Tensor):
    """P = exp(s - LSE) on J(i), 0 elsewhere; log P on J(i), 0 elsewhere."""
    lse_safe = torch.where(torch.isinf(lse), torch.zeros_like(lse), lse)
    logp = torch.where(mask, s - lse_safe[:, None], torch.zeros_like(s))
    p = torch.where(mask, torch.exp(logp), torch.zeros_like(s))
    return p, logp


def _block_kl(s_t, s_s, mask, lse_t, lse_s):
    p_t, logp_t = _probs(s_t, lse_t, mask)
    p_s, logp_s = _probs(s_s, lse_s, mask)
    kl = (p_t * (logp_t - logp_s)).sum(dim=1)
    return kl, p_t, p_s


def oracle_fwd(q_t, k_t, q_s, k_s, scale_t: float, scale_s: float, causal: bool,
               row_block: int = 1024):
    """Per-row KL(P_T || P_S), LSE_T and LSE_S, float64 tensors of shape [B, H, N_Q]."""
    B, H, n_q, _ = q_t.shape
    n_k = k_t.shape[2]
    kl = torch.empty(B, H, n_q, dtype=F64)
    lse_t = torch.empty(B, H, n_q, dtype=F64)
    lse_s = torch.empty(B, H, n_q, dtype=F64)
    for b in range(B):
        for h in range(H):
            kt, ks = _f64(k_t[b, h]), _f64(k_s[b, h])
            for r0 in range(0, n_q, row_block):
                rows = torch.arange(r0, min(n_q, r0 + row_block))
                st, ss, mask, lt, ls = _row_block_stats(
                    _f64(q_t[b, h, rows]), kt, _f64(q_s[b, h, rows]), ks,
                    rows, scale_t, scale_s, causal, n_q)
                k_row, _, _ = _block_kl(st, ss, mask, lt, ls)
                kl[b, h, rows] = k_row
                lse_t[b, h, rows] = lt
                lse_s[b, h, rows] = ls
    return kl, lse_t, lse_s


def oracle_bwd(q_t, k_t, q_s, k_s, scale_t: float, scale_s: float, causal: bool, g,
               row_block: int = 1024):
    """dQ_S [B,H,N_Q,d_S] and dK_S [B,H,N_K,d_S] (float64) of sum_i g[i] * KL[i]."""
    B, H, n_q, d_s = q_s.shape
    n_k = k_s.shape[2]
    dq = torch.zeros(B, H, n_q, d_s, dtype=F64)
    dk = torch.zeros(B, H, n_k, d_s, dtype=F64)
    for b in range(B):
        for h in range(H):
            kt, ks = _f64(k_t[b, h]), _f64(k_s[b, h])
            for r0 in range(0, n_q, row_block):
                rows = torch.arange(r0, min(n_q, r0 + row_block))
                qs = _f64(q_s[b, h, rows])
                st, ss, mask, lt, ls = _row_block_stats(
                    _f64(q_t[b, h, rows]), kt, qs, ks, rows, scale_t, scale_s, causal, n_q)
                _, p_t, p_s = _block_kl(st, ss, mask, lt, ls)
                gi = _f64(g[b, h, rows])
                ds = gi[:, None] * scale_s * (p_s - p_t)
                dq[b, h, rows] = ds @ ks
                dk[b, h] += ds.T @ qs
    return dq, dk


def oracle_rows(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, g,
                rows: Sequence[Tuple[int, int]]):
    """KL, LSE_T, LSE_S and the dQ_S row for selected (bh, i) query rows.

    Each row needs only its own scores, so this is the per-row definition
    evaluated on a sample (used for parity at full size).
    Returns (kl [R], lse_t [R], lse_s [R], dq [R, d_S]) in float64.
    """
    B, H, n_q, _ = q_t.shape
    n_k = k_t.shape[2]
    qt2 = q_t.reshape(B * H, n_q, -1)
    kt2 = k_t.reshape(B * H, n_k, -1)
    qs2 = q_s.reshape(B * H, n_q, -1)
    ks2 = k_s.reshape(B * H, n_k, -1)
    g2 = g.reshape(B * H, n_q)
    kl, lt_o, ls_o, dq = [], [], [], []
    by_head = {}
    for bh, i in rows:
        by_head.setdefault(bh, []).append(i)
    order = []
    for bh, idx in by_head.items():
        rr = torch.tensor(idx)
        kt, ks = _f64(kt2[bh]), _f64(ks2[bh])
        st, ss, mask, lt, ls = _row_block_stats(
            _f64(qt2[bh, rr]), kt, _f64(qs2[bh, rr]), ks, rr, scale_t, scale_s, causal, n_q)
        k_row, p_t, p_s = _block_kl(st, ss, mask, lt, ls)
        ds = _f64(g2[bh, rr])[:, None] * scale_s * (p_s - p_t)
        kl.append(k_row); lt_o.append(lt); ls_o.append(ls); dq.append(ds @ ks)
        order += [(bh, i) for i in idx]
    pos = {r: n for n, r in enumerate(order)}
    perm = torch.tensor([pos[tuple(r)] for r in rows])
    cat = lambda xs: torch.cat(xs)[perm]
    return cat(kl), cat(lt_o), cat(ls_o), cat(dq)


def oracle_dk_rows(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, g, bh: int,
                   keys: Sequence[int], row_block: int = 2048):
    """dK_S rows for selected keys of one head (float64 [len(keys), d_S]).

    dK_S[j] = sum_i dS[i, j] q_S[i] needs P_T[i, j] and P_S[i, j] for every
    query row i, so every row's LSE is computed here from the full row.
    """
    B, H, n_q, d_s = q_s.shape
    n_k = k_s.shape[2]
    qt = q_t.reshape(B * H, n_q, -1)[bh]
    qs = q_s.reshape(B * H, n_q, -1)[bh]
    kt = _f64(k_t.reshape(B * H, n_k, -1)[bh])
    ks = _f64(k_s.reshape(B * H, n_k, -1)[bh])
    gg = g.reshape(B * H, n_q)[bh]
    sel = torch.tensor(list(keys))
    out = torch.zeros(len(sel), d_s, dtype=F64)
    for r0 in range(0, n_q, row_block):
        rows = torch.arange(r0, min(n_q, r0 + row_block))
        qsr = _f64(qs[rows])
        st, ss, mask, lt, ls = _row_block_stats(
            _f64(qt[rows]), kt, qsr, ks, rows, scale_t, scale_s, causal, n_q)
        _, p_t, p_s = _block_kl(st, ss, mask, lt, ls)
        ds = _f64(gg[rows])[:, None] * scale_s * (p_s - p_t)
        out += ds[:, sel].T @ qsr
    return out


def _sampled_ds(g_rows, scale_s, p_s, p_t):
    """dS rows of sampled query rows: g_i * scale_S * (P_S[i, :] - P_T[i, :])."""
    return g_rows[:, None] * scale_s * (p_s - p_t)


def oracle_row_work(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, g,
                    rows: Sequence[Tuple[int, int]]):
    """Whole forward + backward work of selected query rows (CPU-baseline timing).

    For each sampled row: its KL and LSEs, its dQ_S row, and its contribution
    dS[i, :]^T q_S[i] to dK_S. Returns (kl [R], dq [R, d_S], dk_acc [N_K, d_S]),
    where dk_acc is the sum of those contributions over every sampled row (rows of
    different heads added together, so nothing is optimised away; a row listed twice
    contributes twice).
    """
    kl, _, _, dq = oracle_rows(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, g, rows)
    B, H, n_q, d_s = q_s.shape
    n_k = k_s.shape[2]
    qs2 = q_s.reshape(B * H, n_q, -1)
    qt2 = q_t.reshape(B * H, n_q, -1)
    kt2 = k_t.reshape(B * H, n_k, -1)
    ks2 = k_s.reshape(B * H, n_k, -1)
    g2 = g.reshape(B * H, n_q)
    dk_acc = torch.zeros(n_k, d_s, dtype=F64)
    for bh, i in rows:
        rr = torch.tensor([i])
        qsr = _f64(qs2[bh, rr])
        st, ss, mask, lt, ls = _row_block_stats(
            _f64(qt2[bh, rr]), _f64(kt2[bh]), qsr, _f64(ks2[bh]), rr,
            scale_t, scale_s, causal, n_q)
        _, p_t, p_s = _block_kl(st, ss, mask, lt, ls)
        ds = _sampled_ds(_f64(g2[bh, rr]), scale_s, p_s, p_t)
        dk_acc += ds.T @ qsr
    return kl, dq, dk_acc


def row_pair_count(n_q: int, n_k: int, causal: bool, i: int) -> int:
    """|J(i)|: number of keys query row i attends to."""
    if not causal:
        return n_k
    return max(0, min(n_k, i + n_k - n_q + 1))


def oracle_bwd_teacher(q_t, k_t, q_s, k_s, scale_t: float, scale_s: float, causal: bool, g,
                       row_block: int = 1024):
    """dQ_T [B,H,N_Q,d_T] and dK_T [B,H,N_K,d_T] (float64) of sum_i g[i] * KL[i].

    For a trainable teacher. With the student fixed, KL_i = sum_j P_T (s_T - log P_S) - LSE_T,
    so dKL_i/ds_T[i,j] = P_T[i,j] * ((s_T - s_S)[i,j] - E_i) with
    E_i = sum_j P_T[i,j] (s_T - s_S)[i,j] (= KL_i + LSE_T,i - LSE_S,i), and
    dS_T[i,j] = g[i] * scale_T * P_T[i,j] * ((s_T - s_S)[i,j] - E_i) on J(i), else 0;
    dQ_T = dS_T K_T, dK_T = dS_T^T Q_T.
    """
    B, H, n_q, d_t = q_t.shape
    n_k = k_t.shape[2]
    dq = torch.zeros(B, H, n_q, d_t, dtype=F64)
    dk = torch.zeros(B, H, n_k, d_t, dtype=F64)
    for b in range(B):
        for h in range(H):
            kt, ks = _f64(k_t[b, h]), _f64(k_s[b, h])
            for r0 in range(0, n_q, row_block):
                rows = torch.arange(r0, min(n_q, r0 + row_block))
                qt = _f64(q_t[b, h, rows])
                st, ss, mask, lt, ls = _row_block_stats(
                    qt, kt, _f64(q_s[b, h, rows]), ks, rows, scale_t, scale_s, causal, n_q)
                p_t, _ = _probs(st, lt, mask)
                diff = torch.where(mask, st - ss, torch.zeros_like(st))
                e = (p_t * diff).sum(dim=1)
                gi = _f64(g[b, h, rows])
                ds = gi[:, None] * scale_t * p_t * (diff - e[:, None])
                ds = torch.where(mask, ds, torch.zeros_like(ds))
                dq[b, h, rows] = ds @ kt
                dk[b, h] += ds.T @ qt
    return dq, dk


# ------------------------------------------------ grouped-query attention (GQA)
#
# Query head h of H reads K head h // (H / H_kv) (teacher and student may group their
# K heads differently). The KL of a query head is unchanged; the gradient of a shared K
# head is the sum over the query heads of its group.

def expand_kv(k, h_q: int):
    """[B, H_kv, N, d] -> [B, H_q, N, d], query head h reading K head h // (H_q / H_kv)."""
    return k.repeat_interleave(h_q // k.shape[1], dim=1)


def group_sum_kv(dk, h_kv: int):
    """[B, H_q, N, d] -> [B, H_kv, N, d]: sum over the query heads sharing a K head."""
    B, H, N, d = dk.shape
    return dk.reshape(B, h_kv, H // h_kv, N, d).sum(dim=2)


def oracle_fwd_gqa(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, row_block: int = 1024):
    H = q_t.shape[1]
    return oracle_fwd(q_t, expand_kv(k_t, H), q_s, expand_kv(k_s, H), scale_t, scale_s, causal,
                      row_block)


def oracle_bwd_gqa(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, g, row_block: int = 1024):
    """dQ_S [B,H,N_Q,d_S], dK_S [B,H_kv_S,N_K,d_S] with grouped K heads."""
    H = q_t.shape[1]
    dq, dk = oracle_bwd(q_t, expand_kv(k_t, H), q_s, expand_kv(k_s, H), scale_t, scale_s,
                        causal, g, row_block)
    return dq, group_sum_kv(dk, k_s.shape[1])


def oracle_bwd_teacher_gqa(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, g,
                           row_block: int = 1024):
    """dQ_T [B,H,N_Q,d_T], dK_T [B,H_kv_T,N_K,d_T] with grouped K heads."""
    H = q_t.shape[1]
    dq, dk = oracle_bwd_teacher(q_t, expand_kv(k_t, H), q_s, expand_kv(k_s, H), scale_t,
                                scale_s, causal, g, row_block)
    return dq, group_sum_kv(dk, k_t.shape[1])


# ------------------------------------------------ packed variable-length sequences
#
# B sequences of different lengths share one packed tensor: sequence b owns query rows
# cu_q[b] .. cu_q[b+1]-1 and key rows cu_k[b] .. cu_k[b+1]-1 (token-major, [total, heads,
# d]). Each sequence is an independent problem with its own causal alignment (bottom-right
# within the sequence: j <= i + n_k(b) - n_q(b)); no query attends to another sequence's
# keys. Row outputs and g are [H, total_q]. Query heads read K heads as in GQA.

def _seq_bounds(cu):
    cu = [int(c) for c in cu]
    if len(cu) < 2 or cu[0] != 0 or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must start at 0 and be non-decreasing")
    return list(zip(cu[:-1], cu[1:]))


def _seq_heads_first(x, lo, hi):
    """Rows lo..hi-1 of a packed [total, heads, d] tensor as a [1, heads, n, d] problem."""
    return x[lo:hi].permute(1, 0, 2).unsqueeze(0)


def oracle_fwd_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, scale_t, scale_s, causal,
                      row_block: int = 1024):
    """KL, LSE_T, LSE_S as float64 [H, total_q] for packed sequences."""
    H, total_q = q_t.shape[1], q_t.shape[0]
    kl = torch.zeros(H, total_q, dtype=F64)
    lse_t = torch.full((H, total_q), NEG_INF, dtype=F64)
    lse_s = torch.full((H, total_q), NEG_INF, dtype=F64)
    seq_q, seq_k = _seq_bounds(cu_q), _seq_bounds(cu_k)
    if len(seq_q) != len(seq_k):
        raise ValueError("cu_q and cu_k must describe the same number of sequences")
    for (q0, q1), (k0, k1) in zip(seq_q, seq_k):
        if q1 == q0 or k1 == k0:
            continue  # no rows, or rows with no keys: KL 0, LSE -inf (already set)
        out = oracle_fwd_gqa(_seq_heads_first(q_t, q0, q1), _seq_heads_first(k_t, k0, k1),
                             _seq_heads_first(q_s, q0, q1), _seq_heads_first(k_s, k0, k1),
                             scale_t, scale_s, causal, row_block)
        for dst, src in zip((kl, lse_t, lse_s), out):
            dst[:, q0:q1] = src[0]
    return kl, lse_t, lse_s


def _bwd_varlen(fn, q_t, k_t, q_s, k_s, cu_q, cu_k, scale_t, scale_s, causal, g, side,
                row_block):
    q_g, k_g = (q_t, k_t) if side == "teacher" else (q_s, k_s)
    dq = torch.zeros(q_g.shape, dtype=F64)
    dk = torch.zeros(k_g.shape, dtype=F64)
    for (q0, q1), (k0, k1) in zip(_seq_bounds(cu_q), _seq_bounds(cu_k)):
        if q1 == q0 or k1 == k0:
            continue
        gb = g[:, q0:q1].unsqueeze(0)
        dq_b, dk_b = fn(_seq_heads_first(q_t, q0, q1), _seq_heads_first(k_t, k0, k1),
                        _seq_heads_first(q_s, q0, q1), _seq_heads_first(k_s, k0, k1),
                        scale_t, scale_s, causal, gb, row_block)
        dq[q0:q1] = dq_b[0].permute(1, 0, 2)
        dk[k0:k1] = dk_b[0].permute(1, 0, 2)
    return dq, dk


def oracle_bwd_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, scale_t, scale_s, causal, g,
                      row_block: int = 1024):
    """dQ_S [total_q, H, d_S], dK_S [total_k, H_kv_S, d_S] (float64); g is [H, total_q]."""
    return _bwd_varlen(oracle_bwd_gqa, q_t, k_t, q_s, k_s, cu_q, cu_k, scale_t, scale_s,
                       causal, g, "student", row_block)


def oracle_bwd_teacher_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, scale_t, scale_s, causal, g,
                              row_block: int = 1024):
    """dQ_T [total_q, H, d_T], dK_T [total_k, H_kv_T, d_T] (float64); g is [H, total_q]."""
    return _bwd_varlen(oracle_bwd_teacher_gqa, q_t, k_t, q_s, k_s, cu_q, cu_k, scale_t,
                       scale_s, causal, g, "teacher", row_block)


# ------------------------------------------------ context parallelism over N_K
#
# The keys of a sequence (N_K_total of them) are split into contiguous shards; shard r
# holds keys k_offset .. k_offset + n_shard - 1. Per query row, a shard summarises what it
# saw in a state, in base-2 units (t_X = s_X / ln 2):
#   m_X = max_j t_X[j],   l_X = sum_j 2^(t_X[j] - m_X)      (X = T, S)
#   A   = sum_j 2^(t_T[j] - m_T) * (t_T[j] - t_S[j])
# over the shard's allowed keys (global index j allowed iff j <= i + N_K_total - N_Q when
# causal); a row with no allowed key in the shard has m = -inf, l = 0, A = 0. States merge
# by rescaling to the larger maximum and adding, which is associative, and the merged
# state gives LSE_X = ln2 * (m_X + log2 l_X) and KL = ln2 * (A / l_T + m_S - m_T +
# log2 l_S - log2 l_T), the same KL as the unsplit definition.

LN2 = math.log(2.0)


def _shard_scores(q_t, k_t, q_s, k_s, b, h, scale_t, scale_s, causal, k_offset, n_k_total):
    qt, qs = _f64(q_t[b, h]), _f64(q_s[b, h])
    kt, ks = _f64(k_t[b, h]), _f64(k_s[b, h])
    n_q = qt.shape[0]
    i = torch.arange(n_q)[:, None]
    j = k_offset + torch.arange(kt.shape[0])[None, :]
    mask = (j <= i + (n_k_total - n_q)) if causal else torch.ones(n_q, kt.shape[0],
                                                                    dtype=torch.bool)
    return scale_t * (qt @ kt.T), scale_s * (qs @ ks.T), mask, qt, qs, kt, ks


def oracle_partial_state(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset: int,
                         n_k_total: int):
    """State planes (m_T, m_S, l_T, l_S, A) as float64 [5, B, H, N_Q] of one key shard
    (k_* hold the shard's keys; grouped K heads are expanded)."""
    B, H, n_q, _ = q_t.shape
    k_t, k_s = expand_kv(k_t, H), expand_kv(k_s, H)
    out = torch.zeros(5, B, H, n_q, dtype=F64)
    if k_t.shape[2] == 0:  # an empty shard: the identity state
        out[:2] = NEG_INF
        return out
    for b in range(B):
        for h in range(H):
            s_t, s_s, mask, *_ = _shard_scores(q_t, k_t, q_s, k_s, b, h, scale_t, scale_s,
                                               causal, k_offset, n_k_total)
            t_t = torch.where(mask, s_t / LN2, torch.full_like(s_t, NEG_INF))
            t_s = torch.where(mask, s_s / LN2, torch.full_like(s_s, NEG_INF))
            m_t, m_s = t_t.max(dim=1).values, t_s.max(dim=1).values
            live = mask.any(dim=1)
            mt0 = torch.where(live, m_t, torch.zeros_like(m_t))
            ms0 = torch.where(live, m_s, torch.zeros_like(m_s))
            e_t = torch.where(mask, torch.exp2(t_t - mt0[:, None]), torch.zeros_like(t_t))
            e_s = torch.where(mask, torch.exp2(t_s - ms0[:, None]), torch.zeros_like(t_s))
            diff = torch.where(mask, s_t / LN2 - s_s / LN2, torch.zeros_like(s_t))
            out[0, b, h] = m_t
            out[1, b, h] = m_s
            out[2, b, h] = e_t.sum(dim=1)
            out[3, b, h] = e_s.sum(dim=1)
            out[4, b, h] = (e_t * diff).sum(dim=1)
    return out


def oracle_merge_states(states):
    """Merge [R, 5, ...] shard states and finalise: (KL, LSE_T, LSE_S) float64."""
    st = states.to(F64)
    m_t, m_s = st[:, 0].max(dim=0).values, st[:, 1].max(dim=0).values
    empty_t = torch.isinf(m_t) & (m_t < 0)
    empty_s = torch.isinf(m_s) & (m_s < 0)
    mt0 = torch.where(empty_t, torch.zeros_like(m_t), m_t)
    ms0 = torch.where(empty_s, torch.zeros_like(m_s), m_s)
    w_t = torch.exp2(st[:, 0] - mt0)  # -inf - m -> weight 0
    w_s = torch.exp2(st[:, 1] - ms0)
    l_t = (st[:, 2] * w_t).sum(dim=0)
    l_s = (st[:, 3] * w_s).sum(dim=0)
    a = (st[:, 4] * w_t).sum(dim=0)
    empty = l_t == 0
    l_t1, l_s1 = torch.where(empty, torch.ones_like(l_t), l_t), torch.where(empty, torch.ones_like(l_s), l_s)
    kl = LN2 * (a / l_t1 + (ms0 - mt0) + torch.log2(l_s1) - torch.log2(l_t1))
    lse_t = LN2 * (mt0 + torch.log2(l_t1))
    lse_s = LN2 * (ms0 + torch.log2(l_s1))
    kl = torch.where(empty, torch.zeros_like(kl), kl)
    lse_t = torch.where(empty, torch.full_like(lse_t, NEG_INF), lse_t)
    lse_s = torch.where(empty, torch.full_like(lse_s, NEG_INF), lse_s)
    return kl, lse_t, lse_s


def _bwd_shard(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset, n_k_total, kl, lse_t,
               lse_s, g, teacher):
    B, H, n_q, _ = q_t.shape
    h_kv = (k_t if teacher else k_s).shape[1]
    k_t, k_s = expand_kv(k_t, H), expand_kv(k_s, H)
    q_g, k_g = (q_t, k_t) if teacher else (q_s, k_s)
    dq = torch.zeros(q_g.shape, dtype=F64)
    dk = torch.zeros(k_g.shape, dtype=F64)
    for b in range(B):
        for h in range(H):
            s_t, s_s, mask, qt, qs, kt, ks = _shard_scores(q_t, k_t, q_s, k_s, b, h, scale_t,
                                                          scale_s, causal, k_offset, n_k_total)
            lt, ls = _f64(lse_t[b, h]), _f64(lse_s[b, h])
            p_t, _ = _probs(s_t, lt, mask)
            p_s, _ = _probs(s_s, ls, mask)
            gi = _f64(g[b, h])[:, None]
            if teacher:
                e = _f64(kl[b, h]) + torch.where(torch.isinf(lt), torch.zeros_like(lt), lt - ls)
                ds = gi * scale_t * p_t * ((s_t - s_s) - e[:, None])
                ds = torch.where(mask, ds, torch.zeros_like(ds))
                dq[b, h], dk[b, h] = ds @ kt, ds.T @ qt
            else:
                ds = gi * scale_s * (p_s - p_t)
                dq[b, h], dk[b, h] = ds @ ks, ds.T @ qs
    return dq, group_sum_kv(dk, h_kv)


def oracle_bwd_shard(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset: int,
                     n_k_total: int, lse_t, lse_s, g):
    """Student gradients of one key shard with the global LSE_T / LSE_S: the shard's part
    of dQ_S (summed over shards it gives dQ_S) and dK_S of the shard's keys."""
    return _bwd_shard(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset, n_k_total, None,
                      lse_t, lse_s, g, teacher=False)


def oracle_bwd_teacher_shard(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset: int,
                             n_k_total: int, kl, lse_t, lse_s, g):
    """Trainable-teacher gradients of one key shard with the global KL and LSEs."""
    return _bwd_shard(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset, n_k_total, kl,
                      lse_t, lse_s, g, teacher=True)
