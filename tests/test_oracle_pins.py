"""Pins for the fp64 oracle, against things other than itself (CPU only).

Each test states what fixes the expected value: brute force from the
definition, a library routine (torch log_softmax / kl_div + autograd), closed
forms, invariances, finite differences. Together they make a dropped term, a
wrong sign, a wrong index, a wrong causal alignment or a transposed operand in
the oracle fail at least one test (see test_planted_mistakes_are_caught).
"""
import math

import pytest
import torch

from oracle import streamkl_oracle as O
from workloads import WORKLOADS, make_inputs

F64 = torch.float64


def rand_case(B, H, nq, nk, dt, ds, seed, bf16=True, spread=1.0):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: (spread * torch.randn(*s, generator=g, dtype=torch.float32))
    q_t, k_t = mk(B, H, nq, dt), mk(B, H, nk, dt)
    q_s, k_s = mk(B, H, nq, ds), mk(B, H, nk, ds)
    gg = torch.rand(B, H, nq, generator=g) + 0.5
    if bf16:
        q_t, k_t, q_s, k_s = (x.to(torch.bfloat16) for x in (q_t, k_t, q_s, k_s))
    return q_t, k_t, q_s, k_s, gg


# ---------------------------------------------------------------- brute force

def brute_force(q_t, k_t, q_s, k_s, st, ss, causal, g):
    """Pure-Python loops straight from the definition (no max shift, no matmul).

    KL_i = sum_j p_T log(p_T / p_S) with p = exp(s) / sum exp(s) over the keys
    j <= i + N_K - N_Q (causal) or all keys. dQ_S and dK_S are the derivatives
    of sum_i g_i KL_i, using dKL_i/ds_S[i,j] = p_S - p_T.
    """
    B, H, nq, dt = q_t.shape
    nk, ds_ = k_t.shape[2], q_s.shape[3]
    L = lambda t: t.double().tolist()
    QT, KT, QS, KS, G = L(q_t), L(k_t), L(q_s), L(k_s), L(g)
    kl = [[[0.0] * nq for _ in range(H)] for _ in range(B)]
    lt = [[[0.0] * nq for _ in range(H)] for _ in range(B)]
    ls = [[[0.0] * nq for _ in range(H)] for _ in range(B)]
    dq = [[[[0.0] * ds_ for _ in range(nq)] for _ in range(H)] for _ in range(B)]
    dk = [[[[0.0] * ds_ for _ in range(nk)] for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(nq):
                js = [j for j in range(nk) if (not causal) or j <= i + nk - nq]
                if not js:
                    lt[b][h][i] = ls[b][h][i] = float("-inf")
                    continue
                sT = {j: st * sum(QT[b][h][i][c] * KT[b][h][j][c] for c in range(dt)) for j in js}
                sS = {j: ss * sum(QS[b][h][i][c] * KS[b][h][j][c] for c in range(ds_)) for j in js}
                zT = sum(math.exp(v) for v in sT.values())
                zS = sum(math.exp(v) for v in sS.values())
                pT = {j: math.exp(sT[j]) / zT for j in js}
                pS = {j: math.exp(sS[j]) / zS for j in js}
                kl[b][h][i] = sum(pT[j] * math.log(pT[j] / pS[j]) for j in js)
                lt[b][h][i], ls[b][h][i] = math.log(zT), math.log(zS)
                for j in js:
                    dsij = G[b][h][i] * ss * (pS[j] - pT[j])
                    for c in range(ds_):
                        dq[b][h][i][c] += dsij * KS[b][h][j][c]
                        dk[b][h][j][c] += dsij * QS[b][h][i][c]
    T = lambda x: torch.tensor(x, dtype=F64)
    return T(kl), T(lt), T(ls), T(dq), T(dk)


@pytest.mark.parametrize("nq,nk,causal", [(5, 5, False), (5, 5, True), (6, 3, True),
                                          (3, 6, True), (4, 7, False), (1, 1, True)])
def test_brute_force_tiny(nq, nk, causal):
    q_t, k_t, q_s, k_s, g = rand_case(2, 2, nq, nk, 3, 2, seed=nq * 31 + nk + causal)
    st, ss = 0.7, 1.3
    ref = brute_force(q_t, k_t, q_s, k_s, st, ss, causal, g)
    kl, lt, ls = O.oracle_fwd(q_t, k_t, q_s, k_s, st, ss, causal, row_block=2)
    dq, dk = O.oracle_bwd(q_t, k_t, q_s, k_s, st, ss, causal, g, row_block=2)
    for got, want in zip((kl, lt, ls, dq, dk), ref):
        fin = torch.isfinite(want)
        assert torch.equal(fin, torch.isfinite(got))
        assert torch.equal(got[~fin], want[~fin])
        torch.testing.assert_close(got[fin], want[fin], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------- library routine

MASKED = -1.0e4  # finite stand-in for -inf: exp underflows to exactly 0 in fp64, no NaN grads


def _masked_scores(s, nq, nk, causal):
    if not causal:
        return s
    bad = torch.arange(nk)[None, :] > torch.arange(nq)[:, None] + nk - nq
    return torch.where(bad, torch.full_like(s, MASKED), s)


def library_kl(q_t, k_t, q_s, k_s, st, ss, causal, g):
    """torch log_softmax + kl_div (log_target) in fp64, autograd for the student gradients.

    Masked scores use a large finite value so that every gradient entry is finite and
    compared; rows with no allowed key become uniform over masked keys (P_T = P_S, so KL
    and gradients are 0 there, matching the empty-row reading) and are excluded from
    the LSE comparison by the caller.
    """
    qs = q_s.double().requires_grad_(True)
    ks = k_s.double().requires_grad_(True)
    nq, nk = q_t.shape[2], k_t.shape[2]
    s_t = _masked_scores(st * q_t.double() @ k_t.double().transpose(-1, -2), nq, nk, causal)
    s_s = _masked_scores(ss * qs @ ks.transpose(-1, -2), nq, nk, causal)
    lp_t = torch.log_softmax(s_t, -1)
    lp_s = torch.log_softmax(s_s, -1)
    # kl_div(input=log q, target=log p, log_target=True) = p * (log p - log q)
    kl = torch.nn.functional.kl_div(lp_s, lp_t, reduction="none", log_target=True).sum(-1)
    (kl * g.double()).sum().backward()
    return kl.detach(), torch.logsumexp(s_t, -1).detach(), torch.logsumexp(s_s, -1).detach(), qs.grad, ks.grad


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dims", [(8, 8, 16, 16), (16, 9, 8, 4), (9, 16, 4, 8)])
def test_against_library(causal, dims):
    nq, nk, dt, ds = dims
    q_t, k_t, q_s, k_s, g = rand_case(1, 3, nq, nk, dt, ds, seed=sum(dims) + causal)
    st, ss = 1 / math.sqrt(dt), 1 / math.sqrt(ds)
    kl_r, lt_r, ls_r, dq_r, dk_r = library_kl(q_t, k_t, q_s, k_s, st, ss, causal, g)
    kl, lt, ls = O.oracle_fwd(q_t, k_t, q_s, k_s, st, ss, causal, row_block=5)
    dq, dk = O.oracle_bwd(q_t, k_t, q_s, k_s, st, ss, causal, g, row_block=5)
    ok = torch.isfinite(lt)  # rows with at least one allowed key
    torch.testing.assert_close(kl, kl_r, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(lt[ok], lt_r[ok], rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(ls[ok], ls_r[ok], rtol=1e-12, atol=1e-12)
    assert torch.all(torch.isfinite(dq_r)) and torch.all(torch.isfinite(dk_r))
    torch.testing.assert_close(dq, dq_r, rtol=1e-10, atol=1e-12)
    torch.testing.assert_close(dk, dk_r, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------------- closed forms

def test_two_key_bernoulli_closed_form():
    """Two keys: softmax over two scores is a Bernoulli law; KL and dS are closed-form."""
    # d = 2, keys e1 and e2, so s[i, j] = scale * q[i, j].
    q_t = torch.tensor([[[[1.5, -0.5], [0.25, 2.0], [0.0, 0.0]]]], dtype=F64)
    q_s = torch.tensor([[[[0.5, 0.5], [-1.0, 1.0], [3.0, -2.0]]]], dtype=F64)
    k = torch.tensor([[[[1.0, 0.0], [0.0, 1.0]]]], dtype=F64)
    st, ss = 0.8, 1.7
    g = torch.tensor([[[1.0, 0.5, 2.0]]], dtype=F64)
    kl, lt, ls = O.oracle_fwd(q_t, k, q_s, k, st, ss, False)
    dq, dk = O.oracle_bwd(q_t, k, q_s, k, st, ss, False, g)
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    for i in range(3):
        a = sig(st * (q_t[0, 0, i, 0] - q_t[0, 0, i, 1]).item())
        b = sig(ss * (q_s[0, 0, i, 0] - q_s[0, 0, i, 1]).item())
        want = a * math.log(a / b) + (1 - a) * math.log((1 - a) / (1 - b))
        assert abs(kl[0, 0, i].item() - want) < 1e-13 * max(1.0, abs(want))
        want_lt = math.log(math.exp(st * q_t[0, 0, i, 0].item()) + math.exp(st * q_t[0, 0, i, 1].item()))
        assert abs(lt[0, 0, i].item() - want_lt) < 1e-13 * max(1.0, abs(want_lt))
        # dKL/ds_S[i,0] = b - a, dKL/ds_S[i,1] = a - b; dQ_S[i] = g*scale_S*(b-a, a-b)
        gi = g[0, 0, i].item()
        torch.testing.assert_close(dq[0, 0, i], torch.tensor([gi * ss * (b - a), gi * ss * (a - b)], dtype=F64),
                                   rtol=1e-13, atol=1e-15)


def test_uniform_student_closed_form():
    """scale_S = 0 makes P_S uniform on J(i): KL = log|J(i)| - H(P_T)."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 2, 12, 12, 8, 8, seed=7)
    for causal in (False, True):
        kl, lt, ls = O.oracle_fwd(q_t, k_t, q_s, k_s, 0.9, 0.0, causal)
        for h in range(2):
            for i in range(12):
                n = O.row_pair_count(12, 12, causal, i)
                s = [0.9 * float(q_t[0, h, i].double() @ k_t[0, h, j].double()) for j in range(n)]
                z = sum(math.exp(v) for v in s)
                p = [math.exp(v) / z for v in s]
                ent = -sum(x * math.log(x) for x in p)
                assert abs(kl[0, h, i].item() - (math.log(n) - ent)) < 1e-12
                assert abs(ls[0, h, i].item() - math.log(n)) < 1e-12


def test_both_scales_zero_gives_zero():
    q_t, k_t, q_s, k_s, g = rand_case(1, 1, 9, 9, 4, 4, seed=3)
    kl, _, _ = O.oracle_fwd(q_t, k_t, q_s, k_s, 0.0, 0.0, True)
    assert torch.all(kl.abs() < 1e-15)


def test_causal_row_zero_single_key():
    """Causal with N_Q = N_K: row 0 sees key 0 only, so KL = 0, LSE = s[0,0], dQ row 0 = 0."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 2, 10, 10, 4, 4, seed=11)
    kl, lt, ls = O.oracle_fwd(q_t, k_t, q_s, k_s, 0.5, 0.5, True)
    dq, dk = O.oracle_bwd(q_t, k_t, q_s, k_s, 0.5, 0.5, True, g)
    assert torch.all(kl[:, :, 0] == 0)
    want = 0.5 * (q_t[0, :, 0].double() * k_t[0, :, 0].double()).sum(-1)
    torch.testing.assert_close(lt[0, :, 0], want, rtol=1e-14, atol=1e-14)
    assert torch.all(dq[:, :, 0] == 0)


def test_empty_rows_when_more_queries_than_keys():
    """Causal, N_Q > N_K: rows i < N_Q - N_K see no key (KL 0, LSE -inf, zero gradient)."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 1, 7, 4, 4, 4, seed=5)
    kl, lt, ls = O.oracle_fwd(q_t, k_t, q_s, k_s, 0.5, 0.5, True)
    dq, dk = O.oracle_bwd(q_t, k_t, q_s, k_s, 0.5, 0.5, True, g)
    assert torch.all(kl[0, 0, :3] == 0)
    assert torch.all(torch.isneginf(lt[0, 0, :3])) and torch.all(torch.isneginf(ls[0, 0, :3]))
    assert torch.all(torch.isfinite(lt[0, 0, 3:]))
    assert torch.all(dq[0, 0, :3] == 0)
    assert torch.all(kl[0, 0, 3] == 0)  # row 3 sees key 0 only


# --------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_gibbs_nonnegative(causal):
    for seed in range(4):
        q_t, k_t, q_s, k_s, g = rand_case(2, 2, 33, 29, 16, 8, seed=seed, spread=2.0)
        kl, _, _ = O.oracle_fwd(q_t, k_t, q_s, k_s, 0.3, 0.4, causal, row_block=7)
        assert torch.all(kl >= -1e-13)
        assert kl.max() > 0.01


def test_identical_inputs_give_zero():
    q_t, k_t, _, _, g = rand_case(1, 2, 20, 20, 8, 8, seed=9)
    for causal in (False, True):
        kl, lt, ls = O.oracle_fwd(q_t, k_t, q_t, k_t, 0.35, 0.35, causal)
        dq, dk = O.oracle_bwd(q_t, k_t, q_t, k_t, 0.35, 0.35, causal, g)
        assert torch.all(kl == 0)
        assert torch.equal(lt, ls)
        assert torch.all(dq == 0) and torch.all(dk == 0)


def test_key_shift_invariance_and_dk_sums_to_zero():
    """Adding one vector c to every student key shifts each row's student scores
    by a constant, which softmax ignores: KL is unchanged. Because sum_j dS[i,j] = 0
    for every row, sum_j dK_S[j] = sum_i (sum_j dS[i,j]) q_S[i] = 0."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 2, 15, 15, 8, 8, seed=21, bf16=False)
    q_t, k_t, q_s, k_s = (x.double() for x in (q_t, k_t, q_s, k_s))
    c = torch.randn(8, generator=torch.Generator().manual_seed(1), dtype=F64)
    for causal in (False, True):
        kl1, _, _ = O.oracle_fwd(q_t, k_t, q_s, k_s, 0.4, 0.6, causal)
        kl2, _, _ = O.oracle_fwd(q_t, k_t, q_s, k_s + c, 0.4, 0.6, causal)
        torch.testing.assert_close(kl1, kl2, rtol=1e-11, atol=1e-12)
        dq, dk = O.oracle_bwd(q_t, k_t, q_s, k_s, 0.4, 0.6, causal, g)
        assert dk.sum(dim=2).abs().max() < 1e-12
        assert dk.abs().max() > 1e-3


def test_online_identity_matches_materialised_form():
    """KL_i = E_{P_T}[s_T - s_S] - LSE_T + LSE_S (the identity the forward streams)."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 2, 17, 17, 8, 8, seed=2)
    st, ss = 0.5, 0.7
    for causal in (False, True):
        kl, lt, ls = O.oracle_fwd(q_t, k_t, q_s, k_s, st, ss, causal)
        for h in range(2):
            s_t = st * q_t[0, h].double() @ k_t[0, h].double().T
            s_s = ss * q_s[0, h].double() @ k_s[0, h].double().T
            for i in range(17):
                n = O.row_pair_count(17, 17, causal, i)
                p = torch.exp(s_t[i, :n] - lt[0, h, i])
                e = (p * (s_t[i, :n] - s_s[i, :n])).sum()
                assert abs((e - lt[0, h, i] + ls[0, h, i]).item() - kl[0, h, i].item()) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(causal):
    """Central differences of sum_i g_i KL_i w.r.t. entries of Q_S and K_S."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 1, 6, 7, 4, 3, seed=13, bf16=False)
    q_t, k_t, q_s, k_s = (x.double() for x in (q_t, k_t, q_s, k_s))
    g = g.double()
    st, ss = 0.6, 0.9
    dq, dk = O.oracle_bwd(q_t, k_t, q_s, k_s, st, ss, causal, g)
    loss = lambda qs, ks: float((O.oracle_fwd(q_t, k_t, qs, ks, st, ss, causal)[0] * g).sum())
    h = 1e-6
    for (i, c) in [(0, 0), (2, 1), (5, 2), (3, 0)]:
        e = torch.zeros_like(q_s); e[0, 0, i, c] = h
        fd = (loss(q_s + e, k_s) - loss(q_s - e, k_s)) / (2 * h)
        assert abs(fd - dq[0, 0, i, c].item()) <= 1e-6 * max(1.0, abs(fd))
    for (j, c) in [(0, 0), (3, 2), (6, 1)]:
        e = torch.zeros_like(k_s); e[0, 0, j, c] = h
        fd = (loss(q_s, k_s + e) - loss(q_s, k_s - e)) / (2 * h)
        assert abs(fd - dk[0, 0, j, c].item()) <= 1e-6 * max(1.0, abs(fd))


# ------------------------------------------------------ sampled-row helpers

def test_sampled_rows_match_full():
    w = WORKLOADS["tiny_n256_d64"].with_sizes(H=3, N_Q=70, N_K=70, causal=True)
    x = make_inputs(w)
    args = (x["q_t"], x["k_t"], x["q_s"], x["k_s"], w.scale_T, w.scale_S, w.causal)
    kl, lt, ls = O.oracle_fwd(*args, row_block=16)
    dq, dk = O.oracle_bwd(*args, x["g"], row_block=16)
    rows = [(0, 0), (2, 69), (1, 33), (0, 5)]
    kl_r, lt_r, ls_r, dq_r = O.oracle_rows(*args, x["g"], rows)
    for n, (bh, i) in enumerate(rows):
        assert kl_r[n] == kl.view(-1, 70)[bh, i]
        assert lt_r[n] == lt.view(-1, 70)[bh, i]
        torch.testing.assert_close(dq_r[n], dq.view(3, 70, -1)[bh, i], rtol=1e-13, atol=1e-15)
    keys = [0, 17, 69]
    dk_r = O.oracle_dk_rows(*args, x["g"], 1, keys, row_block=16)
    torch.testing.assert_close(dk_r, dk.view(3, 70, -1)[1, keys], rtol=1e-12, atol=1e-14)


# --------------------------------------------------- planted mistakes (CPU)

def _mutants():
    """Plausible one-line mistakes, each planted in a copy of one oracle helper."""
    orig_stats = O._row_block_stats

    def wrong_causal(i, n_q, n_k, causal):  # top-left alignment instead of bottom-right
        j = torch.arange(n_k)
        if not causal:
            return torch.ones(len(i), n_k, dtype=torch.bool)
        return j[None, :] <= i[:, None]

    def lse_no_max(s):  # drops the max term of the log-sum-exp
        m = s.max(dim=1).values
        return torch.log(torch.exp(s - m[:, None]).sum(dim=1))

    def probs_sign(s, lse, mask):  # wrong sign: exp(s + LSE)
        logp = torch.where(mask, s + lse[:, None], torch.zeros_like(s))
        return torch.where(mask, torch.exp(logp), torch.zeros_like(s)), logp

    def kl_dropped_term(s_t, s_s, mask, lse_t, lse_s):  # drops the -log P_S term
        p_t, logp_t = O._probs(s_t, lse_t, mask)
        p_s, _ = O._probs(s_s, lse_s, mask)
        return (p_t * logp_t).sum(dim=1), p_t, p_s

    def teacher_keys_for_student(qt, kt, qs, ks, rows, st, ss, causal, n_q):  # wrong operand
        return orig_stats(qt, kt, qs, kt[:, : ks.shape[1]], rows, st, ss, causal, n_q)

    return [("allowed", wrong_causal), ("_logsumexp", lse_no_max), ("_probs", probs_sign),
            ("_block_kl", kl_dropped_term), ("_row_block_stats", teacher_keys_for_student)]


def test_planted_mistakes_are_caught(monkeypatch):
    """Each planted oracle mistake must break the brute-force pin (N_Q != N_K, causal)."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 1, 4, 6, 3, 2, seed=99)
    ref = brute_force(q_t, k_t, q_s, k_s, 0.7, 1.1, True, g)
    mutants = _mutants()
    for name, fn in mutants:
        with monkeypatch.context() as m:
            m.setattr(O, name, fn)
            kl, lt, ls = O.oracle_fwd(q_t, k_t, q_s, k_s, 0.7, 1.1, True)
            dq, dk = O.oracle_bwd(q_t, k_t, q_s, k_s, 0.7, 1.1, True, g)
            same = all(torch.allclose(a, b, rtol=1e-9, atol=1e-12, equal_nan=True)
                       for a, b in zip((kl, lt, ls, dq, dk), ref))
            assert not same, f"planted mistake in {name} was not caught"


# ------------------------------------------------- trainable-teacher gradient

@pytest.mark.parametrize("causal", [False, True])
def test_teacher_grad_against_library_autograd(causal):
    """dQ_T, dK_T from torch log_softmax/kl_div autograd w.r.t. the teacher inputs."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 2, 9, 11, 8, 4, seed=31 + causal)
    st, ss = 0.45, 0.6
    qt = q_t.double().requires_grad_(True)
    kt = k_t.double().requires_grad_(True)
    s_t = _masked_scores(st * qt @ kt.transpose(-1, -2), 9, 11, causal)
    s_s = _masked_scores(ss * q_s.double() @ k_s.double().transpose(-1, -2), 9, 11, causal)
    terms = torch.nn.functional.kl_div(torch.log_softmax(s_s, -1), torch.log_softmax(s_t, -1),
                                       reduction="none", log_target=True)
    (terms.sum(-1) * g.double()).sum().backward()
    assert torch.all(torch.isfinite(qt.grad)) and torch.all(torch.isfinite(kt.grad))
    dq, dk = O.oracle_bwd_teacher(q_t, k_t, q_s, k_s, st, ss, causal, g, row_block=4)
    torch.testing.assert_close(dq, qt.grad, rtol=1e-10, atol=1e-12)
    torch.testing.assert_close(dk, kt.grad, rtol=1e-10, atol=1e-12)


def test_teacher_grad_finite_differences_and_invariants():
    q_t, k_t, q_s, k_s, g = rand_case(1, 1, 5, 6, 3, 3, seed=41, bf16=False)
    q_t, k_t, q_s, k_s, g = (x.double() for x in (q_t, k_t, q_s, k_s, g))
    st, ss = 0.8, 0.7
    dq, dk = O.oracle_bwd_teacher(q_t, k_t, q_s, k_s, st, ss, True, g)
    loss = lambda qt, kt: float((O.oracle_fwd(qt, kt, q_s, k_s, st, ss, True)[0] * g).sum())
    h = 1e-6
    for (i, c) in [(1, 0), (4, 2)]:
        e = torch.zeros_like(q_t); e[0, 0, i, c] = h
        fd = (loss(q_t + e, k_t) - loss(q_t - e, k_t)) / (2 * h)
        assert abs(fd - dq[0, 0, i, c].item()) <= 1e-6 * max(1.0, abs(fd))
    for (j, c) in [(0, 1), (5, 0)]:
        e = torch.zeros_like(k_t); e[0, 0, j, c] = h
        fd = (loss(q_t, k_t + e) - loss(q_t, k_t - e)) / (2 * h)
        assert abs(fd - dk[0, 0, j, c].item()) <= 1e-6 * max(1.0, abs(fd))
    # sum_j dS_T[i, j] = 0 for every row, so the teacher key gradients sum to zero
    assert dk.sum(dim=2).abs().max() < 1e-12
    # identical teacher and student: zero gradient for the teacher as well
    dq0, dk0 = O.oracle_bwd_teacher(q_t, k_t, q_t, k_t, st, st, True, g)
    assert dq0.abs().max() < 1e-15 and dk0.abs().max() < 1e-15


# ------------------------------------------------ grouped-query attention (GQA)

def brute_force_gqa(q_t, k_t, q_s, k_s, st, ss, causal, g):
    """Pure-Python loops with explicit K-head indices: query head h reads teacher K head
    h // (H / H_kv_T) and student K head h // (H / H_kv_S); dK of a K head sums over the
    query heads that read it."""
    B, H, nq, dt = q_t.shape
    hkt, hks = k_t.shape[1], k_s.shape[1]
    nk, ds_ = k_t.shape[2], q_s.shape[3]
    L = lambda t: t.double().tolist()
    QT, KT, QS, KS, G = L(q_t), L(k_t), L(q_s), L(k_s), L(g)
    kl = [[[0.0] * nq for _ in range(H)] for _ in range(B)]
    dk = [[[[0.0] * ds_ for _ in range(nk)] for _ in range(hks)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            ht, hs = h // (H // hkt), h // (H // hks)
            for i in range(nq):
                js = [j for j in range(nk) if (not causal) or j <= i + nk - nq]
                if not js:
                    continue
                sT = {j: st * sum(QT[b][h][i][c] * KT[b][ht][j][c] for c in range(dt)) for j in js}
                sS = {j: ss * sum(QS[b][h][i][c] * KS[b][hs][j][c] for c in range(ds_)) for j in js}
                zT = sum(math.exp(v) for v in sT.values())
                zS = sum(math.exp(v) for v in sS.values())
                pT = {j: math.exp(sT[j]) / zT for j in js}
                pS = {j: math.exp(sS[j]) / zS for j in js}
                kl[b][h][i] = sum(pT[j] * math.log(pT[j] / pS[j]) for j in js)
                for j in js:
                    dsij = G[b][h][i] * ss * (pS[j] - pT[j])
                    for c in range(ds_):
                        dk[b][hs][j][c] += dsij * QS[b][h][i][c]
    return torch.tensor(kl, dtype=F64), torch.tensor(dk, dtype=F64)


@pytest.mark.parametrize("hkt,hks", [(2, 1), (1, 2), (4, 4), (4, 2)])
def test_gqa_against_brute_force(hkt, hks):
    g = torch.Generator().manual_seed(7 * hkt + hks)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    q_t, k_t = mk(1, 4, 5, 3), mk(1, hkt, 6, 3)
    q_s, k_s = mk(1, 4, 5, 2), mk(1, hks, 6, 2)
    gg = torch.rand(1, 4, 5, generator=g) + 0.5
    kl_r, dk_r = brute_force_gqa(q_t, k_t, q_s, k_s, 0.8, 1.2, True, gg)
    kl, _, _ = O.oracle_fwd_gqa(q_t, k_t, q_s, k_s, 0.8, 1.2, True)
    dq, dk = O.oracle_bwd_gqa(q_t, k_t, q_s, k_s, 0.8, 1.2, True, gg)
    torch.testing.assert_close(kl, kl_r, rtol=1e-12, atol=1e-13)
    torch.testing.assert_close(dk, dk_r, rtol=1e-11, atol=1e-13)
    assert dq.shape == q_s.shape and dk.shape == k_s.shape


def test_gqa_shared_key_finite_differences():
    """Both query heads of a group move with a shared K entry: dK sums their parts."""
    g = torch.Generator().manual_seed(3)
    q_t, k_t = torch.randn(1, 4, 5, 3, generator=g, dtype=F64), torch.randn(1, 4, 6, 3, generator=g, dtype=F64)
    q_s, k_s = torch.randn(1, 4, 5, 3, generator=g, dtype=F64), torch.randn(1, 2, 6, 3, generator=g, dtype=F64)
    gg = torch.rand(1, 4, 5, generator=g, dtype=F64)
    dq, dk = O.oracle_bwd_gqa(q_t, k_t, q_s, k_s, 0.5, 0.9, False, gg)
    dqt, dkt = O.oracle_bwd_teacher_gqa(q_t, k_t[:, :1], q_s, k_s, 0.5, 0.9, False, gg)
    loss = lambda kt, ks: float((O.oracle_fwd_gqa(q_t, kt, q_s, ks, 0.5, 0.9, False)[0] * gg).sum())
    h = 1e-6
    for (hk, j, c) in [(0, 1, 0), (1, 5, 2)]:
        e = torch.zeros_like(k_s); e[0, hk, j, c] = h
        fd = (loss(k_t, k_s + e) - loss(k_t, k_s - e)) / (2 * h)
        assert abs(fd - dk[0, hk, j, c].item()) <= 1e-6 * max(1.0, abs(fd))
    kt1 = k_t[:, :1]
    for (j, c) in [(0, 2), (4, 1)]:
        e = torch.zeros_like(kt1); e[0, 0, j, c] = h
        fd = (loss(kt1 + e, k_s) - loss(kt1 - e, k_s)) / (2 * h)
        assert abs(fd - dkt[0, 0, j, c].item()) <= 1e-6 * max(1.0, abs(fd))


# ------------------------------------------------ packed variable-length sequences

def brute_force_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, st, ss, causal, g):
    """Pure-Python loops over packed [total, heads, d] rows with explicit token indices.

    Query token i of sequence b (rows cu_q[b] <= i < cu_q[b+1]) sees key token j of the
    same sequence iff not causal or (j - cu_k[b]) <= (i - cu_q[b]) + n_k(b) - n_q(b).
    Returns KL and LSE_T as [H, total_q], dQ_S [total_q, H, d_S], dK_S [total_k, H_kv_S, d_S].
    """
    tq, H, dt = q_t.shape
    tk, hkt, _ = k_t.shape
    hks, ds_ = k_s.shape[1], k_s.shape[2]
    L = lambda t: t.double().tolist()
    QT, KT, QS, KS, G = L(q_t), L(k_t), L(q_s), L(k_s), L(g)
    kl = [[0.0] * tq for _ in range(H)]
    lt = [[float("-inf")] * tq for _ in range(H)]
    dq = [[[0.0] * ds_ for _ in range(H)] for _ in range(tq)]
    dk = [[[0.0] * ds_ for _ in range(hks)] for _ in range(tk)]
    for b in range(len(cu_q) - 1):
        nq, nk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for h in range(H):
            ht, hs = h // (H // hkt), h // (H // hks)
            for i in range(cu_q[b], cu_q[b + 1]):
                js = [j for j in range(cu_k[b], cu_k[b + 1])
                      if (not causal) or (j - cu_k[b]) <= (i - cu_q[b]) + nk - nq]
                if not js:
                    continue
                sT = {j: st * sum(QT[i][h][c] * KT[j][ht][c] for c in range(dt)) for j in js}
                sS = {j: ss * sum(QS[i][h][c] * KS[j][hs][c] for c in range(ds_)) for j in js}
                zT = sum(math.exp(v) for v in sT.values())
                zS = sum(math.exp(v) for v in sS.values())
                pT = {j: math.exp(sT[j]) / zT for j in js}
                pS = {j: math.exp(sS[j]) / zS for j in js}
                kl[h][i] = sum(pT[j] * math.log(pT[j] / pS[j]) for j in js)
                lt[h][i] = math.log(zT)
                for j in js:
                    dsij = G[h][i] * ss * (pS[j] - pT[j])
                    for c in range(ds_):
                        dq[i][h][c] += dsij * KS[j][hs][c]
                        dk[j][hs][c] += dsij * QS[i][h][c]
    T = lambda x: torch.tensor(x, dtype=F64)
    return T(kl), T(lt), T(dq), T(dk)


def varlen_case(lq, lk, H, hkt, hks, dt, ds, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    tq, tk = sum(lq), sum(lk)
    cu_q = [0] + list(torch.tensor(lq).cumsum(0).tolist())
    cu_k = [0] + list(torch.tensor(lk).cumsum(0).tolist())
    return (mk(tq, H, dt), mk(tk, hkt, dt), mk(tq, H, ds), mk(tk, hks, ds), cu_q, cu_k,
            torch.rand(H, tq, generator=g) + 0.5)


# sequences with: equal lengths, n_q > n_k (empty causal rows), n_q < n_k, no queries,
# no keys, a single token
VARLEN_LENS = [([3, 5, 0, 4, 1, 2], [3, 2, 4, 6, 1, 0])]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hkt,hks", [(2, 2), (1, 2)])
def test_varlen_against_brute_force(causal, hkt, hks):
    lq, lk = VARLEN_LENS[0]
    q_t, k_t, q_s, k_s, cu_q, cu_k, gg = varlen_case(lq, lk, 2, hkt, hks, 3, 2, 11 + hkt)
    kl_r, lt_r, dq_r, dk_r = brute_force_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, 0.7, 1.1,
                                                causal, gg)
    kl, lt, _ = O.oracle_fwd_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, 0.7, 1.1, causal)
    dq, dk = O.oracle_bwd_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, 0.7, 1.1, causal, gg)
    torch.testing.assert_close(kl, kl_r, rtol=1e-12, atol=1e-13)
    torch.testing.assert_close(lt, lt_r, rtol=1e-12, atol=1e-13)
    torch.testing.assert_close(dq, dq_r, rtol=1e-11, atol=1e-13)
    torch.testing.assert_close(dk, dk_r, rtol=1e-11, atol=1e-13)
    assert dq.shape == q_s.shape and dk.shape == k_s.shape


def test_varlen_sequences_are_independent_and_match_padded_runs():
    """A sequence's outputs equal those of the same tokens run alone in the [B, H, N, d]
    layout, and do not move when another sequence's tokens change."""
    lq, lk = [4, 6], [5, 6]
    q_t, k_t, q_s, k_s, cu_q, cu_k, gg = varlen_case(lq, lk, 2, 2, 2, 3, 3, 5)
    kl, _, _ = O.oracle_fwd_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, 0.9, 0.6, True)
    alone = lambda x, lo, hi: x[lo:hi].permute(1, 0, 2).unsqueeze(0)
    kl1, _, _ = O.oracle_fwd(alone(q_t, 4, 10), alone(k_t, 5, 11), alone(q_s, 4, 10),
                             alone(k_s, 5, 11), 0.9, 0.6, True)
    torch.testing.assert_close(kl[:, 4:10], kl1[0], rtol=0, atol=0)
    k_s2 = k_s.clone()
    k_s2[:5] = torch.randn(5, 2, 3).to(torch.bfloat16)
    kl2, _, _ = O.oracle_fwd_varlen(q_t, k_t, q_s, k_s2, cu_q, cu_k, 0.9, 0.6, True)
    assert torch.equal(kl2[:, 4:], kl[:, 4:]) and not torch.equal(kl2[:, :4], kl[:, :4])


def test_varlen_teacher_finite_differences():
    lq, lk = [3, 4], [5, 4]
    g = torch.Generator().manual_seed(9)
    mk = lambda *s: torch.randn(*s, generator=g, dtype=F64)
    q_t, k_t, q_s, k_s = mk(7, 2, 3), mk(9, 1, 3), mk(7, 2, 2), mk(9, 2, 2)
    cu_q, cu_k = [0, 3, 7], [0, 5, 9]
    gg = torch.rand(2, 7, generator=g, dtype=F64)
    dq, dk = O.oracle_bwd_teacher_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, 0.8, 1.3, True, gg)
    loss = lambda qt, kt: float((O.oracle_fwd_varlen(qt, kt, q_s, k_s, cu_q, cu_k, 0.8, 1.3,
                                                     True)[0] * gg).sum())
    h = 1e-6
    for (i, hh, c) in [(1, 0, 2), (6, 1, 0)]:
        e = torch.zeros_like(q_t); e[i, hh, c] = h
        fd = (loss(q_t + e, k_t) - loss(q_t - e, k_t)) / (2 * h)
        assert abs(fd - dq[i, hh, c].item()) <= 1e-6 * max(1.0, abs(fd))
    for (j, c) in [(0, 1), (4, 2), (8, 0)]:
        e = torch.zeros_like(k_t); e[j, 0, c] = h
        fd = (loss(q_t, k_t + e) - loss(q_t, k_t - e)) / (2 * h)
        assert abs(fd - dk[j, 0, c].item()) <= 1e-6 * max(1.0, abs(fd))


def test_varlen_one_sequence_mistake_is_caught(monkeypatch):
    """Treating the packed tensor as one sequence (no boundaries) fails the brute force."""
    lq, lk = [3, 4], [4, 3]
    q_t, k_t, q_s, k_s, cu_q, cu_k, gg = varlen_case(lq, lk, 2, 2, 2, 3, 2, 21)
    kl_r, _, _, _ = brute_force_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, 0.7, 1.1, True, gg)
    monkeypatch.setattr(O, "_seq_bounds", lambda cu: [(0, int(cu[-1]))])
    kl, _, _ = O.oracle_fwd_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, 0.7, 1.1, True)
    assert not torch.allclose(kl, kl_r, rtol=1e-6, atol=1e-8)


def test_varlen_rejects_bad_offsets():
    q = torch.zeros(4, 1, 2)
    with pytest.raises(ValueError):
        O.oracle_fwd_varlen(q, q, q, q, [0, 3, 2, 4], [0, 1, 2, 4], 1.0, 1.0, False)
    with pytest.raises(ValueError):
        O.oracle_fwd_varlen(q, q, q, q, [1, 4], [0, 4], 1.0, 1.0, False)


# ------------------------------------------------ context parallelism over N_K

def brute_force_state(q_t, k_t, q_s, k_s, st, ss, causal, k_offset, n_k_total):
    """Shard state from its definition with pure-Python loops, base-2 units."""
    B, H, nq, dt = q_t.shape
    n_sh, ds_ = k_t.shape[2], q_s.shape[3]
    L = lambda t: t.double().tolist()
    QT, KT, QS, KS = L(q_t), L(k_t), L(q_s), L(k_s)
    out = [[[[0.0] * nq for _ in range(H)] for _ in range(B)] for _ in range(5)]
    for b in range(B):
        for h in range(H):
            for i in range(nq):
                js = [j for j in range(n_sh)
                      if (not causal) or (k_offset + j) <= i + n_k_total - nq]
                if not js:
                    out[0][b][h][i] = out[1][b][h][i] = float("-inf")
                    continue
                tT = {j: st * sum(QT[b][h][i][c] * KT[b][h][j][c] for c in range(dt)) / math.log(2)
                      for j in js}
                tS = {j: ss * sum(QS[b][h][i][c] * KS[b][h][j][c] for c in range(ds_)) / math.log(2)
                      for j in js}
                mT, mS = max(tT.values()), max(tS.values())
                out[0][b][h][i], out[1][b][h][i] = mT, mS
                out[2][b][h][i] = sum(2.0 ** (tT[j] - mT) for j in js)
                out[3][b][h][i] = sum(2.0 ** (tS[j] - mS) for j in js)
                out[4][b][h][i] = sum(2.0 ** (tT[j] - mT) * (tT[j] - tS[j]) for j in js)
    return torch.tensor(out, dtype=F64)


@pytest.mark.parametrize("causal", [False, True])
def test_partial_state_against_brute_force(causal):
    q_t, k_t, q_s, k_s, _ = rand_case(1, 2, 5, 9, 3, 2, seed=61)
    sh = slice(6, 9)  # causal: row i sees global keys j <= i + 4, so rows 0, 1 see none
    ref = brute_force_state(q_t, k_t[:, :, sh], q_s, k_s[:, :, sh], 0.8, 1.3, causal, 6, 9)
    got = O.oracle_partial_state(q_t, k_t[:, :, sh], q_s, k_s[:, :, sh], 0.8, 1.3, causal, 6, 9)
    fin = torch.isfinite(ref)
    assert torch.equal(fin, torch.isfinite(got))
    torch.testing.assert_close(got[fin], ref[fin], rtol=1e-12, atol=1e-12)
    if causal:  # the identity state
        assert torch.all(got[2:, :, :, :2] == 0) and torch.all(torch.isinf(got[:2, :, :, :2]))
        assert torch.all(torch.isfinite(got[:, :, :, 2:]))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cuts", [[0, 11], [0, 4, 11], [0, 1, 7, 11], [0, 5, 5, 11]])
def test_merged_shards_equal_the_unsplit_oracle(causal, cuts):
    q_t, k_t, q_s, k_s, g = rand_case(2, 2, 8, 11, 4, 3, seed=62)
    args = (0.7, 1.1, causal)
    states = torch.stack([
        O.oracle_partial_state(q_t, k_t[:, :, a:b], q_s, k_s[:, :, a:b], *args, a, 11)
        for a, b in zip(cuts, cuts[1:])])
    kl, lt, ls = O.oracle_merge_states(states)
    kl_r, lt_r, ls_r = O.oracle_fwd(q_t, k_t, q_s, k_s, *args)
    torch.testing.assert_close(kl, kl_r, rtol=1e-11, atol=1e-12)
    torch.testing.assert_close(lt, lt_r, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(ls, ls_r, rtol=1e-12, atol=1e-12)
    # merge order does not matter
    kl2, _, _ = O.oracle_merge_states(states.flip(0))
    torch.testing.assert_close(kl2, kl, rtol=1e-13, atol=1e-14)
    # shard gradients: dQ parts sum to dQ, dK shards concatenate to dK (student, teacher)
    dq_r, dk_r = O.oracle_bwd(q_t, k_t, q_s, k_s, *args, g)
    dqt_r, dkt_r = O.oracle_bwd_teacher(q_t, k_t, q_s, k_s, *args, g)
    parts = [O.oracle_bwd_shard(q_t, k_t[:, :, a:b], q_s, k_s[:, :, a:b], *args, a, 11, lt_r,
                                ls_r, g) for a, b in zip(cuts, cuts[1:])]
    tparts = [O.oracle_bwd_teacher_shard(q_t, k_t[:, :, a:b], q_s, k_s[:, :, a:b], *args, a, 11,
                                         kl_r, lt_r, ls_r, g) for a, b in zip(cuts, cuts[1:])]
    torch.testing.assert_close(sum(p[0] for p in parts), dq_r, rtol=1e-10, atol=1e-12)
    torch.testing.assert_close(torch.cat([p[1] for p in parts], dim=2), dk_r, rtol=1e-10,
                               atol=1e-12)
    torch.testing.assert_close(sum(p[0] for p in tparts), dqt_r, rtol=1e-10, atol=1e-12)
    torch.testing.assert_close(torch.cat([p[1] for p in tparts], dim=2), dkt_r, rtol=1e-10,
                               atol=1e-12)


def test_merge_identity_and_grouped_heads():
    """A shard that no row can see merges as the identity; grouped K heads work per shard."""
    q_t, k_t, q_s, k_s, g = rand_case(1, 4, 6, 10, 3, 3, seed=63)
    k_t, k_s = k_t[:, :2], k_s[:, :1]
    st = [O.oracle_partial_state(q_t, k_t[:, :, a:b], q_s, k_s[:, :, a:b], 0.9, 0.6, True, a, 10)
          for a, b in [(0, 6), (6, 10)]]
    empty = O.oracle_partial_state(q_t, k_t[:, :, :2], q_s, k_s[:, :, :2], 0.9, 0.6, True, 50, 10)
    assert torch.all(torch.isinf(empty[:2])) and torch.all(empty[2:] == 0)
    kl, lt, _ = O.oracle_merge_states(torch.stack(st))
    kl_e, lt_e, _ = O.oracle_merge_states(torch.stack(st + [empty]))
    assert torch.equal(kl, kl_e) and torch.equal(lt, lt_e)
    kl_r, _, _ = O.oracle_fwd_gqa(q_t, k_t, q_s, k_s, 0.9, 0.6, True)
    torch.testing.assert_close(kl, kl_r, rtol=1e-11, atol=1e-12)


# ------------------------------------------------ timed CPU-baseline row work

def _row_work_case():
    q_t, k_t, q_s, k_s, g = rand_case(2, 2, 13, 17, 6, 5, seed=71)
    args = (q_t, k_t, q_s, k_s, 0.6, 0.9, True)
    # distinct (bh, i) rows: several per head, rows 0 (5 keys) and N_Q-1 (all 17 keys)
    rows = [(0, 0), (0, 5), (1, 12), (3, 7), (2, 3), (3, 12), (1, 0)]
    return args, g, rows


def _row_work_expected(args, g, rows):
    """What oracle_row_work must return, from the full oracle_fwd / oracle_bwd.

    KL and dQ rows are read off the full outputs. The summed dK contribution of the
    sampled rows is the dK of oracle_bwd with the upstream weights of every other row set
    to 0 (dK_S = sum_i g_i dS-row_i^T q_S[i] is linear in g), added over the heads.
    """
    B, H, n_q = g.shape
    kl_f, _, _ = O.oracle_fwd(*args)
    dq_f, _ = O.oracle_bwd(*args, g)
    g_sel = torch.zeros_like(g).view(B * H, n_q)
    for bh, i in rows:
        g_sel[bh, i] = g.view(B * H, n_q)[bh, i]
    _, dk_sel = O.oracle_bwd(*args, g_sel.view_as(g))
    n_k, d_s = dk_sel.shape[2], dk_sel.shape[3]
    kl = torch.stack([kl_f.view(B * H, n_q)[bh, i] for bh, i in rows])
    dq = torch.stack([dq_f.view(B * H, n_q, -1)[bh, i] for bh, i in rows])
    return kl, dq, dk_sel.view(B * H, n_k, d_s).sum(0)


def test_row_work_matches_full_oracle():
    """oracle_row_work (the timed CPU baseline and reference arm) does the same work as
    the full oracle: its KL, dQ rows and summed dK contributions equal oracle_fwd /
    oracle_bwd restricted to the sampled rows (N_Q != N_K, causal, ragged rows)."""
    args, g, rows = _row_work_case()
    kl, dq, dk = O.oracle_row_work(*args, g, rows)
    kl_e, dq_e, dk_e = _row_work_expected(args, g, rows)
    torch.testing.assert_close(kl, kl_e, rtol=1e-12, atol=1e-14)
    torch.testing.assert_close(dq, dq_e, rtol=1e-12, atol=1e-14)
    torch.testing.assert_close(dk, dk_e, rtol=1e-12, atol=1e-14)
    assert dk.abs().max() > 1e-3  # the sampled rows do contribute


def test_row_work_dropped_weight_is_caught(monkeypatch):
    """A planted mistake in the row work's dS (upstream weight g dropped) breaks the pin."""
    args, g, rows = _row_work_case()
    kl_e, dq_e, dk_e = _row_work_expected(args, g, rows)
    with monkeypatch.context() as m:
        m.setattr(O, "_sampled_ds", lambda g_rows, scale_s, p_s, p_t: scale_s * (p_s - p_t))
        _, _, dk = O.oracle_row_work(*args, g, rows)
    assert not torch.allclose(dk, dk_e, rtol=1e-6, atol=1e-9)
