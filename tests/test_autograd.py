"""autograd wrapper and loss reductions: values and gradients vs the fp64 oracle."""
import math

import pytest
import torch

from attention_kl_divergence_fwd_b200 import autograd as ska
from workloads import WORKLOADS, make_inputs


def test_unknown_reduction_rejected_before_any_launch():
    with pytest.raises(ValueError):
        ska.attention_kl_loss(None, None, None, None, reduction="avg")


def test_reduce_kl_defines_g():
    kl = torch.arange(24, dtype=torch.float32).reshape(2, 3, 4).requires_grad_(True)
    for red, g in [("sum", 1.0), ("mean", 1.0 / 24), ("batchmean", 0.5)]:
        kl.grad = None
        ska.reduce_kl(kl, red).backward()
        assert torch.allclose(kl.grad, torch.full_like(kl, g))
    assert ska.reduce_kl(kl, "none") is kl


@pytest.mark.gpu
@pytest.mark.parametrize("reduction", ["mean", "sum", "batchmean"])
def test_loss_and_grads_match_oracle(reduction):
    from oracle import oracle_bwd, oracle_fwd
    w = WORKLOADS["b2h16_n4096_d128_causal"].with_sizes(B=2, H=2, N_Q=300, N_K=300)
    x = make_inputs(w, seed=17)
    d = {k: v.cuda() for k, v in x.items()}
    q_s = d["q_s"].clone().requires_grad_(True)
    k_s = d["k_s"].clone().requires_grad_(True)
    loss = ska.attention_kl_loss(d["q_t"], d["k_t"], q_s, k_s, w.scale_T, w.scale_S, True,
                                 reduction)
    loss.backward()
    args = (x["q_t"], x["k_t"], x["q_s"], x["k_s"], w.scale_T, w.scale_S, True)
    kl, _, _ = oracle_fwd(*args)
    n = kl.numel()
    g = {"sum": 1.0, "mean": 1.0 / n, "batchmean": 1.0 / w.B}[reduction]
    ref_loss = kl.sum() * g
    assert abs(loss.item() - ref_loss.item()) <= 1e-4 * max(1.0, abs(ref_loss.item()))
    dq, dk = oracle_bwd(*args, torch.full_like(x["g"], g))
    rel = lambda a, b: ((a.double().cpu() - b).norm() / b.norm()).item()
    assert q_s.grad.dtype == torch.bfloat16 and k_s.grad.dtype == torch.bfloat16
    assert rel(q_s.grad, dq) < 1.5e-2
    assert rel(k_s.grad, dk) < 1.5e-2


@pytest.mark.gpu
def test_trainable_teacher_grads_match_oracle():
    from oracle import oracle_bwd_teacher
    w = WORKLOADS["b2h16_n4096_d128_causal"].with_sizes(B=1, H=2, N_Q=260, N_K=260)
    x = make_inputs(w, seed=23)
    d = {k: v.cuda() for k, v in x.items()}
    q_t = d["q_t"].clone().requires_grad_(True)
    k_t = d["k_t"].clone().requires_grad_(True)
    ska.attention_kl_loss(q_t, k_t, d["q_s"], d["k_s"], w.scale_T, w.scale_S, True,
                          "sum").backward()
    dq, dk = oracle_bwd_teacher(x["q_t"], x["k_t"], x["q_s"], x["k_s"], w.scale_T, w.scale_S,
                                True, torch.ones_like(x["g"]))
    rel = lambda a, b: ((a.double().cpu() - b).norm() / b.norm()).item()
    assert rel(q_t.grad, dq) < 1.5e-2 and rel(k_t.grad, dk) < 1.5e-2


@pytest.mark.gpu
def test_default_scales_and_frozen_teacher():
    w = WORKLOADS["tiny_n256_d64"]
    x = make_inputs(w)
    d = {k: v.cuda() for k, v in x.items()}
    q_s = d["q_s"].clone().requires_grad_(True)
    kl = ska.attention_kl(d["q_t"], d["k_t"], q_s, d["k_s"])  # scales default to 1/sqrt(64)
    kl.sum().backward()
    assert q_s.grad is not None and d["q_t"].grad is None
    kl2 = ska.attention_kl(d["q_t"], d["k_t"], d["q_s"], d["k_s"], 1 / math.sqrt(64),
                           1 / math.sqrt(64))
    assert torch.equal(kl.detach(), kl2)


@pytest.mark.gpu
@pytest.mark.parametrize("reduction", ["mean", "batchmean"])
def test_varlen_loss_and_grads_match_oracle(reduction):
    from oracle import oracle_bwd_teacher_varlen, oracle_bwd_varlen, oracle_fwd_varlen
    from workloads import make_varlen_inputs
    lens_q, lens_k = [150, 0, 270, 33], [150, 20, 200, 80]
    x = make_varlen_inputs(lens_q, lens_k, 4, 2, 4, 128, 64, seed=31)
    d = {k: v.cuda() for k, v in x.items()}
    q_t = d["q_t"].clone().requires_grad_(True)
    q_s = d["q_s"].clone().requires_grad_(True)
    k_s = d["k_s"].clone().requires_grad_(True)
    st, ss = 0.09, 0.125
    loss = ska.attention_kl_varlen_loss(q_t, d["k_t"], q_s, k_s, d["cu_q"], d["cu_k"], 270, 200,
                                        st, ss, True, reduction)
    loss.backward()
    args = (x["q_t"], x["k_t"], x["q_s"], x["k_s"], x["cu_q"].tolist(), x["cu_k"].tolist(), st,
            ss, True)
    kl, _, _ = oracle_fwd_varlen(*args)
    g = 1.0 / kl.numel() if reduction == "mean" else 1.0 / len(lens_q)
    assert abs(loss.item() - kl.sum().item() * g) <= 1e-4 * max(1.0, abs(kl.sum().item() * g))
    gg = torch.full_like(x["g"], g)
    rel = lambda a, b: ((a.double().cpu() - b).norm() / b.norm()).item()
    dq, dk = oracle_bwd_varlen(*args, gg)
    assert rel(q_s.grad, dq) < 1.5e-2 and rel(k_s.grad, dk) < 1.5e-2
    dqt, _ = oracle_bwd_teacher_varlen(*args, gg)
    assert rel(q_t.grad, dqt) < 1.5e-2
