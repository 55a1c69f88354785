"""autograd wrapper and loss reductions: values and gradients vs the fp64 oracle.

The wrapper returns gradients in the dtype of the inputs (bf16), so each gradient is the
library's fp32 gradient rounded once to bf16. The tests check exactly that (element by element
within one rounding of a direct call of the entry point), hold the fp32 gradient to the 1e-2 relative
Frobenius bound of the parity tests, and hold the bf16 gradient to that bound plus what
one rounding can add: bf16 keeps 8 significant bits, so round-to-nearest changes each
element by at most 2^-8 of its magnitude and the whole tensor by at most 2^-8 of its norm.
"""
import math

import pytest
import torch

from attention_kl_divergence_fwd_b200 import autograd as ska
from workloads import WORKLOADS, make_inputs

GRAD_TOL = 1e-2                 # fp32 gradients of the library vs the oracle
BF16_TOL = GRAD_TOL + 2.0 ** -8  # the same after one rounding to bf16 (about 1.39e-2)


def _rel(a, b):
    return ((a.double().cpu() - b).norm() / b.norm()).item()


def _one_rounding(grad_bf16, ref32):
    """Each element of the bf16 gradient is the fp32 one rounded to nearest: within 2^-8 of
    its magnitude (plus a sliver for the run-to-run order of the dQ reduce-adds)."""
    err = (grad_bf16.float() - ref32).abs()
    bound = (2.0 ** -8 + 1e-5) * ref32.abs() + 1e-6 * ref32.abs().max()
    return bool((err <= bound).all())


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
    assert q_s.grad.dtype == torch.bfloat16 and k_s.grad.dtype == torch.bfloat16
    # the wrapper's gradient is the entry point's fp32 gradient rounded once
    from attention_kl_divergence_fwd_b200 import streamkl_bwd, streamkl_fwd
    _, lse_t, lse_s = streamkl_fwd(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T,
                                   w.scale_S, True)
    gg = torch.full((w.B, w.H, w.N_Q), g, dtype=torch.float32, device="cuda")
    dq32, dk32 = streamkl_bwd(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T, w.scale_S,
                              True, lse_t, lse_s, gg)
    assert _one_rounding(q_s.grad, dq32) and _one_rounding(k_s.grad, dk32)
    assert _rel(dq32, dq) < GRAD_TOL and _rel(dk32, dk) < GRAD_TOL
    assert _rel(q_s.grad, dq) < BF16_TOL and _rel(k_s.grad, dk) < BF16_TOL


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
    from attention_kl_divergence_fwd_b200 import streamkl_bwd_teacher, streamkl_fwd
    kl, lse_t, lse_s = streamkl_fwd(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T,
                                    w.scale_S, True)
    gg = torch.ones(w.B, w.H, w.N_Q, dtype=torch.float32, device="cuda")
    dq32, dk32 = streamkl_bwd_teacher(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T,
                                      w.scale_S, True, kl, lse_t, lse_s, gg)
    assert _one_rounding(q_t.grad, dq32) and _one_rounding(k_t.grad, dk32)
    assert _rel(dq32, dq) < GRAD_TOL and _rel(dk32, dk) < GRAD_TOL
    assert _rel(q_t.grad, dq) < BF16_TOL and _rel(k_t.grad, dk) < BF16_TOL


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
    dq, dk = oracle_bwd_varlen(*args, gg)
    assert _rel(q_s.grad, dq) < BF16_TOL and _rel(k_s.grad, dk) < BF16_TOL
    dqt, _ = oracle_bwd_teacher_varlen(*args, gg)
    assert _rel(q_t.grad, dqt) < BF16_TOL


@pytest.mark.gpu
def test_status_check_raises_on_device_error():
    """With status checks on, an error the kernel records on the device (here packed offsets
    that decrease, found by the forward kernel) surfaces as StreamKLError from the wrapper;
    with them off, the call returns and the error stays readable through device_status()."""
    import attention_kl_divergence_fwd_b200 as skl
    from workloads import make_varlen_inputs
    x = make_varlen_inputs([100, 100, 100], [100, 100, 100], 2, 2, 2, 64, 64, seed=8)
    d = {k: v.cuda() for k, v in x.items()}
    bad = torch.tensor([0, 200, 100, 300], dtype=torch.int32, device="cuda")
    args = (d["q_t"], d["k_t"], d["q_s"], d["k_s"], bad, d["cu_k"], 200, 100, 0.125, 0.125,
            False)
    try:
        ska.set_check_status(True)
        with pytest.raises(skl.StreamKLError) as e:
            ska.attention_kl_varlen(*args)
        assert e.value.status == 1  # STREAMKL_ERR_INVALID_ARG, cleared by the read
        ska.set_check_status(False)
        ska.attention_kl_varlen(*args)
        assert skl.device_status() == 1
        assert skl.device_status() == 0
    finally:
        ska.set_check_status(False)
