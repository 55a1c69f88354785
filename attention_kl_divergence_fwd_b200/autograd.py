"""PyTorch autograd wrapper over the StreamKL C ABI, with the usual loss reductions.

    loss = attention_kl_loss(q_t, k_t, q_s, k_s, causal=True, reduction="mean")
    loss.backward()          # fills q_s.grad and k_s.grad; q_t/k_t too if they require grad

The forward calls ``streamkl_fwd`` (per-row KL plus the two log-sum-exps it saves for
backward); the backward calls ``streamkl_bwd`` with g = dLoss/dKL per row, which the
reduction determines: 1 for "sum", 1/(B*H*N_Q) for "mean", 1/B for "batchmean". Only
the O(B*H*N_Q) row vector is touched by PyTorch; every O(N_Q*N_K) step runs in the CUDA
kernels and nothing of that size is ever allocated.

Packed variable-length batches use ``attention_kl_varlen`` / ``attention_kl_varlen_loss``
(q_* [total_q, H, d], k_* [total_k, H_kv, d], int32 cu_seqlens on the device); there
"batchmean" divides by the number of sequences.

Errors found on the device (a pipeline wait that ran out, malformed packed offsets) are
recorded in the library's device error word and the kernel returns early, leaving some
outputs unwritten; the launch itself still succeeds. The wrappers check that word after
every forward and backward when status checks are on (``set_check_status(True)`` or the
environment variable STREAMKL_CHECK_STATUS=1) and raise ``StreamKLError``. The check
synchronises the stream, so it is off by default; with it off, poll
``attention_kl_divergence_fwd_b200.device_status()`` yourself (for instance once per
training step) before trusting the step's gradients.
"""
from __future__ import annotations

import math
import os
from typing import Optional

import torch

from . import (StreamKLError, device_status, streamkl_bwd, streamkl_bwd_gqa, streamkl_bwd_teacher,
               streamkl_bwd_teacher_gqa, streamkl_bwd_teacher_varlen, streamkl_bwd_varlen,
               streamkl_fwd, streamkl_fwd_gqa, streamkl_fwd_varlen)

REDUCTIONS = ("none", "sum", "mean", "batchmean")

_check_status = os.environ.get("STREAMKL_CHECK_STATUS", "0") not in ("", "0")


def set_check_status(enabled: bool) -> None:
    """Turn the device-status check after every wrapped forward and backward on or off."""
    global _check_status
    _check_status = bool(enabled)


def _after_launch(where: str, device) -> None:
    """Raise StreamKLError when status checks are on and the device reported an error."""
    if _check_status:
        with torch.cuda.device(device):
            st = device_status()
        if st != 0:
            raise StreamKLError(st, where)


class StreamKLFunction(torch.autograd.Function):
    """Row-wise KL(P_T || P_S) of two attention maps.

    Gradients flow to Q_S and K_S (streamkl_bwd) and, when the teacher inputs require
    grad, to Q_T and K_T as well (streamkl_bwd_teacher). K tensors with fewer heads than
    the queries select the grouped-query (GQA) entry points.
    """

    @staticmethod
    def forward(ctx, q_t, k_t, q_s, k_s, scale_t: float, scale_s: float, causal: bool):
        gqa = k_t.shape[1] != q_t.shape[1] or k_s.shape[1] != q_s.shape[1]
        fwd = streamkl_fwd_gqa if gqa else streamkl_fwd
        kl, lse_t, lse_s = fwd(q_t, k_t, q_s, k_s, scale_t, scale_s, causal)
        _after_launch("attention_kl forward", q_t.device)
        ctx.save_for_backward(q_t, k_t, q_s, k_s, kl, lse_t, lse_s)
        ctx.params = (scale_t, scale_s, causal, gqa)
        ctx.mark_non_differentiable(lse_t, lse_s)
        return kl, lse_t, lse_s

    @staticmethod
    def backward(ctx, g_kl, _g_lse_t=None, _g_lse_s=None):
        q_t, k_t, q_s, k_s, kl, lse_t, lse_s = ctx.saved_tensors
        scale_t, scale_s, causal, gqa = ctx.params
        g = g_kl.detach().to(torch.float32).contiguous()
        need_t = ctx.needs_input_grad[0] or ctx.needs_input_grad[1]
        need_s = ctx.needs_input_grad[2] or ctx.needs_input_grad[3]
        dq_t = dk_t = dq_s = dk_s = None
        if need_s:
            bwd = streamkl_bwd_gqa if gqa else streamkl_bwd
            dq_s, dk_s = bwd(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, lse_t, lse_s, g)
            dq_s, dk_s = dq_s.to(q_s.dtype), dk_s.to(k_s.dtype)
        if need_t:
            bwd_t = streamkl_bwd_teacher_gqa if gqa else streamkl_bwd_teacher
            dq_t, dk_t = bwd_t(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, kl, lse_t, lse_s, g)
            dq_t, dk_t = dq_t.to(q_t.dtype), dk_t.to(k_t.dtype)
        _after_launch("attention_kl backward", q_t.device)
        return dq_t, dk_t, dq_s, dk_s, None, None, None


def attention_kl(q_t, k_t, q_s, k_s, scale_t: Optional[float] = None,
                 scale_s: Optional[float] = None, causal: bool = False):
    """Per-row KL [B, H, N_Q] (fp32), differentiable w.r.t. q_s, k_s (and q_t, k_t).

    Default scales are 1/sqrt(d) of each side. Tensors: bf16 [B, H, N, d] on one GPU.
    """
    scale_t = 1.0 / math.sqrt(q_t.shape[-1]) if scale_t is None else float(scale_t)
    scale_s = 1.0 / math.sqrt(q_s.shape[-1]) if scale_s is None else float(scale_s)
    kl, _, _ = StreamKLFunction.apply(q_t.contiguous(), k_t.contiguous(), q_s.contiguous(),
                                      k_s.contiguous(), scale_t, scale_s, bool(causal))
    return kl


def reduce_kl(kl: torch.Tensor, reduction: str = "mean") -> torch.Tensor:
    """Reduce per-row KL [B, H, N_Q] to a loss; the reduction fixes g = dLoss/dKL."""
    if reduction == "none":
        return kl
    if reduction == "sum":
        return kl.sum()
    if reduction == "mean":
        return kl.mean()
    if reduction == "batchmean":
        return kl.sum() / kl.shape[0]
    raise ValueError(f"reduction must be one of {REDUCTIONS}, got {reduction!r}")


def attention_kl_loss(q_t, k_t, q_s, k_s, scale_t: Optional[float] = None,
                      scale_s: Optional[float] = None, causal: bool = False,
                      reduction: str = "mean") -> torch.Tensor:
    """Attention-distillation loss: reduction of the row-wise KL(P_T || P_S)."""
    if reduction not in REDUCTIONS:
        raise ValueError(f"reduction must be one of {REDUCTIONS}, got {reduction!r}")
    return reduce_kl(attention_kl(q_t, k_t, q_s, k_s, scale_t, scale_s, causal), reduction)


class StreamKLVarlenFunction(torch.autograd.Function):
    """Row-wise KL over packed variable-length sequences; KL is [H, total_q]."""

    @staticmethod
    def forward(ctx, q_t, k_t, q_s, k_s, cu_q, cu_k, max_q: int, max_k: int, scale_t: float,
                scale_s: float, causal: bool):
        H, tq = q_t.shape[1], q_t.shape[0]
        # Rows that belong to no sequence are not written by the kernel: start them at 0
        # (KL) so that reductions over the whole tensor ignore them.
        kl = torch.zeros(H, tq, device=q_t.device, dtype=torch.float32)
        kl, lse_t, lse_s = streamkl_fwd_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k, max_q, max_k,
                                               scale_t, scale_s, causal, kl=kl)
        _after_launch("attention_kl_varlen forward", q_t.device)
        ctx.save_for_backward(q_t, k_t, q_s, k_s, cu_q, cu_k, kl, lse_t, lse_s)
        ctx.params = (max_q, max_k, scale_t, scale_s, causal)
        ctx.mark_non_differentiable(lse_t, lse_s)
        return kl, lse_t, lse_s

    @staticmethod
    def backward(ctx, g_kl, _g_lse_t=None, _g_lse_s=None):
        q_t, k_t, q_s, k_s, cu_q, cu_k, kl, lse_t, lse_s = ctx.saved_tensors
        a = (q_t, k_t, q_s, k_s, cu_q, cu_k) + ctx.params
        g = g_kl.detach().to(torch.float32).contiguous()
        dq_t = dk_t = dq_s = dk_s = None
        if ctx.needs_input_grad[2] or ctx.needs_input_grad[3]:
            dq_s, dk_s = streamkl_bwd_varlen(*a, lse_t, lse_s, g)
            dq_s, dk_s = dq_s.to(q_s.dtype), dk_s.to(k_s.dtype)
        if ctx.needs_input_grad[0] or ctx.needs_input_grad[1]:
            dq_t, dk_t = streamkl_bwd_teacher_varlen(*a, kl, lse_t, lse_s, g)
            dq_t, dk_t = dq_t.to(q_t.dtype), dk_t.to(k_t.dtype)
        _after_launch("attention_kl_varlen backward", q_t.device)
        return dq_t, dk_t, dq_s, dk_s, None, None, None, None, None, None, None


def attention_kl_varlen(q_t, k_t, q_s, k_s, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                        max_seqlen_k: int, scale_t: Optional[float] = None,
                        scale_s: Optional[float] = None, causal: bool = False):
    """Per-row KL [H, total_q] (fp32) of packed sequences, differentiable like
    ``attention_kl``. Rows outside every sequence are 0."""
    scale_t = 1.0 / math.sqrt(q_t.shape[-1]) if scale_t is None else float(scale_t)
    scale_s = 1.0 / math.sqrt(q_s.shape[-1]) if scale_s is None else float(scale_s)
    kl, _, _ = StreamKLVarlenFunction.apply(
        q_t.contiguous(), k_t.contiguous(), q_s.contiguous(), k_s.contiguous(),
        cu_seqlens_q.to(torch.int32).contiguous(), cu_seqlens_k.to(torch.int32).contiguous(),
        int(max_seqlen_q), int(max_seqlen_k), scale_t, scale_s, bool(causal))
    return kl


def attention_kl_varlen_loss(q_t, k_t, q_s, k_s, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                             max_seqlen_k: int, scale_t: Optional[float] = None,
                             scale_s: Optional[float] = None, causal: bool = False,
                             reduction: str = "mean") -> torch.Tensor:
    """Reduction of the packed row-wise KL: "mean" over the H*total_q rows, "batchmean"
    divided by the number of sequences B."""
    if reduction not in REDUCTIONS:
        raise ValueError(f"reduction must be one of {REDUCTIONS}, got {reduction!r}")
    kl = attention_kl_varlen(q_t, k_t, q_s, k_s, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                             max_seqlen_k, scale_t, scale_s, causal)
    if reduction == "batchmean":
        return kl.sum() / (cu_seqlens_q.numel() - 1)
    return reduce_kl(kl, reduction)
