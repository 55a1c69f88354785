"""Context parallelism over N_K: the keys of a sequence are split across ranks.

Each rank holds every query row (Q_T, Q_S) and one contiguous shard of the keys
(K_T, K_S rows k_offset .. k_offset + N_K_shard - 1 of N_K_total). The one-pass forward
leaves an online per-row state that merges associatively ("StreamKL: Fast and
Memory-Efficient KL Divergence for Boosting Attention Distillation", abstract: the forward
reduces both distributions together, online, in one pass), so the exchange is small:

  forward : state_r = streamkl_fwd_partial(shard r)          [5, B, H, N_Q] fp32 per rank
            all-gather the states (20 bytes per row per rank), then
            streamkl_merge_partial -> KL, LSE_T, LSE_S (identical on every rank)
  backward: streamkl_bwd_shard(shard r, merged LSEs, g) -> dK of the shard (final) and
            the shard's part of dQ; all-reduce(sum) of dQ over the ranks.

Nothing of size N_Q x N_K exists on any rank, and no rank holds another rank's keys.
The collectives run on the process group given (NCCL on GPUs). ``ops`` selects the
compute: the CUDA library by default.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Optional

import torch
import torch.distributed as dist


@dataclasses.dataclass(frozen=True)
class ShardOps:
    """The per-shard computations (the CUDA library's by default)."""
    fwd_partial: Callable   # (q_t, k_t, q_s, k_s, st, ss, causal, k_offset, n_k_total) -> state
    merge: Callable         # (states [R, 5, B, H, N_Q]) -> (kl, lse_t, lse_s)
    bwd_shard: Callable     # (..., k_offset, n_k_total, lse_t, lse_s, g) -> (dq_part, dk)
    bwd_teacher_shard: Callable  # (..., k_offset, n_k_total, kl, lse_t, lse_s, g) -> (dq, dk)


def cuda_ops() -> ShardOps:
    from . import (streamkl_bwd_shard, streamkl_bwd_teacher_shard, streamkl_fwd_partial,
                   streamkl_merge_partial)
    return ShardOps(streamkl_fwd_partial, streamkl_merge_partial, streamkl_bwd_shard,
                    streamkl_bwd_teacher_shard)


def _world(group) -> int:
    return dist.get_world_size(group) if dist.is_initialized() else 1


def _all_gather_stacked(t: torch.Tensor, group) -> torch.Tensor:
    """[R, *t.shape] with rank r's tensor at index r."""
    R = _world(group)
    out = torch.empty((R,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    if R == 1:
        out[0].copy_(t)
        return out
    dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group)
    return out


def _status_check(where: str, device, group) -> None:
    """With status checks on (see ``autograd.set_check_status``): read this rank's device
    error word and take the maximum over the group, so that every rank raises together
    and none is left waiting in the next collective."""
    from . import StreamKLError, device_status
    from . import autograd as _ag
    if not _ag._check_status:
        return
    with torch.cuda.device(device):
        st = device_status()
    if _world(group) > 1:
        t = torch.tensor([st], dtype=torch.int32, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
        st = int(t.item())
    if st != 0:
        raise StreamKLError(st, where)


def cp_forward(q_t, k_t, q_s, k_s, scale_t: float, scale_s: float, causal: bool,
               k_offset: int, n_k_total: int, group=None, ops: Optional[ShardOps] = None):
    """KL, LSE_T, LSE_S [B, H, N_Q] of the whole key range, on every rank of ``group``."""
    ops = ops or cuda_ops()
    state = ops.fwd_partial(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset, n_k_total)
    return ops.merge(_all_gather_stacked(state, group))


def cp_backward(q_t, k_t, q_s, k_s, scale_t: float, scale_s: float, causal: bool,
                k_offset: int, n_k_total: int, lse_t, lse_s, g, group=None,
                ops: Optional[ShardOps] = None, teacher: bool = False, kl=None):
    """(dQ, dK_shard): dQ of all keys (all-reduced over the ranks) and dK of this rank's
    keys, for the student (teacher=False) or a trainable teacher (teacher=True)."""
    ops = ops or cuda_ops()
    if teacher:
        dq, dk = ops.bwd_teacher_shard(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset,
                                       n_k_total, kl, lse_t, lse_s, g)
    else:
        dq, dk = ops.bwd_shard(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset,
                               n_k_total, lse_t, lse_s, g)
    if _world(group) > 1:
        dist.all_reduce(dq, op=dist.ReduceOp.SUM, group=group)
    return dq, dk


class ContextParallelKL(torch.autograd.Function):
    """Row-wise KL with the keys sharded over ``group``; gradients as StreamKLFunction.

    dQ gradients are all-reduced (every rank returns the full dQ for its replicated
    queries); dK gradients belong to the rank's own key shard.
    """

    @staticmethod
    def forward(ctx, q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset, n_k_total, group):
        kl, lse_t, lse_s = cp_forward(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset,
                                      n_k_total, group)
        _status_check("attention_kl_context_parallel forward", q_t.device, group)
        ctx.save_for_backward(q_t, k_t, q_s, k_s, kl, lse_t, lse_s)
        ctx.params = (scale_t, scale_s, causal, k_offset, n_k_total, group)
        ctx.mark_non_differentiable(lse_t, lse_s)
        return kl, lse_t, lse_s

    @staticmethod
    def backward(ctx, g_kl, _g_lse_t=None, _g_lse_s=None):
        q_t, k_t, q_s, k_s, kl, lse_t, lse_s = ctx.saved_tensors
        scale_t, scale_s, causal, k_offset, n_k_total, group = ctx.params
        g = g_kl.detach().to(torch.float32).contiguous()
        a = (q_t, k_t, q_s, k_s, scale_t, scale_s, causal, k_offset, n_k_total, lse_t, lse_s, g)
        # Every rank takes the same collective steps in the same order: the student
        # backward first, then the teacher backward, each decided by flags that are the
        # same on every rank (whether the inputs require grad).
        dq_t = dk_t = dq_s = dk_s = None
        if ctx.needs_input_grad[2] or ctx.needs_input_grad[3]:
            dq_s, dk_s = cp_backward(*a, group=group)
            dq_s, dk_s = dq_s.to(q_s.dtype), dk_s.to(k_s.dtype)
        if ctx.needs_input_grad[0] or ctx.needs_input_grad[1]:
            dq_t, dk_t = cp_backward(*a, group=group, teacher=True, kl=kl)
            dq_t, dk_t = dq_t.to(q_t.dtype), dk_t.to(k_t.dtype)
        _status_check("attention_kl_context_parallel backward", q_t.device, group)
        return dq_t, dk_t, dq_s, dk_s, None, None, None, None, None, None


def attention_kl_context_parallel(q_t, k_t, q_s, k_s, k_offset: int, n_k_total: int,
                                  scale_t: Optional[float] = None,
                                  scale_s: Optional[float] = None, causal: bool = False,
                                  group=None):
    """Per-row KL [B, H, N_Q] with this rank's key shard; call on every rank of ``group``."""
    scale_t = 1.0 / math.sqrt(q_t.shape[-1]) if scale_t is None else float(scale_t)
    scale_s = 1.0 / math.sqrt(q_s.shape[-1]) if scale_s is None else float(scale_s)
    kl, _, _ = ContextParallelKL.apply(q_t.contiguous(), k_t.contiguous(), q_s.contiguous(),
                                       k_s.contiguous(), scale_t, scale_s, bool(causal),
                                       int(k_offset), int(n_k_total), group)
    return kl


def even_shards(n_k_total: int, world: int):
    """Contiguous (k_offset, n_k_shard) of each rank: sizes differ by at most one key tile
    of 128 so the TMA tiles of every shard but the last stay full."""
    tiles = -(-n_k_total // 128)
    if tiles < world:
        raise ValueError(f"{n_k_total} keys make {tiles} tiles of 128: too few for {world} ranks")
    base, extra = divmod(tiles, world)
    out, start = [], 0
    for r in range(world):
        n = (base + (1 if r < extra else 0)) * 128
        n = max(0, min(n, n_k_total - start))
        out.append((start, n))
        start += n
    return out
