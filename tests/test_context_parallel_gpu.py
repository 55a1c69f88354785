"""Context parallelism end to end on one GPU: two ranks, each running the CUDA shard kernels
on its own key shard, joined by the real exchange code (cp_forward / cp_backward) over a
world-size-2 gloo group, against the unsplit fp64 oracle.

Both ranks are processes on cuda:0; their kernels never wait on one another (each shard
kernel is independent), only the host-side collectives do. gloo runs the all-gather of the
row states and the all-reduce of the dQ parts on CPU tensors, so the shard operations
below copy their GPU outputs to the host where the exchange happens, and the merged
states back to the GPU for the merge kernel: the same calls and the same order as with
NCCL, the bytes only take a detour through host memory.
"""
import math
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

KL_ABS, KL_REL = 1e-4, 2e-3
LSE_ABS, LSE_REL = 1e-4, 1e-5
GRAD_REL = 1e-2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case(seed=41):
    """B=1, H=2, 300 queries, 700 keys (ragged tiles), d_T=128, d_S=64; student near the
    teacher's scale, upstream weights in [0.5, 1.5)."""
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    B, H, nq, nk = 1, 2, 300, 700
    return (mk(B, H, nq, 128), mk(B, H, nk, 128), mk(B, H, nq, 64), mk(B, H, nk, 64),
            torch.rand(B, H, nq, generator=g) + 0.5)


SCALE_T, SCALE_S = 1 / math.sqrt(128), 1 / 8


def _host_boundary_ops():
    """The CUDA shard operations, with their outputs moved to the host for the gloo
    exchange and the gathered states moved back for the merge kernel."""
    import attention_kl_divergence_fwd_b200 as skl
    from attention_kl_divergence_fwd_b200.context_parallel import ShardOps

    def fwd_partial(*a):
        return skl.streamkl_fwd_partial(*a).cpu()

    def merge(states):
        return skl.streamkl_merge_partial(states.cuda().contiguous())

    def bwd_shard(*a):
        dq, dk = skl.streamkl_bwd_shard(*a)
        return dq.cpu(), dk.cpu()

    def bwd_teacher_shard(*a):
        dq, dk = skl.streamkl_bwd_teacher_shard(*a)
        return dq.cpu(), dk.cpu()

    return ShardOps(fwd_partial, merge, bwd_shard, bwd_teacher_shard)


def _worker(rank, world, port, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        import attention_kl_divergence_fwd_b200 as skl
        from attention_kl_divergence_fwd_b200.context_parallel import (cp_backward, cp_forward,
                                                                       even_shards)
        torch.cuda.set_device(0)
        q_t, k_t, q_s, k_s, g = _case()
        nk = k_t.shape[2]
        k0, n = even_shards(nk, world)[rank]
        sh = slice(k0, k0 + n)
        d = lambda t: t.cuda().contiguous()
        a = (d(q_t), d(k_t[:, :, sh]), d(q_s), d(k_s[:, :, sh]), SCALE_T, SCALE_S, causal, k0,
             nk)
        ops = _host_boundary_ops()
        kl, lt, ls = cp_forward(*a, ops=ops)
        dq, dk = cp_backward(*a, lt, ls, d(g), ops=ops)
        dqt, dkt = cp_backward(*a, lt, ls, d(g), ops=ops, teacher=True, kl=kl)
        torch.cuda.synchronize()
        status = skl.device_status()
        out[rank] = {"shard": (k0, n), "kl": kl.cpu(), "lt": lt.cpu(), "ls": ls.cpu(), "dq": dq,
                     "dk": dk, "dqt": dqt, "dkt": dkt, "status": status}
    finally:
        dist.destroy_process_group()


def _check_kl(got, ref):
    err = (got.double() - ref).abs()
    assert bool(((err <= KL_ABS) | (err <= KL_REL * ref.abs())).all()), err.max().item()


def _check_lse(got, ref):
    err = (got.double() - ref).abs()
    assert bool((err <= LSE_ABS + LSE_REL * ref.abs()).all()), err.max().item()


def _rel(got, ref):
    return ((got.double() - ref).norm() / ref.norm()).item()


@pytest.mark.timeout(600)
@pytest.mark.parametrize("causal", [True, False])
def test_context_parallel_two_ranks_cuda_kernels_and_exchange(causal):
    from oracle import oracle_bwd, oracle_bwd_teacher, oracle_fwd
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), causal, out), nprocs=world,
                       join=True, start_method="spawn")
    q_t, k_t, q_s, k_s, g = _case()
    args = (q_t, k_t, q_s, k_s, SCALE_T, SCALE_S, causal)
    kl, lt, ls = oracle_fwd(*args)
    dq, dk = oracle_bwd(*args, g)
    dqt, dkt = oracle_bwd_teacher(*args, g)
    shards = []
    for r in range(world):
        o = out[r]
        assert o["status"] == 0
        _check_kl(o["kl"], kl)
        _check_lse(o["lt"], lt)
        _check_lse(o["ls"], ls)
        assert _rel(o["dq"], dq) <= GRAD_REL and _rel(o["dqt"], dqt) <= GRAD_REL
        k0, n = o["shard"]
        shards.append((k0, n))
        assert _rel(o["dk"], dk[:, :, k0:k0 + n]) <= GRAD_REL
        assert _rel(o["dkt"], dkt[:, :, k0:k0 + n]) <= GRAD_REL
    # both ranks hold the same merged rows and the same all-reduced dQ
    assert torch.equal(out[0]["kl"], out[1]["kl"]) and torch.equal(out[0]["dq"], out[1]["dq"])
    assert shards == [(0, 384), (384, 316)]
