"""Context-parallel plumbing on CPU: world_size 2 over gloo, keys split across the ranks.

The per-shard computations are the fp64 oracle's (injected through ShardOps), so this
checks the exchange itself: the all-gather of row states and their merge in the forward,
the all-reduce of the dQ parts in the backward, and the shard bookkeeping, against the
unsplit oracle. The CUDA shard kernels are checked against the oracle in the GPU tests.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from attention_kl_divergence_fwd_b200.context_parallel import (ShardOps, cp_backward, cp_forward,
                                                               even_shards)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def oracle_ops():
    from oracle import (oracle_bwd_shard, oracle_bwd_teacher_shard, oracle_merge_states,
                        oracle_partial_state)
    return ShardOps(oracle_partial_state, oracle_merge_states, oracle_bwd_shard,
                    oracle_bwd_teacher_shard)


def _case(seed=5):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    B, H, nq, nk = 1, 2, 160, 300
    return (mk(B, H, nq, 8), mk(B, H, nk, 8), mk(B, H, nq, 6), mk(B, H, nk, 6),
            torch.rand(B, H, nq, generator=g) + 0.5)


def _worker(rank, world, port, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q_t, k_t, q_s, k_s, g = _case()
        nk = k_t.shape[2]
        k0, n = even_shards(nk, world)[rank]
        sh = slice(k0, k0 + n)
        ops = oracle_ops()
        a = (q_t, k_t[:, :, sh].contiguous(), q_s, k_s[:, :, sh].contiguous(), 0.35, 0.4, causal,
             k0, nk)
        kl, lt, ls = cp_forward(*a, ops=ops)
        dq, dk = cp_backward(*a, lt, ls, g, ops=ops)
        dqt, dkt = cp_backward(*a, lt, ls, g, ops=ops, teacher=True, kl=kl)
        out[rank] = {"shard": (k0, n), "kl": kl, "lt": lt, "dq": dq, "dk": dk, "dqt": dqt,
                     "dkt": dkt}
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("causal", [True, False])
def test_context_parallel_gloo_world2_matches_unsplit_oracle(causal):
    from oracle import oracle_bwd, oracle_bwd_teacher, oracle_fwd
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), causal, out), nprocs=world, join=True)
    q_t, k_t, q_s, k_s, g = _case()
    args = (q_t, k_t, q_s, k_s, 0.35, 0.4, causal)
    kl, lt, _ = oracle_fwd(*args)
    dq, dk = oracle_bwd(*args, g)
    dqt, dkt = oracle_bwd_teacher(*args, g)
    shards = []
    for r in range(world):
        o = out[r]
        torch.testing.assert_close(o["kl"], kl, rtol=1e-10, atol=1e-12)
        torch.testing.assert_close(o["lt"], lt, rtol=1e-12, atol=1e-12)
        torch.testing.assert_close(o["dq"], dq, rtol=1e-9, atol=1e-12)
        torch.testing.assert_close(o["dqt"], dqt, rtol=1e-9, atol=1e-12)
        k0, n = o["shard"]
        shards.append((k0, n))
        torch.testing.assert_close(o["dk"], dk[:, :, k0:k0 + n], rtol=1e-9, atol=1e-12)
        torch.testing.assert_close(o["dkt"], dkt[:, :, k0:k0 + n], rtol=1e-9, atol=1e-12)
    assert shards == [(0, 256), (256, 44)]


def test_even_shards():
    assert even_shards(16384, 4) == [(0, 4096), (4096, 4096), (8192, 4096), (12288, 4096)]
    assert even_shards(1000, 3) == [(0, 384), (384, 384), (768, 232)]
    with pytest.raises(ValueError):
        even_shards(200, 3)
