"""Multi-rank plumbing of bench.py on CPU: world_size 2 over gloo (no GPU).

Heads are independent in StreamKL, so N GPUs run N independent replicas (weak
scaling) with no data-path collective; the only cross-rank operations are the
barrier around the timed region and the max-over-ranks of the measured time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank)
    bench.barrier(w)
    # Rank r pretends its timed region took 10 + r ms: the job time is the slowest rank.
    t = bench.max_over_ranks(10.0 + r, w)
    out[rank] = t
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_gloo_world2():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert dict(out) == {0: 11.0, 1: 11.0}


def test_weak_scaling_value_counts_every_rank():
    """value = N x (per-rank flops) / max-over-ranks time."""
    import bench
    from workloads import WORKLOADS, flops_bwd, flops_fwd
    w = WORKLOADS["long_b1h32_n16384_d128_causal"]
    per_rank = flops_fwd(w) + flops_bwd(w)
    assert per_rank == pytest.approx(6.597e12, rel=1e-3)  # 2.20 TFLOP fwd + 4.40 TFLOP bwd
    cfg = bench.config_of(w, 4)
    assert cfg["workload"] == w.name and "replicas" in cfg["parallelism"]
