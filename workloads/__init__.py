"""Seeded synthetic inputs for the StreamKL attention-KL primitive.

This module only draws random tensors. It holds none of the method's arithmetic
(no scores, no softmax, no KL), so both the fp64 oracle and the CUDA path can be
fed from it without sharing any computation.

The five workloads follow the synthetic attention shapes the method is measured
on ("StreamKL: Fast and Memory-Efficient KL Divergence for Boosting Attention
Distillation", abstract: long-context attention distillation between a teacher
and a student attention map). The pages print no workload table, so the shapes,
value distributions and seeds here are a plain reading of those workloads:

* teacher Q and K are standard normal, rounded to bf16;
* the student is either the teacher plus sigma * N(0, 1) noise (added in fp32 to
  the bf16 teacher values, then rounded to bf16) or an independent N(0, 1) draw;
* g (the upstream gradient dLoss/dKL per query row) is 1, 1/N_Q or U(0, 1).

Draw order from one ``torch.Generator('cpu')`` seeded with ``1000 + k`` for
workload k: Q_T, K_T, then either (noise_Q, noise_K) or (Q_S, K_S), then g.
All tensors are contiguous row-major [B, H, N, d] (d innermost).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int            # 1-based position in the workload list; seeds are 1000 + index
    B: int
    H: int
    N_Q: int
    N_K: int
    d_T: int
    d_S: int
    scale_T: float
    scale_S: float
    causal: bool
    student: str          # "perturb" (teacher + sigma * noise) or "independent"
    sigma: float
    g: str                # "ones", "uniform" or "inv_nq"

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def bh(self) -> int:
        return self.B * self.H

    def with_sizes(self, **kw) -> "Workload":
        """Same recipe at other sizes (used for small parity cases)."""
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_n256_d64", 1, 1, 1, 256, 256, 64, 64, 1 / 8, 1 / 8, False,
                 "perturb", 0.5, "ones"),
        Workload("b2h16_n4096_d128_causal", 2, 2, 16, 4096, 4096, 128, 128,
                 1 / math.sqrt(128), 1 / math.sqrt(128), True, "perturb", 0.3, "uniform"),
        Workload("long_b1h32_n16384_d128_causal", 3, 1, 32, 16384, 16384, 128, 128,
                 1 / math.sqrt(128), 1 / math.sqrt(128), True, "independent", 0.0, "inv_nq"),
        Workload("mismatch_b4h32_n8192_dT128_dS64", 4, 4, 32, 8192, 8192, 128, 64,
                 1 / (2 * math.sqrt(128)), 1 / 8, False, "independent", 0.0, "ones"),
        Workload("extreme_b1h8_n65536_d128_causal", 5, 1, 8, 65536, 65536, 128, 128,
                 1 / math.sqrt(128), 1 / math.sqrt(128), True, "perturb", 0.2, "ones"),
    ]
}

WORKLOAD_LIST = sorted(WORKLOADS.values(), key=lambda w: w.index)


def make_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw the inputs of workload ``w`` on the CPU.

    Returns bf16 tensors ``q_t, k_t`` ([B,H,N_Q|N_K,d_T]), ``q_s, k_s``
    ([B,H,N_Q|N_K,d_S]) and the fp32 upstream gradient ``g`` ([B,H,N_Q]).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)

    def normal(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q_t = normal(w.B, w.H, w.N_Q, w.d_T).to(torch.bfloat16)
    k_t = normal(w.B, w.H, w.N_K, w.d_T).to(torch.bfloat16)
    if w.student == "perturb":
        if w.d_S != w.d_T:
            raise ValueError("a perturbed student needs d_S == d_T")
        nq = normal(w.B, w.H, w.N_Q, w.d_S)
        nk = normal(w.B, w.H, w.N_K, w.d_S)
        q_s = (q_t.float() + w.sigma * nq).to(torch.bfloat16)
        k_s = (k_t.float() + w.sigma * nk).to(torch.bfloat16)
    elif w.student == "independent":
        q_s = normal(w.B, w.H, w.N_Q, w.d_S).to(torch.bfloat16)
        k_s = normal(w.B, w.H, w.N_K, w.d_S).to(torch.bfloat16)
    else:
        raise ValueError(f"unknown student recipe {w.student!r}")

    if w.g == "ones":
        g = torch.ones(w.B, w.H, w.N_Q, dtype=torch.float32)
    elif w.g == "inv_nq":
        g = torch.full((w.B, w.H, w.N_Q), 1.0 / w.N_Q, dtype=torch.float32)
    elif w.g == "uniform":
        g = torch.rand(w.B, w.H, w.N_Q, generator=gen, dtype=torch.float32)
    else:
        raise ValueError(f"unknown g recipe {w.g!r}")
    return {"q_t": q_t.contiguous(), "k_t": k_t.contiguous(),
            "q_s": q_s.contiguous(), "k_s": k_s.contiguous(), "g": g.contiguous()}


def sample_rows(w: Workload, count: int = 256, seed: Optional[int] = None):
    """Seeded (bh, i) query rows for sampled checks at full size.

    Uniform without replacement over all B*H*N_Q rows, plus row 0 and row N_Q-1
    of the first sampled head so both ends of the causal triangle are covered.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(1234 + w.index if seed is None else seed)
    total = w.bh * w.N_Q
    flat = torch.randperm(total, generator=gen)[:count].tolist()
    rows = [(f // w.N_Q, f % w.N_Q) for f in flat]
    bh0 = rows[0][0]
    for extra in [(bh0, 0), (bh0, w.N_Q - 1)]:
        if extra not in rows:
            rows[-1 if extra[1] else -2] = extra
    return sorted(set(rows))


def sample_keys(w: Workload, heads: int = 2, keys: int = 64, seed: Optional[int] = None):
    """Seeded (bh, [key indices]) for sampled dK_S checks (includes key 0 and N_K-1)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(4321 + w.index if seed is None else seed)
    bhs = torch.randperm(w.bh, generator=gen)[:heads].tolist()
    out = []
    for bh in bhs:
        ks = torch.randperm(w.N_K, generator=gen)[:keys].tolist()
        ks[0], ks[-1] = 0, w.N_K - 1
        out.append((bh, sorted(set(ks))))
    return out


def flops_fwd(w: Workload) -> float:
    """Counted forward FLOPs: 2*|J|*(d_T + d_S) per query row (two QK^T contractions)."""
    return 2.0 * allowed_pairs(w) * (w.d_T + w.d_S) * w.bh


def flops_bwd(w: Workload) -> float:
    """Counted backward FLOPs: 2*|J|*(d_T + 3*d_S) per row (S_T, S_S, dQ_S, dK_S)."""
    return 2.0 * allowed_pairs(w) * (w.d_T + 3 * w.d_S) * w.bh


def flops_bwd_teacher(w: Workload) -> float:
    """Counted trainable-teacher backward FLOPs: 2*|J|*(3*d_T + d_S) per row
    (S_T, S_S, dQ_T, dK_T)."""
    return 2.0 * allowed_pairs(w) * (3 * w.d_T + w.d_S) * w.bh


def allowed_pairs(w: Workload) -> float:
    """Number of (i, j) pairs per head that the method counts.

    Non-causal: N_Q*N_K. Causal: the counting convention halves it (N_Q*N_K/2),
    as the throughput convention of attention kernels does.
    """
    return w.N_Q * w.N_K / (2.0 if w.causal else 1.0)


# ------------------------------------------------ packed variable-length sequences

def varlen_lengths(total: int, min_len: int, max_len: int, seed: int):
    """Seeded sequence lengths, uniform in [min_len, max_len], summing to ``total``
    (the last one is cut to fit): the length mix of a packed training batch."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    lens, left = [], total
    while left > 0:
        n = int(torch.randint(min_len, max_len + 1, (1,), generator=gen))
        n = min(n, left)
        lens.append(n)
        left -= n
    return lens


def cu_seqlens(lens):
    """[B+1] int32 offsets of packed sequences with the given lengths."""
    out = [0]
    for n in lens:
        out.append(out[-1] + int(n))
    return torch.tensor(out, dtype=torch.int32)


def make_varlen_inputs(lens_q, lens_k, H: int, H_kv_T: int, H_kv_S: int, d_T: int, d_S: int,
                       seed: int, sigma: Optional[float] = 0.3) -> Dict[str, torch.Tensor]:
    """Packed inputs: q_* [total_q, H, d], k_* [total_k, H_kv, d] (bf16), g [H, total_q]
    fp32 U(0, 1) and the offsets cu_q, cu_k (int32 [B+1]).

    The student is the teacher plus sigma * N(0, 1) when the shapes allow it (same head
    dims and K head counts; sigma not None), else an independent N(0, 1) draw. Draw order:
    Q_T, K_T, then (noise_Q, noise_K) or (Q_S, K_S), then g.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    tq, tk = int(sum(lens_q)), int(sum(lens_k))

    def normal(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q_t = normal(tq, H, d_T).to(torch.bfloat16)
    k_t = normal(tk, H_kv_T, d_T).to(torch.bfloat16)
    if sigma is not None and d_S == d_T and H_kv_S == H_kv_T:
        q_s = (q_t.float() + sigma * normal(tq, H, d_S)).to(torch.bfloat16)
        k_s = (k_t.float() + sigma * normal(tk, H_kv_S, d_S)).to(torch.bfloat16)
    else:
        q_s = normal(tq, H, d_S).to(torch.bfloat16)
        k_s = normal(tk, H_kv_S, d_S).to(torch.bfloat16)
    g = torch.rand(H, tq, generator=gen, dtype=torch.float32)
    return {"q_t": q_t, "k_t": k_t, "q_s": q_s, "k_s": k_s, "g": g,
            "cu_q": cu_seqlens(lens_q), "cu_k": cu_seqlens(lens_k)}


def varlen_pairs(lens_q, lens_k, causal: bool) -> float:
    """(i, j) pairs per head counted for FLOPs: per sequence n_q*n_k, halved when causal
    (the same convention as allowed_pairs)."""
    return sum(a * b / (2.0 if causal else 1.0) for a, b in zip(lens_q, lens_k))
