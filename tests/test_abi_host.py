"""C-ABI library: loads, exports every declared symbol, host-side argument checks.

No CUDA call is made here: every case below is rejected on the host before any
launch, so these run on a machine without a GPU.
"""
import ctypes
import os
import re
import subprocess

import pytest

import attention_kl_divergence_fwd_b200 as skl
from attention_kl_divergence_fwd_b200 import build as skl_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "streamkl.h")


@pytest.fixture(scope="module")
def lib():
    skl_build.build()
    return skl.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(streamkl_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_exports():
    assert declared_functions() == sorted(skl.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", skl.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (streamkl_[a-z0-9_]+)\b", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code in range(6):
        assert skl.status_string(code)
    assert skl.version() >= 100


P = 1 << 12  # a fake, 16-byte aligned, non-null address: never dereferenced on these paths


def fwd(**kw):
    a = dict(q_t=P, k_t=P, q_s=P, k_s=P, B=1, H=1, N_Q=128, N_K=128, d_T=128, d_S=128,
             scale_T=0.1, scale_S=0.1, causal=False, kl=P, lse_t=P, lse_s=P, stream=0)
    a.update(kw)
    return skl.streamkl_fwd_raw(**a)


def bwd(**kw):
    a = dict(q_t=P, k_t=P, q_s=P, k_s=P, B=1, H=1, N_Q=128, N_K=128, d_T=128, d_S=128,
             scale_T=0.1, scale_S=0.1, causal=False, lse_t=P, lse_s=P, g=P, dq_s=P, dk_s=P,
             stream=0)
    a.update(kw)
    return skl.streamkl_bwd_raw(**a)


def bwd_teacher(**kw):
    a = dict(q_t=P, k_t=P, q_s=P, k_s=P, B=1, H=1, N_Q=128, N_K=128, d_T=128, d_S=128,
             scale_T=0.1, scale_S=0.1, causal=False, kl=P, lse_t=P, lse_s=P, g=P, dq_t=P,
             dk_t=P, stream=0)
    a.update(kw)
    return skl.streamkl_bwd_teacher_raw(**a)


@pytest.mark.parametrize("fn", [fwd, bwd, bwd_teacher])
def test_host_validation(lib, fn):
    assert fn(q_t=0) == 1
    assert fn(k_s=0) == 1
    assert fn(B=0) == 1
    assert fn(N_Q=0) == 1
    assert fn(N_K=-5) == 1
    assert fn(scale_T=float("nan")) == 1
    assert fn(scale_S=float("inf")) == 1
    assert fn(d_T=96) == 2
    assert fn(d_S=32) == 2
    assert fn(d_T=256) == 2
    assert fn(B=1 << 12, H=1 << 12) == 2          # B*H beyond the grid limit
    assert fn(H=4096, N_Q=1 << 20) == 2            # B*H*N beyond int32 row indices
    assert fn(q_t=P + 8) == 3
    assert fn(k_s=P + 2) == 3


def test_gqa_head_groups_validated(lib):
    def fwd_gqa(H, hkt, hks):
        return lib.streamkl_fwd_gqa(P, P, P, P, 1, H, hkt, hks, 128, 128, 128, 128, 0.1, 0.1, 0,
                                    P, P, P, 0)
    assert fwd_gqa(8, 3, 8) == 2     # 3 does not divide 8
    assert fwd_gqa(8, 8, 0) == 2     # no K heads
    assert fwd_gqa(8, 4, 16) == 2    # more K heads than query heads
    assert lib.streamkl_bwd_gqa(P, P, P, P, 1, 6, 4, 2, 128, 128, 128, 128, 0.1, 0.1, 0,
                                P, P, P, P, P, 0) == 2
    assert lib.streamkl_bwd_teacher_gqa(P, P, P, P, 1, 6, 3, 5, 128, 128, 128, 128, 0.1, 0.1,
                                        0, P, P, P, P, P, P, 0) == 2
    assert lib.streamkl_fwd_gqa(0, P, P, P, 1, 8, 4, 2, 128, 128, 128, 128, 0.1, 0.1, 0,
                                P, P, P, 0) == 1


def test_host_validation_outputs(lib):
    assert fwd(kl=0) == 1
    assert fwd(lse_s=P + 4) == 3
    assert bwd(g=0) == 1
    assert bwd(dk_s=P + 12) == 3
    assert bwd(lse_t=0) == 1
    assert bwd_teacher(kl=0) == 1
    assert bwd_teacher(kl=P + 4) == 3
    assert bwd_teacher(dk_t=P + 8) == 3


def fwd_varlen(lib, **kw):
    a = dict(q_t=P, k_t=P, q_s=P, k_s=P, cu_q=P, cu_k=P, B=2, H=4, H_kv_T=4, H_kv_S=2,
             total_q=300, total_k=280, max_q=200, max_k=200, d_T=128, d_S=64, scale_T=0.1,
             scale_S=0.1, causal=1, kl=P, lse_t=P, lse_s=P, stream=0)
    a.update(kw)
    return lib.streamkl_fwd_varlen(*a.values())


def bwd_varlen(lib, teacher=False, **kw):
    a = dict(q_t=P, k_t=P, q_s=P, k_s=P, cu_q=P, cu_k=P, B=2, H=4, H_kv_T=4, H_kv_S=2,
             total_q=300, total_k=280, max_q=200, max_k=200, d_T=128, d_S=64, scale_T=0.1,
             scale_S=0.1, causal=1)
    if teacher:
        a["kl"] = P
    a.update(dict(lse_t=P, lse_s=P, g=P, dq=P, dk=P, stream=0))
    a.update(kw)
    fn = lib.streamkl_bwd_teacher_varlen if teacher else lib.streamkl_bwd_varlen
    return fn(*a.values())


@pytest.mark.parametrize("call", ["fwd", "bwd", "bwd_teacher"])
def test_varlen_host_validation(lib, call):
    fn = {"fwd": lambda **kw: fwd_varlen(lib, **kw),
          "bwd": lambda **kw: bwd_varlen(lib, **kw),
          "bwd_teacher": lambda **kw: bwd_varlen(lib, teacher=True, **kw)}[call]
    assert fn(cu_q=0) == 1
    assert fn(cu_k=0) == 1
    assert fn(B=0) == 1
    assert fn(total_q=-1) == 1
    assert fn(total_k=-3) == 1
    assert fn(max_q=-1) == 1
    assert fn(q_t=0) == 1                       # rows but no Q
    assert fn(k_s=0) == 1                       # keys but no K
    assert fn(scale_S=float("nan")) == 1
    assert fn(d_T=96) == 2
    assert fn(H_kv_T=3) == 2                    # 3 does not divide 4
    assert fn(H=64, H_kv_T=64, H_kv_S=64, total_q=1 << 25) == 2   # H*total_q >= 2^31
    assert fn(cu_q=P + 2) == 3
    assert fn(k_t=P + 8) == 3


def test_varlen_host_validation_outputs(lib):
    assert fwd_varlen(lib, kl=0) == 1
    assert fwd_varlen(lib, lse_t=P + 4) == 3
    assert bwd_varlen(lib, g=0) == 1
    assert bwd_varlen(lib, dq=0) == 1
    assert bwd_varlen(lib, dk=P + 4) == 3
    assert bwd_varlen(lib, teacher=True, kl=0) == 1


def test_varlen_without_query_rows_is_a_no_op(lib):
    # No query rows: nothing to compute or write, so no CUDA call is made at all.
    assert fwd_varlen(lib, q_t=0, q_s=0, kl=0, lse_t=0, lse_s=0, total_q=0, max_q=0) == 0


def test_shard_host_validation(lib):
    def fwd_partial(k_offset=0, n_sh=128, n_tot=256, state=P, **kw):
        a = dict(q_t=P, k_t=P, q_s=P, k_s=P, B=1, H=2, H_kv_T=2, H_kv_S=1, N_Q=128)
        a.update(kw)
        return lib.streamkl_fwd_partial(*a.values(), n_sh, k_offset, n_tot, 128, 128, 0.1, 0.1,
                                        1, state, 0)
    assert fwd_partial(k_offset=-1) == 1
    assert fwd_partial(k_offset=200) == 1          # shard runs past N_K_total
    assert fwd_partial(n_sh=0) == 1
    assert fwd_partial(state=0) == 1
    assert fwd_partial(state=P + 4) == 3
    assert fwd_partial(q_t=0) == 1
    assert fwd_partial(H_kv_S=3) == 2
    assert lib.streamkl_bwd_shard(P, P, P, P, 1, 2, 2, 2, 128, 128, 200, 256, 128, 128, 0.1, 0.1,
                                  1, P, P, P, P, P, 0) == 1
    assert lib.streamkl_bwd_teacher_shard(P, P, P, P, 1, 2, 2, 2, 128, 128, 0, 256, 128, 128,
                                          0.1, 0.1, 1, 0, P, P, P, P, P, 0) == 1
    assert lib.streamkl_merge_partial(P, 0, 100, P, P, P, 0) == 1
    assert lib.streamkl_merge_partial(P, 2, 0, P, P, P, 0) == 1
    assert lib.streamkl_merge_partial(P + 4, 2, 100, P, P, P, 0) == 3
    assert lib.streamkl_merge_partial(0, 2, 100, P, P, P, 0) == 1


def test_diagnostics_host_validation(lib):
    # Rejected on the host before any launch: null pointers, odd sizes, probe times out of range.
    assert lib.streamkl_sm_clock_probe(0, 20000, 0) == 1
    assert lib.streamkl_sm_clock_probe(P, 999, 0) == 1
    assert lib.streamkl_sm_clock_probe(P, 10000001, 0) == 1
    assert lib.streamkl_exp2_eval(0, P, P, 8, 0) == 1
    assert lib.streamkl_exp2_eval(P, P, P, 7, 0) == 1
