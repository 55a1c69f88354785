"""Python binding of the StreamKL C ABI (include/streamkl.h).

Argument marshalling only: every step of the forward and backward runs in the CUDA
library ``lib/libstreamkl.so``. PyTorch supplies device memory and the stream. There
is no CPU fallback: if the library is missing, importing the functions raises.

    kl, lse_t, lse_s = streamkl_fwd(q_t, k_t, q_s, k_s, scale_T, scale_S, causal)
    dq_s, dk_s = streamkl_bwd(q_t, k_t, q_s, k_s, scale_T, scale_S, causal, lse_t, lse_s, g)
    dq_t, dk_t = streamkl_bwd_teacher(q_t, k_t, q_s, k_s, scale_T, scale_S, causal,
                                      kl, lse_t, lse_s, g)      # trainable teacher only

Tensors: bf16 [B, H, N, d] contiguous on one CUDA device (d in {64, 128}); row
statistics and g fp32 [B, H, N_Q]; gradients fp32.

The ``*_gqa`` variants take K tensors with fewer heads than Q (grouped-query attention).
The ``*_varlen`` variants take packed sequences: q_* [total_q, H, d], k_* [total_k, H_kv, d],
int32 offsets cu_seqlens_q / cu_seqlens_k [B+1] on the device, row statistics and g
[H, total_q]; gradients keep the packed shapes of Q and K.
"""
from __future__ import annotations

import ctypes
import functools
import os
from typing import Optional, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libstreamkl.so")

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "MISALIGNED", 4: "LAUNCH", 5: "TIMEOUT"}
EXPORTS = ("streamkl_fwd", "streamkl_bwd", "streamkl_bwd_teacher", "streamkl_fwd_gqa",
           "streamkl_bwd_gqa", "streamkl_bwd_teacher_gqa", "streamkl_fwd_varlen",
           "streamkl_bwd_varlen", "streamkl_bwd_teacher_varlen", "streamkl_fwd_partial",
           "streamkl_merge_partial", "streamkl_bwd_shard", "streamkl_bwd_teacher_shard",
           "streamkl_watchdog_selftest", "streamkl_exp2_eval", "streamkl_sm_clock_probe",
           "streamkl_status_string",
           "streamkl_device_status", "streamkl_version")


class StreamKLError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}: {status_string(status)}")


_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"StreamKL CUDA library not built: {path} "
                      "(run python -m attention_kl_divergence_fwd_b200.build)")
    lib = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.streamkl_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, f, i, vp, vp, vp, vp]
    lib.streamkl_fwd.restype = i
    lib.streamkl_bwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, f, i, vp, vp, vp, vp, vp, vp]
    lib.streamkl_bwd.restype = i
    lib.streamkl_bwd_teacher.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, f, i, vp, vp, vp,
                                         vp, vp, vp, vp]
    lib.streamkl_bwd_teacher.restype = i
    lib.streamkl_fwd_gqa.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, f, i, vp, vp, vp,
                                     vp]
    lib.streamkl_fwd_gqa.restype = i
    lib.streamkl_bwd_gqa.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, f, i, vp, vp, vp,
                                     vp, vp, vp]
    lib.streamkl_bwd_gqa.restype = i
    lib.streamkl_bwd_teacher_gqa.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, f, i, vp,
                                             vp, vp, vp, vp, vp, vp]
    lib.streamkl_bwd_teacher_gqa.restype = i
    # varlen: q_t, k_t, q_s, k_s, cu_q, cu_k, B, H, H_kv_T, H_kv_S, total_q, total_k,
    # max_q, max_k, d_T, d_S, scale_T, scale_S, causal, then the outputs / row inputs.
    head = [vp] * 6 + [i] * 10 + [f, f, i]
    lib.streamkl_fwd_varlen.argtypes = head + [vp, vp, vp, vp]
    lib.streamkl_fwd_varlen.restype = i
    lib.streamkl_bwd_varlen.argtypes = head + [vp, vp, vp, vp, vp, vp]
    lib.streamkl_bwd_varlen.restype = i
    lib.streamkl_bwd_teacher_varlen.argtypes = head + [vp, vp, vp, vp, vp, vp, vp]
    lib.streamkl_bwd_teacher_varlen.restype = i
    # shard entry points: q_t, k_t, q_s, k_s, B, H, H_kv_T, H_kv_S, N_Q, N_K_shard, k_offset,
    # N_K_total, d_T, d_S, scale_T, scale_S, causal, then the outputs / row inputs.
    shead = [vp] * 4 + [i] * 10 + [f, f, i]
    lib.streamkl_fwd_partial.argtypes = shead + [vp, vp]
    lib.streamkl_fwd_partial.restype = i
    lib.streamkl_merge_partial.argtypes = [vp, i, ctypes.c_longlong, vp, vp, vp, vp]
    lib.streamkl_merge_partial.restype = i
    lib.streamkl_bwd_shard.argtypes = shead + [vp, vp, vp, vp, vp, vp]
    lib.streamkl_bwd_shard.restype = i
    lib.streamkl_bwd_teacher_shard.argtypes = shead + [vp, vp, vp, vp, vp, vp, vp]
    lib.streamkl_bwd_teacher_shard.restype = i
    lib.streamkl_exp2_eval.argtypes = [vp, vp, vp, ctypes.c_longlong, vp]
    lib.streamkl_exp2_eval.restype = i
    lib.streamkl_sm_clock_probe.argtypes = [vp, ctypes.c_longlong, vp]
    lib.streamkl_sm_clock_probe.restype = i
    lib.streamkl_watchdog_selftest.argtypes = [vp]
    lib.streamkl_watchdog_selftest.restype = i
    lib.streamkl_status_string.argtypes = [i]
    lib.streamkl_status_string.restype = ctypes.c_char_p
    lib.streamkl_device_status.argtypes = [vp]
    lib.streamkl_device_status.restype = i
    lib.streamkl_version.argtypes = []
    lib.streamkl_version.restype = i
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().streamkl_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise StreamKLError(status, where)


def _on_device(fn):
    """Runs a tensor-level entry point on the CUDA device of its tensor arguments: all of
    them (and a given stream) must be on one device, which is made current for the call so
    that the default stream and the launch are on that device."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        import torch
        ts = [a for a in list(args) + list(kwargs.values()) if isinstance(a, torch.Tensor)]
        devs = {t.device for t in ts}
        if len(devs) > 1:
            raise ValueError(f"{fn.__name__}: tensors on different devices: "
                             f"{sorted(str(d) for d in devs)}")
        if not ts or next(iter(devs)).type != "cuda":
            return fn(*args, **kwargs)  # the entry point's own checks reject non-CUDA input
        dev = next(iter(devs))
        stream = kwargs.get("stream")
        if stream is not None and stream.device != dev:
            raise ValueError(f"{fn.__name__}: stream on {stream.device}, tensors on {dev}")
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)
    return wrapper


def _stream_ptr(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _shape(q_t, k_t, q_s, k_s):
    import torch
    for name, t in (("q_t", q_t), ("k_t", k_t), ("q_s", q_s), ("k_s", k_s)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-D bf16 CUDA tensor [B,H,N,d]")
    B, H, n_q, d_t = q_t.shape
    n_k = k_t.shape[2]
    d_s = q_s.shape[3]
    if tuple(k_t.shape) != (B, H, n_k, d_t) or tuple(q_s.shape) != (B, H, n_q, d_s) or \
            tuple(k_s.shape) != (B, H, n_k, d_s):
        raise ValueError("inconsistent shapes")
    return B, H, n_q, n_k, d_t, d_s


def streamkl_fwd_raw(q_t: int, k_t: int, q_s: int, k_s: int, B: int, H: int, N_Q: int, N_K: int,
                     d_T: int, d_S: int, scale_T: float, scale_S: float, causal: bool,
                     kl: int, lse_t: int, lse_s: int, stream: int = 0) -> int:
    """The C entry point with plain pointers; returns the status code."""
    return load_library().streamkl_fwd(q_t, k_t, q_s, k_s, B, H, N_Q, N_K, d_T, d_S,
                                       float(scale_T), float(scale_S), int(bool(causal)),
                                       kl, lse_t, lse_s, stream)


def streamkl_bwd_raw(q_t: int, k_t: int, q_s: int, k_s: int, B: int, H: int, N_Q: int, N_K: int,
                     d_T: int, d_S: int, scale_T: float, scale_S: float, causal: bool,
                     lse_t: int, lse_s: int, g: int, dq_s: int, dk_s: int, stream: int = 0) -> int:
    return load_library().streamkl_bwd(q_t, k_t, q_s, k_s, B, H, N_Q, N_K, d_T, d_S,
                                       float(scale_T), float(scale_S), int(bool(causal)),
                                       lse_t, lse_s, g, dq_s, dk_s, stream)


def streamkl_bwd_teacher_raw(q_t: int, k_t: int, q_s: int, k_s: int, B: int, H: int, N_Q: int,
                             N_K: int, d_T: int, d_S: int, scale_T: float, scale_S: float,
                             causal: bool, kl: int, lse_t: int, lse_s: int, g: int, dq_t: int,
                             dk_t: int, stream: int = 0) -> int:
    return load_library().streamkl_bwd_teacher(q_t, k_t, q_s, k_s, B, H, N_Q, N_K, d_T, d_S,
                                               float(scale_T), float(scale_S),
                                               int(bool(causal)), kl, lse_t, lse_s, g, dq_t,
                                               dk_t, stream)


@_on_device
def streamkl_fwd(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float, causal: bool,
                 kl=None, lse_t=None, lse_s=None, stream=None):
    """Per-row KL(P_T || P_S), LSE_T, LSE_S (fp32 [B,H,N_Q]) on the current stream."""
    import torch
    B, H, n_q, n_k, d_t, d_s = _shape(q_t, k_t, q_s, k_s)
    dev = q_t.device
    mk = lambda: torch.empty(B, H, n_q, device=dev, dtype=torch.float32)
    kl = mk() if kl is None else _check_out(kl, (B, H, n_q), "kl")
    lse_t = mk() if lse_t is None else _check_out(lse_t, (B, H, n_q), "lse_t")
    lse_s = mk() if lse_s is None else _check_out(lse_s, (B, H, n_q), "lse_s")
    st = streamkl_fwd_raw(q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(),
                          B, H, n_q, n_k, d_t, d_s, scale_T, scale_S, causal,
                          kl.data_ptr(), lse_t.data_ptr(), lse_s.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_fwd")
    return kl, lse_t, lse_s


@_on_device
def streamkl_bwd(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float, causal: bool,
                 lse_t, lse_s, g, dq_s=None, dk_s=None, stream=None):
    """dQ_S [B,H,N_Q,d_S] and dK_S [B,H,N_K,d_S] (fp32) of sum_i g_i KL_i."""
    import torch
    B, H, n_q, n_k, d_t, d_s = _shape(q_t, k_t, q_s, k_s)
    dev = q_t.device
    for name, t in (("lse_t", lse_t), ("lse_s", lse_s), ("g", g)):
        if t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != (B, H, n_q):
            raise ValueError(f"{name} must be contiguous fp32 [B,H,N_Q]")
    dq_s = (torch.empty(B, H, n_q, d_s, device=dev, dtype=torch.float32) if dq_s is None
            else _check_out(dq_s, (B, H, n_q, d_s), "dq_s"))
    dk_s = (torch.empty(B, H, n_k, d_s, device=dev, dtype=torch.float32) if dk_s is None
            else _check_out(dk_s, (B, H, n_k, d_s), "dk_s"))
    st = streamkl_bwd_raw(q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(),
                          B, H, n_q, n_k, d_t, d_s, scale_T, scale_S, causal,
                          lse_t.data_ptr(), lse_s.data_ptr(), g.data_ptr(),
                          dq_s.data_ptr(), dk_s.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_bwd")
    return dq_s, dk_s


@_on_device
def streamkl_bwd_teacher(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float, causal: bool,
                         kl, lse_t, lse_s, g, dq_t=None, dk_t=None, stream=None):
    """dQ_T [B,H,N_Q,d_T] and dK_T [B,H,N_K,d_T] (fp32) of sum_i g_i KL_i (trainable teacher)."""
    import torch
    B, H, n_q, n_k, d_t, d_s = _shape(q_t, k_t, q_s, k_s)
    dev = q_t.device
    for name, t in (("kl", kl), ("lse_t", lse_t), ("lse_s", lse_s), ("g", g)):
        if t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != (B, H, n_q):
            raise ValueError(f"{name} must be contiguous fp32 [B,H,N_Q]")
    dq_t = (torch.empty(B, H, n_q, d_t, device=dev, dtype=torch.float32) if dq_t is None
            else _check_out(dq_t, (B, H, n_q, d_t), "dq_t"))
    dk_t = (torch.empty(B, H, n_k, d_t, device=dev, dtype=torch.float32) if dk_t is None
            else _check_out(dk_t, (B, H, n_k, d_t), "dk_t"))
    st = streamkl_bwd_teacher_raw(q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(),
                                  k_s.data_ptr(), B, H, n_q, n_k, d_t, d_s, scale_T, scale_S,
                                  causal, kl.data_ptr(), lse_t.data_ptr(), lse_s.data_ptr(),
                                  g.data_ptr(), dq_t.data_ptr(), dk_t.data_ptr(),
                                  _stream_ptr(stream))
    _check(st, "streamkl_bwd_teacher")
    return dq_t, dk_t


def _shape_gqa(q_t, k_t, q_s, k_s):
    """Shapes with grouped K heads: k_t [B,H_kv_T,N_K,d_T], k_s [B,H_kv_S,N_K,d_S]."""
    import torch
    for name, t in (("q_t", q_t), ("k_t", k_t), ("q_s", q_s), ("k_s", k_s)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-D bf16 CUDA tensor [B,H,N,d]")
    B, H, n_q, d_t = q_t.shape
    h_kt, n_k = k_t.shape[1], k_t.shape[2]
    h_ks, d_s = k_s.shape[1], q_s.shape[3]
    if tuple(k_t.shape) != (B, h_kt, n_k, d_t) or tuple(q_s.shape) != (B, H, n_q, d_s) or \
            tuple(k_s.shape) != (B, h_ks, n_k, d_s):
        raise ValueError("inconsistent shapes")
    return B, H, h_kt, h_ks, n_q, n_k, d_t, d_s


@_on_device
def streamkl_fwd_gqa(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float, causal: bool,
                     kl=None, lse_t=None, lse_s=None, stream=None):
    """streamkl_fwd with grouped K heads (k_* may have fewer heads than q_*)."""
    import torch
    B, H, h_kt, h_ks, n_q, n_k, d_t, d_s = _shape_gqa(q_t, k_t, q_s, k_s)
    dev = q_t.device
    mk = lambda: torch.empty(B, H, n_q, device=dev, dtype=torch.float32)
    kl = mk() if kl is None else _check_out(kl, (B, H, n_q), "kl")
    lse_t = mk() if lse_t is None else _check_out(lse_t, (B, H, n_q), "lse_t")
    lse_s = mk() if lse_s is None else _check_out(lse_s, (B, H, n_q), "lse_s")
    st = load_library().streamkl_fwd_gqa(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), B, H, h_kt, h_ks, n_q,
        n_k, d_t, d_s, float(scale_T), float(scale_S), int(bool(causal)), kl.data_ptr(),
        lse_t.data_ptr(), lse_s.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_fwd_gqa")
    return kl, lse_t, lse_s


@_on_device
def streamkl_bwd_gqa(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float, causal: bool,
                     lse_t, lse_s, g, dq_s=None, dk_s=None, stream=None):
    """streamkl_bwd with grouped K heads; dk_s has the student's K-head count."""
    import torch
    B, H, h_kt, h_ks, n_q, n_k, d_t, d_s = _shape_gqa(q_t, k_t, q_s, k_s)
    _check_rows((("lse_t", lse_t), ("lse_s", lse_s), ("g", g)), (B, H, n_q))
    dev = q_t.device
    dq_s = (torch.empty(B, H, n_q, d_s, device=dev, dtype=torch.float32) if dq_s is None
            else _check_out(dq_s, (B, H, n_q, d_s), "dq_s"))
    dk_s = (torch.empty(B, h_ks, n_k, d_s, device=dev, dtype=torch.float32) if dk_s is None
            else _check_out(dk_s, (B, h_ks, n_k, d_s), "dk_s"))
    st = load_library().streamkl_bwd_gqa(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), B, H, h_kt, h_ks, n_q,
        n_k, d_t, d_s, float(scale_T), float(scale_S), int(bool(causal)), lse_t.data_ptr(),
        lse_s.data_ptr(), g.data_ptr(), dq_s.data_ptr(), dk_s.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_bwd_gqa")
    return dq_s, dk_s


@_on_device
def streamkl_bwd_teacher_gqa(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float, causal: bool,
                             kl, lse_t, lse_s, g, dq_t=None, dk_t=None, stream=None):
    """streamkl_bwd_teacher with grouped K heads; dk_t has the teacher's K-head count."""
    import torch
    B, H, h_kt, h_ks, n_q, n_k, d_t, d_s = _shape_gqa(q_t, k_t, q_s, k_s)
    _check_rows((("kl", kl), ("lse_t", lse_t), ("lse_s", lse_s), ("g", g)), (B, H, n_q))
    dev = q_t.device
    dq_t = (torch.empty(B, H, n_q, d_t, device=dev, dtype=torch.float32) if dq_t is None
            else _check_out(dq_t, (B, H, n_q, d_t), "dq_t"))
    dk_t = (torch.empty(B, h_kt, n_k, d_t, device=dev, dtype=torch.float32) if dk_t is None
            else _check_out(dk_t, (B, h_kt, n_k, d_t), "dk_t"))
    st = load_library().streamkl_bwd_teacher_gqa(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), B, H, h_kt, h_ks, n_q,
        n_k, d_t, d_s, float(scale_T), float(scale_S), int(bool(causal)), kl.data_ptr(),
        lse_t.data_ptr(), lse_s.data_ptr(), g.data_ptr(), dq_t.data_ptr(), dk_t.data_ptr(),
        _stream_ptr(stream))
    _check(st, "streamkl_bwd_teacher_gqa")
    return dq_t, dk_t


def _check_rows(named, shape) -> None:
    import torch
    for name, t in named:
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or \
                tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor of shape {tuple(shape)}")


def _check_out(t, shape, name):
    import torch
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or \
            tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor of shape {tuple(shape)}")
    return t


def _shape_varlen(q_t, k_t, q_s, k_s, cu_q, cu_k):
    """Packed shapes: q_* [total_q, H, d], k_* [total_k, H_kv, d], cu_* int32 [B+1]."""
    import torch
    for name, t in (("q_t", q_t), ("k_t", k_t), ("q_s", q_s), ("k_s", k_s)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 3-D bf16 CUDA tensor [total, heads, d]")
    for name, t in (("cu_seqlens_q", cu_q), ("cu_seqlens_k", cu_k)):
        if t.dtype != torch.int32 or not t.is_cuda or t.dim() != 1 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 1-D int32 CUDA tensor [B+1]")
    if cu_q.numel() != cu_k.numel() or cu_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B+1 >= 2 entries")
    total_q, H, d_t = q_t.shape
    total_k, h_kt = k_t.shape[0], k_t.shape[1]
    h_ks, d_s = k_s.shape[1], q_s.shape[2]
    if tuple(k_t.shape) != (total_k, h_kt, d_t) or tuple(q_s.shape) != (total_q, H, d_s) or \
            tuple(k_s.shape) != (total_k, h_ks, d_s):
        raise ValueError("inconsistent shapes")
    return cu_q.numel() - 1, H, h_kt, h_ks, total_q, total_k, d_t, d_s


@_on_device
def streamkl_fwd_varlen(q_t, k_t, q_s, k_s, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                        max_seqlen_k: int, scale_T: float, scale_S: float, causal: bool,
                        kl=None, lse_t=None, lse_s=None, stream=None):
    """streamkl_fwd over packed sequences: KL, LSE_T, LSE_S fp32 [H, total_q]. Rows that
    belong to no sequence are not written."""
    import torch
    B, H, h_kt, h_ks, tq, tk, d_t, d_s = _shape_varlen(q_t, k_t, q_s, k_s, cu_seqlens_q,
                                                        cu_seqlens_k)
    dev = q_t.device
    mk = lambda: torch.empty(H, tq, device=dev, dtype=torch.float32)
    kl = mk() if kl is None else _check_out(kl, (H, tq), "kl")
    lse_t = mk() if lse_t is None else _check_out(lse_t, (H, tq), "lse_t")
    lse_s = mk() if lse_s is None else _check_out(lse_s, (H, tq), "lse_s")
    st = load_library().streamkl_fwd_varlen(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), cu_seqlens_q.data_ptr(),
        cu_seqlens_k.data_ptr(), B, H, h_kt, h_ks, tq, tk, int(max_seqlen_q), int(max_seqlen_k),
        d_t, d_s, float(scale_T), float(scale_S), int(bool(causal)), kl.data_ptr(),
        lse_t.data_ptr(), lse_s.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_fwd_varlen")
    return kl, lse_t, lse_s


@_on_device
def streamkl_bwd_varlen(q_t, k_t, q_s, k_s, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                        max_seqlen_k: int, scale_T: float, scale_S: float, causal: bool,
                        lse_t, lse_s, g, dq_s=None, dk_s=None, stream=None):
    """streamkl_bwd over packed sequences: dQ_S [total_q, H, d_S], dK_S [total_k, H_kv_S, d_S]."""
    import torch
    B, H, h_kt, h_ks, tq, tk, d_t, d_s = _shape_varlen(q_t, k_t, q_s, k_s, cu_seqlens_q,
                                                        cu_seqlens_k)
    _check_rows((("lse_t", lse_t), ("lse_s", lse_s), ("g", g)), (H, tq))
    dev = q_t.device
    dq_s = (torch.empty(tq, H, d_s, device=dev, dtype=torch.float32) if dq_s is None
            else _check_out(dq_s, (tq, H, d_s), "dq_s"))
    dk_s = (torch.empty(tk, h_ks, d_s, device=dev, dtype=torch.float32) if dk_s is None
            else _check_out(dk_s, (tk, h_ks, d_s), "dk_s"))
    st = load_library().streamkl_bwd_varlen(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), cu_seqlens_q.data_ptr(),
        cu_seqlens_k.data_ptr(), B, H, h_kt, h_ks, tq, tk, int(max_seqlen_q), int(max_seqlen_k),
        d_t, d_s, float(scale_T), float(scale_S), int(bool(causal)), lse_t.data_ptr(),
        lse_s.data_ptr(), g.data_ptr(), dq_s.data_ptr(), dk_s.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_bwd_varlen")
    return dq_s, dk_s


@_on_device
def streamkl_bwd_teacher_varlen(q_t, k_t, q_s, k_s, cu_seqlens_q, cu_seqlens_k,
                                max_seqlen_q: int, max_seqlen_k: int, scale_T: float,
                                scale_S: float, causal: bool, kl, lse_t, lse_s, g, dq_t=None,
                                dk_t=None, stream=None):
    """streamkl_bwd_teacher over packed sequences: dQ_T [total_q, H, d_T], dK_T
    [total_k, H_kv_T, d_T]."""
    import torch
    B, H, h_kt, h_ks, tq, tk, d_t, d_s = _shape_varlen(q_t, k_t, q_s, k_s, cu_seqlens_q,
                                                        cu_seqlens_k)
    _check_rows((("kl", kl), ("lse_t", lse_t), ("lse_s", lse_s), ("g", g)), (H, tq))
    dev = q_t.device
    dq_t = (torch.empty(tq, H, d_t, device=dev, dtype=torch.float32) if dq_t is None
            else _check_out(dq_t, (tq, H, d_t), "dq_t"))
    dk_t = (torch.empty(tk, h_kt, d_t, device=dev, dtype=torch.float32) if dk_t is None
            else _check_out(dk_t, (tk, h_kt, d_t), "dk_t"))
    st = load_library().streamkl_bwd_teacher_varlen(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), cu_seqlens_q.data_ptr(),
        cu_seqlens_k.data_ptr(), B, H, h_kt, h_ks, tq, tk, int(max_seqlen_q), int(max_seqlen_k),
        d_t, d_s, float(scale_T), float(scale_S), int(bool(causal)), kl.data_ptr(),
        lse_t.data_ptr(), lse_s.data_ptr(), g.data_ptr(), dq_t.data_ptr(), dk_t.data_ptr(),
        _stream_ptr(stream))
    _check(st, "streamkl_bwd_teacher_varlen")
    return dq_t, dk_t


@_on_device
def streamkl_fwd_partial(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float, causal: bool,
                         k_offset: int, n_k_total: int, state=None, stream=None):
    """Row state of one key shard (k_* hold the shard's keys): fp32 [5, B, H, N_Q], planes
    m_T, m_S, l_T, l_S, A in base-2 units."""
    import torch
    B, H, h_kt, h_ks, n_q, n_k, d_t, d_s = _shape_gqa(q_t, k_t, q_s, k_s)
    state = (torch.empty(5, B, H, n_q, device=q_t.device, dtype=torch.float32) if state is None
             else _check_out(state, (5, B, H, n_q), "state"))
    st = load_library().streamkl_fwd_partial(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), B, H, h_kt, h_ks, n_q,
        n_k, int(k_offset), int(n_k_total), d_t, d_s, float(scale_T), float(scale_S),
        int(bool(causal)), state.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_fwd_partial")
    return state


@_on_device
def streamkl_merge_partial(states, kl=None, lse_t=None, lse_s=None, stream=None):
    """Merge gathered shard states [R, 5, B, H, N_Q] into KL, LSE_T, LSE_S [B, H, N_Q]."""
    import torch
    if states.dtype != torch.float32 or not states.is_cuda or not states.is_contiguous() or \
            states.dim() != 5 or states.shape[1] != 5:
        raise ValueError("states must be a contiguous fp32 CUDA tensor [R, 5, B, H, N_Q]")
    R, _, B, H, n_q = states.shape
    mk = lambda: torch.empty(B, H, n_q, device=states.device, dtype=torch.float32)
    kl = mk() if kl is None else _check_out(kl, (B, H, n_q), "kl")
    lse_t = mk() if lse_t is None else _check_out(lse_t, (B, H, n_q), "lse_t")
    lse_s = mk() if lse_s is None else _check_out(lse_s, (B, H, n_q), "lse_s")
    st = load_library().streamkl_merge_partial(states.data_ptr(), R, B * H * n_q, kl.data_ptr(),
                                               lse_t.data_ptr(), lse_s.data_ptr(),
                                               _stream_ptr(stream))
    _check(st, "streamkl_merge_partial")
    return kl, lse_t, lse_s


@_on_device
def streamkl_bwd_shard(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float, causal: bool,
                       k_offset: int, n_k_total: int, lse_t, lse_s, g, dq_s=None, dk_s=None,
                       stream=None):
    """Student gradients of one key shard with the merged LSEs: the shard's part of dQ_S
    [B,H,N_Q,d_S] (sum over shards = dQ_S) and dK_S of its keys [B,H_kv_S,N_K_shard,d_S]."""
    import torch
    B, H, h_kt, h_ks, n_q, n_k, d_t, d_s = _shape_gqa(q_t, k_t, q_s, k_s)
    _check_rows((("lse_t", lse_t), ("lse_s", lse_s), ("g", g)), (B, H, n_q))
    dev = q_t.device
    dq_s = (torch.empty(B, H, n_q, d_s, device=dev, dtype=torch.float32) if dq_s is None
            else _check_out(dq_s, (B, H, n_q, d_s), "dq_s"))
    dk_s = (torch.empty(B, h_ks, n_k, d_s, device=dev, dtype=torch.float32) if dk_s is None
            else _check_out(dk_s, (B, h_ks, n_k, d_s), "dk_s"))
    st = load_library().streamkl_bwd_shard(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), B, H, h_kt, h_ks, n_q,
        n_k, int(k_offset), int(n_k_total), d_t, d_s, float(scale_T), float(scale_S),
        int(bool(causal)), lse_t.data_ptr(), lse_s.data_ptr(), g.data_ptr(), dq_s.data_ptr(),
        dk_s.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_bwd_shard")
    return dq_s, dk_s


@_on_device
def streamkl_bwd_teacher_shard(q_t, k_t, q_s, k_s, scale_T: float, scale_S: float,
                               causal: bool, k_offset: int, n_k_total: int, kl, lse_t, lse_s, g,
                               dq_t=None, dk_t=None, stream=None):
    """Trainable-teacher gradients of one key shard with the merged KL and LSEs."""
    import torch
    B, H, h_kt, h_ks, n_q, n_k, d_t, d_s = _shape_gqa(q_t, k_t, q_s, k_s)
    _check_rows((("kl", kl), ("lse_t", lse_t), ("lse_s", lse_s), ("g", g)), (B, H, n_q))
    dev = q_t.device
    dq_t = (torch.empty(B, H, n_q, d_t, device=dev, dtype=torch.float32) if dq_t is None
            else _check_out(dq_t, (B, H, n_q, d_t), "dq_t"))
    dk_t = (torch.empty(B, h_kt, n_k, d_t, device=dev, dtype=torch.float32) if dk_t is None
            else _check_out(dk_t, (B, h_kt, n_k, d_t), "dk_t"))
    st = load_library().streamkl_bwd_teacher_shard(
        q_t.data_ptr(), k_t.data_ptr(), q_s.data_ptr(), k_s.data_ptr(), B, H, h_kt, h_ks, n_q,
        n_k, int(k_offset), int(n_k_total), d_t, d_s, float(scale_T), float(scale_S),
        int(bool(causal)), kl.data_ptr(), lse_t.data_ptr(), lse_s.data_ptr(), g.data_ptr(),
        dq_t.data_ptr(), dk_t.data_ptr(), _stream_ptr(stream))
    _check(st, "streamkl_bwd_teacher_shard")
    return dq_t, dk_t


def watchdog_selftest(stream=None) -> None:
    """Let one bounded pipeline wait expire on purpose (about 2 s); device_status() then
    reports STREAMKL_ERR_TIMEOUT (5)."""
    _check(load_library().streamkl_watchdog_selftest(_stream_ptr(stream)),
           "streamkl_watchdog_selftest")


@_on_device
def exp2_eval(x, stream=None):
    """The forward's FMA-pipe 2^x on a float32 CUDA tensor with an even number of elements:
    (scalar form, packed-pair form)."""
    import torch
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous() or x.numel() % 2:
        raise ValueError("x must be a contiguous float32 CUDA tensor with an even size")
    y1, y2 = torch.empty_like(x), torch.empty_like(x)
    _check(load_library().streamkl_exp2_eval(x.data_ptr(), y1.data_ptr(), y2.data_ptr(),
                                             x.numel(), _stream_ptr(stream)), "streamkl_exp2_eval")
    return y1, y2


def sm_clock_probe(out, ns: int = 20000, stream=None) -> None:
    """Enqueue the SM clock probe on the stream: out (int64 CUDA tensor of 2) receives the
    clock ticks and nanoseconds of a ~`ns` ns spin; out[0] / out[1] * 1000 is the SM MHz."""
    import torch
    if out.dtype != torch.int64 or not out.is_cuda or not out.is_contiguous() or out.numel() < 2:
        raise ValueError("out must be a contiguous int64 CUDA tensor of at least 2 elements")
    _check(load_library().streamkl_sm_clock_probe(out.data_ptr(), int(ns), _stream_ptr(stream)),
           "streamkl_sm_clock_probe")


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the library's device error status."""
    return load_library().streamkl_device_status(_stream_ptr(stream))


def version() -> int:
    return load_library().streamkl_version()
