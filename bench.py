"""StreamKL benchmark: forward + backward throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one StreamKL forward (KL, LSE_T, LSE_S per row) + one backward (dQ_S, dK_S)
over the whole workload, inputs resident in HBM. Default workload: B=1, H=32,
N_Q=N_K=16384, d=128, causal (long context). Multi-GPU runs (torchrun) are weak
scaling: every rank runs its own copy of the workload (heads are independent, so
there is no data-path collective); time is the max over ranks.

Prints one JSON line (rank 0). FLOPs are counted per head as 2*N_Q*N_K*(d_T+d_S)
forward and 2*N_Q*N_K*(d_T+3*d_S) backward, halved when causal.
"""
from __future__ import annotations

import argparse
import contextlib
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import (WORKLOADS, flops_bwd, flops_bwd_teacher, flops_fwd, make_inputs,  # noqa: E402
                       make_varlen_inputs, varlen_lengths, varlen_pairs)

METRIC = "fwd/bwd TFLOP/s and % of B200 bf16 peak at N=16K,d=128; ms per fwd+bwd"
DEFAULT_WORKLOAD = "long_b1h32_n16384_d128_causal"
FWD_FMA_EXP_SHARE = 1.0 / 16.0  # share of the forward's exponentials computed on the FMA pipe


def clocks_mhz_or(clk, default=1965.0):
    """Median SM clock sampled during the timed region (MHz), else the B200's maximum."""
    try:
        v = float(clk["sm_mhz"]) if clk else 0.0
    except (KeyError, TypeError, ValueError):
        v = 0.0
    return v if v > 0 else default


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock, power and clock-event reasons of this process's GPU, sampled through NVML
    every few milliseconds from a background thread while the timed region runs. The GPU
    is found by its PCI bus id (NVML does not follow CUDA_VISIBLE_DEVICES); read-only."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []
        self.error = None
        self.thread = None
        self.stop_flag = False

    def _handle(self, nv):
        prop = torch.cuda.get_device_properties(self.cuda_index)
        bus = f"{prop.pci_domain_id:08X}:{prop.pci_bus_id:02X}:{prop.pci_device_id:02X}.0"
        return nv.nvmlDeviceGetHandleByPciBusId(bus.encode()), bus

    def _run(self, nv, h):
        while not self.stop_flag:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception as e:  # keep whatever was sampled
                self.error = repr(e)
                return
            time.sleep(self.period)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h, self.bus = self._handle(nv)
            self.nv = nv
        except Exception as e:
            self.error = f"NVML unavailable: {e!r}"
            return
        self.thread = threading.Thread(target=self._run, args=(self.nv, h), daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.samples and self.error is None and time.time() - t0 < 2.0:
            time.sleep(0.001)

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "no sampler"]}
        self.stop_flag = True
        self.thread.join(timeout=2.0)
        rows = list(self.samples)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "no samples"]}
        masks = {name: getattr(self.nv, attr, 0) for name, attr in self.REASONS}
        reasons = sorted({name for r in rows for name, m in masks.items() if m and (r[3] & m)})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows),
                "power_w_median": statistics.median(r[2] for r in rows),
                "power_w_max": max(r[2] for r in rows),
                "samples": len(rows), "gpu_pci_bus_id": self.bus, "source": "NVML",
                "reasons": reasons}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


@contextlib.contextmanager
def nvtx(name: str):
    """An NVTX range around a region of the bench (visible in Nsight timelines; a no-op
    without a profiler attached)."""
    torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        torch.cuda.nvtx.range_pop()


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_baseline(w, budget_s: float = 12.0, seed: int = 77):
    """The fp64 oracle as it stands, timed on this host's cores on sampled query rows.

    Each sampled row does its full forward + backward work: its KL and LSEs, its dQ_S
    row and its contribution to dK_S. FLOPs are counted with the same convention as
    the GPU (2*|J(i)|*(d_T+d_S) + 2*|J(i)|*(d_T+3*d_S) per row)."""
    from oracle import oracle_row_work, row_pair_count
    x = make_inputs(w) if w.bh * w.N_Q * (w.d_T + w.d_S) * 2 < (3 << 30) else None
    if x is None:
        raise RuntimeError("workload too large for the CPU baseline")
    gen = torch.Generator().manual_seed(seed)
    args = (x["q_t"], x["k_t"], x["q_s"], x["k_s"], w.scale_T, w.scale_S, w.causal, x["g"])
    done_rows, flops, elapsed = 0, 0.0, 0.0
    batch = 16
    while elapsed < budget_s:
        flat = torch.randint(0, w.bh * w.N_Q, (batch,), generator=gen).tolist()
        rows = [(f // w.N_Q, f % w.N_Q) for f in flat]
        t0 = time.perf_counter()
        oracle_row_work(*args, rows)
        elapsed += time.perf_counter() - t0
        for _, i in rows:
            n = row_pair_count(w.N_Q, w.N_K, w.causal, i)
            flops += 2.0 * n * (w.d_T + w.d_S) + 2.0 * n * (w.d_T + 3 * w.d_S)
        done_rows += batch
    cores = torch.get_num_threads()
    return {"value": flops / elapsed / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{done_rows} uniformly sampled query rows of {w.name} (fwd + bwd work of "
                      f"each row, fp64, torch CPU ops), {elapsed:.1f} s",
            "seconds": elapsed, "host_cores": len(os.sched_getaffinity(0))}


def run_reference(args, world, rank):
    """Reference arm: the fp64 oracle on the host cores (rank 0 only)."""
    w = WORKLOADS[args.workload]
    if rank != 0:
        return
    # The whole run (warm-up and timed steps) spends about args.ref_seconds on the host.
    per_step = max(0.5, args.ref_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(w, budget_s=min(per_step, 3.0), seed=11)
    vals, secs = [], 0.0
    for k in range(args.steps):
        cb = cpu_baseline(w, budget_s=per_step, seed=100 + k)
        vals.append(cb["value"])
        secs += cb["seconds"]
    value = statistics.mean(vals)
    cb["value"] = value
    cb["sample"] = f"{args.steps} steps, each {cb['sample']}"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_of(w, world), "cpu_baseline": cb,
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def config_of(w, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "N_Q": w.N_Q, "N_K": w.N_K, "d_T": w.d_T,
            "d_S": w.d_S, "causal": w.causal, "scale_T": w.scale_T, "scale_S": w.scale_S,
            "per_rank": "full workload per rank (heads are independent)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": l2_note(w)}


L2_BYTES = 126 * 1000 * 1000


def l2_note(w):
    """How the timed loop treats L2 (no flush between steps; say whether the inputs exceed it)."""
    inputs = 2 * w.bh * (w.N_Q * (w.d_T + w.d_S) + w.N_K * (w.d_T + w.d_S))
    if inputs > L2_BYTES:
        return (f"no flush: each step reads {inputs / 1e6:.0f} MB of bf16 inputs, more than "
                f"the 126 MB L2")
    return (f"no flush: the {inputs / 1e6:.1f} MB of bf16 inputs fit in the 126 MB L2 "
            f"(a small parity case, not the metric's workload)")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-eager", action="store_true",
                    help="skip the PyTorch eager materialising comparator")
    ap.add_argument("--no-variants", action="store_true",
                    help="time only the step (skip the teacher, grouped-query, packed and "
                         "context-parallel legs), e.g. for a small profiler capture")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="host time of the cpu_baseline leg of this arm")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="total host time of the --impl reference arm")
    args = ap.parse_args()

    if args.impl == "reference":
        # The reference arm is the host-side oracle: rank 0 alone runs it, no process group.
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")),
                      int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup()

    import attention_kl_divergence_fwd_b200 as skl
    skl.load_library()
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    x = make_inputs(w)
    d = {k: v.to(dev) for k, v in x.items()}
    B, H, nq, nk = w.B, w.H, w.N_Q, w.N_K
    kl = torch.empty(B, H, nq, device=dev)
    lt, ls = torch.empty_like(kl), torch.empty_like(kl)
    dq = torch.empty(B, H, nq, w.d_S, device=dev)
    dk = torch.empty(B, H, nk, w.d_S, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        skl.streamkl_fwd(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T, w.scale_S, w.causal,
                         kl=kl, lse_t=lt, lse_s=ls)
        if ev is not None:
            ev[1].record(stream)
        skl.streamkl_bwd(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T, w.scale_S, w.causal,
                         lt, ls, d["g"], dq_s=dq, dk_s=dk)
        if ev is not None:
            ev[2].record(stream)

    with nvtx("warm-up"):
        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize()
    if skl.device_status() != 0:
        raise RuntimeError("kernel watchdog fired during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    # The SM clock the kernels actually ran at, measured by the library's probe (clock64
    # ticks over global-timer nanoseconds) just before the first and just after the last
    # timed step, outside the timed region: NVML's sampled clock misses the fast drops a
    # sustained load causes.
    probe = torch.zeros(2, 2, dtype=torch.int64, device=dev)
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with nvtx("timed steps"):
        skl.sm_clock_probe(probe[0], 20000)
        t_start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t_end.record(stream)
        skl.sm_clock_probe(probe[1], 20000)
        torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    if clk is not None:
        pr = probe.cpu().tolist()
        clk["sm_mhz_probe"] = {"before": round(pr[0][0] / pr[0][1] * 1e3, 1),
                               "after": round(pr[1][0] / pr[1][1] * 1e3, 1),
                               "how": "clock64 ticks / globaltimer ns of one warp spinning "
                                      "20 us, launched right before and right after the "
                                      "timed steps (outside the timed region)"}
    if skl.device_status() != 0:
        raise RuntimeError("kernel watchdog fired during the timed region")

    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    fwd_ms = max_over_ranks(fwd_ms, world)
    bwd_ms = max_over_ranks(bwd_ms, world)
    ms_step = total_ms / args.steps
    ff, fb = flops_fwd(w), flops_bwd(w)
    value = world * (ff + fb) * args.steps / (total_ms * 1e-3) / 1e12

    peaks, peak_kind = load_peaks()
    peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    fwd_tf = ff / (fwd_ms * 1e-3) / 1e12
    bwd_tf = fb / (bwd_ms * 1e-3) / 1e12
    dominant = "bwd" if bwd_ms >= fwd_ms else "fwd"
    traffic = load_traffic(w.name, dominant)
    # The timed region is tens of milliseconds and the clocks stay at their maximum (see
    # "clocks"), so the denominator is the burst cuBLAS figure; the fraction of the
    # sustained (power-capped, seconds-long loop) figure is reported beside it.
    achieved = bwd_tf if dominant == "bwd" else fwd_tf
    roof = {"kernel": f"streamkl_{dominant}_kernel", "bound": "tensor",
            "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
            "frac": achieved / peak_burst, "traffic": traffic,
            "peak_kind": f"{peak_kind} bf16 dense, burst (short timed region at full clocks)",
            "frac_of_sustained_peak": achieved / peak_sus}

    # Second roofline of the forward: its statistics warps are bound by the exponential unit
    # (MUFU), two exponentials per (row, key) pair, of which the kernel sends 1/16 to the
    # FMA pipe as a polynomial. Peak: 16 ex2 per clock per SM at the sampled SM clock.
    pairs = ff / (2.0 * (w.d_T + w.d_S))
    mufu_ex2 = 2.0 * pairs * (1.0 - FWD_FMA_EXP_SHARE)
    sm_hz = (clocks_mhz_or(clk) * 1e6)
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    mufu_peak = 16.0 * n_sm * sm_hz
    fwd_mufu = {"bound": "mufu", "achieved": mufu_ex2 / (fwd_ms * 1e-3) / 1e12,
                "peak": mufu_peak / 1e12, "unit": "Tex2/s",
                "frac": (mufu_ex2 / (fwd_ms * 1e-3)) / mufu_peak,
                "peak_kind": f"16 ex2/clock/SM x {n_sm} SMs x {sm_hz / 1e6:.0f} MHz (sampled)"}

    bwd_t_ms, gqa, varlen, cp = None, None, None, None
    if not args.no_variants:
        bwd_t_ms, gqa, varlen, cp = run_variants(skl, args, w, d, dev, stream, world, kl, lt,
                                                 ls, dq)

    eager = None
    if rank == 0 and not args.no_eager:
        skl.streamkl_fwd(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T, w.scale_S, w.causal,
                         kl=kl, lse_t=lt, lse_s=ls)  # the buffers held the variants' rows
        with nvtx("eager comparator"):
            eager = run_eager(w, d, kl, dev, stream, fwd_ms, bwd_ms)

    e2e = None
    if not args.no_e2e:
        with nvtx("end to end"):
            e2e = run_e2e(skl, w, x, dev, stream, args.steps, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with nvtx("cpu baseline"):
            cpu = cpu_baseline(w, budget_s=args.cpu_seconds)

    if rank == 0:
        out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
               "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
               "dtype": "bf16", "data": "synthetic", "config": config_of(w, world),
               "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
               "fwd_frac_peak": fwd_tf / peak_burst, "bwd_frac_peak": bwd_tf / peak_burst,
               "fwd_frac_sustained_peak": fwd_tf / peak_sus,
               "bwd_frac_sustained_peak": bwd_tf / peak_sus,
               "roofline": roof, "fwd_mufu": fwd_mufu, "cpu_baseline": cpu, "e2e": e2e,
               "clocks": clk,
               "gqa": gqa, "varlen": varlen, "context_parallel": cp, "eager_baseline": eager,
               "bwd_teacher_ms": bwd_t_ms,
               "bwd_teacher_tflops": (flops_bwd_teacher(w) / (bwd_t_ms * 1e-3) / 1e12
                                      if bwd_t_ms else None),
               "gpu_launches": 2 * args.steps,
               "extra_hbm_bytes": 3 * 4 * w.bh * w.N_Q,
               "impl": "ours"}
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_variants(skl, args, w, d, dev, stream, world, kl, lt, ls, dq):
    """The legs timed beside the step: trainable-teacher backward, grouped-query variant,
    packed variable-length batch, context-parallel key shards."""
    B, H, nq, nk = w.B, w.H, w.N_Q, w.N_K
    ff, fb = flops_fwd(w), flops_bwd(w)
    # Trainable-teacher backward (streamkl_bwd_teacher), timed on its own: not part of the
    # step (the teacher is frozen in the measured workload), reported beside it.
    dq_t = torch.empty(B, H, nq, w.d_T, device=dev)
    dk_t = torch.empty(B, H, nk, w.d_T, device=dev)
    for _ in range(2):
        skl.streamkl_bwd_teacher(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T, w.scale_S,
                                 w.causal, kl, lt, ls, d["g"], dq_t=dq_t, dk_t=dk_t)
    torch.cuda.synchronize()
    te0, te1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    te0.record(stream)
    for _ in range(args.steps):
        skl.streamkl_bwd_teacher(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T, w.scale_S,
                                 w.causal, kl, lt, ls, d["g"], dq_t=dq_t, dk_t=dk_t)
    te1.record(stream)
    torch.cuda.synchronize()
    bwd_t_ms = max_over_ranks(te0.elapsed_time(te1) / args.steps, world)
    del dq_t, dk_t

    # Grouped-query variant of the same workload (student K heads shared by 4 query heads),
    # timed on its own and reported beside the step.
    gqa = None
    if w.H % 4 == 0:
        k_s4 = d["k_s"][:, : w.H // 4].contiguous()
        dk4 = torch.empty(B, w.H // 4, nk, w.d_S, device=dev)
        ga = (d["q_t"], d["k_t"], d["q_s"], k_s4, w.scale_T, w.scale_S, w.causal)
        for _ in range(2):
            skl.streamkl_fwd_gqa(*ga, kl=kl, lse_t=lt, lse_s=ls)
            skl.streamkl_bwd_gqa(*ga, lt, ls, d["g"], dq_s=dq, dk_s=dk4)
        torch.cuda.synchronize()
        ge = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ge[0].record(stream)
        for _ in range(args.steps):
            skl.streamkl_fwd_gqa(*ga, kl=kl, lse_t=lt, lse_s=ls)
        ge[1].record(stream)
        for _ in range(args.steps):
            skl.streamkl_bwd_gqa(*ga, lt, ls, d["g"], dq_s=dq, dk_s=dk4)
        ge[2].record(stream)
        torch.cuda.synchronize()
        gf = max_over_ranks(ge[0].elapsed_time(ge[1]) / args.steps, world)
        gb = max_over_ranks(ge[1].elapsed_time(ge[2]) / args.steps, world)
        gqa = {"student_kv_heads": w.H // 4, "fwd_ms": gf, "bwd_ms": gb,
               "fwd_tflops": ff / (gf * 1e-3) / 1e12, "bwd_tflops": fb / (gb * 1e-3) / 1e12}
        del k_s4, dk4

    with nvtx("packed sequences"):
        varlen = run_varlen(skl, w, dev, stream, args.steps, world) if w.d_T == w.d_S else None
    with nvtx("context-parallel shards"):
        cp = run_context_parallel(skl, w, d, dev, stream, args.steps, world)
    return bwd_t_ms, gqa, varlen, cp


def run_varlen(skl, w, dev, stream, steps, world, tokens=65536, lo=512, hi=8192):
    """Packed variable-length batch with the workload's heads and head dims: seeded
    sequence lengths uniform in [lo, hi] filling ``tokens`` rows, timed on its own."""
    lens = varlen_lengths(tokens, lo, hi, seed=2024)
    x = make_varlen_inputs(lens, lens, w.H, w.H, w.H, w.d_T, w.d_S, seed=2025)
    d = {k: v.to(dev) for k, v in x.items()}
    a = (d["q_t"], d["k_t"], d["q_s"], d["k_s"], d["cu_q"], d["cu_k"], max(lens), max(lens),
         w.scale_T, w.scale_S, w.causal)
    kl = torch.empty(w.H, tokens, device=dev)
    lt, ls = torch.empty_like(kl), torch.empty_like(kl)
    dq = torch.empty(tokens, w.H, w.d_S, device=dev)
    dk = torch.empty(tokens, w.H, w.d_S, device=dev)
    for _ in range(3):
        skl.streamkl_fwd_varlen(*a, kl=kl, lse_t=lt, lse_s=ls)
        skl.streamkl_bwd_varlen(*a, lt, ls, d["g"], dq_s=dq, dk_s=dk)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record(stream)
    for _ in range(steps):
        skl.streamkl_fwd_varlen(*a, kl=kl, lse_t=lt, lse_s=ls)
    ev[1].record(stream)
    for _ in range(steps):
        skl.streamkl_bwd_varlen(*a, lt, ls, d["g"], dq_s=dq, dk_s=dk)
    ev[2].record(stream)
    torch.cuda.synchronize()
    if skl.device_status() != 0:
        raise RuntimeError("kernel watchdog fired in the packed-sequence run")
    fms = max_over_ranks(ev[0].elapsed_time(ev[1]) / steps, world)
    bms = max_over_ranks(ev[1].elapsed_time(ev[2]) / steps, world)
    pairs = varlen_pairs(lens, lens, w.causal) * w.H
    ff, fb = 2 * pairs * (w.d_T + w.d_S), 2 * pairs * (w.d_T + 3 * w.d_S)
    return {"tokens": tokens, "sequences": len(lens), "lengths": f"seeded uniform {lo}..{hi}",
            "fwd_ms": fms, "bwd_ms": bms, "fwd_tflops": ff / (fms * 1e-3) / 1e12,
            "bwd_tflops": fb / (bms * 1e-3) / 1e12}


def run_context_parallel(skl, w, d, dev, stream, steps, world, shards=4):
    """The workload with its keys split into ``shards`` contiguous shards, run one after
    another on this GPU as the shard ranks of a context-parallel group would run them
    side by side: partial forwards, the merge of their states, shard backwards. The
    all-gather / all-reduce between ranks is not part of it (one GPU)."""
    from attention_kl_divergence_fwd_b200.context_parallel import even_shards
    shards = min(shards, -(-w.N_K // 128))  # at least one 128-key tile per shard
    if shards < 2:
        return None
    cuts = even_shards(w.N_K, shards)
    ks = [(d["k_t"][:, :, a:a + n].contiguous(), d["k_s"][:, :, a:a + n].contiguous(), a)
          for a, n in cuts]
    B, H, nq = w.B, w.H, w.N_Q
    states = torch.empty(shards, 5, B, H, nq, device=dev)
    kl = torch.empty(B, H, nq, device=dev)
    lt, ls = torch.empty_like(kl), torch.empty_like(kl)
    dq = torch.empty(B, H, nq, w.d_S, device=dev)
    dks = [torch.empty(B, H, kt.shape[2], w.d_S, device=dev) for kt, _, _ in ks]
    base = (d["q_t"], d["q_s"])

    def fwd():
        for r, (kt, kss, a) in enumerate(ks):
            skl.streamkl_fwd_partial(base[0], kt, base[1], kss, w.scale_T, w.scale_S, w.causal,
                                     a, w.N_K, state=states[r])

    def merge():
        skl.streamkl_merge_partial(states, kl=kl, lse_t=lt, lse_s=ls)

    def bwd():
        for r, (kt, kss, a) in enumerate(ks):
            skl.streamkl_bwd_shard(base[0], kt, base[1], kss, w.scale_T, w.scale_S, w.causal, a,
                                   w.N_K, lt, ls, d["g"], dq_s=dq, dk_s=dks[r])

    for _ in range(3):
        fwd(); merge(); bwd()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    ev[0].record(stream)
    for _ in range(steps):
        fwd()
    ev[1].record(stream)
    for _ in range(steps):
        merge()
    ev[2].record(stream)
    for _ in range(steps):
        bwd()
    ev[3].record(stream)
    torch.cuda.synchronize()
    if skl.device_status() != 0:
        raise RuntimeError("kernel watchdog fired in the context-parallel run")
    t = [max_over_ranks(ev[i].elapsed_time(ev[i + 1]) / steps, world) for i in range(3)]
    merge_bytes = (shards * 20 + 12) * B * H * nq
    return {"shards": shards, "fwd_partial_ms": t[0], "merge_ms": t[1], "bwd_shard_ms": t[2],
            "fwd_tflops": flops_fwd(w) / ((t[0] + t[1]) * 1e-3) / 1e12,
            "bwd_tflops": flops_bwd(w) / (t[2] * 1e-3) / 1e12,
            "merge_gbs": merge_bytes / (t[1] * 1e-3) / 1e9}


def run_e2e(skl, w, x, dev, stream, steps, world):
    """Same metric through the public API from and to pinned host buffers: every step
    copies its inputs host->device, runs forward + backward, and copies its whole result,
    the KL rows and the student gradients dQ_S and dK_S, device->host. Three streams
    overlap: step k's input copy (second stream) runs beside step k-1's kernels, and step
    k-1's result copy (third stream) beside step k's kernels; inputs and outputs are
    double-buffered on the device, so the step time is bound by the slower PCIe direction."""
    host = {k: v.pin_memory() for k, v in x.items()}
    bufs = [{k: torch.empty_like(v, device=dev) for k, v in x.items()} for _ in range(2)]
    out_shapes = {"kl": (w.B, w.H, w.N_Q), "lse_t": (w.B, w.H, w.N_Q),
                  "lse_s": (w.B, w.H, w.N_Q), "dq": (w.B, w.H, w.N_Q, w.d_S),
                  "dk": (w.B, w.H, w.N_K, w.d_S)}
    outs = [{k: torch.empty(sh, device=dev) for k, sh in out_shapes.items()} for _ in range(2)]
    result = ("kl", "dq", "dk")  # what the step returns to the host
    host_out = [{k: torch.empty(out_shapes[k]).pin_memory() for k in result} for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(host_out[0][k].numel() * 4 for k in result)
    copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]    # step's kernels done with buffer set b
    drained = [torch.cuda.Event() for _ in range(2)]  # result of buffer set b is on the host

    def one(k):
        b = k & 1
        d, o = bufs[b], outs[b]
        with torch.cuda.stream(copy_in):
            copy_in.wait_event(freed[b])  # step k-2's kernels are done with input buffer b
            for name in d:
                d[name].copy_(host[name], non_blocking=True)
            copied[b].record(copy_in)
        stream.wait_event(copied[b])
        stream.wait_event(drained[b])  # step k-2's result has left output buffer b
        skl.streamkl_fwd(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T, w.scale_S,
                         w.causal, kl=o["kl"], lse_t=o["lse_t"], lse_s=o["lse_s"],
                         stream=stream)
        skl.streamkl_bwd(d["q_t"], d["k_t"], d["q_s"], d["k_s"], w.scale_T, w.scale_S,
                         w.causal, o["lse_t"], o["lse_s"], d["g"], dq_s=o["dq"], dk_s=o["dk"],
                         stream=stream)
        freed[b].record(stream)
        with torch.cuda.stream(copy_out):
            copy_out.wait_event(freed[b])
            for name in result:
                host_out[b][name].copy_(o[name], non_blocking=True)
            drained[b].record(copy_out)

    for b in range(2):
        freed[b].record(stream)
        drained[b].record(stream)
    for k in range(2):
        one(k)
    torch.cuda.synchronize()
    barrier(world)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    copy_in.wait_event(a)  # the first timed copy starts inside the timed region
    for k in range(steps):
        one(k)
    stream.wait_stream(copy_out)  # the last result copy ends inside the timed region
    e.record(stream)
    torch.cuda.synchronize()
    if skl.device_status() != 0:
        raise RuntimeError("kernel watchdog fired in the end-to-end run")
    ms = max_over_ranks(a.elapsed_time(e), world)
    value = world * (flops_fwd(w) + flops_bwd(w)) * steps / (ms * 1e-3) / 1e12
    return {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms / steps,
            "returned": "KL rows, dQ_S and dK_S (fp32) to pinned host memory every step",
            "pipeline": "input copies, kernels and result copies on three streams, inputs and "
                        "outputs double-buffered on the device"}


def run_eager(w, d, kl_fused, dev, stream, fwd_ms, bwd_ms, steps=2, budget_bytes=24 << 30):
    """The materialising comparator the pages measure against, timed on the same GPU:
    plain PyTorch eager ops that form both N_Q x N_K score matrices (bf16 matmul as under
    autocast, then fp32), both log-softmaxes and the row-wise KL, and differentiate
    sum_i g_i KL_i with autograd for dQ_S and dK_S. Heads are processed in chunks sized
    to the memory budget (the whole batch at once does not fit for long sequences).
    Returns times per step, the speedups of the fused kernels over it and the peak extra
    memory of one chunk, and the largest difference of its per-row KL from the fused
    forward's (its scores are rounded to bf16, the fused kernels keep them in fp32); a
    "skipped" note when a single head would not fit the budget."""
    nq, nk = w.N_Q, w.N_K
    per_head = 36 * nq * nk  # fp32 N_Q x N_K tensors live at the peak (measured ~32 B/pair)
    if per_head > budget_bytes:
        return {"skipped": f"one head needs about {per_head / 2**30:.0f} GiB of score matrices"}
    hc = max(1, min(w.bh, budget_bytes // per_head))
    qt, kt = d["q_t"].flatten(0, 1), d["k_t"].flatten(0, 1)
    qs, ks = d["q_s"].flatten(0, 1), d["k_s"].flatten(0, 1)
    g = d["g"].flatten(0, 1)
    allowed = None
    if w.causal:  # bottom-right aligned: key j is visible to query i iff j <= i + N_K - N_Q
        i = torch.arange(nq, device=dev)[:, None]
        j = torch.arange(nk, device=dev)[None, :]
        allowed = j <= i + (nk - nq)

    def chunk(a, b, ev):
        q_s = qs[a:b].detach().requires_grad_(True)
        k_s = ks[a:b].detach().requires_grad_(True)
        ev[0].record(stream)
        s_t = torch.matmul(qt[a:b], kt[a:b].transpose(-1, -2)).float() * w.scale_T
        s_s = torch.matmul(q_s, k_s.transpose(-1, -2)).float() * w.scale_S
        if allowed is not None:
            s_t = s_t.masked_fill(~allowed, float("-inf"))
            s_s = s_s.masked_fill(~allowed, float("-inf"))
        lp_t = torch.log_softmax(s_t, dim=-1)
        lp_s = torch.log_softmax(s_s, dim=-1)
        terms = lp_t.exp() * (lp_t - lp_s)
        if allowed is not None:
            terms = torch.where(allowed, terms, 0.0)
        kl = terms.sum(-1)
        ev[1].record(stream)
        (kl * g[a:b]).sum().backward()
        ev[2].record(stream)
        return kl

    def one_step(evs):
        diff = 0.0
        for n, a in enumerate(range(0, w.bh, hc)):
            b = min(w.bh, a + hc)
            kl = chunk(a, b, evs[n] if evs else [torch.cuda.Event() for _ in range(3)])
            if not evs:
                ref = kl_fused.flatten(0, 1)[a:b]
                diff = max(diff, (kl.detach() - ref).abs().max().item())
        return diff

    n_chunks = (w.bh + hc - 1) // hc
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    diff = one_step(None)  # warm-up, compared with the fused forward
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated(dev) - base
    f_ms = b_ms = 0.0
    for _ in range(steps):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_chunks)]
        one_step(evs)
        torch.cuda.synchronize()
        f_ms += sum(e[0].elapsed_time(e[1]) for e in evs)
        b_ms += sum(e[1].elapsed_time(e[2]) for e in evs)
    f_ms, b_ms = f_ms / steps, b_ms / steps
    return {"kind": "torch eager, both softmaxes materialised (bf16 scores, fp32 softmax/KL)",
            "heads_per_chunk": hc, "fwd_ms": f_ms, "bwd_ms": b_ms,
            "speedup_fwd": f_ms / fwd_ms, "speedup_bwd": b_ms / bwd_ms,
            "peak_extra_bytes": peak, "max_abs_kl_diff_vs_fused": diff}


def load_traffic(workload: str, which: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, if any."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        return d.get(workload, {}).get(which)
    except Exception:
        return None


if __name__ == "__main__":
    main()
