"""bench.py's reference arm (the fp64 oracle on the host cores) on CPU: one JSON line with
the contract's keys, and no GPU touched."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
         "--warmup", "1", "--ref-seconds", "3", "--workload", "tiny_n256_d64"],
        capture_output=True, text=True, timeout=300, cwd=ROOT,
        env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny_n256_d64"


def test_eager_comparator_computes_the_kl(monkeypatch):
    """The materialising comparator of bench.py (run here on CPU tensors with the CUDA event
    and memory calls stubbed) forms the same per-row KL as the oracle, up to the bf16
    rounding of its scores, for causal and full attention."""
    import dataclasses

    import torch

    sys.path.insert(0, ROOT)
    import bench
    from oracle import oracle_fwd
    from workloads import WORKLOADS, make_inputs

    class Ev:
        def __init__(self, **kw):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 1.0

    monkeypatch.setattr(torch.cuda, "Event", Ev)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "memory_allocated", lambda *a: 0)
    monkeypatch.setattr(torch.cuda, "reset_peak_memory_stats", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "max_memory_allocated", lambda *a: 0)
    for causal in (False, True):
        w = dataclasses.replace(WORKLOADS["tiny_n256_d64"], causal=causal)
        x = make_inputs(w)
        kl, _, _ = oracle_fwd(x["q_t"], x["k_t"], x["q_s"], x["k_s"], w.scale_T, w.scale_S,
                              causal)
        r = bench.run_eager(w, x, kl.float(), torch.device("cpu"), None, 2.0, 4.0, steps=1)
        assert r["max_abs_kl_diff_vs_fused"] < 0.02, r
        assert r["speedup_fwd"] == 0.5 and r["speedup_bwd"] == 0.25
        assert r["heads_per_chunk"] == 1
    big = dataclasses.replace(WORKLOADS["extreme_b1h8_n65536_d128_causal"])
    assert "skipped" in bench.run_eager(big, {}, None, torch.device("cpu"), None, 1.0, 1.0)


def test_bench_helpers():
    """The config's L2 note and the clock used for the exponential-unit roofline."""
    sys.path.insert(0, ROOT)
    import bench
    from workloads import WORKLOADS

    assert "fit in the 126 MB L2" in bench.l2_note(WORKLOADS["tiny_n256_d64"])
    assert "537 MB" in bench.l2_note(WORKLOADS["long_b1h32_n16384_d128_causal"])
    assert bench.clocks_mhz_or(None) == 1965.0
    assert bench.clocks_mhz_or({"sm_mhz": 1804.0}) == 1804.0
    assert bench.clocks_mhz_or({"sm_mhz": None}) == 1965.0
