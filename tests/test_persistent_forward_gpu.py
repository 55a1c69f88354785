"""The forward's two grid forms give the same results, bit for bit (needs a B200).

The launch planner runs the forward as a persistent grid (one CTA per SM walking a
heaviest-first snake of work units) when a dense problem has at most 8 units per SM, and as
one CTA per unit otherwise. The arithmetic of a row is the same in both, so KL, LSE_T, LSE_S
(and the raw row state of a key shard) must agree exactly. STREAMKL_FWD_PERSIST forces a
form; it is read once per process, so each form runs in a process of its own.
"""
import math
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import sys, torch
import attention_kl_divergence_fwd_b200 as skl
from workloads import WORKLOADS, make_inputs
base = WORKLOADS["b2h16_n4096_d128_causal"]
cases = [
    dict(B=1, H=7, N_Q=700, N_K=700, causal=True),
    dict(B=2, H=3, N_Q=517, N_K=333, d_T=64, d_S=128, causal=True, scale_T=0.125,
         scale_S=0.0884, student="independent"),
    dict(B=1, H=2, N_Q=200, N_K=700, d_T=64, d_S=64, causal=False, scale_T=0.125,
         scale_S=0.125, student="independent"),
    dict(B=3, H=4, N_Q=1000, N_K=1000, causal=True),
]
out = {}
for n, c in enumerate(cases):
    w = base.with_sizes(**c)
    x = {k: v.cuda() for k, v in make_inputs(w, seed=50 + n).items()}
    kl, lt, ls = skl.streamkl_fwd(x["q_t"], x["k_t"], x["q_s"], x["k_s"], w.scale_T,
                                  w.scale_S, w.causal)
    out[f"c{n}"] = torch.stack([kl, lt, ls]).cpu()
# grouped-query K heads (teacher 2, student 4 of 8 query heads)
w = base.with_sizes(B=2, H=8, N_Q=640, N_K=640, causal=True)
x = {k: v.cuda() for k, v in make_inputs(w, seed=61).items()}
kl, lt, ls = skl.streamkl_fwd_gqa(x["q_t"], x["k_t"][:, :2].contiguous(), x["q_s"],
                                  x["k_s"][:, :4].contiguous(), w.scale_T, w.scale_S, True)
out["gqa"] = torch.stack([kl, lt, ls]).cpu()
# planted keys lift some rows' scores far above their first tiles (the lazy fold keeps a
# tile with sums up to 2^44 and refolds one that would reach 2^64)
w = base.with_sizes(B=1, H=2, N_Q=640, N_K=640, causal=False)
x = make_inputs(w, seed=21)
for side, h, plants in (("t", 0, ((500, 600, 3.0), (560, 620, 8.0))),
                        ("s", 1, ((450, 610, 3.0), (530, 630, 8.0)))):
    for key, row, gain in plants:
        x["k_" + side][0, h, key] = (x["q_" + side][0, h, row].float() * gain).to(torch.bfloat16)
x = {k: v.cuda() for k, v in x.items()}
kl, lt, ls = skl.streamkl_fwd(x["q_t"], x["k_t"], x["q_s"], x["k_s"], w.scale_T, w.scale_S, False)
out["jumps"] = torch.stack([kl, lt, ls]).cpu()
# a key shard's raw row state (context parallelism): keys 384..767 of 1000
w = base.with_sizes(B=1, H=3, N_Q=1000, N_K=1000, causal=True)
x = {k: v.cuda() for k, v in make_inputs(w, seed=62).items()}
st = skl.streamkl_fwd_partial(x["q_t"], x["k_t"][:, :, 384:768].contiguous(), x["q_s"],
                              x["k_s"][:, :, 384:768].contiguous(), w.scale_T, w.scale_S, True,
                              384, 1000)
out["shard"] = st.cpu()
assert skl.device_status() == 0
torch.save(out, sys.argv[1])
"""


def _run(form: str, path: str):
    env = dict(os.environ)
    env["STREAMKL_FWD_PERSIST"] = form
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    subprocess.run([sys.executable, "-c", _CHILD, path], env=env, cwd=ROOT, check=True,
                   timeout=300)
    return torch.load(path)


def test_persistent_and_grid_forward_agree_bitwise(tmp_path):
    from attention_kl_divergence_fwd_b200 import build
    build.build()
    grid = _run("0", str(tmp_path / "grid.pt"))
    pers = _run("1", str(tmp_path / "pers.pt"))
    assert grid.keys() == pers.keys()
    for k in grid:
        assert torch.equal(grid[k], pers[k]), k


def test_persistent_forward_matches_oracle(tmp_path):
    """The persistent form against the fp64 oracle on a causal case with a ragged tail."""
    from oracle import oracle_fwd
    from workloads import WORKLOADS, make_inputs
    from attention_kl_divergence_fwd_b200 import build
    build.build()
    pers = _run("1", str(tmp_path / "pers.pt"))
    w = WORKLOADS["b2h16_n4096_d128_causal"].with_sizes(B=1, H=7, N_Q=700, N_K=700, causal=True)
    x = make_inputs(w, seed=50)
    kl, lt, ls = oracle_fwd(x["q_t"], x["k_t"], x["q_s"], x["k_s"], w.scale_T, w.scale_S, True)
    got = pers["c0"].double()
    err = (got[0] - kl).abs()
    assert bool(((err <= 1e-4) | (err <= 2e-3 * kl.abs())).all()), err.max().item()
    for i, ref in ((1, lt), (2, ls)):
        assert bool(((got[i] - ref).abs() <= 1e-4 + 1e-5 * ref.abs()).all())
