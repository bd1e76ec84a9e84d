"""The benchmark's reference arm (the CPU oracle timed on bounded slices) on CPU: the
slices cover every touched expert's intermediate features exactly once, and in the bf16
format (where no per-tensor scale couples them) their outputs add up to the oracle's
whole expert networks."""
from __future__ import annotations

import numpy as np

import bench
from oracle import fused_moe_oracle as O
from mixture_experts_layer_26_b200 import inputs as minp


def test_slices_cover_the_layer_and_add_up(monkeypatch):
    s = minp.MoEShape(T=6, H=256, I=512, E=4, top_k=2, wdtype="bf16", n_shared=1)
    inp = minp.make_inputs(s, seed=3)
    # a small work budget per step, so that every expert is cut into several blocks
    monkeypatch.setattr(bench.OracleSlices, "WORK_PER_STEP", 3.0 * s.H * 200 * 128)
    sl2 = bench.OracleSlices(inp)
    ids, w, counts, offsets, rows, inv, a_perm, s1 = sl2.prep
    for e in sl2.touched:
        blocks = sorted((f0, f1) for ee, f0, f1 in sl2.slices if ee == e)
        assert blocks[0][0] == 0 and blocks[-1][1] == s.I
        assert all(b[1] == c[0] for b, c in zip(blocks, blocks[1:]))
        assert len(blocks) > 1
    # the whole layer's expert outputs, from the oracle in one go
    d = bench.np_inputs(inp)
    y_full, *_ = O.experts(a_perm, offsets, rows, w, d["w13"], d["w2"], s.H, s.I, s.E_all,
                           False, s1)
    y_sum = np.zeros_like(y_full)
    for _ in range(len(sl2.slices)):
        e, y = sl2.step()
        y_sum[offsets[e]:offsets[e + 1]] += y
    assert np.abs(y_sum - y_full).max() <= 1e-9 * np.abs(y_full).max()


import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", ["tiny_bf16", "inv_rope_fp8_partial"])
def test_reference_arm_prints_one_contract_line(workload):
    """`bench.py --impl reference` runs the oracle on the host cores only and prints one
    JSON line with the contract's keys (the end-to-end number equals the value, no copies)."""
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", workload,
                        "--steps", "2", "--warmup", "3"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "cpu_baseline", "e2e", "config"):
        assert key in j, key
    assert j["impl"] == "reference" and j["value"] > 0 and j["steps"] == 2
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"]["value"] == j["value"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
