"""Writes tests/golden/tiny_bf16_seed0.json from the CPU oracle alone.

The pages print no worked example, so this fixture is a regression record of
the oracle on the tiny bf16 workload (T=4, H=256, I=512, E=8, k=2, seed 0); it
is not an independent pin.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import fused_moe_oracle as O  # noqa: E402
from mixture_experts_layer_26_b200 import inputs as minp  # noqa: E402


def main():
    s = minp.shape("tiny_bf16")
    inp = minp.make_inputs(s, seed=0)
    r = O.fused_moe(minp.bf16_bits(inp.x), minp.bf16_bits(inp.router_w), minp.bf16_bits(inp.w13),
                    minp.bf16_bits(inp.w2), s.top_k, fp8=False)
    doc = {
        "workload": "tiny bf16 MoE, T=4 H=256 I=512 E=8 k=2, seed 0",
        "written_by": "tests/golden/make_golden.py (CPU oracle only)",
        "topk_ids": r["topk_ids"].tolist(),
        "topk_w": [[float(v) for v in row] for row in r["topk_w"]],
        "counts": r["counts"].tolist(),
        "sorted_rows": r["sorted_rows"].tolist(),
        "out_bf16_bits": [[int(v) for v in row] for row in r["out"]],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_bf16_seed0.json")
    with open(path, "w") as f:
        json.dump(doc, f, separators=(",", ":"))
        f.write("\n")


if __name__ == "__main__":
    main()
