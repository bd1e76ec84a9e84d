"""Writes tests/golden/inv_rope_tiny_seed0.json from the inverse-RoPE CPU oracle alone.

The pages print no worked example, so this fixture is a regression record of the oracle
on a tiny case (T=5, 3 heads of 64, partial rotary 32, half split, 11 positions, seed 0);
it is not an independent pin.  Run from the repository root:
    python tests/golden/make_golden_rope.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import inv_rope_fp8_oracle as RO  # noqa: E402
from mixture_experts_layer_26_b200 import inputs as minp  # noqa: E402

SHAPE = dict(T=5, n_heads=3, head_dim=64, rot_dim=32, style=0, max_pos=11)


def main():
    s = minp.RopeShape(**SHAPE)
    inp = minp.make_rope_inputs(s, seed=0)
    r = RO.inv_rope_fp8_quant(minp.bf16_bits(inp.x), inp.positions.numpy(), inp.cos_sin.numpy(),
                              s.rot_dim, s.style)
    doc = {
        "workload": "inverse RoPE + per-head FP8, T=5 heads=3 head_dim=64 rot_dim=32 half split, "
                    "max_pos 11, seed 0",
        "written_by": "tests/golden/make_golden_rope.py (CPU oracle only)",
        "shape": SHAPE,
        "codes": r["q"].tolist(),
        "scales": [[float(v) for v in row] for row in r["scales"]],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "inv_rope_tiny_seed0.json")
    with open(path, "w") as f:
        json.dump(doc, f, separators=(",", ":"))
        f.write("\n")


if __name__ == "__main__":
    main()
