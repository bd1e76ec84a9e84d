"""GPU parity of the fused inverse-rotary + per-head FP8 quantisation kernel (through the
C ABI) against its CPU oracle on the same seeded inputs.

Bar: the e4m3 codes and the per-head scales are bit-exact (both sides evaluate y in
fp32 in the same order without fused multiply-adds, and take every code from that fp32
value).  Small cases cover every head size, both pair layouts, partial rotary, head
counts that do not fill the kernel's four-head step, all-zero heads and ragged token
counts; the full-size cases run the three workloads at their real shapes.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import inv_rope_fp8_oracle as RO
from mixture_experts_layer_26_b200 import inputs as minp

capi = pytest.importorskip("mixture_experts_layer_26_b200.capi")

pytestmark = pytest.mark.gpu


def run_gpu(inp: minp.RopeInputs, positions=None):
    s = inp.shape
    d = capi.make_rope_dims(s.T, s.n_heads, s.head_dim, s.rot_dim, s.style, s.max_pos)
    x = inp.x.cuda()
    pos = (inp.positions if positions is None else positions).cuda()
    cs = inp.cos_sin.cuda()
    q = torch.full((s.T, s.n_heads, s.head_dim), 0xAB, dtype=torch.uint8, device="cuda")
    sc = torch.full((s.T, s.n_heads), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.fused_inv_rope_fp8_quant_per_head(d, x, pos, cs, q, sc, st)
    torch.cuda.synchronize()
    return q.cpu().numpy(), sc.cpu().numpy(), int(st.item())


def run_oracle(inp: minp.RopeInputs, positions=None):
    s = inp.shape
    xb = inp.x.view(torch.int16).numpy().view(np.uint16)
    pos = (inp.positions if positions is None else positions).numpy()
    return RO.inv_rope_fp8_quant(xb, pos, inp.cos_sin.numpy(), s.rot_dim, s.style)


SMALL = [
    # T, n_heads, head_dim, rot_dim, style
    (37, 5, 128, 128, 0),   # heads not a multiple of the four-head step, ragged T
    (19, 3, 64, 64, 0),
    (11, 2, 256, 256, 0),
    (23, 6, 128, 64, 0),    # partial rotary: coordinates 64..127 pass through
    (29, 4, 256, 32, 0),    # smallest rotary span for head_dim 256 (2 * 8)
    (17, 7, 128, 64, 1),    # interleaved pairs, partial
    (13, 4, 64, 64, 1),
    (9, 1, 256, 128, 1),
    (1, 1, 128, 8, 0),      # one token, one head, the shortest rotary span for 128
    (21, 9, 128, 128, 1),   # interleaved, full rotary, a second head group of one head
    (15, 12, 64, 64, 0),    # half split, full rotary, head groups of eight and four
]


@pytest.mark.parametrize("T,nh,hd,rot,style", SMALL)
def test_small_cases_match_oracle_bit_exact(T, nh, hd, rot, style):
    s = minp.RopeShape(T=T, n_heads=nh, head_dim=hd, rot_dim=rot, style=style, max_pos=257)
    inp = minp.make_rope_inputs(s, seed=T)
    q, sc, st = run_gpu(inp)
    ref = run_oracle(inp)
    assert st == capi.FMOE_OK
    assert np.array_equal(sc, ref["scales"])
    assert np.array_equal(q, ref["q"])


def test_zero_heads_and_position_zero():
    s = minp.RopeShape(T=12, n_heads=4, head_dim=128, rot_dim=128, max_pos=64)
    inp = minp.make_rope_inputs(s, seed=4)
    inp.x[2, 1].zero_()
    inp.x[5].zero_()
    inp.positions[7] = 0
    q, sc, st = run_gpu(inp)
    ref = run_oracle(inp)
    assert np.array_equal(sc, ref["scales"]) and np.array_equal(q, ref["q"])
    assert sc[2, 1] == 1.0 and np.all(RO.e4m3_decode(q[2, 1]) == 0)


def test_out_of_range_positions_are_reported_and_read_as_zero():
    s = minp.RopeShape(T=8, n_heads=4, head_dim=128, rot_dim=128, max_pos=32)
    inp = minp.make_rope_inputs(s, seed=2)
    bad = inp.positions.clone()
    bad[3] = 32
    bad[6] = -5
    q, sc, st = run_gpu(inp, bad)
    assert st == capi.FMOE_ERR_DEVICE_BOUNDS
    fixed = bad.clone()
    fixed[3] = 0
    fixed[6] = 0
    ref = run_oracle(inp, fixed)
    assert np.array_equal(q, ref["q"]) and np.array_equal(sc, ref["scales"])


@pytest.mark.parametrize("workload", sorted(minp.ROPE_WORKLOADS))
def test_full_size_workloads_bit_exact(workload):
    inp = minp.make_rope_inputs(minp.rope_shape(workload), seed=0)
    q, sc, st = run_gpu(inp)
    ref = run_oracle(inp)
    assert st == capi.FMOE_OK
    assert np.array_equal(sc, ref["scales"])
    assert np.array_equal(q, ref["q"])
