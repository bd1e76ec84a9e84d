"""Pins for the inverse-rotary + per-head FP8 oracle: checks against things other than
the oracle itself.

* the inverse rotation against complex multiplication by exp(-i*theta) in fp64;
* the round trip: rotating by +theta (an independent real formula) then applying the
  oracle gives the start back; rotations keep every pair's norm;
* special cases: position 0 leaves x unchanged exactly, coordinates past rot_dim pass
  through, the interleaved layout is the half-split one on permuted coordinates;
* per-head quantisation: the largest |y| of a head becomes code +-448 exactly, the
  dequantised values stay within half an e4m3 step, an all-zero head has scale 1;
* brute force: element-by-element Python loops on a tiny case.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import inv_rope_fp8_oracle as RO
from mixture_experts_layer_26_b200 import inputs as minp


def _case(T=6, nh=3, hd=64, rot=64, style=0, seed=0, max_pos=97):
    s = minp.RopeShape(T=T, n_heads=nh, head_dim=hd, rot_dim=rot, style=style, max_pos=max_pos)
    inp = minp.make_rope_inputs(s, seed=seed)
    xb = inp.x.view(torch.int16).numpy().view(np.uint16)
    return s, inp, xb, inp.positions.numpy(), inp.cos_sin.numpy()


@pytest.mark.parametrize("style", [0, 1])
def test_inverse_rotation_is_complex_multiplication(style):
    s, inp, xb, pos, cs = _case(style=style)
    y = RO.inv_rope(xb, pos, cs, s.rot_dim, style)
    x = inp.x.to(torch.float64).numpy()
    half = s.rot_dim // 2
    a = np.arange(half) if style == 0 else 2 * np.arange(half)
    b = a + half if style == 0 else a + 1
    c = cs[pos][:, None, :half].astype(np.float64)
    sn = cs[pos][:, None, half:].astype(np.float64)
    z = (x[:, :, a] + 1j * x[:, :, b]) * (c - 1j * sn)        # times exp(-i theta)
    assert np.abs(y[:, :, a] - z.real).max() <= 1e-6 * np.abs(z.real).max()
    assert np.abs(y[:, :, b] - z.imag).max() <= 1e-6 * np.abs(z.imag).max()


def test_round_trip_and_norms():
    s, inp, xb, pos, cs = _case(T=8, nh=2, hd=128, rot=128, seed=3)
    rng = np.random.default_rng(5)
    y0 = rng.standard_normal((s.T, s.n_heads, s.head_dim))
    half = s.rot_dim // 2
    c = cs[pos][:, None, :half].astype(np.float64)
    sn = cs[pos][:, None, half:].astype(np.float64)
    fwd = y0.copy()                                            # rotate by +theta
    fwd[:, :, :half] = y0[:, :, :half] * c - y0[:, :, half:] * sn
    fwd[:, :, half:] = y0[:, :, :half] * sn + y0[:, :, half:] * c
    xbits = torch.from_numpy(fwd).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    y = RO.inv_rope(xbits, pos, cs, s.rot_dim, 0)
    # bf16 rounding of the rotated input bounds the error (relative 2^-8 per element)
    assert np.abs(y - y0).max() <= 2.0 ** -7 * np.abs(y0).max()
    x = RO.bf16_to_f32(xbits).astype(np.float64)
    n_in = x[:, :, :half] ** 2 + x[:, :, half:] ** 2
    n_out = y[:, :, :half].astype(np.float64) ** 2 + y[:, :, half:].astype(np.float64) ** 2
    assert np.abs(n_in - n_out).max() <= 1e-5 * n_in.max()


def test_position_zero_and_pass_through_are_exact():
    s, inp, xb, pos, cs = _case(T=5, nh=2, hd=128, rot=64, style=0)
    pos0 = np.zeros_like(pos)
    y = RO.inv_rope(xb, pos0, cs, s.rot_dim, 0)
    assert np.array_equal(y, RO.bf16_to_f32(xb))             # cos 1, sin 0: x itself
    y = RO.inv_rope(xb, pos, cs, s.rot_dim, 0)
    assert np.array_equal(y[:, :, 64:], RO.bf16_to_f32(xb)[:, :, 64:])


def test_interleaved_layout_is_a_permutation_of_the_half_split_one():
    s, inp, xb, pos, cs = _case(T=4, nh=2, hd=64, rot=64, style=1)
    perm = np.concatenate([np.arange(0, 64, 2), np.arange(1, 64, 2)])   # evens, then odds
    y1 = RO.inv_rope(xb, pos, cs, 64, 1)
    y0 = RO.inv_rope(xb[:, :, perm], pos, cs, 64, 0)
    assert np.array_equal(y1[:, :, perm], y0)


def test_per_head_quantisation_properties():
    s, inp, xb, pos, cs = _case(T=7, nh=4, hd=128, rot=128, seed=2)
    xb = xb.copy()
    xb[3, 1, :] = 0                                           # one all-zero head
    r = RO.inv_rope_fp8_quant(xb, pos, cs, s.rot_dim, 0)
    y, q, sc = r["y"], r["q"], r["scales"]
    deq = RO.e4m3_decode(q)
    amax = np.abs(y).max(axis=2)
    for t in range(s.T):
        for h in range(s.n_heads):
            if amax[t, h] == 0:
                # signed zeros from the rotation encode as 0x00 / 0x80: all decode to 0
                assert sc[t, h] == 1.0 and np.all(deq[t, h] == 0)
                continue
            assert sc[t, h] == np.float32(amax[t, h]) / np.float32(448)
            assert np.abs(deq[t, h]).max() == 448.0           # the largest element
            # round to nearest: within half a step (relative 2^-4) or the subnormal step
            err = np.abs(deq[t, h] * sc[t, h] - y[t, h])
            bound = np.maximum(np.abs(y[t, h]) * 2.0 ** -4, 2.0 ** -10 * sc[t, h]) * 1.0001
            assert np.all(err <= bound)


def test_bruteforce_tiny():
    s, inp, xb, pos, cs = _case(T=2, nh=2, hd=8, rot=8, style=0, seed=7, max_pos=11)
    r = RO.inv_rope_fp8_quant(xb, pos, cs, s.rot_dim, 0)
    x = inp.x.to(torch.float32).numpy()
    f = np.float32
    for t in range(2):
        for h in range(2):
            y = [0.0] * 8
            for i in range(4):
                c, sn = f(cs[pos[t], i]), f(cs[pos[t], 4 + i])
                xa, xb_ = f(x[t, h, i]), f(x[t, h, 4 + i])
                y[i] = f(f(xa * c) + f(xb_ * sn))
                y[4 + i] = f(f(-f(xa * sn)) + f(xb_ * c))
            assert [float(v) for v in r["y"][t, h]] == [float(v) for v in y]
            m = max(abs(v) for v in y)
            inv = f(f(448) / f(m))
            ref = torch.tensor([float(f(v * inv)) for v in y], dtype=torch.float32) \
                .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(r["q"][t, h], ref)


def test_inverse_scale_is_one_division_448_over_amax():
    """P3: inv = 448/amax (one fp32 division), not 1/(amax/448): pick an amax where the
    two differ and a value whose e4m3 code depends on which one is used; the expected
    code comes from torch's cast of the fp32 product."""
    f = np.float32
    a = f(1.11)
    inv_a, inv_b = f(f(448) / a), f(f(1) / f(a / f(448)))
    assert inv_a != inv_b
    mids = [(RO.e4m3_decode(np.uint8(c)) + RO.e4m3_decode(np.uint8(c + 1))) / 2
            for c in range(8, 126)]
    v = None
    for m in mids:
        for cand in (np.nextafter(f(m / inv_a), f(0)), f(m / inv_a), np.nextafter(f(m / inv_a), f(9))):
            cand = f(cand)
            if cand < a and RO.e4m3_encode(f(cand * inv_a)) != RO.e4m3_encode(f(cand * inv_b)):
                v = cand
                break
        if v is not None:
            break
    assert v is not None
    y = np.zeros((1, 1, 64), np.float32)
    y[0, 0, 0], y[0, 0, 1] = a, v
    q, sc = RO.quant_per_head(y)
    want = torch.tensor([float(f(v * inv_a))]).to(torch.float8_e4m3fn).view(torch.uint8).item()
    assert q[0, 0, 1] == want and sc[0, 0] == f(a / f(448))


def test_tiny_regression_golden():
    """The oracle against its own committed record (tests/golden/make_golden_rope.py):
    catches an unintended change of the oracle's arithmetic, not a wrong reading."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "inv_rope_tiny_seed0.json")
    doc = json.load(open(path))
    s = minp.RopeShape(**doc["shape"])
    inp = minp.make_rope_inputs(s, seed=0)
    r = RO.inv_rope_fp8_quant(minp.bf16_bits(inp.x), inp.positions.numpy(), inp.cos_sin.numpy(),
                              s.rot_dim, s.style)
    assert r["q"].tolist() == doc["codes"]
    assert [[float(v) for v in row] for row in r["scales"]] == doc["scales"]
