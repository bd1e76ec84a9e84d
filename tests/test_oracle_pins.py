"""Pins for the CPU oracle: checks against things other than the oracle itself.

* the e4m3fn and bf16 codecs against torch's casts (a library routine),
  exhaustively over bf16 bit patterns and on random and tie values;
* the canonical router summation order against hand-derived sums on inputs
  built so that different orders give different fp32 results;
* routing against closed forms (integer logits, k = E full softmax);
* the whole layer against the independent brute-force per-token loops on tiny
  shapes, and against closed forms built from one-hot weights;
* invariants (weights sum to 1, counts sum to T*k, the permutation is a stable
  bijection, selected logits dominate the unselected ones).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import fused_moe_oracle as O
from mixture_experts_layer_26_b200 import inputs as minp
from bruteforce import brute_force, exact_logits, grouped_routing as brute_grouped
from helpers import np_inputs, run_oracle, max_rel_err, tiny_shape, bf16_bits_to_float, torch_bf16_bits


# ----------------------------------------------------------------------------- codecs

def _torch_e4m3(v32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(v32, dtype=np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert nan.sum() == 2                      # 0x7F and 0xFF
    assert np.array_equal(got[~nan], ref[~nan])
    assert O.e4m3_decode(np.uint8(0x7E)) == 448.0
    assert O.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9


def test_e4m3_encode_every_bf16_pattern_matches_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = bf16_bits_to_float(bits)
    keep = np.isfinite(v) & (np.abs(v) < 464.0)     # torch turns >= 464 into NaN
    v = v[keep]
    assert np.array_equal(O.e4m3_encode(v), _torch_e4m3(v))


def test_e4m3_encode_random_and_ties_match_torch():
    rng = np.random.default_rng(1)
    u = rng.uniform(-463.9, 463.9, 500_000).astype(np.float32)
    lg = (np.sign(rng.standard_normal(500_000)) *
          np.exp2(rng.uniform(-14, 8.85, 500_000))).astype(np.float32)
    pos = O.E4M3_TABLE[:127]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)     # exact ties
    ties = np.concatenate([mids, -mids])
    for v in (u, lg, ties):
        assert np.array_equal(O.e4m3_encode(v), _torch_e4m3(v))


def test_e4m3_saturation_and_signs():
    v = np.array([448, 449, 463.99, 464, 1e6, -1e6, np.inf, -np.inf], dtype=np.float32)
    assert list(O.e4m3_encode(v)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]
    assert O.e4m3_encode(np.float32(-0.0)) == 0x80
    assert O.e4m3_encode(np.float32(-1e-10)) == 0x80
    assert O.e4m3_encode(np.float32(np.nan)) == 0x7F
    # the smallest subnormal is 2^-9; half of it is a tie that goes to the even code 0
    assert O.e4m3_encode(np.float32(2.0 ** -10)) == 0x00
    assert O.e4m3_encode(np.float32(3 * 2.0 ** -10)) == 0x02


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(200_000) * np.exp2(rng.uniform(-30, 30, 200_000))).astype(np.float32)
    # exact ties: odd multiples of 2^-8 just above 1
    ties = (1.0 + (2 * np.arange(1, 200) + 1) * 2.0 ** -9).astype(np.float32)
    for arr in (v, ties, -ties):
        assert np.array_equal(O.f32_to_bf16(arr), torch_bf16_bits(arr))
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = bf16_bits_to_float(bits)
    ok = np.isfinite(f)
    assert np.array_equal(O.bf16_to_f32(bits)[ok],
                          torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
                          .to(torch.float32).numpy()[ok])


# ----------------------------------------------------------------------------- router

def _bits(v) -> np.ndarray:
    return torch_bf16_bits(np.asarray(v, dtype=np.float32))


def _single_logit(prod_pairs, H):
    """x, w rows (bf16 bits) whose products are the given {column: (x, w)}."""
    x = np.zeros((1, H), np.float32)
    w = np.zeros((1, H), np.float32)
    for col, (a, b) in prod_pairs.items():
        x[0, col], w[0, col] = a, b
    return _bits(x), _bits(w)


def test_canonical_order_butterfly():
    # Products 2^24 at column 0 (lane 0), 1 at column 128 (lane 16),
    # 1 at column 8 (lane 1), -2^24 at column 136 (lane 17).
    # Butterfly off=16: p0 = 2^24 + 1 = 2^24 (tie to even), p1 = 1 - 2^24 = -16777215;
    # off=8,4,2 add zeros; off=1: 2^24 - 16777215 = 1.
    # Plain ascending summation would give 0, the exact sum is 2.
    x, w = _single_logit({0: (4096, 4096), 128: (1, 1), 8: (1, 1), 136: (-4096, 4096)}, 256)
    assert O.router_logits(x, w)[0, 0] == np.float32(1.0)
    assert math.fsum(bf16_bits_to_float(x)[0] * bf16_bits_to_float(w)[0]) == 2.0


def test_canonical_order_butterfly_direction():
    # Products 2^24 (column 0, lane 0), 1 (column 128, lane 16), 1 (column 136, lane 17).
    # Offsets 16 first: p0 = 2^24 + 1 -> 2^24, p1 = 0 + 1 = 1; last step 2^24 + 1 -> 2^24.
    # Offset 1 first would pair lanes 16 and 17 (1 + 1 = 2) and end at 2^24 + 2.
    x, w = _single_logit({0: (4096, 4096), 128: (1, 1), 136: (1, 1)}, 256)
    assert O.router_logits(x, w)[0, 0] == np.float32(16777216.0)


def test_canonical_order_chunks_interleave_over_lanes():
    # H = 512: column 8 is chunk 1, owned by lane 1 (not lane 0).  Products 2^24 at
    # column 0, 1 at columns 8 and 9: lane 1 holds 2 exactly, final 2^24 + 2.
    # If lane 0 owned columns 0..15 each +1 would be lost and the sum would be 2^24.
    x, w = _single_logit({0: (4096, 4096), 8: (1, 1), 9: (1, 1)}, 512)
    assert O.router_logits(x, w)[0, 0] == np.float32(16777218.0)


def test_canonical_order_within_lane():
    # H = 512: lane 0 owns chunk 0 (columns 0..7) and chunk 32 (columns 256..263).
    # Ascending: 1 + 1 = 2, then 2 + 2^24 = 16777218 (exact).
    # Chunk 32 first would give 2^24 + 1 -> 2^24, + 1 -> 2^24.
    x, w = _single_logit({0: (1, 1), 1: (1, 1), 256: (4096, 4096)}, 512)
    assert O.router_logits(x, w)[0, 0] == np.float32(16777218.0)
    # Element order inside a chunk: 2^24 then 1 then 1 -> 2^24 (each +1 is a tie to even)
    x, w = _single_logit({0: (4096, 4096), 1: (1, 1), 2: (1, 1)}, 256)
    assert O.router_logits(x, w)[0, 0] == np.float32(16777216.0)


def test_router_integer_logits_closed_form():
    # Token t has x = e_t (one-hot), so logit[t,e] = Wr[e,t] exactly.
    T, E, H, k = 4, 6, 256, 3
    Wr = np.zeros((E, H), np.float32)
    table = np.array([[3, 1, 4, 1, 5, 9],     # token 0: 9,5,4 -> experts 5,4,2
                      [2, 7, 1, 8, 2, 8],     # token 1: tie 8,8 -> experts 3,5 then 7 -> 1
                      [0, 0, 0, 0, 0, 0],     # token 2: all tie -> experts 0,1,2
                      [-1, -2, -3, -4, -5, -6]], np.float32)
    for t in range(T):
        Wr[:, t] = table[t]
    x = np.zeros((T, H), np.float32)
    x[np.arange(T), np.arange(T)] = 1.0
    ids, w, logits = O.router(_bits(x), _bits(Wr), k)
    assert np.array_equal(logits, table)
    assert ids.tolist() == [[5, 4, 2], [3, 5, 1], [0, 1, 2], [0, 1, 2]]
    for t in range(T):
        l = [table[t][e] for e in ids[t]]
        z = sum(math.exp(v - l[0]) for v in l)
        ref = [math.exp(v - l[0]) / z for v in l]
        assert np.allclose(w[t], ref, rtol=1e-7, atol=0)


def test_router_k_equals_E_is_full_softmax():
    s = tiny_shape(5, 256, 256, 4, 4, "bf16")
    x, wr = minp.make_activations(s, seed=3)
    ids, w, _ = O.router(minp.bf16_bits(x), minp.bf16_bits(wr), 4)
    ex = exact_logits(minp.bf16_bits(x), minp.bf16_bits(wr))
    for t in range(5):
        m = max(ex[t])
        z = math.fsum(math.exp(v - m) for v in ex[t])
        ref = [math.exp(ex[t][e] - m) / z for e in ids[t]]
        assert np.allclose(w[t], ref, rtol=2e-6, atol=0)
        assert sorted(ids[t].tolist()) == [0, 1, 2, 3]


@pytest.mark.parametrize("seed,T,H,E,k,std", [(0, 16, 256, 8, 2, None), (1, 9, 512, 32, 4, None),
                                              (2, 7, 768, 64, 8, 1.0)])
def test_router_matches_exact_logits(seed, T, H, E, k, std):
    s = tiny_shape(T, H, 128, E, k, "fp8", router_std=std)
    x, wr = minp.make_activations(s, seed=seed)
    xb, wb = minp.bf16_bits(x), minp.bf16_bits(wr)
    ids, w, logits = O.router(xb, wb, k)
    ex = np.array(exact_logits(xb, wb))
    absprod = np.abs(bf16_bits_to_float(xb)).astype(np.float64) @ \
        np.abs(bf16_bits_to_float(wb)).astype(np.float64).T
    bound = (H // 32 + 5) * 2.0 ** -24 * absprod          # fp32 summation error bound
    assert np.all(np.abs(logits - ex) <= bound)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-ex[t][e], e))
        gap = ex[t][order[k - 1]] - ex[t][order[k]] if k < E else np.inf
        assert gap > 2 * bound[t].max()                  # the seeds have clear margins
        assert ids[t].tolist() == order[:k]


# ----------------------------------------------------------------------------- invariants

@pytest.mark.parametrize("seed,T,E,k", [(0, 33, 8, 2), (1, 64, 32, 8), (2, 1, 4, 4), (3, 200, 16, 1)])
def test_routing_invariants(seed, T, E, k):
    s = tiny_shape(T, 256, 128, E, k, "fp8")
    x, wr = minp.make_activations(s, seed=seed)
    ids, w, logits = O.router(minp.bf16_bits(x), minp.bf16_bits(wr), k)
    assert np.allclose(w.astype(np.float64).sum(1), 1.0, atol=4 * 2.0 ** -24 * k)
    assert np.all(w > 0)
    for t in range(T):
        assert len(set(ids[t].tolist())) == k
        sel = logits[t, ids[t]]
        assert np.all(np.diff(sel) <= 0)                          # descending
        uns = np.delete(logits[t], ids[t])
        if uns.size:
            assert sel.min() >= uns.max()
    counts, offsets, rows, inv = O.permute(ids, E)
    R = T * k
    assert counts.sum() == R and offsets[0] == 0 and offsets[-1] == R
    assert np.array_equal(np.sort(rows), np.arange(R))
    assert np.array_equal(rows[inv], np.arange(R))
    flat = ids.reshape(-1)
    for e in range(E):
        seg = rows[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)   # grouped and stable


def test_zero_tokens():
    s = tiny_shape(0, 256, 128, 4, 2, "fp8")
    inp = minp.make_inputs(s)
    r = run_oracle(O, inp)
    assert r["out"].shape == (0, 256) and r["counts"].sum() == 0


def test_act_scales_rules():
    assert O.act_scales(np.float32(0)) == (1.0, 1.0)
    # the inverse scale is the single division 448/amax (R4), which for amax = 3
    # differs from the reciprocal of the rounded scale 1/(amax/448)
    a = np.float32(1.11)
    _, inv = O.act_scales(a)
    assert inv == np.float32(403.6036)
    assert inv != np.float32(np.float32(1.0) / np.float32(a / np.float32(448)))
    s, inv = O.act_scales(np.float32(3.5))
    assert s == np.float32(3.5) / np.float32(448) and inv == np.float32(448) / np.float32(3.5)
    s, inv = O.act_scales(np.float32(3.5), static_scale=0.25)
    assert s == np.float32(0.25) and inv == np.float32(4.0)


# ----------------------------------------------------------------------------- whole layer

BRUTE_CASES = [
    # (seed, T, H, I, E, k, wdtype)
    (0, 4, 256, 256, 8, 2, "fp8"),
    (1, 3, 256, 256, 1, 1, "fp8"),     # single expert: a dense gated MLP
    (2, 2, 256, 256, 4, 4, "fp8"),     # k = E: every expert, full softmax
    (3, 4, 256, 256, 8, 2, "bf16"),
    (4, 3, 256, 256, 1, 1, "bf16"),
    (5, 2, 256, 128, 4, 4, "bf16"),
]


@pytest.mark.parametrize("seed,T,H,I,E,k,wdtype", BRUTE_CASES)
def test_oracle_matches_bruteforce(seed, T, H, I, E, k, wdtype):
    s = tiny_shape(T, H, I, E, k, wdtype)
    inp = minp.make_inputs(s, seed=seed)
    d = np_inputs(inp)
    r = run_oracle(O, inp)
    b = brute_force(d["x_bits"], d["wr_bits"], d["w13"], d["w2"], k, d["fp8"],
                    d["w13_scale"], d["w2_scale"])
    assert r["topk_ids"].tolist() == b["ids"]
    assert np.allclose(r["topk_w"], np.array(b["weights"]), rtol=1e-6, atol=0)
    if E == 1:
        assert np.all(r["topk_w"] == 1.0)
    hb = np.array([b["h"][(t, j)] for t in range(T) for j in range(k)], np.float32)
    h_or = r["h"][r["inv_perm"]]                     # back to (t, j) order
    assert np.abs(h_or - hb).max() <= 1e-6 * np.abs(hb).max()
    out_o = bf16_bits_to_float(r["out"])
    out_b = np.array(b["out"])
    # identical up to a one-ulp bf16 flip from fp64 summation order differences
    assert max_rel_err(out_o, out_b) <= 2.0 ** -8
    assert np.mean(out_o == out_b) >= 0.99


def _onehot_case(fp8: bool):
    """Experts whose rows are one-hot, so the layer has a closed form.

    Expert e: W1[n] picks column a_e(n), W3[n] picks column b_e(n), W2[m] picks
    row c_e(m) of h.  Then g_n = x[a(n)], u_n = x[b(n)], h_n = SiLU(g_n) * u_n and
    Y[m] = h[c(m)]: a swapped gate/up half, a transposed W2 or a wrong expert
    index changes the result."""
    T, H, I, E, k = 3, 256, 128, 3, 2
    rng = np.random.default_rng(7)
    x = rng.standard_normal((T, H)).astype(np.float32)
    wr = rng.standard_normal((E, H)).astype(np.float32) / 16
    a = rng.integers(0, H, (E, I))
    b = rng.integers(0, H, (E, I))
    c = rng.integers(0, I, (E, H))
    w13 = np.zeros((E, 2 * I, H), np.float32)
    w2 = np.zeros((E, H, I), np.float32)
    for e in range(E):
        w13[e, np.arange(I), a[e]] = 1.0
        w13[e, I + np.arange(I), b[e]] = 1.0
        w2[e, np.arange(H), c[e]] = 1.0
    xb, wrb = _bits(x), _bits(wr)
    if fp8:
        one = np.uint8(0x38)                           # e4m3 code of 1.0
        q13 = np.where(w13 == 1.0, one, np.uint8(0)).astype(np.uint8)
        q2 = np.where(w2 == 1.0, one, np.uint8(0)).astype(np.uint8)
        s13 = np.array([0.75, 1.5, 0.5], np.float32)
        s2 = np.array([2.0, 0.25, 1.25], np.float32)
        return xb, wrb, q13, q2, s13, s2, a, b, c, k
    return xb, wrb, _bits(w13), _bits(w2), None, None, a, b, c, k


@pytest.mark.parametrize("fp8", [False, True])
def test_onehot_experts_closed_form(fp8):
    xb, wrb, w13, w2, s13, s2, a, b, c, k = _onehot_case(fp8)
    r = O.fused_moe(xb, wrb, w13, w2, k, fp8=fp8, w13_scale=s13, w2_scale=s2)
    xf = bf16_bits_to_float(xb).astype(np.float64)
    T, H = xf.shape
    ids, w = r["topk_ids"], r["topk_w"]
    if fp8:
        amax = np.float32(np.abs(bf16_bits_to_float(xb)).max())
        s1, inv1 = np.float32(amax / np.float32(448)), np.float32(np.float32(448) / amax)
        q = lambda v, inv: torch.from_numpy((np.asarray(v, np.float32) * inv).astype(np.float32)) \
            .to(torch.float8_e4m3fn).to(torch.float64).numpy()
        xa = q(bf16_bits_to_float(xb), inv1)           # dequantised codes, unscaled
    hs = {}
    for t in range(T):
        for j, e in enumerate(ids[t]):
            if fp8:
                sc = float(np.float32(s1 * s13[e]))
                g, u = xa[t, a[e]] * sc, xa[t, b[e]] * sc
            else:
                g, u = xf[t, a[e]], xf[t, b[e]]
            hs[(t, j)] = (g / (1 + np.exp(-g)) * u).astype(np.float32)
    out = np.zeros((T, H))
    if fp8:
        amax2 = np.float32(max(np.abs(v).max() for v in hs.values()))
        s2g, inv2 = np.float32(amax2 / np.float32(448)), np.float32(np.float32(448) / amax2)
    for t in range(T):
        for j, e in enumerate(ids[t]):
            if fp8:
                hq = q(hs[(t, j)], inv2)
                Y = hq[c[e]] * float(np.float32(s2g * s2[e]))
            else:
                hb = torch.from_numpy(hs[(t, j)]).to(torch.bfloat16).to(torch.float64).numpy()
                Y = hb[c[e]]
            out[t] += float(w[t, j]) * Y
    ref = torch.from_numpy(out.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()
    got = bf16_bits_to_float(r["out"])
    assert np.array_equal(got, ref)


def test_silu_zero_gives_zero_output():
    s = tiny_shape(4, 256, 128, 4, 2, "fp8")
    inp = minp.make_inputs(s, seed=5)
    d = np_inputs(inp)
    w13 = d["w13"].copy()
    w13[:, :128, :] = 0                               # gate rows zero -> g = 0 -> h = 0
    r = O.fused_moe(d["x_bits"], d["wr_bits"], w13, d["w2"], 2, fp8=True,
                    w13_scale=d["w13_scale"], w2_scale=d["w2_scale"])
    assert np.all(r["h"] == 0) and np.all(bf16_bits_to_float(r["out"]) == 0)


def test_static_scales_follow_their_definition():
    s = tiny_shape(4, 256, 128, 4, 2, "fp8")
    inp = minp.make_inputs(s, seed=6)
    dyn = run_oracle(O, inp)
    a1 = 0.0123
    st = run_oracle(O, inp, a1_scale=a1, a2_scale=float(dyn["s2"]))
    inv = np.float32(np.float32(1.0) / np.float32(a1))
    xrows = bf16_bits_to_float(minp.bf16_bits(inp.x))[st["sorted_rows"] // 2]
    ref = torch.from_numpy(np.clip(xrows * inv, -448, 448).astype(np.float32)) \
        .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(st["a_perm"], ref)
    assert st["s1"] == np.float32(a1) and st["s2"] == dyn["s2"]


def test_tiny_bf16_regression_golden():
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_bf16_seed0.json")
    doc = json.load(open(path))
    s = minp.shape("tiny_bf16")
    r = run_oracle(O, minp.make_inputs(s, seed=0))
    assert r["topk_ids"].tolist() == doc["topk_ids"]
    assert r["counts"].tolist() == doc["counts"]
    assert r["sorted_rows"].tolist() == doc["sorted_rows"]
    assert r["out"].astype(int).tolist() == doc["out_bf16_bits"]


# ----------------------------------------------------------------------------- grouped routing

def _sig(v):
    return 1.0 / (1.0 + math.exp(-v))


def _onehot_router(table):
    """x = e_t, router_w[:, t] = table[t]: logit[t, e] = table[t][e] exactly."""
    table = np.asarray(table, np.float32)
    T, E = table.shape
    H = 256
    x = np.zeros((T, H), np.float32)
    x[np.arange(T), np.arange(T)] = 1.0
    wr = np.zeros((E, H), np.float32)
    wr[:, :T] = table.T
    return _bits(x), _bits(wr)


def test_grouped_routing_closed_form():
    # 8 experts in 4 groups of 2, keep 2 groups, pick 2 experts.
    # token 0: expert 7 has the largest score but its group {6, 7} scores s(-1)+s(5)
    # = 1.262, below {0, 1}: s(4)+s(3) = 1.935 and {4, 5}: 2 s(2) = 1.762, so the
    # choice is experts 0 then 1.  token 1: all equal -> groups 0, 1 -> experts 0, 1.
    table = [[4, 3, 0, 0, 2, 2, -1, 5],
             [1, 1, 1, 1, 1, 1, 1, 1]]
    xb, wb = _onehot_router(table)
    ids, w, s, sb = O.router_grouped(xb, wb, 2, n_group=4, topk_group=2, routed_scaling=2.5)
    assert ids.tolist() == [[0, 1], [0, 1]]
    ref0 = [_sig(4) / (_sig(4) + _sig(3)) * 2.5, _sig(3) / (_sig(4) + _sig(3)) * 2.5]
    assert np.allclose(w[0], ref0, rtol=1e-6, atol=0)
    assert np.allclose(w[1], [1.25, 1.25], rtol=1e-7, atol=0)
    # a bias of +1 on expert 7 lifts group {6, 7} to s(-1) + s(5) + 1 = 2.262: the kept
    # groups become {6, 7} and {0, 1}; by biased score expert 7 then expert 0, and the
    # weights use the unbiased scores
    bias = np.zeros(8, np.float32)
    bias[7] = 1.0
    ids, w, _, sb = O.router_grouped(xb, wb, 2, n_group=4, topk_group=2, bias=bias)
    assert ids[0].tolist() == [7, 0]
    assert np.allclose(w[0], [_sig(5) / (_sig(5) + _sig(4)), _sig(4) / (_sig(5) + _sig(4))],
                       rtol=1e-6, atol=0)
    assert sb[0, 7] == np.float32(np.float32(_sig(5)) + np.float32(1.0))


def test_grouped_sigmoid_is_fp64_rounded_once():
    l = np.array([[-3.5, 0.0, 0.1234567, 7.25, -20.0, 40.0]], np.float32)
    got = O.sigmoid_scores(l)
    ref = np.array([[_sig(float(v)) for v in l[0]]], np.float64).astype(np.float32)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("seed,T,E,G,M,k", [(0, 12, 16, 4, 2, 4), (1, 9, 32, 8, 3, 6),
                                            (2, 5, 64, 8, 4, 8)])
def test_grouped_routing_matches_bruteforce(seed, T, E, G, M, k):
    s_ = tiny_shape(T, 256, 128, E, k, "fp8", router_std=0.5)
    x, wr = minp.make_activations(s_, seed=seed)
    xb, wb = minp.bf16_bits(x), minp.bf16_bits(wr)
    rng = np.random.default_rng(seed)
    bias = (rng.standard_normal(E) * 0.05).astype(np.float32)
    ids, w, s, sb = O.router_grouped(xb, wb, k, n_group=G, topk_group=M, bias=bias,
                                     routed_scaling=2.5)
    # the brute force starts from the same fp32 logits (pinned by the canonical-order
    # tests) and redoes the sigmoid, grouping, selection and weights on its own
    logits = O.router_logits(xb, wb)
    bids, bw = brute_grouped(logits, k, G, M, bias, 2.5)
    assert ids.tolist() == bids
    assert np.allclose(w, np.array(bw), rtol=1e-6, atol=0)
    eg = E // G
    for t in range(T):
        assert np.isclose(float(w[t].astype(np.float64).sum()), 2.5, rtol=1e-6)
        assert len(set(ids[t].tolist())) == k
        groups = sb[t].reshape(G, eg)
        gscore = np.sort(groups, axis=1)[:, -1] + np.sort(groups, axis=1)[:, -2]
        kept = set(sorted(range(G), key=lambda g: (-gscore[g], g))[:M])
        assert {int(e) // eg for e in ids[t]} <= kept


# ----------------------------------------------------------------------------- shared experts

@pytest.mark.parametrize("seed,T,H,I,E,k,ns,wdtype", [
    (6, 3, 256, 256, 4, 2, 1, "fp8"),
    (7, 2, 256, 128, 4, 1, 2, "bf16"),
    (8, 3, 256, 256, 1, 1, 1, "fp8"),   # one routed expert (weight 1) plus one shared
])
def test_shared_experts_match_bruteforce(seed, T, H, I, E, k, ns, wdtype):
    s = tiny_shape(T, H, I, E, k, wdtype, n_shared=ns)
    inp = minp.make_inputs(s, seed=seed)
    d = np_inputs(inp)
    r = run_oracle(O, inp)
    b = brute_force(d["x_bits"], d["wr_bits"], d["w13"], d["w2"], k, d["fp8"],
                    d["w13_scale"], d["w2_scale"], n_shared=ns)
    assert r["topk_ids"].tolist() == b["ids"]
    assert np.allclose(r["topk_w"], np.array(b["weights"]), rtol=1e-6, atol=0)
    assert np.array_equal(r["counts"][E:], np.full(ns, T))          # every token, once each
    hb = np.array([b["h"][(t, j)] for t in range(T) for j in range(k + ns)], np.float32)
    h_or = r["h"][r["inv_perm"]]
    assert np.abs(h_or - hb).max() <= 1e-6 * np.abs(hb).max()
    out_o = bf16_bits_to_float(r["out"])
    assert max_rel_err(out_o, np.array(b["out"])) <= 2.0 ** -8


def test_shared_slots_follow_the_routed_ones_with_weight_one():
    # grouped routing with routed_scaling 2.5: routed weights sum to 2.5, the shared
    # slots keep weight exactly 1 and come last, in expert order
    s = tiny_shape(6, 256, 128, 16, 3, "fp8", router_std=1.0, grouped=(4, 2, 2.5), n_shared=2)
    inp = minp.make_inputs(s, seed=3)
    r = run_oracle(O, inp)
    ids, w = r["topk_ids"], r["topk_w"]
    assert ids.shape == (6, 5) and w.shape == (6, 5)
    assert np.all(ids[:, 3:] == np.array([16, 17])) and np.all(ids[:, :3] < 16)
    assert np.all(w[:, 3:] == np.float32(1.0))
    assert np.allclose(w[:, :3].sum(axis=1), 2.5, rtol=1e-6)
    assert np.all(r["counts"][16:] == 6)


def test_shared_expert_adds_a_dense_gated_mlp():
    """bf16 format (no per-tensor scale couples the rows): the layer's unrounded output
    with the shared expert minus the output without it is the shared expert's dense
    gated MLP of every token, computed here with torch in float64."""
    T, H, I, E, k = 5, 256, 128, 6, 2
    s1 = tiny_shape(T, H, I, E, k, "bf16", n_shared=1)
    inp = minp.make_inputs(s1, seed=9)
    d = np_inputs(inp)
    with_s = run_oracle(O, inp)
    without = O.fused_moe(d["x_bits"], d["wr_bits"], d["w13"][:E], d["w2"][:E], k, fp8=False)
    assert np.array_equal(with_s["topk_ids"][:, :k], without["topk_ids"])
    diff = with_s["out64"] - without["out64"]
    x = torch.from_numpy(bf16_bits_to_float(d["x_bits"]).astype(np.float64))
    w13 = torch.from_numpy(bf16_bits_to_float(d["w13"][E]).astype(np.float64))
    w2 = torch.from_numpy(bf16_bits_to_float(d["w2"][E]).astype(np.float64))
    gu = x @ w13.T
    h = (torch.nn.functional.silu(gu[:, :I]) * gu[:, I:]).to(torch.float32)
    h = h.to(torch.bfloat16).to(torch.float64)                      # R7: h rounded to bf16
    y = (h @ w2.T).numpy()
    assert np.abs(diff - y).max() <= 1e-9 * np.abs(y).max()


# ----------------------------------------------------------------------------- sharding

def _shard(w13, w2, r, n):
    """Plain numpy slices of shard r of n over the intermediate features (independent of
    the package's torch helper)."""
    I = w2.shape[2]
    m = I // n
    cols = np.arange(r * m, (r + 1) * m)
    return np.concatenate([w13[:, cols], w13[:, I + cols]], axis=1), w2[:, :, cols], cols


@pytest.mark.parametrize("n", [2, 4])
@pytest.mark.parametrize("wdtype", ["fp8", "bf16"])
def test_sharded_expert_networks_reassemble_the_layer(n, wdtype):
    """Splitting the intermediate features over n shards, each given the max |h| of the
    whole layer (amax2), reproduces the unsharded layer: every shard's h and its codes
    are the unsharded columns bit for bit, and the shards' outputs add up to the
    unsharded output (the contraction over I splits into a sum over shards)."""
    T, H, I, E, k = 9, 256, 512, 4, 2
    s = tiny_shape(T, H, I, E, k, wdtype)
    inp = minp.make_inputs(s, seed=21)
    d = np_inputs(inp)
    fp8 = d["fp8"]
    full = run_oracle(O, inp)
    ids, w = full["topk_ids"], full["topk_w"]
    a_perm, s1 = full["a_perm"], full["s1"]
    amax_full = np.float32(np.abs(full["h"]).max())
    y_sum = np.zeros_like(full["y"])
    local_codes_differ = False
    for r in range(n):
        w13_r, w2_r, cols = _shard(d["w13"], d["w2"], r, n)
        y_r, h_r, hq_r, s2_r = O.experts(a_perm, full["offsets"], full["sorted_rows"], w, w13_r,
                                         w2_r, H, I // n, E, fp8, s1, d["w13_scale"],
                                         d["w2_scale"], amax2=amax_full if fp8 else None)
        assert np.array_equal(h_r, full["h"][:, cols])
        assert np.array_equal(hq_r, full["hq"][:, cols])
        assert s2_r == full["s2"]
        y_sum += y_r
        if fp8:   # a shard scaled by its own max would quantise differently
            _, _, hq_own, _ = O.experts(a_perm, full["offsets"], full["sorted_rows"], w, w13_r,
                                        w2_r, H, I // n, E, fp8, s1, d["w13_scale"],
                                        d["w2_scale"])
            local_codes_differ |= not np.array_equal(hq_own, hq_r)
    assert np.abs(y_sum - full["y"]).max() <= 1e-12 * np.abs(full["y"]).max()
    if fp8:
        assert local_codes_differ
    # amax2 equal to the call's own max is the default
    y_a, _, hq_a, _ = O.experts(a_perm, full["offsets"], full["sorted_rows"], w, d["w13"], d["w2"],
                                H, I, E, fp8, s1, d["w13_scale"], d["w2_scale"],
                                amax2=amax_full if fp8 else None)
    assert np.array_equal(hq_a, full["hq"]) and np.array_equal(y_a, full["y"])
