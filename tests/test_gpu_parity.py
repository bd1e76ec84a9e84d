"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same
seeded inputs.

Bars: routing ids, per-expert counts, offsets, the permutation, its inverse, max |x|,
the activation scale and the quantised activation bytes are bit-exact; routing
weights within 1e-6 relative; layer outputs within a normwise max relative error of
2e-2 (FP8 format) or 5e-3 (bf16 format).

Small cases span several tiles and ragged tails in every dimension; the full-size
cases run the five workloads at their real shapes in the launch configuration the
benchmark times (AUTO variant), and both variants are forced on the same inputs.
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

from oracle import fused_moe_oracle as O
from mixture_experts_layer_26_b200 import inputs as minp
from helpers import (run_oracle, max_rel_err, bf16_bits_to_float, tiny_shape, grouped_args,
                     report_errors)

capi = pytest.importorskip("mixture_experts_layer_26_b200.capi")

pytestmark = pytest.mark.gpu

TOL = {"fp8": 2e-2, "bf16": 5e-3}


def dev_inputs(inp: minp.MoEInputs):
    d = dict(x=inp.x.cuda(), router_w=inp.router_w.cuda(), w13=inp.w13.cuda(), w2=inp.w2.cuda())
    d["w13_scale"] = inp.w13_scale.cuda() if inp.w13_scale is not None else None
    d["w2_scale"] = inp.w2_scale.cuda() if inp.w2_scale is not None else None
    d["routing"] = routing_of(inp)
    return d


def routing_of(inp):
    s = inp.shape
    if s.grouped is None:
        return capi.make_softmax_routing(s.n_shared) if s.n_shared else None
    n_group, topk_group, scaling = s.grouped
    return capi.make_routing(n_group, topk_group, scaling, inp.router_bias.cuda(),
                             n_shared=s.n_shared)


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run_steps(inp, g, variant="auto", a1=0.0, a2=0.0):
    s = inp.shape
    fp8 = s.wdtype == "fp8"
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, fp8, variant, routing=g.get("routing"))
    ws = capi.alloc_workspace(dims)
    R = s.R
    dev = "cuda"
    ids = torch.empty(R, dtype=torch.int32, device=dev)
    tw = torch.empty(R, dtype=torch.float32, device=dev)
    counts = torch.empty(s.E_all, dtype=torch.int32, device=dev)
    offsets = torch.empty(s.E_all + 1, dtype=torch.int32, device=dev)
    rows = torch.empty(R, dtype=torch.int32, device=dev)
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    a_perm = torch.empty(R, s.H, dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    y = torch.empty(R, s.H, dtype=torch.float32, device=dev)
    out = torch.empty(s.T, s.H, dtype=torch.bfloat16, device=dev)
    sc = capi.make_scales(g["w13_scale"], g["w2_scale"], a1, a2)
    capi.fused_moe_route(dims, g["x"], g["router_w"], ids, tw, ws)
    capi.fused_moe_permute(dims, ids, g["x"], sc, counts, offsets, rows, inv, a_perm, ws)
    capi.fused_moe_experts(dims, a_perm, offsets, rows, tw, g["w13"], g["w2"], sc, y, ws)
    capi.fused_moe_combine(dims, y, inv, out)
    torch.cuda.synchronize()
    assert capi.fused_moe_get_device_status(ws) == capi.FMOE_OK
    fs, ints = capi.fused_moe_debug_scalars(ws)
    K = s.top_k + s.n_shared  # slots per token: routed, then shared
    return dict(topk_ids=ids.cpu().numpy().reshape(s.T, K),
                topk_w=tw.cpu().numpy().reshape(s.T, K),
                counts=counts.cpu().numpy(), offsets=offsets.cpu().numpy(),
                sorted_rows=rows.cpu().numpy(), inv_perm=inv.cpu().numpy(),
                a_perm=a_perm.cpu().numpy() if fp8 else bits16(a_perm),
                y=y.cpu().numpy(), out=bits16(out), scalars=fs, plan=ints)


def run_fused(inp, g, variant="auto", a1=0.0, a2=0.0):
    s = inp.shape
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, s.wdtype == "fp8", variant,
                          routing=g.get("routing"))
    ws = capi.alloc_workspace(dims)
    out = torch.empty(s.T, s.H, dtype=torch.bfloat16, device="cuda")
    sc = capi.make_scales(g["w13_scale"], g["w2_scale"], a1, a2)
    capi.fused_moe(dims, g["x"], g["router_w"], g["w13"], g["w2"], sc, out, ws)
    torch.cuda.synchronize()
    assert capi.fused_moe_get_device_status(ws) == capi.FMOE_OK
    return bits16(out), capi.fused_moe_debug_scalars(ws)


def check_routing(gpu, ref):
    assert np.array_equal(gpu["topk_ids"], ref["topk_ids"])
    assert np.allclose(gpu["topk_w"], ref["topk_w"], rtol=1e-6, atol=1e-9)
    assert np.array_equal(gpu["counts"], ref["counts"])
    assert np.array_equal(gpu["offsets"], ref["offsets"])
    assert np.array_equal(gpu["sorted_rows"], ref["sorted_rows"])
    assert np.array_equal(gpu["inv_perm"], ref["inv_perm"])
    assert np.float32(gpu["scalars"]["amax_x"]) == ref["amax_x"]


def check_layer(gpu, ref, wdtype):
    """Normwise max relative error against the oracle's result before its final bf16
    rounding (two independently bf16-rounded outputs may differ by a whole bf16 ulp,
    up to 2^-7 of the max, more than the bf16 bound itself)."""
    tol = TOL[wdtype]
    err_y = max_rel_err(gpu["y"], ref["y"])
    err = max_rel_err(bf16_bits_to_float(gpu["out"]), ref["out64"])
    report_errors(os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0],
                  bf16_bits_to_float(gpu["out"]), ref["out64"])
    assert err_y <= tol, err_y
    assert err <= tol, err
    return err


# ------------------------------------------------------------------ small cases

SMALL = [
    # id, (T, H, I, E, k, wdtype), extra shape kwargs
    ("tiny_bf16", (4, 256, 512, 8, 2, "bf16"), {}),
    ("fp8_ragged", (37, 512, 384, 8, 2, "fp8"), {}),
    ("fp8_many_experts", (100, 768, 256, 32, 4, "fp8"), {}),
    ("fp8_multichunk", (300, 256, 256, 4, 2, "fp8"), {}),
    ("bf16_multichunk", (300, 256, 384, 4, 2, "bf16"), {}),
    ("fp8_single_token", (1, 512, 256, 8, 2, "fp8"), {}),
    ("fp8_empty_experts", (3, 256, 128, 64, 2, "fp8"), {}),
    ("fp8_k_equals_E", (5, 256, 256, 4, 4, "fp8"), {}),
    ("fp8_single_expert", (9, 256, 256, 1, 1, "fp8"), {}),
    ("fp8_adversarial", (40, 512, 256, 16, 2, "fp8"), {"adversarial": True}),
    ("fp8_dsv3_gate", (64, 512, 256, 64, 8, "fp8"), {"router_std": 1.0}),
    ("fp8_grouped", (64, 512, 256, 64, 8, "fp8"), {"router_std": 1.0, "grouped": (8, 4, 2.5)}),
    ("bf16_grouped_small_groups", (24, 256, 256, 32, 4, "bf16"), {"grouped": (16, 3, 1.0)}),
    # more than 256 rows per expert: several CTA-pair chunks with ragged tails
    ("fp8_pair_chunks", (700, 512, 384, 2, 1, "fp8"), {}),
    ("bf16_pair_chunks", (600, 256, 256, 3, 2, "bf16"), {}),
    # shared experts (every token, weight 1, after the routed slots)
    ("fp8_shared", (37, 512, 384, 8, 2, "fp8"), {"n_shared": 1}),
    ("bf16_shared_two", (21, 256, 256, 6, 2, "bf16"), {"n_shared": 2}),
    ("fp8_grouped_shared", (64, 512, 256, 64, 8, "fp8"),
     {"router_std": 1.0, "grouped": (8, 4, 2.5), "n_shared": 1}),
    ("fp8_shared_pair_chunks", (300, 256, 256, 4, 2, "fp8"), {"n_shared": 1}),
    # E >= 128: four experts per router warp, experts split over CTAs (last-CTA hand-off),
    # a last expert group that is not full, grouped routing with a shared expert
    ("fp8_experts_128", (13, 512, 256, 128, 4, "fp8"), {"router_std": 1.0}),
    ("fp8_experts_130", (9, 1024, 128, 130, 3, "fp8"), {}),
    ("bf16_grouped_shared_160", (20, 1024, 256, 160, 6, "bf16"),
     {"grouped": (8, 3, 1.5), "n_shared": 1}),
    # the tiled router (many token x expert tiles): 32-token tiles over <= 8 experts with a
    # ragged last tile and expert rows past E; 16-token tiles over groups of 32 experts
    # handed to each tile's last CTA, a ragged last expert group; grouped routing
    ("fp8_router_tiled_e6", (3999, 512, 128, 6, 2, "fp8"), {}),
    ("bf16_router_tiled_e130", (1000, 512, 128, 130, 3, "bf16"), {}),
    ("fp8_router_tiled_grouped", (1600, 512, 128, 64, 6, "fp8"),
     {"router_std": 1.0, "grouped": (8, 3, 2.5), "n_shared": 1}),
    # more than 32 slots per token: the swap-AB output is combined by its own launch
    ("fp8_many_slots", (6, 256, 128, 40, 34, "fp8"), {}),
]


@pytest.fixture(scope="module")
def small_cases():
    cache = {}

    def get(name):
        if name not in cache:
            _, (T, H, I, E, k, wd), kw = next(c for c in SMALL if c[0] == name)
            inp = minp.make_inputs(tiny_shape(T, H, I, E, k, wd, **kw), seed=11)
            cache[name] = (inp, dev_inputs(inp), run_oracle(O, inp))
        return cache[name]
    return get


@pytest.mark.parametrize("variant", ["swap_ab", "normal", "normal_pair"])
@pytest.mark.parametrize("name", [c[0] for c in SMALL])
def test_small_steps_match_oracle(small_cases, name, variant):
    inp, g, ref = small_cases(name)
    gpu = run_steps(inp, g, variant)
    check_routing(gpu, ref)
    assert np.array_equal(gpu["a_perm"], ref["a_perm"])            # quantised rows, bit-exact
    if inp.shape.wdtype == "fp8":
        assert np.float32(gpu["scalars"]["s1"]) == ref["s1"]
        assert np.float32(gpu["scalars"]["inv1"]) == ref["inv1"]
        assert abs(gpu["scalars"]["s2"] / ref["s2"] - 1) < 1e-5
    check_layer(gpu, ref, inp.shape.wdtype)
    if name == "fp8_adversarial":
        assert set(ref["topk_ids"][:, 0]) == {0} and set(ref["topk_ids"][:, 1]) == {1}


@pytest.mark.parametrize("name", ["tiny_bf16", "fp8_ragged", "fp8_multichunk"])
def test_small_fused_equals_steps_and_variants_agree(small_cases, name):
    inp, g, ref = small_cases(name)
    tol = TOL[inp.shape.wdtype]
    out_a, _ = run_fused(inp, g, "auto")
    out_s, _ = run_fused(inp, g, "swap_ab")
    out_n, _ = run_fused(inp, g, "normal")
    steps = run_steps(inp, g, "auto")
    assert np.array_equal(out_a, steps["out"])                     # same kernels, same order
    fa, fs, fn = (bf16_bits_to_float(o) for o in (out_a, out_s, out_n))
    # swap-AB == normal (transposed product): each variant is held to tol against the oracle
    # (test_small_steps_match_oracle), so by the triangle inequality they differ by at most
    # 2 * tol in the same normwise measure
    assert max_rel_err(fs, fn) <= 2 * tol
    assert max_rel_err(fa, ref["out64"]) <= tol
    # deterministic: a second call gives the same bits
    out_a2, _ = run_fused(inp, g, "auto")
    assert np.array_equal(out_a, out_a2)


@pytest.mark.parametrize("name", ["tiny_bf16", "fp8_ragged", "fp8_multichunk", "fp8_pair_chunks",
                                  "bf16_pair_chunks", "fp8_many_experts", "fp8_shared_pair_chunks"])
def test_pair_variant_equals_normal(small_cases, name):
    """The CTA-pair kernel runs the normal variant's tiles with the same K order and the
    same epilogue arithmetic: identical output bits."""
    inp, g, _ = small_cases(name)
    out_n, _ = run_fused(inp, g, "normal")
    out_p, _ = run_fused(inp, g, "normal_pair")
    assert np.array_equal(out_n, out_p)


@pytest.mark.parametrize("name", ["fp8_ragged", "fp8_shared", "bf16_grouped_shared_160"])
def test_tensor_level_call_equals_dims_call(small_cases, name):
    """capi.moe (dims from the tensor shapes, its own workspace) gives the same bits as
    fused_moe with explicit dims."""
    inp, g, ref = small_cases(name)
    out_d, _ = run_fused(inp, g, "auto")
    out_t = capi.moe(g["x"], g["router_w"], g["w13"], g["w2"], inp.shape.top_k,
                     g["w13_scale"], g["w2_scale"], routing=g.get("routing"))
    torch.cuda.synchronize()
    assert np.array_equal(bits16(out_t), out_d)


@pytest.mark.parametrize("variant", ["auto", "normal_pair"])
def test_static_scales(small_cases, variant):
    inp, g, _ = small_cases("fp8_ragged")
    ref = run_oracle(O, inp, a1_scale=0.02, a2_scale=0.003)
    gpu = run_steps(inp, g, variant, a1=0.02, a2=0.003)
    check_routing(gpu, ref)
    assert np.array_equal(gpu["a_perm"], ref["a_perm"])
    assert gpu["scalars"]["s1"] == np.float32(0.02) and gpu["scalars"]["s2"] == np.float32(0.003)
    check_layer(gpu, ref, "fp8")


@pytest.mark.parametrize("name,launches", [
    # T=1: router (+ permutation, plan, gather), the split-K first contraction, its finish,
    # the quantisation of h, the second contraction, the finish + combine of its partials
    ("fp8_single_token", ["router_permute_gather", "gemm1_swapab", "finalize1", "quant_h",
                          "gemm2_swapab", "combine_partials"]),
    ("fp8_ragged", ["router_permute_gather", "gemm1_swapab", "finalize1", "quant_h",
                    "gemm2_swapab", "combine_partials"]),
    # 34 slots per token
    ("fp8_many_slots", ["router_permute_gather", "gemm1_swapab", "finalize1", "quant_h",
                        "gemm2_swapab", "combine_partials"]),
    ("bf16_shared_two", ["router_permute_gather", "gemm1_swapab", "finalize1", "gemm2_swapab",
                         "combine_partials"]),
    ("fp8_grouped_shared", None),
])
def test_swap_repeat_and_reinit(small_cases, name, launches):
    """Repeated swap-AB calls on one workspace, with its header re-initialised in between
    or not, give identical bits, within tolerance of the oracle and equal to the
    step-by-step path (separate finish and combine); the launch list of a profiled call is
    the documented one and as long as fused_moe_launches_per_call says."""
    inp, g, ref = small_cases(name)
    s = inp.shape
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, s.wdtype == "fp8", "swap_ab",
                          routing=g.get("routing"))
    ws = capi.alloc_workspace(dims)
    sc = capi.make_scales(g["w13_scale"], g["w2_scale"])
    outs = []
    for i in range(4):
        if i == 2:
            capi.fused_moe_workspace_init(ws)
        out = torch.full((s.T, s.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        capi.fused_moe(dims, g["x"], g["router_w"], g["w13"], g["w2"], sc, out, ws)
        torch.cuda.synchronize()
        assert capi.fused_moe_get_device_status(ws) == capi.FMOE_OK
        outs.append(bits16(out))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    assert max_rel_err(bf16_bits_to_float(outs[0]), ref["out64"]) <= TOL[s.wdtype]
    steps = run_steps(inp, g, "swap_ab")
    assert np.array_equal(outs[0], steps["out"])
    if launches is not None:
        out = torch.empty(s.T, s.H, dtype=torch.bfloat16, device="cuda")
        got = [n for n, _ in capi.fused_moe_profile(dims, g["x"], g["router_w"], g["w13"],
                                                    g["w2"], sc, out, ws)]
        assert got == launches
        assert len(got) == capi.fused_moe_launches_per_call(dims)
        torch.cuda.synchronize()
        assert np.array_equal(bits16(out), outs[0])


def test_host_io_matches_device_call(small_cases):
    inp, g, ref = small_cases("fp8_ragged")
    s = inp.shape
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, True)
    ws = capi.alloc_workspace(dims)
    x_host = inp.x.clone().pin_memory()
    out_host = torch.empty(s.T, s.H, dtype=torch.bfloat16).pin_memory()
    sc = capi.make_scales(g["w13_scale"], g["w2_scale"])
    capi.fused_moe_host_io(dims, x_host, g["router_w"], g["w13"], g["w2"], sc, out_host, ws)
    out_dev, _ = run_fused(inp, g, "auto")
    assert np.array_equal(out_host.view(torch.int16).numpy().view(np.uint16), out_dev)


def test_out_of_range_expert_ids_are_reported(small_cases):
    inp, g, _ = small_cases("fp8_ragged")
    s = inp.shape
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, True)
    ws = capi.alloc_workspace(dims)
    ids = torch.zeros(s.R, dtype=torch.int32, device="cuda")
    ids[5] = s.E + 3                                               # invalid id
    R = s.R
    bufs = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (s.E, s.E + 1, R, R)]
    a_perm = torch.empty(R, s.H, dtype=torch.uint8, device="cuda")
    capi.fused_moe_permute(dims, ids, g["x"], None, *bufs, a_perm, ws)
    torch.cuda.synchronize()
    assert capi.fused_moe_get_device_status(ws) == capi.FMOE_ERR_DEVICE_BOUNDS
    capi.fused_moe_workspace_init(ws)
    assert capi.fused_moe_get_device_status(ws) == capi.FMOE_OK


# ------------------------------------------------------------------ full-size workloads

FULL = [("mixtral_fp8_decode", T) for T in (1, 8, 32, 64)] + \
       [("dsv3_fp8_decode", T) for T in (16, 64, 256)] + \
       [("swapab_stress_fp8", 8), ("swapab_adversarial_fp8", 8), ("prefill_fp8", 4096)] + \
       [("mixtral_bf16_decode", T) for T in (1, 8, 64)] + [("prefill_bf16", 4096)] + \
       [("dsv3_grouped_fp8_decode", T) for T in (16, 64, 256)]


@pytest.fixture(scope="module")
def full_weights():
    """Weights of the most recent workload (one set on the device at a time)."""
    state = {}

    def get(workload):
        if state.get("name") != workload:
            state.clear()
            torch.cuda.empty_cache()
            s = minp.shape(workload)
            w13, w2, s13, s2 = minp.make_weights(s, seed=0)
            state.update(name=workload, host=(w13, w2, s13, s2),
                         dev=dict(w13=w13.cuda(), w2=w2.cuda(),
                                  w13_scale=None if s13 is None else s13.cuda(),
                                  w2_scale=None if s2 is None else s2.cuda()))
        return state
    return get


@pytest.mark.parametrize("workload,T", FULL, ids=[f"{w}-T{t}" for w, t in FULL])
def test_full_size_matches_oracle(full_weights, workload, T):
    st = full_weights(workload)
    s = minp.shape(workload, T)
    x, wr = minp.make_activations(s, seed=0)
    w13, w2, s13, s2 = st["host"]
    inp = minp.MoEInputs(s, x, wr, w13, w2, s13, s2, minp.make_router_bias(s, seed=0))
    g = dict(st["dev"], x=x.cuda(), router_w=wr.cuda(), routing=routing_of(inp))
    ref = run_oracle(O, inp)
    gpu = run_steps(inp, g, "auto")
    check_routing(gpu, ref)
    assert np.array_equal(gpu["a_perm"], ref["a_perm"])
    check_layer(gpu, ref, s.wdtype)
    out_f, _ = run_fused(inp, g, "auto")
    assert np.array_equal(out_f, gpu["out"])
    if workload == "swapab_adversarial_fp8":
        assert ref["counts"][0] == T and ref["counts"][1] == T
    if T <= 64:
        # the other variant on the same inputs
        other = "normal" if (s.R + s.E - 1) // s.E <= 64 else "swap_ab"
        out_o, _ = run_fused(inp, g, other)
        assert max_rel_err(bf16_bits_to_float(out_o), ref["out64"]) <= TOL[s.wdtype]
    if workload.startswith("prefill"):
        # AUTO runs the CTA-pair kernel here; the one-CTA normal kernel gives the same bits
        out_n, _ = run_fused(inp, g, "normal")
        assert np.array_equal(out_n, out_f)


ROUTER_SHAPES = [("mixtral_fp8_decode", T) for T in (1, 64)] + \
                [("dsv3_fp8_decode", T) for T in (16, 256)] + \
                [("dsv3_grouped_fp8_decode", T) for T in (16, 256)] + \
                [("swapab_adversarial_fp8", 8), ("prefill_fp8", 4096)]


@pytest.mark.parametrize("workload,T", ROUTER_SHAPES, ids=[f"{w}-T{t}" for w, t in ROUTER_SHAPES])
def test_router_full_shapes(workload, T):
    """Routing and permutation alone at each workload's real (T, H, E, k), in the launch
    configuration of the full layer: bit-exact ids, counts and permutation."""
    s = minp.shape(workload, T)
    x, wr = minp.make_activations(s, seed=0)
    routing = None
    if s.grouped is None:
        ids_ref, w_ref, _ = O.router(minp.bf16_bits(x), minp.bf16_bits(wr), s.top_k)
        if s.n_shared:
            routing = capi.make_softmax_routing(s.n_shared)
    else:
        bias = minp.make_router_bias(s, seed=0)
        ids_ref, w_ref, _, _ = O.router_grouped(
            minp.bf16_bits(x), minp.bf16_bits(wr), s.top_k, n_group=s.grouped[0],
            topk_group=s.grouped[1], routed_scaling=s.grouped[2], bias=bias.numpy())
        routing = capi.make_routing(*s.grouped, bias.cuda(), n_shared=s.n_shared)
    ids_ref, w_ref = O.append_shared(ids_ref, w_ref, s.E, s.n_shared)
    counts_ref, offs_ref, rows_ref, inv_ref = O.permute(ids_ref, s.E_all)
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, True, routing=routing)
    ws = capi.alloc_workspace(dims)
    R = s.R
    K = s.top_k + s.n_shared
    ids = torch.empty(R, dtype=torch.int32, device="cuda")
    tw = torch.empty(R, dtype=torch.float32, device="cuda")
    bufs = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (s.E_all, s.E_all + 1, R, R)]
    a_perm = torch.empty(R, s.H, dtype=torch.uint8, device="cuda")
    xd = x.cuda()
    for _ in range(2):  # the second call starts from the counters the first one left
        capi.fused_moe_route(dims, xd, wr.cuda(), ids, tw, ws)
        capi.fused_moe_permute(dims, ids, xd, None, *bufs, a_perm, ws)
        torch.cuda.synchronize()
        assert capi.fused_moe_get_device_status(ws) == capi.FMOE_OK
        assert np.array_equal(ids.cpu().numpy().reshape(s.T, K), ids_ref)
        assert np.allclose(tw.cpu().numpy().reshape(s.T, K), w_ref, rtol=1e-6, atol=1e-9)
        for got, ref in zip(bufs, (counts_ref, offs_ref, rows_ref, inv_ref)):
            assert np.array_equal(got.cpu().numpy(), ref)


TIE_CASES = [
    # (T, H, E, k, grouped): the per-warp router with one, two and four experts per warp
    # (E = 256: experts split over CTAs, handed to each token's last CTA), the tiled router
    # with 32-token x 8-expert tiles and with expert groups handed to the tile's last CTA,
    # and grouped sigmoid routing
    (4, 512, 8, 2, None),
    (37, 512, 64, 6, None),
    (20, 1024, 256, 8, None),
    (3000, 512, 8, 2, None),
    (300, 512, 256, 8, None),
    (64, 512, 64, 8, (8, 4, 2.5)),
]


@pytest.mark.parametrize("T,H,E,k,grouped", TIE_CASES)
def test_router_ties_go_to_the_lower_expert(T, H, E, k, grouped):
    """Exact ties in the selection: the upper half of the router rows repeats the lower half
    (equal logits), two rows are zero (logit 0) and token 0 is zero (every logit 0, of either
    sign): the chosen experts, in choice order, are the oracle's, which breaks every tie
    towards the lower expert index, and the weights match."""
    gen = torch.Generator().manual_seed(5)
    x = torch.randn(T, H, generator=gen).to(torch.bfloat16)
    x[0] = 0
    wr = (torch.randn(E, H, generator=gen) / H ** 0.5).to(torch.bfloat16)
    half = E // 2
    wr[half:2 * half] = wr[:half]
    wr[1] = 0
    wr[half + 3] = 0
    xb, wb = minp.bf16_bits(x), minp.bf16_bits(wr)
    routing = None
    if grouped is None:
        ids_ref, w_ref, _ = O.router(xb, wb, k)
    else:
        ids_ref, w_ref, _, _ = O.router_grouped(xb, wb, k, n_group=grouped[0],
                                                topk_group=grouped[1], routed_scaling=grouped[2])
        routing = capi.make_routing(*grouped)
    dims = capi.make_dims(T, H, 256, E, k, True, routing=routing)
    ws = capi.alloc_workspace(dims)
    ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
    tw = torch.empty(T * k, dtype=torch.float32, device="cuda")
    capi.fused_moe_route(dims, x.cuda(), wr.cuda(), ids, tw, ws)
    torch.cuda.synchronize()
    assert capi.fused_moe_get_device_status(ws) == capi.FMOE_OK
    assert np.array_equal(ids.cpu().numpy().reshape(T, k), ids_ref)
    assert np.allclose(tw.cpu().numpy().reshape(T, k), w_ref, rtol=1e-6, atol=1e-9)
    # the ties are real: some token chose both copies of a duplicated router row
    got = ids.cpu().numpy().reshape(T, k)
    assert any(len(set(r) & {e + half for e in r if e < half}) > 0 for r in got)


@pytest.mark.parametrize("name,variant", [("fp8_ragged", "swap_ab"), ("fp8_multichunk", "normal"),
                                          ("bf16_multichunk", "swap_ab"),
                                          ("fp8_pair_chunks", "normal_pair"),
                                          ("bf16_pair_chunks", "normal_pair"),
                                          ("fp8_grouped_shared", "swap_ab")])
def test_poisoned_workspace_and_outputs_are_fully_rewritten(small_cases, name, variant):
    """Workspace (apart from its initialised header) and every output start as NaN
    bytes: a kernel that read a region it had not written, or left an output element
    unwritten, would show up as a NaN or a parity failure."""
    inp, g, ref = small_cases(name)
    s = inp.shape
    fp8 = s.wdtype == "fp8"
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, fp8, variant, routing=g.get("routing"))
    ws = capi.alloc_workspace(dims)
    ws.fill_(0xFF)
    capi.fused_moe_workspace_init(ws)
    out = torch.full((s.T, s.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    sc = capi.make_scales(g["w13_scale"], g["w2_scale"])
    capi.fused_moe(dims, g["x"], g["router_w"], g["w13"], g["w2"], sc, out, ws)
    torch.cuda.synchronize()
    assert capi.fused_moe_get_device_status(ws) == capi.FMOE_OK
    assert not torch.isnan(out.float()).any()
    assert max_rel_err(out.float().cpu().numpy(), ref["out64"]) <= TOL[s.wdtype]


def test_bounded_wait_runs_out_and_context_survives(small_cases):
    """The bounded mbarrier wait every kernel uses gives up after its budget, records
    FMOE_ERR_TIMEOUT and returns; the same context then runs the layer normally."""
    inp, g, ref = small_cases("fp8_ragged")
    s = inp.shape
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, True)
    ws = capi.alloc_workspace(dims)
    capi.fused_moe_selftest_wait(ws, 10_000_000)        # 10 ms
    assert capi.fused_moe_get_device_status(ws) == capi.FMOE_ERR_TIMEOUT
    capi.fused_moe_workspace_init(ws)
    out, _ = run_fused(inp, g, "auto")
    assert max_rel_err(bf16_bits_to_float(out), ref["out64"]) <= TOL["fp8"]
