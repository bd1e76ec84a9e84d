"""Tensor parallelism over the intermediate features on one GPU: the N shards of a
layer run one after another through the C ABI (fused_moe_tp_begin for every shard, the
max of their max |h| words, fused_moe_tp_end for every shard, the sum of their fp32
partial outputs, fused_moe_tp_finish), which is what N ranks do with the two
all-reduces in between.  The result is checked against the oracle of the unsharded layer
at the parity tolerances (2e-2 FP8, 5e-3 bf16); the layer-wide max |h| must equal the
unsharded call's; and with one shard the five steps must give fused_moe's bits."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import fused_moe_oracle as O
from mixture_experts_layer_26_b200 import inputs as minp
from helpers import run_oracle, max_rel_err, bf16_bits_to_float, tiny_shape, report_errors

capi = pytest.importorskip("mixture_experts_layer_26_b200.capi")
from mixture_experts_layer_26_b200 import tp  # noqa: E402

pytestmark = pytest.mark.gpu

TOL = {"fp8": 2e-2, "bf16": 5e-3}


def _dev(inp):
    s = inp.shape
    routing = None
    if s.grouped is not None:
        routing = capi.make_routing(*s.grouped, inp.router_bias.cuda(), n_shared=s.n_shared)
    elif s.n_shared:
        routing = capi.make_softmax_routing(s.n_shared)
    return dict(x=inp.x.cuda(), wr=inp.router_w.cuda(), w13=inp.w13.cuda(), w2=inp.w2.cuda(),
                s13=None if inp.w13_scale is None else inp.w13_scale.cuda(),
                s2=None if inp.w2_scale is None else inp.w2_scale.cuda(), routing=routing)


def run_tp(inp, g, n, variant="auto"):
    """The N shards of one layer call in sequence on this GPU; returns (out bits, the
    layer-wide max |h|, the per-shard maxima)."""
    s = inp.shape
    fp8 = s.wdtype == "fp8"
    dims = capi.make_dims(s.T, s.H, s.I // n, s.E, s.top_k, fp8, variant, routing=g["routing"])
    sc = capi.make_scales(g["s13"], g["s2"])
    shards = [tp.shard_weights(g["w13"], g["w2"], r, n) for r in range(n)]
    ws = [capi.alloc_workspace(dims) for _ in range(n)]
    amax = torch.full((n,), -1.0, dtype=torch.float32, device="cuda")
    parts = torch.empty(n, s.T, s.H, dtype=torch.float32, device="cuda")
    for r in range(n):
        capi.fused_moe_tp_begin(dims, g["x"], g["wr"], shards[r][0], sc, amax[r:r + 1], ws[r])
    local = amax.clone()
    amax.copy_(amax.max().expand(n))              # what the all-reduce MAX leaves on every rank
    for r in range(n):
        capi.fused_moe_tp_end(dims, shards[r][1], sc, amax[r:r + 1], parts[r], ws[r])
    total = parts[0].clone()
    for r in range(1, n):                          # what the all-reduce SUM leaves
        total += parts[r]
    out = torch.empty(s.T, s.H, dtype=torch.bfloat16, device="cuda")
    capi.fused_moe_tp_finish(total, out)
    torch.cuda.synchronize()
    for w in ws:
        assert capi.fused_moe_get_device_status(w) == capi.FMOE_OK
    bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    return bits, float(amax[0].item()), local.cpu().numpy()


def run_unsharded(inp, g, variant="auto"):
    s = inp.shape
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, s.wdtype == "fp8", variant,
                          routing=g["routing"])
    ws = capi.alloc_workspace(dims)
    out = torch.empty(s.T, s.H, dtype=torch.bfloat16, device="cuda")
    capi.fused_moe(dims, g["x"], g["wr"], g["w13"], g["w2"], capi.make_scales(g["s13"], g["s2"]),
                   out, ws)
    torch.cuda.synchronize()
    fs, _ = capi.fused_moe_debug_scalars(ws)
    return out.view(torch.int16).cpu().numpy().view(np.uint16), fs["amax_h"]


SMALL = [
    # id, (T, H, I, E, k, wdtype), extra shape kwargs, shard counts
    ("fp8", (37, 512, 1024, 8, 2, "fp8"), {}, (2, 4, 8)),
    ("bf16", (21, 256, 512, 6, 2, "bf16"), {}, (2, 4)),
    ("fp8_pair_chunks", (700, 512, 512, 2, 1, "fp8"), {}, (2, 4)),
    ("fp8_grouped_shared", (64, 512, 512, 64, 8, "fp8"),
     {"router_std": 1.0, "grouped": (8, 4, 2.5), "n_shared": 1}, (2,)),
]
CASES = [(name, shape, kw, n, variant) for name, shape, kw, ns in SMALL for n in ns
         for variant in ("auto", "swap_ab", "normal", "normal_pair")
         if variant == "auto" or n == ns[0]]


@pytest.fixture(scope="module")
def small():
    cache = {}

    def get(name):
        if name not in cache:
            _, (T, H, I, E, k, wd), kw, _ = next(c for c in SMALL if c[0] == name)
            inp = minp.make_inputs(tiny_shape(T, H, I, E, k, wd, **kw), seed=13)
            cache[name] = (inp, _dev(inp), run_oracle(O, inp))
        return cache[name]
    return get


@pytest.mark.parametrize("name,shape,kw,n,variant", CASES,
                         ids=[f"{c[0]}-N{c[3]}-{c[4]}" for c in CASES])
def test_shards_match_the_unsharded_oracle(small, name, shape, kw, n, variant):
    inp, g, ref = small(name)
    wd = inp.shape.wdtype
    bits, gmax, local = run_tp(inp, g, n, variant)
    err = max_rel_err(bf16_bits_to_float(bits), ref["out64"])
    report_errors(f"tp {name} N={n} {variant}", bf16_bits_to_float(bits), ref["out64"])
    assert err <= TOL[wd], err
    if wd == "fp8":
        _, amax_unsharded = run_unsharded(inp, g, variant)
        assert gmax == float(local.max())
        assert abs(gmax / amax_unsharded - 1) <= 1e-5
        assert abs(gmax / float(np.abs(ref["h"]).max()) - 1) <= 1e-5


@pytest.mark.parametrize("name", ["fp8", "bf16", "fp8_pair_chunks", "fp8_grouped_shared"])
def test_one_shard_is_fused_moe_bit_for_bit(small, name):
    """One shard: begin + end + finish run the one-call layer's kernels and round the same
    fp32 sums, so the bits equal fused_moe's.  Run through the package's TensorParallelMoE
    with no collectives (a group of one)."""
    inp, g, _ = small(name)
    s = inp.shape
    layer = tp.TensorParallelMoE(g["wr"], g["w13"], g["w2"], s.top_k, g["s13"], g["s2"],
                                 routing=g["routing"], reduce_max=lambda t: t,
                                 reduce_sum=lambda t: t)
    out = layer(g["x"])
    torch.cuda.synchronize()
    want, _ = run_unsharded(inp, g)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)


FULL = [("mixtral_fp8_decode", 64, 8), ("mixtral_fp8_decode", 1, 8), ("mixtral_bf16_decode", 8, 4)]


@pytest.mark.parametrize("workload,T,n", FULL, ids=[f"{w}-T{t}-N{n}" for w, t, n in FULL])
def test_full_size_shards_match_oracle(workload, T, n):
    s = minp.shape(workload, T)
    inp = minp.make_inputs(s, seed=0)
    g = _dev(inp)
    ref = run_oracle(O, inp)
    bits, gmax, _ = run_tp(inp, g, n)
    err = max_rel_err(bf16_bits_to_float(bits), ref["out64"])
    report_errors(f"tp {workload} T={T} N={n}", bf16_bits_to_float(bits), ref["out64"])
    assert err <= TOL[s.wdtype], err
    if s.wdtype == "fp8":
        assert abs(gmax / float(np.abs(ref["h"]).max()) - 1) <= 1e-5
