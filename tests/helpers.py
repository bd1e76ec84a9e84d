"""Shared test helpers: numpy views of the seeded inputs and error metrics."""
from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_26_b200 import inputs as minp


def np_inputs(inp: "minp.MoEInputs") -> dict:
    fp8 = inp.shape.wdtype == "fp8"

    def wbits(t):
        return t.numpy() if fp8 else minp.bf16_bits(t)

    return dict(
        x_bits=minp.bf16_bits(inp.x),
        wr_bits=minp.bf16_bits(inp.router_w),
        w13=wbits(inp.w13),
        w2=wbits(inp.w2),
        w13_scale=None if inp.w13_scale is None else inp.w13_scale.numpy(),
        w2_scale=None if inp.w2_scale is None else inp.w2_scale.numpy(),
        fp8=fp8,
        top_k=inp.shape.top_k,
    )


def grouped_args(inp):
    """The oracle's grouped-routing parameters of these inputs (None for softmax)."""
    if inp.shape.grouped is None:
        return None
    n_group, topk_group, scaling = inp.shape.grouped
    return dict(n_group=n_group, topk_group=topk_group, routed_scaling=scaling,
                bias=inp.router_bias.numpy())


def run_oracle(oracle_mod, inp, a1_scale=0.0, a2_scale=0.0):
    d = np_inputs(inp)
    return oracle_mod.fused_moe(d["x_bits"], d["wr_bits"], d["w13"], d["w2"], d["top_k"],
                                fp8=d["fp8"], w13_scale=d["w13_scale"],
                                w2_scale=d["w2_scale"], a1_scale=a1_scale, a2_scale=a2_scale,
                                grouped=grouped_args(inp), n_shared=inp.shape.n_shared)


def bf16_bits_to_float(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def max_rel_err(got, ref) -> float:
    """Normwise max relative error: max|got - ref| / max|ref|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.abs(ref).max()
    if denom == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / denom)


def per_element_err(got, ref) -> float:
    """Per-element relative error max |got - ref| / (|ref| + 1e-3 * rms(ref)), reported for
    information beside the normwise bound (it is not a pass/fail bar)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return float((np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms + 1e-300)).max()) if ref.size else 0.0


# (test id, normwise max relative error, per-element error) of every layer parity check in
# this session; printed at the end of the run (conftest.pytest_terminal_summary)
ERROR_REPORT = []


def report_errors(name: str, got, ref) -> None:
    ERROR_REPORT.append((name, max_rel_err(got, ref), per_element_err(got, ref)))


def tiny_shape(T, H, I, E, k, wdtype, **kw):
    return minp.MoEShape(T=T, H=H, I=I, E=E, top_k=k, wdtype=wdtype, **kw)


def torch_bf16_bits(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)
