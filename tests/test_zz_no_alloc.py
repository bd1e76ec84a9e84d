"""fused_moe_static_workspace: the layer for callers that cannot allocate device
memory (for example a plugin whose host framework owns the whole GPU memory pool,
or code that must not call cudaMalloc/cudaFree because they can synchronise the
device).  It runs with a library-owned device array as its workspace.

Checked through the C ABI against fused_moe with a caller workspace, on two calls in
a row (the array keeps the previous call's contents), within the tolerances the other
parity tests use.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes on its own in a fresh
process."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from mixture_experts_layer_26_b200 import inputs as minp

capi = pytest.importorskip("mixture_experts_layer_26_b200.capi")

pytestmark = pytest.mark.gpu

# The argument checks (null pointers, alignment, unsupported dims, dims beyond the
# array's size) need no GPU and run with the host tests (test_capi_host.py).

CASES = [
    # (T, H, I, E, k, wdtype, tolerance)
    (4, 256, 512, 8, 2, "bf16", 5e-3),
    (37, 512, 384, 8, 2, "fp8", 2e-2),
]


def _max_rel(a: torch.Tensor, b: torch.Tensor) -> float:
    a, b = a.float(), b.float()
    return float((a - b).abs().max() / b.abs().max())


@pytest.mark.parametrize("T,H,I,E,k,wdtype,tol", CASES)
def test_static_workspace_matches_fused_moe_twice(T, H, I, E, k, wdtype, tol):
    s = minp.MoEShape(T=T, H=H, I=I, E=E, top_k=k, wdtype=wdtype)
    fp8 = wdtype == "fp8"
    dims = capi.make_dims(T, H, I, E, k, fp8)
    assert capi.workspace_size(dims) <= capi.STATIC_WS_BYTES
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    outs = []
    for seed in (1, 2):  # two calls in a row with different inputs
        inp = minp.make_inputs(s, seed=seed)
        g = {k2: (None if v is None else v.cuda()) for k2, v in
             dict(x=inp.x, wr=inp.router_w, w13=inp.w13, w2=inp.w2,
                  s13=inp.w13_scale, s2=inp.w2_scale).items()}
        sc = capi.make_scales(g["s13"], g["s2"])
        ref = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        ws = capi.alloc_workspace(dims)
        capi.fused_moe(dims, g["x"], g["wr"], g["w13"], g["w2"], sc, ref, ws)
        out = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        capi.fused_moe_static_workspace(dims, g["x"], g["wr"], g["w13"], g["w2"], sc, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == capi.FMOE_OK
        assert not torch.isnan(out.float()).any()
        assert _max_rel(out, ref) <= tol
        outs.append(out)
    assert not torch.equal(outs[0], outs[1])  # the second call really recomputed
