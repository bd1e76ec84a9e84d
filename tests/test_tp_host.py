"""Tensor parallelism over the intermediate features, host side, on CPU with two gloo
ranks (no GPU): the weight partition, the cross-rank max of max|h| and the sum of the
partial outputs, checked against the oracle of the unsharded layer.

Each rank runs the package's TensorParallelMoE with its real collectives (gloo
all-reduce).  Only the three library calls are stood in for: fakes that compute one
shard's part with the oracle's own steps (route, permute, expert networks on the shard's
weights with the max |h| they are given, combine).  So the test checks the orchestration
the GPU path uses: which slices each rank holds, that the scale of h is taken from the
max over every rank, and that the partial outputs are summed before the one rounding to
bf16."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_26_b200 import inputs as minp

tp = pytest.importorskip("mixture_experts_layer_26_b200.tp",
                         reason="the binding needs libfused_moe.so")

CASES = {
    "fp8": dict(T=9, H=256, I=512, E=4, top_k=2, wdtype="fp8"),
    "bf16": dict(T=7, H=256, I=512, E=4, top_k=2, wdtype="bf16"),
    "fp8_shared": dict(T=5, H=256, I=1024, E=8, top_k=2, wdtype="fp8", n_shared=1),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_weights_partition_the_features():
    s = minp.MoEShape(T=1, H=256, I=512, E=3, top_k=1, wdtype="fp8")
    w13, w2, _, _ = minp.make_weights(s, seed=4)
    for n in (1, 2, 4):
        parts = [tp.shard_weights(w13, w2, r, n) for r in range(n)]
        m = s.I // n
        for a, b in parts:
            assert a.shape == (s.E, 2 * m, s.H) and b.shape == (s.E, s.H, m)
            assert a.is_contiguous() and b.is_contiguous()
        gate = torch.cat([a[:, :m] for a, _ in parts], dim=1)
        up = torch.cat([a[:, m:] for a, _ in parts], dim=1)
        assert torch.equal(torch.cat([gate, up], dim=1), w13)
        assert torch.equal(torch.cat([b for _, b in parts], dim=2), w2)
    with pytest.raises(ValueError):
        tp.shard_weights(w13, w2, 0, 3)       # 512 is not a multiple of 128 * 3
    with pytest.raises(ValueError):
        tp.shard_weights(w13, w2, 2, 2)       # no rank 2 of 2
    with pytest.raises(ValueError):
        tp.shard_weights(w13, w2[:, :, :256], 0, 1)


def _oracle_fakes(capi, O, inp, log):
    """Stand-ins for the three library calls of one shard, built from the oracle's steps.
    `ws` is a dict that carries the shard's state from begin to end, as the workspace
    does on the GPU."""
    s = inp.shape
    fp8 = s.wdtype == "fp8"
    xb, wrb = minp.bf16_bits(inp.x), minp.bf16_bits(inp.router_w)
    bits = (lambda t: t.numpy()) if fp8 else minp.bf16_bits
    sc13 = inp.w13_scale.numpy() if fp8 else None
    sc2 = inp.w2_scale.numpy() if fp8 else None
    K = s.top_k + s.n_shared

    def alloc_workspace(dims, device="cpu"):
        return {}

    def tp_begin(dims, x, router_w, w13, scales, amax_h, ws, stream=None):
        # the descriptor the product builds for one shard: the shard's I, the whole T, E, k
        assert (dims.T, dims.H, dims.I, dims.E, dims.top_k) == \
            (s.T, s.H, w13.shape[1] // 2, s.E, s.top_k)
        assert dims.wdtype == (1 if fp8 else 0)
        assert (dims.routing.contents.n_shared if dims.routing else 0) == s.n_shared
        ids, w, _ = O.router(xb, wrb, s.top_k)
        ids, w = O.append_shared(ids, w, s.E, s.n_shared)
        counts, offsets, rows, inv = O.permute(ids, s.E_all)
        a_perm, s1, _, _ = O.permute_quant(xb, rows, K, fp8)
        Ir = w13.shape[1] // 2
        w2_zero = np.zeros((s.E_all, s.H, Ir), dtype=np.uint8 if fp8 else np.uint16)
        _, h, _, _ = O.experts(a_perm, offsets, rows, w, bits(w13), w2_zero, s.H, Ir, s.E_all,
                               fp8, s1, sc13, sc2)
        ws.update(ids=ids, w=w, offsets=offsets, rows=rows, inv=inv, a_perm=a_perm, s1=s1,
                  w13=bits(w13), Ir=Ir)
        amax_h.fill_(float(np.abs(h).max()) if fp8 else 0.0)
        log.append(("begin", float(amax_h.item())))
        return 0

    def tp_end(dims, w2, scales, amax_h, out_partial, ws, stream=None):
        log.append(("end", float(amax_h.item())))
        y, _, hq, _ = O.experts(ws["a_perm"], ws["offsets"], ws["rows"], ws["w"], ws["w13"],
                                bits(w2), s.H, ws["Ir"], s.E_all, fp8, ws["s1"], sc13, sc2,
                                amax2=np.float32(amax_h.item()) if fp8 else None)
        _, sums = O.combine(y, ws["inv"], s.T, K)
        out_partial.copy_(torch.from_numpy(sums.astype(np.float32)))
        ws["hq"] = hq
        return 0

    def tp_finish(out_sum, out, stream=None):
        log.append(("finish", out_sum.clone()))
        out.copy_(out_sum.to(torch.bfloat16))
        return 0

    capi.alloc_workspace = alloc_workspace
    capi.fused_moe_tp_begin = tp_begin
    capi.fused_moe_tp_end = tp_end
    capi.fused_moe_tp_finish = tp_finish


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mixture_experts_layer_26_b200 import capi, tp as tpm
        from oracle import fused_moe_oracle as O
        s = minp.MoEShape(**CASES[case])
        inp = minp.make_inputs(s, seed=21)
        log = []
        _oracle_fakes(capi, O, inp, log)
        w13_r, w2_r = tpm.shard_weights(inp.w13, inp.w2, rank, world)
        routing = None
        if s.n_shared:
            routing = capi.make_softmax_routing(s.n_shared)
        layer = tpm.TensorParallelMoE(inp.router_w, w13_r, w2_r, s.top_k, inp.w13_scale,
                                      inp.w2_scale, routing=routing)
        out = layer(inp.x)
        ws = next(iter(layer._bufs.values()))[0]
        q.put((rank, out.view(torch.int16).numpy().copy(), log[0][1], log[1][1],
               log[2][1].numpy(), ws["hq"]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", sorted(CASES))
def test_two_gloo_ranks_match_the_unsharded_oracle(case):
    from oracle import fused_moe_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    s = minp.MoEShape(**CASES[case])
    inp = minp.make_inputs(s, seed=21)
    fp8 = s.wdtype == "fp8"
    bits = (lambda t: t.numpy()) if fp8 else minp.bf16_bits
    full = O.fused_moe(minp.bf16_bits(inp.x), minp.bf16_bits(inp.router_w), bits(inp.w13),
                       bits(inp.w2), s.top_k, fp8=fp8,
                       w13_scale=inp.w13_scale.numpy() if fp8 else None,
                       w2_scale=inp.w2_scale.numpy() if fp8 else None, n_shared=s.n_shared)
    amax_full = float(np.abs(full["h"]).max()) if fp8 else 0.0
    local = [r[2] for r in res]
    for rank, out_bits, amax_begin, amax_end, summed, hq in res:
        # the scale of h came from the max over both ranks, which is the layer's max |h|
        assert amax_end == pytest.approx(amax_full, rel=0, abs=0)
        assert amax_end == max(local)
        # each rank's codes are the unsharded layer's codes of its features
        m = s.I // 2
        assert np.array_equal(hq, full["hq"][:, rank * m:(rank + 1) * m])
        # the summed partial outputs are the unsharded sums (fp32 rounding of two terms)
        assert np.abs(summed - full["out64"]).max() <= 2e-6 * np.abs(full["out64"]).max()
        # every rank returns the same bf16 output, that of the unsharded sums
        assert np.array_equal(out_bits, res[0][1])
        ref = torch.from_numpy(summed).to(torch.bfloat16).view(torch.int16).numpy()
        assert np.array_equal(out_bits, ref)
    if fp8:
        assert local[0] != local[1]   # the two halves of h really have different maxima
