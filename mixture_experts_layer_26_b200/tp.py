"""Tensor parallelism of the fused MoE layer over the expert intermediate dimension.

The pages measure their serving result at 8-way tensor parallelism (agentic-affairs.com,
third change; modelsatwork.news, "The three changes") and point out that on multi-GPU
setups every GPU waits for the slowest one (codebridge-ai.com blog "AWS MoE kernel:
WGMMA, Triton, TTFT", section 3).  Here every rank of a process group holds, for every
expert, I/N of the intermediate features: those rows of W1 and W3 and those columns of
W2 (`shard_weights`).  One layer call on N ranks is

    fused_moe_tp_begin   route, permute, first contraction on this rank's features;
                         this rank's max |h|                         (library kernels)
    all-reduce MAX       of that one float: the per-tensor scale of h covers all of h
    fused_moe_tp_end     second contraction and combine into this rank's fp32 partial
                         output [T, H]                               (library kernels)
    all-reduce SUM       of the partial outputs (NCCL over NVLink / NVSwitch)
    fused_moe_tp_finish  out = bf16(sum)                             (library kernel)

Routing and the activation quantisation are computed identically on every rank, so no
routing data crosses the link; the two reductions are the only exchange.  Every kernel is
the library's; this module only orders the calls and the collectives (torch.distributed),
which are the plumbing.  No TMA load of this library ever reads another GPU's memory:
remote data arrives only through the collectives into local buffers.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch

from . import capi


def shard_weights(w13: torch.Tensor, w2: torch.Tensor, rank: int, n_shards: int):
    """Shard `rank` of `n_shards` of the expert weights, as contiguous tensors:
    w13 [E, 2I, H] -> [E, 2I/N, H] (rows r*I/N.. of W1, then the same rows of W3) and
    w2 [E, H, I] -> [E, H, I/N] (columns r*I/N..).  I must be a multiple of 128*N so that
    each shard's I/N is a legal intermediate size of the layer."""
    if w13.dim() != 3 or w2.dim() != 3 or w13.shape[0] != w2.shape[0]:
        raise ValueError("w13 must be [E, 2I, H] and w2 [E, H, I]")
    E, two_i, H = w13.shape
    I = two_i // 2
    if two_i % 2 or tuple(w2.shape) != (E, H, I):
        raise ValueError(f"w13 {tuple(w13.shape)} and w2 {tuple(w2.shape)} do not match")
    if n_shards < 1 or not 0 <= rank < n_shards:
        raise ValueError(f"rank {rank} of {n_shards} shards")
    if I % (128 * n_shards) != 0:
        raise ValueError(f"I = {I} is not a multiple of 128 * {n_shards}")
    n = I // n_shards
    f0 = rank * n
    w13_r = torch.cat([w13[:, f0:f0 + n], w13[:, I + f0:I + f0 + n]], dim=1).contiguous()
    w2_r = w2[:, :, f0:f0 + n].contiguous()
    return w13_r, w2_r


def reduce_amax_(amax: torch.Tensor, group=None) -> torch.Tensor:
    """In place: the max of every rank's max |h| (one fp32 word)."""
    import torch.distributed as dist
    dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def reduce_partial_(partial: torch.Tensor, group=None) -> torch.Tensor:
    """In place: the sum of every rank's partial output."""
    import torch.distributed as dist
    dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


class TensorParallelMoE:
    """One rank's part of a tensor-parallel fused MoE layer.

    router_w [E, H] bf16 (whole), w13_shard / w2_shard from `shard_weights`, the unsharded
    per-expert FP8 scales.  `reduce_max` / `reduce_sum` perform the two exchanges (default:
    all-reduce over `group` with torch.distributed).  Returns out [T, H] bf16, the same on
    every rank."""

    def __init__(self, router_w, w13_shard, w2_shard, top_k, w13_scale=None, w2_scale=None,
                 a1_scale=0.0, a2_scale=0.0, variant="auto", routing=None, group=None,
                 reduce_max: Optional[Callable] = None, reduce_sum: Optional[Callable] = None):
        self.router_w, self.w13, self.w2 = router_w, w13_shard, w2_shard
        self.top_k, self.variant, self.routing = top_k, variant, routing
        self.w13_scale, self.w2_scale = w13_scale, w2_scale
        self.scales = capi.make_scales(w13_scale, w2_scale, a1_scale, a2_scale)
        self.reduce_max = reduce_max or (lambda t: reduce_amax_(t, group))
        self.reduce_sum = reduce_sum or (lambda t: reduce_partial_(t, group))
        self._bufs = {}

    def dims(self, T: int):
        return capi.make_dims(T, self.w13.shape[2], self.w13.shape[1] // 2,
                              self.router_w.shape[0], self.top_k, self.w13.dtype == torch.uint8,
                              self.variant, routing=self.routing)

    def buffers(self, T: int, device):
        """(workspace, amax word, fp32 partial output) for T tokens, kept for reuse."""
        if T not in self._bufs:
            ws = capi.alloc_workspace(self.dims(T), device)
            amax = torch.zeros(1, dtype=torch.float32, device=device)
            partial = torch.empty(T, self.w13.shape[2], dtype=torch.float32, device=device)
            self._bufs[T] = (ws, amax, partial)
        return self._bufs[T]

    def __call__(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
        T, H = x.shape
        if out is None:
            out = torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
        if T == 0:
            return out
        dims = self.dims(T)
        ws, amax, partial = self.buffers(T, x.device)
        capi.fused_moe_tp_begin(dims, x, self.router_w, self.w13, self.scales, amax, ws, stream)
        self.reduce_max(amax)
        capi.fused_moe_tp_end(dims, self.w2, self.scales, amax, partial, ws, stream)
        self.reduce_sum(partial)
        capi.fused_moe_tp_finish(partial, out, stream)
        return out
