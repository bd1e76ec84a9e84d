"""Seeded synthetic inputs for the fused MoE layer.

This module only draws random numbers and lays them out in the formats the layer
consumes. It contains none of the layer's arithmetic (no routing, no permutation,
no contraction). It is shared by the GPU tests, the benchmark and the CPU-side
tests, so that both sides of every parity check read identical bytes.

Shared experts (n_shared > 0) are generated like routed ones and stored after them:
w13 / w2 / scales have E + n_shared experts, router_w has E rows.

Workloads (the MoE shapes named for the method "Mixture-of-Experts kernel
engineering on Amazon SageMaker AI": Mixtral-like and DeepSeek-V3-like experts,
a large expert dimension of 8192 for the Swap-AB case, and a prefill batch):

  x        [T, H]      bf16, N(0, 1)
  router_w [E, H]      bf16, N(0, 1/sqrt(H))   (std 1 for the DeepSeek-like gate)
  w13      [E, 2I, H]  rows 0..I-1 = W1 (gate), rows I..2I-1 = W3 (up), std 1/sqrt(H)
  w2       [E, H, I]   std 1/sqrt(I)

For the FP8 formats each expert's tensor gets one fp32 scale
sw = amax(|W_e|) / 448 and the stored bytes are torch's float8_e4m3fn cast of
clamp(W_e / sw, -448, 448).  The bf16 formats store the bf16 weights directly.

Weights are drawn one expert at a time from generators seeded by (seed, tensor,
expert), so memory stays bounded and any expert can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class MoEShape:
    T: int
    H: int
    I: int
    E: int
    top_k: int
    wdtype: str  # "fp8" or "bf16"
    router_std: Optional[float] = None  # None: 1/sqrt(H)
    adversarial: bool = False
    name: str = ""
    # group-limited sigmoid routing: (n_group, topk_group, routed_scaling); None = softmax
    grouped: Optional[tuple] = None
    # shared experts (every token, weight 1), stored after the E routed experts
    n_shared: int = 0

    @property
    def R(self) -> int:
        return self.T * (self.top_k + self.n_shared)

    @property
    def E_all(self) -> int:
        return self.E + self.n_shared


# The five workloads.  Decode workloads list every batch size they are run at.
WORKLOADS = {
    "tiny_bf16": dict(Ts=(4,), H=256, I=512, E=8, top_k=2, wdtype="bf16"),
    "mixtral_fp8_decode": dict(Ts=(1, 8, 32, 64), H=4096, I=14336, E=8, top_k=2, wdtype="fp8"),
    "dsv3_fp8_decode": dict(Ts=(16, 64, 256), H=7168, I=2048, E=256, top_k=8, wdtype="fp8",
                            router_std=1.0),
    "swapab_stress_fp8": dict(Ts=(8,), H=8192, I=8192, E=16, top_k=2, wdtype="fp8"),
    "swapab_adversarial_fp8": dict(Ts=(8,), H=8192, I=8192, E=16, top_k=2, wdtype="fp8",
                                   adversarial=True),
    "prefill_fp8": dict(Ts=(4096,), H=4096, I=14336, E=8, top_k=2, wdtype="fp8"),
    # the same Mixtral-like shapes with bf16 weights and activations
    "mixtral_bf16_decode": dict(Ts=(1, 8, 32, 64), H=4096, I=14336, E=8, top_k=2, wdtype="bf16"),
    "prefill_bf16": dict(Ts=(4096,), H=4096, I=14336, E=8, top_k=2, wdtype="bf16"),
    # DeepSeek-V3-like shapes with its group-limited sigmoid router (8 groups of 32
    # experts, 4 groups kept, routed scaling 2.5, a seeded selection bias) and its one
    # shared expert of the routed experts' shape
    "dsv3_grouped_fp8_decode": dict(Ts=(16, 64, 256), H=7168, I=2048, E=256, top_k=8,
                                    wdtype="fp8", router_std=1.0, grouped=(8, 4, 2.5),
                                    n_shared=1),
}


def shape(workload: str, T: Optional[int] = None) -> MoEShape:
    w = dict(WORKLOADS[workload])
    Ts = w.pop("Ts")
    if T is None:
        T = Ts[-1]
    return MoEShape(T=T, name=workload, **w)


def _gen(seed: int, tag: int, index: int = 0, device=None) -> torch.Generator:
    g = torch.Generator() if device is None else torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tag * 10_007 + index) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _to_e4m3(w: torch.Tensor):
    """Per-tensor scale and e4m3fn bytes of one fp32 expert tensor (torch's cast)."""
    amax = w.abs().max().to(torch.float32)
    sw = (amax / E4M3_MAX) if amax > 0 else torch.tensor(1.0, device=w.device)
    q = torch.clamp(w / sw, -E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return float(sw), q.view(torch.uint8)


@dataclasses.dataclass
class MoEInputs:
    shape: MoEShape
    x: torch.Tensor          # [T, H] bf16
    router_w: torch.Tensor   # [E, H] bf16
    w13: torch.Tensor        # [E, 2I, H] uint8 (e4m3fn bits) or bf16
    w2: torch.Tensor         # [E, H, I] uint8 (e4m3fn bits) or bf16
    w13_scale: Optional[torch.Tensor]  # [E] fp32 (FP8 formats only)
    w2_scale: Optional[torch.Tensor]   # [E] fp32
    router_bias: Optional[torch.Tensor] = None  # [E] fp32 (grouped routing only)


def make_activations(s: MoEShape, seed: int = 0, T: Optional[int] = None):
    """x [T, H] and router_w [E, H] (bf16).  T defaults to the shape's T."""
    T = s.T if T is None else T
    gx = _gen(seed, 1)
    x = torch.randn(T, s.H, generator=gx, dtype=torch.float32)
    std = s.router_std if s.router_std is not None else 1.0 / math.sqrt(s.H)
    wr = torch.randn(s.E, s.H, generator=_gen(seed, 2), dtype=torch.float32) * std
    if s.adversarial:
        # Every token is pushed towards expert 0, then expert 1: x_t = z_t + 4c with
        # router rows 0 and 1 aligned with c (norms 10 and 5).
        c = torch.randn(s.H, generator=_gen(seed, 7), dtype=torch.float32)
        x = x + 4.0 * c
        cn = c / c.norm()
        wr[0] = 10.0 * cn
        wr[1] = 5.0 * cn
    return x.to(torch.bfloat16), wr.to(torch.bfloat16)


def make_weights(s: MoEShape, seed: int = 0, device=None):
    """Expert weights in the layer's storage format, generated one expert at a time.

    device=None draws on the host (the bytes every parity check uses).  A CUDA device
    draws there with the device's generator, seeded the same way: the same distributions
    and per-expert quantisation but a different random stream, for measurements whose
    weights are too large to draw on the host quickly (the routing depends only on x and
    router_w, which stay host-drawn)."""
    fp8 = s.wdtype == "fp8"
    dt = torch.uint8 if fp8 else torch.bfloat16
    w13 = torch.empty(s.E_all, 2 * s.I, s.H, dtype=dt, device=device)
    w2 = torch.empty(s.E_all, s.H, s.I, dtype=dt, device=device)
    s13 = torch.ones(s.E_all, dtype=torch.float32)
    s2 = torch.ones(s.E_all, dtype=torch.float32)
    for e in range(s.E_all):
        a = torch.randn(2 * s.I, s.H, generator=_gen(seed, 3, e, device), dtype=torch.float32,
                        device=device)
        a *= 1.0 / math.sqrt(s.H)
        b = torch.randn(s.H, s.I, generator=_gen(seed, 4, e, device), dtype=torch.float32,
                        device=device)
        b *= 1.0 / math.sqrt(s.I)
        if fp8:
            s13[e], w13[e] = _to_e4m3(a)
            s2[e], w2[e] = _to_e4m3(b)
        else:
            w13[e] = a.to(torch.bfloat16)
            w2[e] = b.to(torch.bfloat16)
    return w13, w2, (s13 if fp8 else None), (s2 if fp8 else None)


def make_router_bias(s: MoEShape, seed: int = 0) -> Optional[torch.Tensor]:
    """Selection bias of the grouped router: N(0, 0.02) per expert (None otherwise)."""
    if s.grouped is None:
        return None
    return torch.randn(s.E, generator=_gen(seed, 5), dtype=torch.float32) * 0.02


def make_inputs(s: MoEShape, seed: int = 0) -> MoEInputs:
    x, wr = make_activations(s, seed)
    w13, w2, s13, s2 = make_weights(s, seed)
    return MoEInputs(s, x, wr, w13, w2, s13, s2, make_router_bias(s, seed))


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor's bits."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


# ------------------------------------------------------------------------------------
# Inputs of the inverse-rotary + per-head FP8 quantisation kernel
# ------------------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class RopeShape:
    T: int          # tokens
    n_heads: int
    head_dim: int
    rot_dim: int    # rotated leading coordinates of each head (even, <= head_dim)
    style: int = 0  # 0: pairs (i, i + rot_dim/2); 1: pairs (2i, 2i+1)
    max_pos: int = 32768
    base: float = 10000.0
    name: str = ""


# A prefill batch of Mixtral-like attention (32 query heads of 128) on one GPU, the
# same with 8-way tensor parallelism (4 heads per GPU), and a partial-rotary
# interleaved layout.
ROPE_WORKLOADS = {
    "inv_rope_fp8_prefill": dict(T=16384, n_heads=32, head_dim=128, rot_dim=128),
    "inv_rope_fp8_tp8": dict(T=16384, n_heads=4, head_dim=128, rot_dim=128),
    "inv_rope_fp8_partial": dict(T=4096, n_heads=16, head_dim=128, rot_dim=64, style=1),
}


def rope_shape(workload: str, T: Optional[int] = None) -> RopeShape:
    w = dict(ROPE_WORKLOADS[workload])
    if T is not None:
        w["T"] = T
    return RopeShape(name=workload, **w)


@dataclasses.dataclass
class RopeInputs:
    shape: RopeShape
    x: torch.Tensor          # [T, n_heads, head_dim] bf16
    positions: torch.Tensor  # [T] int32
    cos_sin: torch.Tensor    # [max_pos, rot_dim] fp32: rot_dim/2 cosines, then sines


def make_rope_inputs(s: RopeShape, seed: int = 0) -> RopeInputs:
    """x ~ N(0, 1) in bf16; positions drawn uniformly from [0, max_pos); the rotary table
    of a model with the given base: angle(p, i) = p * base^(-2i/rot_dim), evaluated in
    fp64 and stored as fp32 cosines and sines (a cache the model keeps)."""
    x = torch.randn(s.T, s.n_heads, s.head_dim, generator=_gen(seed, 11), dtype=torch.float32)
    pos = torch.randint(0, s.max_pos, (s.T,), generator=_gen(seed, 12), dtype=torch.int64)
    half = s.rot_dim // 2
    inv_freq = s.base ** (-torch.arange(half, dtype=torch.float64) * 2.0 / s.rot_dim)
    ang = torch.arange(s.max_pos, dtype=torch.float64)[:, None] * inv_freq[None, :]
    table = torch.cat([ang.cos(), ang.sin()], dim=1).to(torch.float32).contiguous()
    return RopeInputs(s, x.to(torch.bfloat16), pos.to(torch.int32), table)
