"""Brute-force fused MoE: per-token loops over each token's k experts.

Written independently of the oracle to pin it on tiny inputs.  It shares no
code with the oracle: number formats are decoded and encoded with torch's own
casts (bf16 and float8_e4m3fn, a library routine), sums are exactly rounded
(math.fsum), and the layer is evaluated token by token, expert by expert, the
way the pages describe the unfused baseline ("separate, sequential loop
operations": readmex.ai story "AWS details fused MoE kernel optimizations on
SageMaker", opening section).

The router logits are computed exactly (fsum of exact bf16 products); the
oracle's fp32 logits must select the same experts whenever the gap between the
k-th and (k+1)-th exact logit exceeds the fp32 summation error bound, which the
tests check before comparing.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _bf16_bits_to_float(bits) -> torch.Tensor:
    return torch.from_numpy(np.asarray(bits, dtype=np.uint16).view(np.int16).copy()) \
        .view(torch.bfloat16).to(torch.float64)


def _e4m3_to_float(codes) -> torch.Tensor:
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy()) \
        .view(torch.float8_e4m3fn).to(torch.float64)


def _q_e4m3(v32: float) -> float:
    """Value of the e4m3 code nearest to the fp32 number v32 (clamped to +-448)."""
    t = torch.tensor([min(max(v32, -448.0), 448.0)], dtype=torch.float32)
    return float(t.to(torch.float8_e4m3fn).to(torch.float64)[0])


def _f32(v: float) -> float:
    return float(np.float32(v))


def _bf16(v: float) -> float:
    return float(torch.tensor([v], dtype=torch.float32).to(torch.bfloat16).to(torch.float64)[0])


def exact_logits(x_bits, wr_bits):
    x = _bf16_bits_to_float(x_bits).tolist()
    w = _bf16_bits_to_float(wr_bits).tolist()
    return [[math.fsum(a * b for a, b in zip(xt, we)) for we in w] for xt in x]


def brute_force(x_bits, wr_bits, w13, w2, top_k, fp8, w13_scale=None, w2_scale=None,
                n_shared=0):
    """Returns dict(ids, weights, out [T][H] floats (bf16 values), h [(t,j)] lists).

    n_shared: experts E..E+n_shared-1 of w13/w2 join every token after its k routed
    experts with weight 1 (DeepSeek-V3's always-active shared experts)."""
    x = _bf16_bits_to_float(x_bits).tolist()
    T, H = len(x), len(x[0])
    E = len(wr_bits)
    logits = exact_logits(x_bits, wr_bits)
    ids, weights = [], []
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-logits[t][e], e))[:top_k]
        m = max(logits[t])
        p = [math.exp(l - m) for l in logits[t]]
        z = math.fsum(p)
        p = [v / z for v in p]                       # softmax over all experts
        zs = math.fsum(p[e] for e in order)
        ids.append(order + [E + i for i in range(n_shared)])
        weights.append([_f32(p[e] / zs) for e in order] + [1.0] * n_shared)   # fp32

    if fp8:
        W13 = _e4m3_to_float(w13).tolist()
        W2 = _e4m3_to_float(w2).tolist()
        amax = max(abs(v) for row in x for v in row)
        s1 = float(np.float32(amax) / np.float32(448)) if amax > 0 else 1.0
        inv1 = float(np.float32(448) / np.float32(amax)) if amax > 0 else 1.0
        act = [[_q_e4m3(_f32(v * inv1)) for v in row] for row in x]
    else:
        W13 = _bf16_bits_to_float(w13).tolist()
        W2 = _bf16_bits_to_float(w2).tolist()
        act = x
        s1 = 1.0
    I = len(W2[0][0])

    # first expert network, token by token
    hs = {}
    for t in range(T):
        for j, e in enumerate(ids[t]):
            sc = _f32(s1 * w13_scale[e]) if fp8 else 1.0
            row = []
            for n in range(I):
                g = math.fsum(a * b for a, b in zip(act[t], W13[e][n])) * sc
                u = math.fsum(a * b for a, b in zip(act[t], W13[e][I + n])) * sc
                row.append(_f32(g / (1.0 + math.exp(-g)) * u))
            hs[(t, j)] = row
    if fp8:
        amax2 = max(abs(v) for row in hs.values() for v in row)
        s2 = float(np.float32(amax2) / np.float32(448)) if amax2 > 0 else 1.0
        inv2 = float(np.float32(448) / np.float32(amax2)) if amax2 > 0 else 1.0
        hq = {key: [_q_e4m3(_f32(v * inv2)) for v in row] for key, row in hs.items()}
    else:
        s2 = 1.0
        hq = {key: [_bf16(v) for v in row] for key, row in hs.items()}

    out = []
    for t in range(T):
        acc = [0.0] * H
        for j, e in enumerate(ids[t]):
            sc = _f32(s2 * w2_scale[e]) if fp8 else 1.0
            for mcol in range(H):
                yv = math.fsum(a * b for a, b in zip(hq[(t, j)], W2[e][mcol])) * sc
                acc[mcol] += weights[t][j] * yv
        out.append([_bf16(_f32(v)) for v in acc])
    return dict(ids=ids, weights=weights, logits=logits, out=out, h=hs)


def grouped_routing(logits, top_k, n_group, topk_group, bias=None, routed_scaling=1.0):
    """Group-limited sigmoid routing token by token with Python floats, from given
    fp32 logits (their summation order is pinned separately)."""
    ex = [[float(v) for v in row] for row in logits]
    T, E = len(ex), len(ex[0])
    eg = E // n_group
    b = [0.0] * E if bias is None else [float(v) for v in bias]
    ids, ws = [], []
    for t in range(T):
        s = [_f32(1.0 / (1.0 + math.exp(-_f32(l)))) for l in ex[t]]
        sb = [_f32(s[e] + b[e]) for e in range(E)]
        gs = []
        for g in range(n_group):
            members = sorted(sb[g * eg:(g + 1) * eg], reverse=True)
            gs.append(_f32(members[0] + members[1]))
        kept = sorted(range(n_group), key=lambda g: (-gs[g], g))[:topk_group]
        cand = [e for e in range(E) if e // eg in kept]
        chosen = sorted(cand, key=lambda e: (-sb[e], e))[:top_k]
        tot = math.fsum(s[e] for e in chosen)
        ids.append(chosen)
        ws.append([_f32(s[e] / tot * _f32(routed_scaling)) for e in chosen])
    return ids, ws
