"""CPU oracle for the fused Mixture-of-Experts layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only the tests, the package's smoke check and the benchmark's CPU-baseline /
reference arm use it.  It shares no code with the CUDA library.

Sources.  The method is described on five web pages about one AWS engineering
post on fused MoE kernels:
  [readmex]   readmex.ai story "AWS details fused MoE kernel optimizations on
              SageMaker, up to 10% throughput gain"
  [codebridge] codebridge-ai.com blog "AWS MoE kernel: WGMMA, Triton, TTFT"
  [agentic]   agentic-affairs.com article on the same post
  [n1n]       explore.n1n.ai "Mixture-of-Experts Kernel Engineering on Amazon
              SageMaker AI"
  [modelsatwork] modelsatwork.news "AWS: MoE kernel fixes give up to 10% more
              throughput on H200"
The pages state the problem (a fused MoE merges token routing, data shuffling
and the expert-network computations into one batched GPU operation instead of
separate sequential loops: [readmex] opening section; [agentic] "Swap-AB
targets matrix execution on Hopper") and that FP8 MoE works on per-tensor
("tensor-quantized") scales ([readmex] opening; [agentic] "Triton improves the
FP8 execution path").  They give no formula.  The layer computed here is the
standard softmax-top-k gated-MLP MoE:

  1. logits[t,e] = sum_h x[t,h] * Wr[e,h]                     (router)
  2. the k largest logits per token, in descending order       (top-k)
  3. w = softmax over all E experts, renormalised over the top-k
  4. rows grouped by expert: counts, offsets, a stable permutation
  5. FP8: Aq = e4m3(x * 448/amax|x|)                           (per-tensor)
  6. per expert: g = Aq.W1^T, u = Aq.W3^T (scaled); h = SiLU(g) * u
  7. FP8: hq = e4m3(h * 448/amax|h|)
  8. per expert: Y = hq.W2^T (scaled)
  9. out[t] = bf16( sum_j w[t,j] * Y[row of (t,j)] )

Precision.  Contractions and softmax run in fp64 (the exact result up to fp64
rounding).  Where floating point decides an integer -- the router logits that
choose the top-k, and every e4m3 code -- the oracle takes the decision in fp32,
the precision the layer stores those values in, so that the GPU can match it
bit for bit:
  * router logits are summed in fp32 in one fixed ("canonical") order, spelled
    out in `router_logits`;
  * quantisation multiplies by the fp32 inverse scale in fp32 and rounds the
    fp32 product to e4m3 (round to nearest even, saturating to +-448).

Readings where the pages are silent:
  R1 canonical fp32 summation order of the router logits (see router_logits)
  R2 top-k ties go to the lower expert index; selection is on logits
  R3 permutation is stable by (expert, flattened index t*k+j)
  R4 activation scales are per-tensor dynamic (amax/448) unless a static
     scale > 0 is given; amax == 0 gives scale 1
  R5 one fp32 scale per expert per weight tensor (w13 and w2)
  R6 rows 0..I-1 of w13 are W1 (gate), rows I..2I-1 are W3 (up)
  R7 bf16 format: no quantisation; h is rounded to bf16 before the second
     contraction
  R8 the final sum is rounded fp64 -> fp32 -> bf16 (round to nearest even)
The grouped sigmoid routing of router_grouped (a later variant of step 1-3 for the
DeepSeek-V3-like shapes; the pages name DeepSeek-V3 but do not describe its router) is
taken from DeepSeek-V3's published design; its readings D1-D5 are listed there.
Shared experts (DeepSeek-V3's always-active experts; readings S1-S2 at
append_shared) are experts E..E+n_shared-1 that every token uses with weight 1.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = np.float32(448.0)

# --------------------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------------------


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32: bf16 is the top half of an fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest, ties to even (NaN -> 0x7FC0)."""
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return np.where(np.isnan(x), np.uint16(0x7FC0), r)


def _e4m3_value(code: int) -> float:
    """Value of one OCP e4m3fn code: 1 sign, 4 exponent (bias 7), 3 mantissa bits.
    Exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
# non-negative finite values in code order 0x00..0x7E; they increase with the code
_E4M3_POS = E4M3_TABLE[:127].copy()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """e4m3fn codes (uint8) -> float64 values."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> e4m3fn codes: round to nearest, ties to the even code, and
    clamp finite results to +-448 (saturation); NaN -> 0x7F.  The sign of the
    input is kept, also when the magnitude rounds to zero."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).astype(np.float64)
    a = np.minimum(a, 448.0)
    i = np.searchsorted(_E4M3_POS, a, side="right") - 1          # vals[i] <= a
    i = np.clip(i, 0, 126)
    j = np.minimum(i + 1, 126)
    lo, hi = _E4M3_POS[i], _E4M3_POS[j]
    two_a, mid2 = 2.0 * a, lo + hi                                # exact in fp64
    pick_hi = (two_a > mid2) | ((two_a == mid2) & (i % 2 == 1) & (a != lo))
    code = np.where(a == lo, i, np.where(pick_hi, j, i)).astype(np.uint8)
    code = code | np.where(np.signbit(x), np.uint8(0x80), np.uint8(0))
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)


# --------------------------------------------------------------------------------------
# Step 1-3: router.  [readmex] opening section ("token routing"); [n1n] "2. Triton
# Backend Routing for FP8 Quantization" (expert selection kept on the device).
# --------------------------------------------------------------------------------------


def router_logits(x_bits: np.ndarray, wr_bits: np.ndarray) -> np.ndarray:
    """logits[t,e] = sum_h x[t,h]*Wr[e,h] in fp32, in the canonical order (R1).

    The H products are taken in chunks of 8 consecutive elements.  Chunk c
    belongs to lane c mod 32 (32 lanes); each lane adds its chunks in ascending
    order, the 8 elements of a chunk in ascending order, into an fp32 partial
    that starts at 0.  The 32 partials are then combined by an xor butterfly:
    for off in 16, 8, 4, 2, 1: p[l] = p[l] + p[l ^ off]; the logit is p[0].
    Every bf16*bf16 product is exact in fp32, so only this order matters.
    Requires H % 256 == 0.
    """
    x = bf16_to_f32(x_bits)            # [T, H]
    w = bf16_to_f32(wr_bits)           # [E, H]
    T, H = x.shape
    E = w.shape[0]
    assert H % 256 == 0
    lanes = np.arange(32)
    acc = np.zeros((T, E, 32), dtype=np.float32)
    for s in range(H // 256):                      # chunk index within a lane
        for i in range(8):                         # element within a chunk
            cols = (lanes + 32 * s) * 8 + i        # column of lane l at this step
            prod = x[:, None, cols] * w[None, :, cols]     # fp32, exact
            acc = acc + prod                               # one fp32 rounding
    for off in (16, 8, 4, 2, 1):
        acc = acc + acc[:, :, lanes ^ off]
    return acc[:, :, 0].copy()


def router(x_bits: np.ndarray, wr_bits: np.ndarray, top_k: int):
    """topk_ids [T,k] int32, topk_w [T,k] float32, logits [T,E] float32 (R1, R2).

    Top-k is taken on the logits (softmax is monotonic, so this is the same set
    as on the probabilities), ordered by descending logit, ties to the lower
    expert index.  The weights are the softmax over all E experts renormalised
    over the chosen k, evaluated in fp64 and stored as fp32.
    """
    logits = router_logits(x_bits, wr_bits)
    T, E = logits.shape
    idx = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((idx, -logits), axis=-1)       # primary: -logit, then index
    ids = order[:, :top_k].astype(np.int32)
    l64 = logits.astype(np.float64)
    p = np.exp(l64 - l64.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)               # softmax over all experts
    sel = np.take_along_axis(p, ids, axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)           # renormalised over the top-k
    return ids, w.astype(np.float32), logits


def sigmoid_scores(logits: np.ndarray) -> np.ndarray:
    """Affinities of the grouped routing: sigmoid of the fp32 logits, evaluated in fp64
    and rounded once to fp32 (reading D1)."""
    l64 = np.asarray(logits, dtype=np.float32).astype(np.float64)
    return (1.0 / (1.0 + np.exp(-l64))).astype(np.float32)


def router_grouped(x_bits: np.ndarray, wr_bits: np.ndarray, top_k: int, n_group: int,
                   topk_group: int, bias=None, routed_scaling: float = 1.0):
    """Group-limited sigmoid routing (the DeepSeek-V3 router; readings D1-D5).

    D1 s = fp32(sigmoid(logit)) with the logits of router_logits (canonical order);
    D2 selection scores sb = s + bias[e], one fp32 addition (bias 0 when absent);
    D3 the E experts form n_group groups of E/n_group consecutive experts; a group's
       score is the sum (fp32) of its two largest sb; the topk_group best groups are
       kept, ties to the lower group index;
    D4 top-k experts by sb among the kept groups, descending, ties to the lower index;
    D5 weights: the unbiased s of the chosen experts over their sum (fp64), times
       routed_scaling, stored as fp32.
    Returns topk_ids [T,k] int32, topk_w [T,k] float32, s [T,E], sb [T,E] float32."""
    logits = router_logits(x_bits, wr_bits)
    ids, w, s, sb = grouped_select(logits, top_k, n_group, topk_group, bias, routed_scaling)
    return ids, w, s, sb


def grouped_select(logits, top_k, n_group, topk_group, bias=None, routed_scaling=1.0):
    """Steps D1-D5 of router_grouped on given fp32 logits [T, E]."""
    logits = np.asarray(logits, np.float32)
    T, E = logits.shape
    eg = E // n_group
    assert E % n_group == 0 and eg >= 2 and topk_group * eg >= top_k
    s = sigmoid_scores(logits)
    b = np.zeros(E, np.float32) if bias is None else np.asarray(bias, np.float32)
    sb = (s + b[None, :]).astype(np.float32)
    grp = np.sort(sb.reshape(T, n_group, eg), axis=-1)            # ascending
    gscore = (grp[..., -1] + grp[..., -2]).astype(np.float32)      # two largest
    gidx = np.broadcast_to(np.arange(n_group), (T, n_group))
    keep_g = np.lexsort((gidx, -gscore), axis=-1)[:, :topk_group]
    keep = np.zeros((T, n_group), bool)
    np.put_along_axis(keep, keep_g, True, axis=1)
    masked = np.where(np.repeat(keep, eg, axis=1), sb, -np.inf).astype(np.float32)
    eidx = np.broadcast_to(np.arange(E), (T, E))
    ids = np.lexsort((eidx, -masked), axis=-1)[:, :top_k].astype(np.int32)
    sel = np.take_along_axis(s, ids, axis=1).astype(np.float64)
    w = sel / sel.sum(axis=1, keepdims=True) * float(np.float32(routed_scaling))
    return ids, w.astype(np.float32), s, sb


def append_shared(ids: np.ndarray, w: np.ndarray, E: int, n_shared: int):
    """Routing slots with the shared experts appended (DeepSeek-V3's published design
    adds the output of its always-active shared expert to the routed mixture).

    S1 shared expert s is expert E+s of w13/w2 (and of their scales); every token
       uses it with weight exactly 1 (fp32), outside the renormalisation of the routed
       weights and outside routed_scaling;
    S2 it takes slot k+s of the token, after the k routed slots, so the combine adds
       it last; its rows belong to the layer like any expert's (one per-tensor scale
       for h over all rows).
    Returns ids [T, k+n_shared] int32 and w [T, k+n_shared] float32."""
    if n_shared == 0:
        return ids, w
    T = ids.shape[0]
    sid = np.broadcast_to(np.arange(E, E + n_shared, dtype=np.int32), (T, n_shared))
    sw = np.ones((T, n_shared), np.float32)
    return (np.concatenate([ids, sid], axis=1).astype(np.int32),
            np.concatenate([w, sw], axis=1).astype(np.float32))


# --------------------------------------------------------------------------------------
# Step 4: permutation ("data shuffling": [readmex] opening; irregular access and
# dynamic per-expert batch sizes: [n1n] "The Core Bottlenecks of MoE Inference").
# --------------------------------------------------------------------------------------


def permute(topk_ids: np.ndarray, E: int):
    """counts [E], offsets [E+1], sorted_rows [R], inv_perm [R] (int32), R3.

    sorted_rows lists the flattened indices t*k+j grouped by expert, ascending
    within an expert; inv_perm is its inverse."""
    flat = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    sorted_rows = np.argsort(flat, kind="stable").astype(np.int32)
    inv_perm = np.empty_like(sorted_rows)
    inv_perm[sorted_rows] = np.arange(flat.size, dtype=np.int32)
    return counts, offsets, sorted_rows, inv_perm


# --------------------------------------------------------------------------------------
# Steps 5 and 7: per-tensor FP8 scales ([readmex] opening, "FP8 tensor-quantized";
# [agentic] "Triton improves the FP8 execution path": FP8 tensor scaling).
# --------------------------------------------------------------------------------------


def act_scales(amax: np.float32, static_scale: float = 0.0):
    """(scale, inverse scale) in fp32 (R4): amax/448 and 448/amax, each one fp32
    division; amax == 0 gives (1, 1); a static scale s > 0 gives (s, 1/s)."""
    if static_scale > 0:
        s = np.float32(static_scale)
        return s, np.float32(np.float32(1.0) / s)
    amax = np.float32(amax)
    if amax == 0:
        return np.float32(1.0), np.float32(1.0)
    return np.float32(amax / E4M3_MAX), np.float32(E4M3_MAX / amax)


def quantize(v: np.ndarray, inv_scale: np.float32) -> np.ndarray:
    """e4m3 codes of v * inv_scale, the product taken in fp32."""
    prod = np.asarray(v, dtype=np.float32) * np.float32(inv_scale)
    return e4m3_encode(prod)


def permute_quant(x_bits, sorted_rows, top_k, fp8=True, a1_scale=0.0):
    """The permuted activation rows A[p] = x[sorted_rows[p] // k].

    FP8: returns (Aq codes [R,H] uint8, s1, inv1, amax_x).  bf16: (bits, 1, 1, amax)."""
    x = bf16_to_f32(x_bits)
    amax = np.float32(np.abs(x).max()) if x.size else np.float32(0)
    tok = np.asarray(sorted_rows, dtype=np.int64) // top_k
    if not fp8:
        return np.asarray(x_bits)[tok], np.float32(1), np.float32(1), amax
    s1, inv1 = act_scales(amax, a1_scale)
    return quantize(x[tok], inv1), s1, inv1, amax


# --------------------------------------------------------------------------------------
# Steps 6-8: expert networks ([readmex] opening, "specialized network calculations";
# [agentic] "Triton improves the FP8 execution path": scaling, matrix multiply and
# expert aggregation in one pass).
# --------------------------------------------------------------------------------------


def silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


def experts(a_perm, offsets, sorted_rows, topk_w, w13, w2, H, I, E,
            fp8=True, s1=np.float32(1), w13_scale=None, w2_scale=None, a2_scale=0.0,
            amax2=None):
    """Per-expert gated MLP on the permuted rows.

    Returns y [R,H] float64 (already multiplied by the routing weight of its
    row), h [R,I] float32, hq (codes or bf16 bits) [R,I], s2.
    FP8: g,u = (Aq_e . W1_e^T, Aq_e . W3_e^T) * (s1*sw13[e]) in fp64; h = SiLU(g)*u
    stored as fp32; hq = e4m3(h * inv2) with the global amax of h (R4);
    Y = (hq_e . W2_e^T) * (s2*sw2[e]).  bf16 (R7): no scales; h -> bf16.

    amax2: the max |h| the per-tensor scale of h is taken from; None means the max of
    this call's h.  One shard of the layer split over the intermediate features (the
    tensor parallelism the pages measure at 8 ways: agentic-affairs.com, third change)
    holds a slice of h; given the max over the whole layer's h, its codes are the
    unsharded layer's codes for those features (R4 takes the scale over all of h)."""
    R = a_perm.shape[0]
    A = e4m3_decode(a_perm) if fp8 else bf16_to_f32(a_perm).astype(np.float64)
    h = np.zeros((R, I), dtype=np.float32)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        W = e4m3_decode(w13[e]) if fp8 else bf16_to_f32(w13[e]).astype(np.float64)
        acc = A[r0:r1] @ W.T                                   # [n_e, 2I]
        sc = float(np.float32(s1) * np.float32(w13_scale[e])) if fp8 else 1.0
        g, u = acc[:, :I] * sc, acc[:, I:] * sc                 # R6
        h[r0:r1] = (silu(g) * u).astype(np.float32)
    if fp8:
        if amax2 is None:
            amax2 = np.float32(np.abs(h).max()) if h.size else np.float32(0)
        s2, inv2 = act_scales(np.float32(amax2), a2_scale)
        hq = quantize(h, inv2)
        B = e4m3_decode(hq)
    else:
        s2 = np.float32(1)
        hq = f32_to_bf16(h)
        B = bf16_to_f32(hq).astype(np.float64)
    wrow = np.asarray(topk_w, dtype=np.float32).reshape(-1)[np.asarray(sorted_rows)]
    y = np.zeros((R, H), dtype=np.float64)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        W = e4m3_decode(w2[e]) if fp8 else bf16_to_f32(w2[e]).astype(np.float64)
        sc = float(np.float32(s2) * np.float32(w2_scale[e])) if fp8 else 1.0
        Y = (B[r0:r1] @ W.T) * sc                               # [n_e, H]
        y[r0:r1] = Y * wrow[r0:r1, None].astype(np.float64)
    return y, h, hq, s2


# --------------------------------------------------------------------------------------
# Step 9: combine ("expert aggregation": [codebridge] "2. Backend routing").
# --------------------------------------------------------------------------------------


def combine(y, inv_perm, T, top_k):
    """out[t] = bf16(sum_{j<k} y[inv_perm[t*k+j]]), summed in j order (R8).
    Returns (bf16 bits [T,H], fp64 sums [T,H])."""
    inv = np.asarray(inv_perm, dtype=np.int64).reshape(T, top_k)
    acc = np.zeros((T, y.shape[1]), dtype=np.float64)
    for j in range(top_k):
        acc = acc + y[inv[:, j]]
    return f32_to_bf16(acc.astype(np.float32)), acc


# --------------------------------------------------------------------------------------
# The whole layer
# --------------------------------------------------------------------------------------


def fused_moe(x_bits, wr_bits, w13, w2, top_k, fp8=True, w13_scale=None, w2_scale=None,
              a1_scale=0.0, a2_scale=0.0, grouped=None, n_shared=0):
    """The whole layer on host arrays.  x_bits [T,H] / wr_bits [E,H] are bf16 bit
    patterns (uint16); w13 [E+n_shared,2I,H], w2 [E+n_shared,H,I] are e4m3 codes
    (uint8) or bf16 bits.  grouped: None for softmax top-k routing, else the
    router_grouped parameters.  n_shared: shared experts after the E routed ones.
    Returns a dict with every intermediate the GPU path also exposes; topk_ids /
    topk_w include the shared slots."""
    x_bits = np.asarray(x_bits)
    T, H = x_bits.shape
    E = wr_bits.shape[0]
    I = w2.shape[2]
    if grouped is None:
        ids, w, logits = router(x_bits, wr_bits, top_k)
    else:   # dict(n_group=, topk_group=, bias=, routed_scaling=)
        ids, w, logits, _ = router_grouped(x_bits, wr_bits, top_k, **grouped)
    ids, w = append_shared(ids, w, E, n_shared)
    k_all, E_all = top_k + n_shared, E + n_shared
    counts, offsets, sorted_rows, inv_perm = permute(ids, E_all)
    a_perm, s1, inv1, amax_x = permute_quant(x_bits, sorted_rows, k_all, fp8, a1_scale)
    y, h, hq, s2 = experts(a_perm, offsets, sorted_rows, w, w13, w2, H, I, E_all, fp8, s1,
                           w13_scale, w2_scale, a2_scale)
    out, out64 = combine(y, inv_perm, T, k_all)
    return dict(topk_ids=ids, topk_w=w, logits=logits, amax_x=amax_x, counts=counts,
                offsets=offsets, sorted_rows=sorted_rows, inv_perm=inv_perm,
                a_perm=a_perm, s1=s1, inv1=inv1, h=h, hq=hq, s2=s2, y=y,
                out=out, out64=out64)
