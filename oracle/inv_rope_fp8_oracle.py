"""CPU oracle for the fused inverse-rotary-embedding + per-head FP8 quantisation kernel.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module: only
the tests, the package's smoke check and the benchmark's CPU-baseline / reference arm
use it.  It shares no code with the CUDA library; the e4m3 and bf16 codecs come from
the MoE oracle, where they are pinned against torch's casts.

Source.  The pages name the kernel (`_fused_inv_rope_fp8_quant_per_head`, a fused
rotary-embedding plus FP8-quantisation kernel whose variable-length arguments made
Triton recompile it for every new token count: codebridge-ai.com blog "AWS MoE kernel:
WGMMA, Triton, TTFT", section "3. Kill JIT recompilation"; agentic-affairs.com, third
change) but give no formula, layout or shape.  The plainest reading of the name:

  1. inverse rotary embedding: token t of x [T, n_heads, head_dim] was rotated by the
     angles theta[pos[t], i] of its position; undo it, i.e. rotate every pair of
     coordinates by -theta:
        y_a =  x_a * cos + x_b * sin
        y_b = -x_a * sin + x_b * cos
     pair i of the first rot_dim coordinates is (i, i + rot_dim/2) in the half-split
     layout (style 0) or (2i, 2i+1) in the interleaved layout (style 1); coordinates
     past rot_dim pass through unchanged;
  2. per-head FP8: for every (t, h), amax = max |y| over the head, scale = amax/448,
     q = e4m3(y * 448/amax) rounded to nearest even, saturating; amax == 0 gives
     scale 1.

Readings where the pages are silent:
  P1 the rotary table is an input: cos_sin [max_pos, rot_dim] fp32 holding the rot_dim/2
     cosines then the rot_dim/2 sines of each position (the cache layout rotary
     embeddings keep); positions [T] int32 index it;
  P2 y is evaluated in fp32 with each product and the sum rounded separately, in the
     order written above (no fused multiply-add), so that the GPU's codes can match
     bit for bit (the e4m3 code is an integer decided by an fp32 value);
  P3 one scale per (token, head), from the fp32 y; scale = amax/448 and the inverse
     448/amax are each one fp32 division; the quantised value is the fp32 product
     y * inv rounded to e4m3 (round to nearest even, saturating to +-448);
  P4 the output keeps the input layout: q [T, n_heads, head_dim] e4m3 codes and
     scales [T, n_heads] fp32.
"""
from __future__ import annotations

import numpy as np

from oracle.fused_moe_oracle import bf16_to_f32, e4m3_decode, e4m3_encode  # noqa: F401

E4M3_MAX = np.float32(448.0)


def pair_index(head_dim: int, rot_dim: int, style: int):
    """Coordinates (a, b) of the rot_dim/2 rotated pairs (step 1)."""
    half = rot_dim // 2
    i = np.arange(half)
    if style == 0:
        return i, i + half
    return 2 * i, 2 * i + 1


def inv_rope(x_bits: np.ndarray, positions: np.ndarray, cos_sin: np.ndarray, rot_dim: int,
             style: int = 0) -> np.ndarray:
    """Step 1 in fp32 (P2): y [T, n_heads, head_dim] float32."""
    x = bf16_to_f32(x_bits).astype(np.float32)
    T, nh, hd = x.shape
    half = rot_dim // 2
    cs = np.asarray(cos_sin, np.float32)[np.asarray(positions, np.int64)]   # [T, rot_dim]
    c = cs[:, None, :half]
    s = cs[:, None, half:rot_dim]
    a, b = pair_index(hd, rot_dim, style)
    y = x.copy()
    xa, xb = x[:, :, a], x[:, :, b]
    y[:, :, a] = (xa * c).astype(np.float32) + (xb * s).astype(np.float32)
    y[:, :, b] = (-(xa * s)).astype(np.float32) + (xb * c).astype(np.float32)
    return y.astype(np.float32)


def quant_per_head(y: np.ndarray):
    """Step 2 (P3): codes [T, n_heads, head_dim] uint8, scales [T, n_heads] float32."""
    y = np.asarray(y, np.float32)
    amax = np.abs(y).max(axis=2).astype(np.float32)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1))
    scale = np.where(nz, (safe / E4M3_MAX).astype(np.float32), np.float32(1)).astype(np.float32)
    inv = np.where(nz, (E4M3_MAX / safe).astype(np.float32), np.float32(1)).astype(np.float32)
    q = e4m3_encode((y * inv[:, :, None]).astype(np.float32))
    return q, scale


def inv_rope_fp8_quant(x_bits, positions, cos_sin, rot_dim, style=0):
    """The whole kernel: returns dict(y fp32, q codes, scales)."""
    y = inv_rope(x_bits, positions, cos_sin, rot_dim, style)
    q, scale = quant_per_head(y)
    return dict(y=y, q=q, scales=scale)
