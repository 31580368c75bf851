"""NVFP4 (e2m1 values, e4m3 block scales) quantisation for the oracle. Test
infrastructure.

The Diffusers release blog for FLUX.3 Image Klein ("Smaller GPUs, single
files, and custom LoRA training") ships the transformer as an nvfp4 file, and
the local-run guide (quantised files) says NVFP4 needs a Blackwell GPU. The
pages give no more. READING (the format's plainest definition): every value is
a 4-bit e2m1 code; each run of 16 consecutive values along a row (the GEMM's
K dimension) shares one positive e4m3 scale; one fp32 scale covers the whole
tensor. Value = e2m1(code) x block scale x tensor scale.

e2m1: 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit; exponent field
0 holds the subnormal 0.5; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no
infinities or NaN. Encoding rounds to nearest, ties to even, and saturates to
+-6.

Quantisation decision, in float32 (it decides integer codes):
  tensor scale   g   = amax(tensor) / (448 * 6)        (0 for an all-zero tensor)
  block scale    s_b = e4m3(amax(block) / (6 * g))     (e4m3 round-to-nearest-even, saturating)
  code               = e2m1(x / (decode(s_b) * g))     (0 where the block scale is 0)
each operation one correctly rounded float32 step in that order.

READING for the block's activations (the two GEMM inputs, made at run time):
the second-level fp32 scale g is taken per row (token) instead of per tensor,
so that a row's codes depend on that row alone, as in the rowwise FP8 path
(the 16-value block scales carry the fine-grained range either way). Weights
keep one g per matrix.
"""
from __future__ import annotations

import numpy as np

from .fp8 import e4m3_decode, e4m3_encode

F32 = np.float32
F64 = np.float64
BLOCK = 16
E2M1_MAX = 6.0
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_encode(x) -> np.ndarray:
    """float32 values -> uint8 e2m1 codes in the low 4 bits (sign in bit 3)."""
    x = np.asarray(x, dtype=F32).astype(F64)
    sign = (np.signbit(x).astype(np.uint8) << 3)
    a = np.minimum(np.abs(np.nan_to_num(x, nan=0.0)), E2M1_MAX)
    sub = a < 1.0
    # subnormal range: steps of 0.5 (2 steps = 1.0 = exponent 1, mantissa 0 = code 2)
    code_sub = np.rint(a / 0.5).astype(np.int64)
    an = np.where(sub, 1.0, a)
    e = np.floor(np.log2(an)).astype(np.int64)       # 0, 1 or 2
    frac = np.rint((an / 2.0 ** e - 1.0) * 2.0).astype(np.int64)   # ties to even
    carry = frac == 2
    e = np.where(carry, e + 1, e)
    frac = np.where(carry, 0, frac)
    code_norm = np.minimum((e + 1) * 2 + frac, 7)     # 8 would be past 6: saturate
    code = np.where(sub, code_sub, code_norm).astype(np.uint8)
    return (code | sign).astype(np.uint8)


def e2m1_decode(c) -> np.ndarray:
    c = np.asarray(c, dtype=np.uint8).astype(np.int64)
    mag = E2M1_VALUES[c & 7]
    return np.where(c & 8, -mag, mag)


def tensor_scale(x) -> np.float32:
    amax = F32(np.max(np.abs(np.asarray(x, dtype=F64).astype(F32)))) if np.size(x) else F32(0)
    return F32(amax / F32(448.0 * 6.0))


def quantize(x, g=None, per_row=False):
    """x [..., K] (K a multiple of 16) -> (codes uint8 [..., K], block scales
    as e4m3 codes uint8 [..., K/16], second-level scale float32: one for the
    tensor, or [..., 1] one per row with per_row)."""
    x32 = np.asarray(x, dtype=F64).astype(F32)
    if x32.shape[-1] % BLOCK:
        raise ValueError("the last dimension must be a multiple of 16")
    if per_row:
        g = (np.max(np.abs(x32), axis=-1, keepdims=True) / F32(448.0 * 6.0)).astype(F32)
    else:
        g = tensor_scale(x32) if g is None else F32(g)
    blocks = x32.reshape(x32.shape[:-1] + (x32.shape[-1] // BLOCK, BLOCK))
    amax = np.max(np.abs(blocks), axis=-1)
    gb = np.broadcast_to(np.asarray(g, F32), amax.shape[:-1] + (1,)) if per_row else np.full((1,), g, F32)
    ok = gb > 0
    denom = np.where(ok, F32(6.0) * gb, F32(1.0)).astype(F32)
    sb = np.where(ok, e4m3_encode((amax / denom).astype(F32)), np.uint8(0)).astype(np.uint8)
    sbv = e4m3_decode(sb).astype(F32)
    step = (sbv * gb).astype(F32)
    safe = np.where(step > 0, step, F32(1.0)).astype(F32)
    y = np.where(step[..., None] > 0, blocks / safe[..., None], F32(0.0)).astype(F32)
    codes = e2m1_encode(y).reshape(x32.shape)
    return codes, sb, (g if per_row else F32(g))


def dequantize(codes, sb, g) -> np.ndarray:
    c = e2m1_decode(codes)
    blocks = c.reshape(c.shape[:-1] + (c.shape[-1] // BLOCK, BLOCK))
    g64 = np.asarray(g, F64)
    scale = e4m3_decode(sb) * (g64 if g64.ndim == 0 else g64)
    return (blocks * scale[..., None]).reshape(c.shape)


def fake_quant(x) -> np.ndarray:
    """Quantise with one tensor scale and dequantise."""
    return dequantize(*quantize(x))


def fake_quant_rows(x) -> np.ndarray:
    """Quantise with one second-level scale per row and dequantise (the
    block's activations)."""
    return dequantize(*quantize(x, per_row=True))


def quantize_block_weights(w: dict) -> dict:
    """NVFP4 copy of one block's weights (klein_inputs layout; the blocks of 16
    run along each stored row, the GEMM's K)."""
    return {"w_in_nv": quantize(w["w_in"]), "w_out_nv": quantize(w["w_out"]),
            "q_norm": w["q_norm"], "k_norm": w["k_norm"]}
