"""Rowwise FP8 (e4m3) quantisation for the oracle. Test infrastructure.

The Diffusers release blog for FLUX.3 Image Klein ("Smaller GPUs, single
files, and custom LoRA training") ships the transformer in a rowwise FP8
format besides bf16, and the local-run guide ("The text encoder" / quantised
files) says FP8 runs natively on Blackwell. The pages give no more than that.
READING (the plainest one the name supports): every linear layer of the
blocks keeps its weight as e4m3 codes with one fp32 scale per output row,
and its input activation is quantised the same way at run time, one scale per
token row; the product is the code GEMM times the row scale times the column
scale.

Format: OCP 8-bit floating point, E4M3 ("fn" flavour): 1 sign bit, 4
exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the
subnormals m * 2^-9; no infinities; S.1111.111 is NaN; the largest finite
magnitude is 448. Encoding rounds to nearest, ties to even, and saturates to
+-448 (values beyond it clamp to it).

Quantisation decision, taken in float32 on both sides (it decides integer
codes): amax = max |x| over the row; inv = 448 / amax and scale = amax / 448,
each one correctly rounded float32 division; code = e4m3(fl32(x * inv)).
An all-zero row has scale 0 and codes 0. Dequantised value = decode(code) *
scale (exact in float64).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
F32 = np.float32
F64 = np.float64


def e4m3_encode(x) -> np.ndarray:
    """float32 values -> uint8 e4m3 codes (round to nearest even, saturate)."""
    x = np.asarray(x, dtype=F32).astype(F64)          # exact
    sign = np.signbit(x).astype(np.uint8) << 7
    a = np.abs(x)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, np.minimum(a, E4M3_MAX))   # +inf and > 448 clamp to 448
    code = np.zeros(a.shape, dtype=np.int64)
    # subnormal range: a < 2^-6, grid step 2^-9 (a carry to 8 steps is the
    # smallest normal, 2^-6, which is exponent field 1 mantissa 0 = code 8)
    sub = a < 2.0 ** -6
    code = np.where(sub, np.rint(a / 2.0 ** -9).astype(np.int64), code)
    # normal range: a = 2^e * (1 + f/8), e in [-6, 8]
    an = np.where(sub, 1.0, a)
    e = np.floor(np.log2(an)).astype(np.int64)
    # guard log2 rounding at exact powers of two
    e = np.where(2.0 ** e > an, e - 1, e)
    e = np.where(2.0 ** (e + 1) <= an, e + 1, e)
    frac = np.rint((an / 2.0 ** e - 1.0) * 8.0).astype(np.int64)   # rint = ties to even
    carry = frac == 8
    e = np.where(carry, e + 1, e)
    frac = np.where(carry, 0, frac)
    normal_code = (e + 7) * 8 + frac
    normal_code = np.minimum(normal_code, 0x7E)        # 480 would be NaN: saturate to 448
    code = np.where(sub, code, normal_code)
    out = (code.astype(np.uint8) | sign).astype(np.uint8)
    return np.where(nan, np.uint8(0x7F) | sign, out).astype(np.uint8)


def e4m3_decode(c) -> np.ndarray:
    """uint8 e4m3 codes -> float64 values (NaN for S.1111.111)."""
    c = np.asarray(c, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(ex == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (ex - 7))
    mag = np.where((ex == 0xF) & (m == 7), np.nan, mag)
    return s * mag


def quantize_rowwise(x) -> tuple[np.ndarray, np.ndarray]:
    """x [..., K] -> (codes uint8 [..., K], scale float32 [...]).

    The decision is taken in float32 (module docstring); x is rounded to
    float32 first.
    """
    x32 = np.asarray(x, dtype=F64).astype(F32)
    amax = np.max(np.abs(x32), axis=-1)
    nz = amax > 0
    safe = np.where(nz, amax, F32(1.0)).astype(F32)
    inv = np.where(nz, F32(E4M3_MAX) / safe, F32(0.0)).astype(F32)
    scale = np.where(nz, safe / F32(E4M3_MAX), F32(0.0)).astype(F32)
    y = (x32 * inv[..., None]).astype(F32)
    return e4m3_encode(y), scale


def dequantize(codes, scale) -> np.ndarray:
    """codes [..., K], scale [...] -> float64 [..., K]."""
    return e4m3_decode(codes) * np.asarray(scale, F64)[..., None]


def fake_quant(x) -> np.ndarray:
    """Quantise rowwise and dequantise: the value the FP8 GEMM sees."""
    return dequantize(*quantize_rowwise(x))


def quantize_block_weights(w: dict) -> dict:
    """Rowwise e4m3 copy of one block's weights (klein_inputs layout).

    w_in [27648, 3072] and w_out [3072, 12288] are both stored [out, in], so
    one scale per stored row is one scale per output channel.
    """
    wi_q, wi_s = quantize_rowwise(w["w_in"])
    wo_q, wo_s = quantize_rowwise(w["w_out"])
    return {"w_in_q": wi_q, "w_in_s": wi_s, "w_out_q": wo_q, "w_out_s": wo_s,
            "q_norm": w["q_norm"], "k_norm": w["k_norm"]}


class QuantizedModel:
    """A klein_inputs.ModelWeights whose blocks are served quantised (rowwise
    FP8 by default; `quantize` may be oracle.nvfp4.quantize_block_weights);
    everything else (embedders, modulation, in/out layers) stays as is."""

    def __init__(self, model, quantize=None):
        self.model = model
        self._quantize = quantize if quantize is not None else quantize_block_weights
        self._q: dict = {}

    def __getattr__(self, name):
        return getattr(self.model, name)

    def _quant(self, key, w):
        if key not in self._q:
            self._q[key] = self._quantize(w)
        return self._q[key]

    def stage1(self, mode: str) -> list:
        return [self._quant(("s1", mode, i), w) for i, w in enumerate(self.model.stage1(mode))]

    def joint(self) -> list:
        return [self._quant(("j", i), w) for i, w in enumerate(self.model.joint())]
