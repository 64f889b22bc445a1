"""FP8 (E4M3) per-tensor quantiser in plain NumPy — test infrastructure (see
``oracle/__init__``).

Source: "QuantWAMs: Calibrating at the Right Granularity for World Action
Models" (report), section "During inference": the default backend runs NVFP4
W4A4 and FP8 W8A8 for the Linears that calibration upgrades.  The pages name
the format (FP8, weights and activations) and nothing else.  Readings, one
each:

* elements are E4M3 (the "fn" variant: 4 exponent bits with bias 7, 3 mantissa
  bits, largest magnitude 448, subnormals m * 2**-9, no infinities), the FP8
  format the B200 tensor cores take next to E5M2 and the one with more
  mantissa for activations;
* one fp32 scale per tensor, g = amax / 448 (g = 1 when amax = 0): per call
  for activations, once at prepare for weights, as the NVFP4 arm's per-tensor
  scale;
* the quantiser's fp32 operation order follows the NVFP4 arm's element step
  (reciprocal, then multiply; each one correctly rounded fp32 operation):

      rg = 1 / g;  q_i = T_i * rg;  code_i = sign(T_i) << 7 | E4M3_RNE_satfinite(|q_i|)

* zero codes keep the input's sign bit (-0.0 -> 0x80), as in the NVFP4 arm;
* dequant: e4m3(code & 0x7F) * (-1 if code & 0x80) * g.

The E4M3 encoder is the brute-force nearest-even table search of
``oracle.nvfp4`` (no library float8 cast).
"""
from __future__ import annotations

import numpy as np

from . import nvfp4

F32 = np.float32
#: Largest finite E4M3 magnitude: the per-tensor scale maps amax onto it.
E4M3_MAX = nvfp4.E4M3_MAX


def quantize(T) -> tuple[np.ndarray, np.float32]:
    """Per-tensor FP8 E4M3 quantiser on a fp32 tensor T.  Returns
    ``(codes, g)``: codes uint8 with T's shape (sign bit 7, magnitude code in
    bits 0..6) and the fp32 per-tensor scale g."""
    T = np.asarray(T)
    if T.dtype != np.float32:
        raise TypeError("the quantiser input is fp32 by definition")
    A = np.abs(T).max() if T.size else F32(0)
    g = F32(1.0) if A == 0 else F32(A) / F32(E4M3_MAX)        # RN division
    rg = F32(1.0) / g                                          # RN reciprocal
    q = T * rg                                                 # RN multiply, no FMA
    assert q.dtype == np.float32
    mag = nvfp4.encode_e4m3_satfinite(np.abs(q))
    sign = np.signbit(T).astype(np.uint8) << 7
    return (sign | mag).astype(np.uint8), F32(g)


def decode(codes) -> np.ndarray:
    """Signed float64 value of FP8 E4M3 codes (no NaN codes expected)."""
    codes = np.asarray(codes, dtype=np.int64)
    mag = nvfp4.decode_e4m3(codes & 0x7F)
    return np.where(codes & 0x80, -mag, mag)


def dequantize(codes, g) -> np.ndarray:
    """float64 value of every element: e4m3(code) * g (exact in float64)."""
    return decode(codes) * float(g)
