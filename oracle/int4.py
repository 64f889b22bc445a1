"""INT4 group-64 quantiser of the SVDQuant arm in plain NumPy — test
infrastructure (see ``oracle/__init__``).

Source: "FastWAM UR3 3-task — 4-bit quantisations" (model card), the top
comparison table, SVDQuant column: INT4 elements, groups of 64 on both the
weights and the activations ("W4A4, both at group 64"), the products on integer
tensor cores, exact for 4-bit codes; its "size" row, 4.5798 bits per weight;
and section "Verification — INT4 SVDQuant" (activation scales bit-identical to
the formula, codes within one step).  The pages print neither the scale nor
the rounding.  Readings, one each:

* symmetric signed INT4, levels -8..7, one scale per group of 64 consecutive
  elements along K of one row (a weight's output row, an activation's token);
* the scale is 16-bit, IEEE fp16: 4 bits per element plus 16 bits per 64
  elements is 4.25 bits, and the rank-r branch of the method (bf16 L1 [N, r]
  and L2 [r, K]) adds 512 (1/K + 1/N) bits per weight at r = 32 (0.33 at
  3072 x 3072): the card's 4.58 follows, where 32-bit scales would give 4.83
  and 8-bit ones 4.46;
* each step one correctly rounded fp32 operation, then one fp16 rounding:

      a = max |v| over the group;  t = a / 7;  s = fp16_rn_satfinite(t)
      rs = 1 / s;  code_i = clamp(rint(v_i * rs), -8, 7)    (rint: half to even)
      every code 0 when s == 0 (an all-zero group, or t below half the
      smallest fp16 subnormal)

  a / 7 maps the largest magnitude onto level 7; reciprocal then multiply is
  the order the FP8 arm's reading takes; a t above the largest fp16
  saturates to 65504, and then the clamp decides (the one case that can
  give -8);
* dequant: code * s, exact in float64.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
GROUP = 64
FP16_MAX = 65504.0


def fp16_rn_satfinite(t) -> np.ndarray:
    """fp32 -> nearest fp16 (ties to even), magnitudes beyond the largest
    finite fp16 saturate to +-65504.  Returned as float16."""
    t = np.asarray(t, dtype=np.float32)
    with np.errstate(over="ignore"):
        h = t.astype(np.float16)  # IEEE round to nearest even
    return np.where(np.isinf(h) & np.isfinite(t), np.float16(FP16_MAX) * np.sign(t).astype(np.float16), h)


def quantize(T) -> tuple[np.ndarray, np.ndarray]:
    """Group-64 INT4 quantiser on a fp32 tensor T [rows, K] (K % 64 == 0).
    Returns ``(codes, scales)``: codes int8 [rows, K] in -8..7, scales fp16
    [rows, K / 64]."""
    T = np.asarray(T)
    if T.dtype != np.float32:
        raise TypeError("the quantiser input is fp32 by definition")
    rows, K = T.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 64")
    G = T.reshape(rows, K // GROUP, GROUP)
    a = np.abs(G).max(axis=2)                      # exact
    t = a / F32(7.0)                               # RN division (fp32 / fp32)
    assert t.dtype == np.float32
    s16 = fp16_rn_satfinite(t)
    s = s16.astype(np.float32)                     # exact widening
    with np.errstate(divide="ignore"):
        rs = np.where(s > 0, F32(1.0) / np.where(s > 0, s, F32(1.0)), F32(0.0)).astype(np.float32)  # RN reciprocal
    q = G * rs[:, :, None]                         # RN multiply
    assert q.dtype == np.float32
    codes = np.clip(np.rint(q), -8, 7).astype(np.int8)  # rint: half to even
    codes = np.where((s > 0)[:, :, None], codes, np.int8(0)).astype(np.int8)
    return codes.reshape(rows, K), s16


def dequantize(codes, scales) -> np.ndarray:
    """float64 value of every element: code * s of its group (exact)."""
    codes = np.asarray(codes, dtype=np.float64)
    rows, K = codes.shape
    s = np.asarray(scales, dtype=np.float64)
    return (codes.reshape(rows, K // GROUP, GROUP) * s[:, :, None]).reshape(rows, K)


def group_products(codes_a, codes_b) -> np.ndarray:
    """The integer tensor-core step: P[g, m, n] = sum over group g of
    a[m, k] b[n, k], exact (int64)."""
    A = np.asarray(codes_a, dtype=np.int64)
    B = np.asarray(codes_b, dtype=np.int64)
    M, K = A.shape
    N = B.shape[0]
    Ag = A.reshape(M, K // GROUP, GROUP).transpose(1, 0, 2)
    Bg = B.reshape(N, K // GROUP, GROUP).transpose(1, 2, 0)
    return Ag @ Bg


def group_gemm(codes_a, scales_a, codes_b, scales_b) -> np.ndarray:
    """The INT4 product as the hardware forms it: the exact integer group sums
    P[g] scaled by s_a[m, g] s_b[n, g] and summed over the groups, in
    float64."""
    P = group_products(codes_a, codes_b).astype(np.float64)
    sa = np.asarray(scales_a, dtype=np.float64).T[:, :, None]   # [G, M, 1]
    sb = np.asarray(scales_b, dtype=np.float64).T[:, None, :]   # [G, 1, N]
    return (P * sa * sb).sum(axis=0)
