"""The ASP (deflated form) NVFP4 linear layer in float64 — test infrastructure.

Source: "FastWAM UR3 3-task — 4-bit quantisations" (model card), section
"What ASP is, and what the deflated form means":

    x~ = (x / s) H
    y  = (x~ V)(W~ V)^T + NVFP4GEMM((I - V V^T) x~, W~ (I - V V^T)) + bias

with s the per-channel smoothing vector, H a block Hadamard, V the rank-r
basis (orthonormal columns), and "deflated" meaning the protected subspace is
removed from the 4-bit path on both sides: the branch carries the exact W~V
and the FP4 weight holds W~(I - VV^T).  The branch stays 16-bit (bf16 on the
card; "16-bit low-rank branch" in the Q-WAM abstract) — in this float64 oracle
it is exact.

Readings of points the card leaves open:

* W~ = W diag(s) H: the card writes W~ = W diag(s) without H, but the branch
  pairs x~V with W~V in the same coordinates, and only with H on both sides
  does the layer reduce to x W^T + bias when nothing is quantised.
* H = blockdiag(H_b, ..., H_b), H_b = Sylvester(b) / sqrt(b) in natural order.
* x / s divides activation channels, W diag(s) scales weight input channels.
* The FP4 inputs are cast float64 -> fp32 (round to nearest) and quantised with
  ``oracle.nvfp4.quantize``; activations get a fresh per-tensor scale per call,
  the weight's is fixed at prepare time.
* y is float64 here; the device rounds it once to bf16.

Plain steps only: a library matmul is the one building block; nothing is
blocked, fused or reordered.
"""
from __future__ import annotations

import numpy as np

from . import fp8, int4, nvfp4

FORMATS = ("nvfp4", "fp8", "int4")


def _quantise(T32, fmt: str) -> dict:
    """The chosen 4-bit or 8-bit quantiser on a fp32 tensor, with its float64
    dequantisation: NVFP4 (codes, block scales, g) or FP8 E4M3 (codes, g)."""
    if fmt == "nvfp4":
        codes, scales, g = nvfp4.quantize(T32)
        return {"codes": codes, "scales": scales, "g": g, "deq": nvfp4.dequantize(codes, scales, g)}
    if fmt == "fp8":
        codes, g = fp8.quantize(T32)
        return {"codes": codes, "g": g, "deq": fp8.dequantize(codes, g)}
    if fmt == "int4":
        codes, scales = int4.quantize(T32)
        return {"codes": codes, "scales": scales, "deq": int4.dequantize(codes, scales)}
    raise ValueError(fmt)


def sylvester(b: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix of order b (a power of two):
    S(1) = [1], S(2n) = [[S, S], [S, -S]]."""
    if b < 1 or b & (b - 1):
        raise ValueError("Hadamard block must be a power of two")
    S = np.ones((1, 1))
    while S.shape[0] < b:
        S = np.block([[S, S], [S, -S]])
    return S


def block_hadamard(K: int, b: int) -> np.ndarray:
    """Orthonormal block-diagonal H (K x K) with K/b copies of S(b)/sqrt(b)."""
    if K % b:
        raise ValueError("K must be a multiple of the Hadamard block")
    Hb = sylvester(b) / np.sqrt(b)
    return np.kron(np.eye(K // b), Hb)


def apply_block_hadamard(T, b: int) -> np.ndarray:
    """T H for H = blockdiag(H_b, ...): every b-wide column group of T times
    H_b (the definition of a block-diagonal product; no dense K x K matrix)."""
    T = np.asarray(T, dtype=np.float64)
    rows, K = T.shape
    if K % b:
        raise ValueError("K must be a multiple of the Hadamard block")
    Hb = sylvester(b) / np.sqrt(b)
    return (T.reshape(rows, K // b, b) @ Hb).reshape(rows, K)


def rotate_activation(x, s, b: int) -> np.ndarray:
    """x~ = (x / s) H in float64."""
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    return apply_block_hadamard(x / s[None, :], b)


def rotate_weight(W, s, b: int) -> np.ndarray:
    """W~ = W diag(s) H in float64."""
    W = np.asarray(W, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    return apply_block_hadamard(W * s[None, :], b)


def deflate(T, V):
    """Split rows of T into the rank-r coordinates c = T V and the remainder
    T (I - V V^T) = T - c V^T.  Returns (c, remainder); r = 0 gives (empty, T)."""
    T = np.asarray(T, dtype=np.float64)
    if V is None or np.asarray(V).shape[1] == 0:
        return np.zeros((T.shape[0], 0)), T.copy()
    V = np.asarray(V, dtype=np.float64)
    c = T @ V
    return c, T - c @ V.T


def prepare_weight(W, s, V, b: int, fp4: bool = True, fmt: str = "nvfp4") -> dict:
    """Offline side: W~, the exact branch L = W~V, the deflated weight
    W_d = W~ - L V^T, and its quantisation (codes, scales, g_w).  ``fp4=False``
    replaces the quantiser by the identity; ``fmt="fp8"`` takes the FP8 arm's
    per-tensor E4M3 quantiser instead of NVFP4."""
    Wt = rotate_weight(W, s, b)
    L, Wd = deflate(Wt, V)
    out = {"Wt": Wt, "L": L, "Wd": Wd}
    if fp4:
        out.update(_quantise(Wd.astype(np.float32), fmt))
    else:
        out["deq"] = Wd
    return out


def prepare_weight_shared(W, s, V, b: int, fp4: bool = True) -> dict:
    """Offline side of the shared-weight arm (model card, section "What ASP
    is, and what the deflated form means": the cheaper variant "quantises one
    weight and stores V alone").  Reading: the one quantised weight is W~
    itself, not deflated, and both paths use it: the FP4 product takes
    Q(W~), and the branch weight is formed from that stored weight and V,
    L = deq(Q(W~)) V, so nothing but the FP4 weight and V is stored.  The
    activation side is the deflated one of the main arm."""
    Wt = rotate_weight(W, s, b)
    out = {"Wt": Wt}
    if fp4:
        codes, scales, g = nvfp4.quantize(Wt.astype(np.float32))
        deq = nvfp4.dequantize(codes, scales, g)
        out.update(codes=codes, scales=scales, g=g, deq=deq)
    else:
        deq = Wt
        out["deq"] = deq
    if V is None or np.asarray(V).shape[1] == 0:
        out["L"] = np.zeros((Wt.shape[0], 0))
    else:
        out["L"] = deq @ np.asarray(V, dtype=np.float64)
    return out


def activation_prologue(x, s, V, b: int, fp4: bool = True, fmt: str = "nvfp4", deflated: bool = True) -> dict:
    """Per-call side: x~, u = x~V, z = x~ - u V^T, and the quantisation of z
    (NVFP4, or the FP8 arm's E4M3 with ``fmt="fp8"``).  ``deflated=False``
    (the SVDQuant arm) quantises x~ itself: z = x~."""
    xt = rotate_activation(x, s, b)
    u, z = deflate(xt, V)
    if not deflated:
        z = xt.copy()
    out = {"xt": xt, "u": u, "z": z}
    if fp4:
        out.update(_quantise(z.astype(np.float32), fmt))
    else:
        out["deq"] = z
    return out


def nvfp4_gemm(deq_a, deq_b) -> np.ndarray:
    """NVFP4GEMM on dequantised operands: deq(A) deq(B)^T in float64."""
    return np.asarray(deq_a, dtype=np.float64) @ np.asarray(deq_b, dtype=np.float64).T


def asp_linear(x, W, s, V, bias, b: int, fp4: bool = True, parts: bool = False, variant: str = "deflated",
               fmt: str = "nvfp4"):
    """The whole layer.  ``fp4=False`` replaces both quantisers by the identity
    (used to pin the formula to x W^T + bias).  ``variant="shared"`` takes the
    shared-weight arm's weight side (prepare_weight_shared).  ``fmt="fp8"`` is
    the FP8 W8A8 arm: the same layer with both quantisers FP8 E4M3 per tensor
    (oracle.fp8) and the product taken on those operands.  ``variant=
    "svdquant"`` (with ``fmt="int4"`` and b = 1) is the SVDQuant arm: see
    ``svdquant_linear``."""
    if variant not in ("deflated", "shared", "svdquant"):
        raise ValueError(variant)
    if fmt not in FORMATS or (fmt == "fp8" and variant != "deflated") or ((fmt == "int4") != (variant == "svdquant")):
        raise ValueError(f"format {fmt!r} with variant {variant!r}")
    if variant == "svdquant" and b != 1:
        raise ValueError("the SVDQuant arm has no Hadamard rotation: b = 1")
    if variant == "shared":
        wp = prepare_weight_shared(W, s, V, b, fp4=fp4)
    else:
        wp = prepare_weight(W, s, V, b, fp4=fp4, fmt=fmt)
    ap = activation_prologue(x, s, V, b, fp4=fp4, fmt=fmt, deflated=variant != "svdquant")
    y_fp4 = nvfp4_gemm(ap["deq"], wp["deq"])
    y_lr = ap["u"] @ wp["L"].T
    y = y_fp4 + y_lr
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    if parts:
        return y, {"act": ap, "wt": wp, "y_fp4": y_fp4, "y_lr": y_lr}
    return y


def svdquant_linear(x, W, s, V, bias, fp4: bool = True, parts: bool = False):
    """The SVDQuant W4A4 arm (model card, top table, SVDQuant column; "Verification
    — INT4 SVDQuant"), in this oracle's terms: smoothing x^ = x / s and
    W^ = W diag(s) with no rotation (b = 1); the low-rank branch from the
    rank-r basis V, L = W^ V, so that L V^T is the rank-r truncated SVD of W^
    when V holds its top right singular vectors (calibrating V is out of
    scope: V is an input, as on the ASP arm); the residual R = W^ - L V^T
    quantised INT4 group 64, and the activation x^ itself (not deflated)
    quantised the same way:

        y = deq(Q(x^)) deq(Q(R))^T + (x^ V) L^T + bias

    Without quantisation the two paths add up to x^ W^T^ + bias = x W^T + bias."""
    return asp_linear(x, W, s, V, bias, 1, fp4=fp4, parts=parts, variant="svdquant", fmt="int4")


def rel_fro(a, ref) -> float:
    """||a - ref||_F / ||ref||_F in float64."""
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / (den if den > 0 else 1.0))
