"""Pins of the SVDQuant arm's oracle (oracle.int4 and asp.svdquant_linear)
against what the pages and the mathematics fix, not against a retyping of it:

* the hand-worked example in tests/golden/int4_group64_worked_example.txt
  (model card, top table, SVDQuant column: INT4, group 64);
* brute force: every code is the level nearest to v * rs among -8..7, ties to
  the even level, and every scale is torch's fp16 rounding of amax / 7;
* the largest magnitude of a group lands on +-7 and the dequantisation error
  stays within half a step;
* the integer group sums times the two scales equal the dequantised product;
* the layer without quantisation is x W^T + bias for any V (the branch and
  the residual add back up), and with V from numpy's SVD the branch is the
  rank-r truncated SVD of W diag(s) and the residual holds the rest of its
  spectrum;
* the activation side of the arm is not deflated: the quantiser sees x / s.
"""
import os

import numpy as np
import pytest

from oracle import asp, int4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "int4_group64_worked_example.txt")


def read_golden():
    T = np.zeros((3, 128), dtype=np.float32)
    codes, scales = {}, {}
    for line in open(GOLDEN):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "E":
            r, c = int(f[1]), int(f[2])
            T[r, c] = np.float32(float(f[3]))
            codes[(r, c)] = int(f[4])
        elif f[0] == "S":
            scales[(int(f[1]), int(f[2]))] = float(f[3])
    return T, codes, scales


def test_worked_example():
    T, want_codes, want_scales = read_golden()
    codes, scales = int4.quantize(T)
    assert codes.dtype == np.int8 and scales.dtype == np.float16
    for (r, c), q in want_codes.items():
        assert codes[r, c] == q, (r, c)
    for (r, g), s in want_scales.items():
        assert float(scales[r, g]) == s, (r, g)
    # every element the file does not list is zero and codes to zero
    listed = np.zeros_like(codes, dtype=bool)
    for (r, c) in want_codes:
        listed[r, c] = True
    assert np.all(codes[~listed] == 0)


def brute_force_codes(T, scales):
    """The nearest of the 16 levels to v * rs (fp32, the reciprocal of the
    fp16 scale), ties to the even level; zero where the scale is zero."""
    rows, K = T.shape
    s = scales.astype(np.float32).repeat(64, axis=1)
    with np.errstate(divide="ignore"):
        rs = np.where(s > 0, np.float32(1) / np.where(s > 0, s, 1), 0).astype(np.float32)
    q = (T * rs).astype(np.float64)
    levels = np.arange(-8, 8, dtype=np.float64)
    d = np.abs(q[..., None] - levels)
    best = d.min(axis=-1, keepdims=True)
    cand = np.where(d == best, levels, np.nan)
    # among equal distances (a tie) take the even level
    even = np.where(np.isfinite(cand) & (np.mod(cand, 2) == 0), cand, np.nan)
    pick = np.where(np.isfinite(even).any(axis=-1), np.nanmax(np.where(np.isfinite(even), even, -99), axis=-1),
                    np.nanmax(np.where(np.isfinite(cand), cand, -99), axis=-1))
    return np.where(s > 0, pick, 0).astype(np.int8)


@pytest.mark.parametrize("seed,scale", [(0, 1.0), (1, 1e-3), (2, 300.0), (3, 1e-6)])
def test_codes_are_nearest_levels_and_scales_are_fp16_of_amax_over_7(seed, scale):
    import torch
    rng = np.random.default_rng(seed)
    T = (rng.standard_normal((37, 256)) * scale).astype(np.float32)
    T[3, :64] = 0.0                     # an all-zero group
    T[5, 64:128] *= 1000.0              # a group with an outlier scale
    codes, scales = int4.quantize(T)
    amax = np.abs(T.reshape(37, 4, 64)).max(axis=2)
    t = torch.from_numpy(amax) / 7.0    # fp32 division in torch
    want = t.to(torch.float16)
    want = torch.where(torch.isinf(want), torch.full_like(want, 65504.0), want)  # satfinite
    assert np.array_equal(scales, want.numpy())
    assert np.array_equal(codes, brute_force_codes(T, scales))


def test_group_maximum_is_level_7_and_error_within_half_a_step():
    rng = np.random.default_rng(4)
    T = rng.standard_normal((16, 512)).astype(np.float32)
    codes, scales = int4.quantize(T)
    G = T.reshape(16, 8, 64)
    arg = np.abs(G).argmax(axis=2)
    top = np.take_along_axis(codes.reshape(16, 8, 64), arg[:, :, None], axis=2)[:, :, 0]
    sign = np.sign(np.take_along_axis(G, arg[:, :, None], axis=2)[:, :, 0])
    assert np.all(top == 7 * sign)
    err = np.abs(int4.dequantize(codes, scales) - T.astype(np.float64)).reshape(16, 8, 64)
    step = scales.astype(np.float64)[:, :, None]
    assert np.all(err <= 0.5 * step * (1 + 1e-3))


def test_codes_span_every_level_in_range():
    T = (np.arange(-7, 8, dtype=np.float32) / 7.0).repeat(1)
    T = np.concatenate([T, np.zeros(64 - T.size, dtype=np.float32)])[None, :]
    codes, scales = int4.quantize(T)
    assert float(scales[0, 0]) == float(np.float16(np.float32(1) / np.float32(7)))
    assert list(codes[0, :15]) == list(range(-7, 8))


def test_group_sums_equal_dequantised_product():
    rng = np.random.default_rng(5)
    A = rng.standard_normal((9, 192)).astype(np.float32)
    B = rng.standard_normal((11, 192)).astype(np.float32)
    ca, sa = int4.quantize(A)
    cb, sb = int4.quantize(B)
    # explicit loops for one element, then the whole matrix
    m, n = 4, 7
    acc = 0.0
    for g in range(3):
        P = sum(int(ca[m, 64 * g + k]) * int(cb[n, 64 * g + k]) for k in range(64))
        acc += float(sa[m, g]) * float(sb[n, g]) * P
    full = int4.group_gemm(ca, sa, cb, sb)
    assert abs(full[m, n] - acc) <= 1e-12 * max(1.0, abs(acc))
    ref = int4.dequantize(ca, sa) @ int4.dequantize(cb, sb).T
    assert np.allclose(full, ref, rtol=1e-12, atol=1e-12)
    # the group sums are integers of at most 64 * 8 * 8 in magnitude
    P = int4.group_products(ca, cb)
    assert np.abs(P).max() <= 64 * 64


def test_fp16_saturation_and_underflow():
    s = int4.fp16_rn_satfinite(np.array([65504.0, 65519.0, 65520.0, 1e9, -1e9, 2.0 ** -25, 2.0 ** -24], np.float32))
    assert list(s.astype(np.float64)) == [65504.0, 65504.0, 65504.0, 65504.0, -65504.0, 0.0, 2.0 ** -24]


def layer(seed=6, M=24, K=256, N=48, r=16):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) / np.sqrt(K)
    s = np.exp(rng.uniform(-1, 1, K))
    bias = rng.standard_normal(N)
    Wh = W * s[None, :]
    V = np.linalg.svd(Wh)[2][:r].T           # top right singular vectors of W diag(s)
    return x, W, s, V, bias, Wh


def test_unquantised_arm_is_the_plain_linear():
    x, W, s, V, bias, _ = layer()
    y = asp.svdquant_linear(x, W, s, V, bias, fp4=False)
    assert np.allclose(y, x @ W.T + bias[None, :], rtol=1e-12, atol=1e-10)
    # any orthonormal V, not only the singular one
    rng = np.random.default_rng(7)
    Q = np.linalg.qr(rng.standard_normal((256, 16)))[0]
    y2 = asp.svdquant_linear(x, W, s, Q, bias, fp4=False)
    assert np.allclose(y2, x @ W.T + bias[None, :], rtol=1e-12, atol=1e-10)


def test_branch_is_truncated_svd_and_residual_holds_the_rest():
    x, W, s, V, bias, Wh = layer()
    wp = asp.prepare_weight(W, s, V, 1, fmt="int4")
    U, S, Vt = np.linalg.svd(Wh)
    r = V.shape[1]
    trunc = (U[:, :r] * S[:r]) @ Vt[:r]
    assert np.allclose(wp["L"] @ V.T, trunc, atol=1e-12)
    assert np.allclose(np.linalg.svd(wp["Wd"], compute_uv=False)[: len(S) - r], S[r:], atol=1e-10)
    assert np.allclose(wp["Wd"] @ V, 0.0, atol=1e-12)


def test_activation_side_is_not_deflated():
    x, W, s, V, bias, _ = layer()
    y, parts = asp.svdquant_linear(x, W, s, V, bias, parts=True)
    ap = parts["act"]
    assert np.array_equal(ap["z"], x / s[None, :])
    codes, scales = int4.quantize((x / s[None, :]).astype(np.float32))
    assert np.array_equal(ap["codes"], codes) and np.array_equal(ap["scales"], scales)
    # the product and the branch it adds up from
    want = int4.group_gemm(ap["codes"], ap["scales"], parts["wt"]["codes"], parts["wt"]["scales"])
    want = want + (x / s[None, :]) @ V @ parts["wt"]["L"].T + bias[None, :]
    assert np.allclose(y, want, rtol=1e-12, atol=1e-10)
    # and it is a 4-bit approximation of the layer
    assert asp.rel_fro(y, x @ W.T + bias[None, :]) < 0.2


def test_arm_argument_checks():
    x, W, s, V, bias, _ = layer()
    with pytest.raises(ValueError):
        asp.asp_linear(x, W, s, V, bias, 2, variant="svdquant", fmt="int4")
    with pytest.raises(ValueError):
        asp.asp_linear(x, W, s, V, bias, 1, variant="deflated", fmt="int4")
    with pytest.raises(ValueError):
        asp.asp_linear(x, W, s, V, bias, 1, variant="svdquant", fmt="nvfp4")
