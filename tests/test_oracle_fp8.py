"""Pins for the FP8 (E4M3, per-tensor) quantiser of the W8A8 arm and for the
arm's layer in the oracle (CPU only).

The format is fixed by the QuantWAMs report ("During inference": FP8 W8A8 for
the upgraded Linears) and the E4M3 definition; the scale and op order are the
readings stated in ``oracle/fp8.py``.  Checked against a hand-worked table,
the E4M3 decode of every code, the torch float8_e4m3fn cast (a library pin),
the round-trip error bound, the zero tensor, and explicit sums for a tiny
layer.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_quantised_b200 import workloads
from conftest import read_golden
from oracle import asp, fp8, nvfp4


def _golden(case):
    rows = [r for r in read_golden("fp8_quantizer_worked_example.txt") if r[0] == case]
    return np.array([float(r[1]) for r in rows], dtype=np.float32), np.array([int(r[2], 16) for r in rows])


def test_worked_example_g_equal_one():
    vals, codes = _golden("A")
    T = np.concatenate([vals, np.float32([448.0])])[None, :]   # amax 448 -> g = 1
    c, g = fp8.quantize(T)
    assert g == np.float32(1.0)
    assert np.array_equal(c[0, :len(vals)], codes)


def test_worked_example_scale_order():
    vals, codes = _golden("B")
    c, g = fp8.quantize(vals[None, :])
    assert g == np.float32(3.0) / np.float32(448.0)
    assert np.array_equal(c[0], codes)


def test_decode_every_code():
    # positive codes decode to the E4M3 values, the sign bit negates
    for code in range(127):
        e, m = code >> 3, code & 7
        want = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        assert fp8.decode(code) == want and fp8.decode(code | 0x80) == -want


def test_encoder_matches_torch_float8_cast():
    # library pin: round-to-nearest-even inside the finite range
    rng = np.random.default_rng(3)
    q = np.concatenate([rng.uniform(0, 448, 20000), 2.0 ** rng.uniform(-12, 8.8, 20000)]).astype(np.float32)
    q = q[q <= 448.0]
    ours = nvfp4.encode_e4m3_satfinite(q)
    theirs = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_round_trip_error_bound():
    rng = np.random.default_rng(4)
    T = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-4, 4, (64, 1)))).astype(np.float32)
    c, g = fp8.quantize(T)
    d = fp8.dequantize(c, g)
    q = np.abs(T.astype(np.float64)) / float(g)
    # half a code step: 2^-4 relative for normals (3 mantissa bits), 2^-10
    # absolute for subnormals, in units of g; plus the fp32 roundings of 1 / g
    # and of the product
    half = np.where(q >= 2.0 ** -6, q * 2.0 ** -4, 2.0 ** -10) * float(g)
    assert np.all(np.abs(d - T) <= half * (1 + 1e-6) + 1e-30)
    assert np.abs(d).max() <= 448.0 * float(g) * (1 + 1e-6)


def test_zero_tensor_and_signs():
    T = np.array([[0.0, -0.0, 0.0, -0.0]], dtype=np.float32)
    c, g = fp8.quantize(T)
    assert g == np.float32(1.0) and list(c[0]) == [0x00, 0x80, 0x00, 0x80]


def test_fp8_layer_explicit_sums():
    # r = 0, s = 1, b = 1: quantise x and W per tensor, multiply the decoded
    # codes, scale by g_x g_w, add the bias
    rng = np.random.default_rng(5)
    M, K, N = 5, 64, 7
    x = rng.standard_normal((M, K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    bias = rng.standard_normal(N)
    y = asp.asp_linear(x, W, np.ones(K), None, bias, 1, fmt="fp8")
    ca, ga = fp8.quantize(x)
    cb, gb = fp8.quantize(W)
    for m in range(M):
        for n in range(N):
            acc = sum(float(fp8.decode(ca[m, k])) * float(fp8.decode(cb[n, k])) for k in range(K))
            want = acc * float(ga) * float(gb) + bias[n]
            assert abs(y[m, n] - want) <= 1e-13 * max(1.0, abs(want))


def test_fp8_arm_is_closer_to_the_unquantised_layer():
    # every normal E4M3 element is within 2^-4 relative of its input (3
    # mantissa bits), so the layer's relative error stays below that; E2M1 has
    # one mantissa bit, and the W4A4 arm's error on the same layer is several
    # times larger (3.6x on this one)
    case = workloads.c2_action_attn()
    exact = case.x.astype(np.float64) @ case.W.astype(np.float64).T + case.bias
    e4 = asp.rel_fro(asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, case.b), exact)
    e8 = asp.rel_fro(asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, case.b, fmt="fp8"), exact)
    assert e8 < 2.0 ** -4 and e8 < e4 / 3, (e8, e4)
