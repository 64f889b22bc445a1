"""Pins for the oracle's layer formula (CPU only).

The deflated ASP contract ("FastWAM UR3 3-task — 4-bit quantisations", section
"What ASP is, and what the deflated form means") is checked against what the
mathematics fixes: orthonormality, projector idempotence, exact reduction to
x W^T + bias when nothing is quantised, the r = 0 and r = K special cases, the
"input in span(V)" case, and brute-force summation for the FP4 product.
"""
import numpy as np
import pytest
import scipy.linalg

from oracle import asp, nvfp4
from bit_w4a4_quantised_b200 import workloads


@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128])
def test_hadamard_orthonormal_and_matches_scipy(b):
    S = asp.sylvester(b)
    assert np.array_equal(S, scipy.linalg.hadamard(b))        # library pin
    H = asp.block_hadamard(4 * b, b)
    assert np.abs(H @ H.T - np.eye(4 * b)).max() <= 1e-15


@pytest.mark.parametrize("b", [1, 16, 128])
def test_block_product_equals_dense(b):
    rng = np.random.default_rng(1)
    T = rng.standard_normal((5, 256))
    assert np.abs(asp.apply_block_hadamard(T, b) - T @ asp.block_hadamard(256, b)).max() < 1e-13


def test_generated_basis_is_orthonormal():
    case = workloads.c1_tiny()
    V = case.V.astype(np.float64)
    assert np.abs(V.T @ V - np.eye(V.shape[1])).max() < 1e-6       # fp32 storage
    G = np.random.default_rng(0).standard_normal((256, 32))
    Q, _ = np.linalg.qr(G)
    assert np.abs(Q.T @ Q - np.eye(32)).max() < 1e-12
    P = np.eye(256) - Q @ Q.T
    assert np.abs(P @ P - P).max() < 1e-12                           # idempotent


def test_deflated_weight_is_orthogonal_to_basis():
    case = workloads.c1_tiny()
    Q, _ = np.linalg.qr(np.random.default_rng(2).standard_normal((case.K, 32)))
    wp = asp.prepare_weight(case.W, case.s, Q, case.b, fp4=False)
    assert np.abs(wp["Wd"] @ Q).max() < 1e-12 * np.abs(wp["Wt"]).max() * case.K


@pytest.mark.parametrize("r", [0, 16, 32])
@pytest.mark.parametrize("b", [1, 16, 128])
def test_identity_quantiser_gives_plain_linear(r, b):
    rng = np.random.default_rng(r + b)
    M, K, N = 12, 256, 40
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) * 0.02
    s = np.exp(rng.uniform(-1, 1, K))
    V = np.linalg.qr(rng.standard_normal((K, r)))[0] if r else np.zeros((K, 0))
    bias = rng.standard_normal(N) * 0.01
    y = asp.asp_linear(x, W, s, V, bias, b, fp4=False)
    ref = x @ W.T + bias
    assert asp.rel_fro(y, ref) < 1e-12


def test_rank_K_gives_unquantised_product():
    # I - VV^T = 0: the FP4 path carries only rounding noise, y = x W^T + bias
    rng = np.random.default_rng(4)
    for K in (16, 32, 64):
        M, N = 8, 24
        x = rng.standard_normal((M, K))
        W = rng.standard_normal((N, K)) * 0.02
        s = np.exp(rng.uniform(-1, 1, K))
        V = np.linalg.qr(rng.standard_normal((K, K)))[0]
        bias = rng.standard_normal(N) * 0.01
        y = asp.asp_linear(x, W, s, V, bias, 16 if K >= 16 else 1)
        assert asp.rel_fro(y, x @ W.T + bias) < 1e-12


def test_input_in_span_gives_exact_low_rank_product():
    # b = 1 (H = I), power-of-two s and identity-column V make every step exact:
    # z == 0 bit for bit, the FP4 side takes the all-zero path, and y equals the
    # exact low-rank product plus bias
    rng = np.random.default_rng(6)
    M, K, N, r = 16, 64, 32, 8
    cols = rng.choice(K, r, replace=False)
    V = np.zeros((K, r))
    V[cols, np.arange(r)] = 1.0
    s = 2.0 ** rng.integers(-3, 4, K)
    xt = np.zeros((M, K))
    xt[:, cols] = rng.standard_normal((M, r))
    x = xt * s
    W = rng.standard_normal((N, K)) * 0.02
    bias = rng.standard_normal(N) * 0.01
    y, parts = asp.asp_linear(x, W, s, V, bias, 1, parts=True)
    act = parts["act"]
    assert np.all(act["z"] == 0) and act["g"] == 1.0
    assert np.all(act["scales"] == 0) and np.all(act["codes"] == 0)
    assert np.array_equal(parts["y_fp4"], np.zeros((M, N)))
    Wt = W * s
    assert np.array_equal(y, (xt @ V) @ (Wt @ V).T + bias)


def test_input_in_span_with_rotation_and_qr_basis():
    rng = np.random.default_rng(8)
    M, K, N, r, b = 16, 256, 32, 32, 128
    V = np.linalg.qr(rng.standard_normal((K, r)))[0]
    s = np.exp(rng.uniform(-1, 1, K))
    xt = rng.standard_normal((M, r)) @ V.T
    x = asp.apply_block_hadamard(xt, b) * s      # H is symmetric and orthonormal
    W = rng.standard_normal((N, K)) * 0.02
    act = asp.activation_prologue(x, s, V, b, fp4=False)
    assert np.abs(act["z"]).max() < 1e-13 * np.abs(xt).max()
    y = asp.asp_linear(x, W, s, V, None, b, fp4=False)
    assert asp.rel_fro(y, xt @ asp.rotate_weight(W, s, b).T) < 1e-12


def test_rank0_s1_b1_is_textbook_nvfp4_gemm():
    # with r = 0, s = 1, b = 1 the layer is quantise(x), quantise(W), then
    # dequantise-and-multiply; checked against explicit per-element sums
    rng = np.random.default_rng(10)
    M, K, N = 6, 64, 5
    x = rng.standard_normal((M, K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    bias = rng.standard_normal(N)
    y = asp.asp_linear(x, W, np.ones(K), None, bias, 1)
    ca, sa, ga = nvfp4.quantize(x)
    cb, sb, gb = nvfp4.quantize(W)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                ia, ib = int(ca[m, k]), int(cb[n, k])
                va = nvfp4.E2M1_MAGNITUDES[ia & 7] * (-1.0 if ia >> 3 else 1.0)
                vb = nvfp4.E2M1_MAGNITUDES[ib & 7] * (-1.0 if ib >> 3 else 1.0)
                acc += va * nvfp4.E4M3_MAGNITUDES[sa[m, k // 16]] * vb * nvfp4.E4M3_MAGNITUDES[sb[n, k // 16]]
            want = acc * float(ga) * float(gb) + bias[n]
            assert abs(y[m, n] - want) <= 1e-13 * max(1.0, abs(want))


def test_fp4_gemm_brute_force_16x16_exact():
    # integer-exact: with g = 1 every product and partial sum is exact in f64
    rng = np.random.default_rng(12)
    ca = rng.integers(0, 16, (16, 16)).astype(np.uint8)
    cb = rng.integers(0, 16, (16, 16)).astype(np.uint8)
    sa = rng.integers(0, 127, (16, 1)).astype(np.uint8)
    sb = rng.integers(0, 127, (16, 1)).astype(np.uint8)
    got = asp.nvfp4_gemm(nvfp4.dequantize(ca, sa, 1.0), nvfp4.dequantize(cb, sb, 1.0))
    for m in range(16):
        for n in range(16):
            acc = 0.0
            for k in range(16):
                acc += (float(nvfp4.decode_e2m1(ca[m, k])) * nvfp4.E4M3_MAGNITUDES[sa[m, 0]]
                        * float(nvfp4.decode_e2m1(cb[n, k])) * nvfp4.E4M3_MAGNITUDES[sb[n, 0]])
            assert got[m, n] == acc


def test_c1_error_budget():
    # the full oracle on the tiny config stays near the unquantised layer:
    # FP4 noise only, well inside a few percent
    case = workloads.c1_tiny()
    y = asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, case.b)
    ref = case.x.astype(np.float64) @ case.W.astype(np.float64).T + case.bias
    err = asp.rel_fro(y, ref)
    assert 1e-3 < err < 0.2


# ---------------------------------------------------------------------------
# The shared-weight arm (one quantised weight W~, branch weight deq(Q(W~)) V).
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("r", [16, 32])
@pytest.mark.parametrize("b", [1, 16, 128])
def test_shared_identity_quantiser_gives_plain_linear(r, b):
    # z W~^T + u (W~V)^T = x~ W~^T - u V^T W~^T + u V^T W~^T = x W^T
    rng = np.random.default_rng(100 + r + b)
    M, K, N = 12, 256, 40
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) * 0.02
    s = np.exp(rng.uniform(-1, 1, K))
    V = np.linalg.qr(rng.standard_normal((K, r)))[0]
    bias = rng.standard_normal(N) * 0.01
    y = asp.asp_linear(x, W, s, V, bias, b, fp4=False, variant="shared")
    assert asp.rel_fro(y, x @ W.T + bias) < 1e-12


def test_shared_rank0_is_the_deflated_arm():
    # with no subspace both arms quantise the same W~ and have no branch
    case = workloads.custom(16, 256, 48, 0, 16, seed=101, n_outliers=2)
    a = asp.asp_linear(case.x, case.W, case.s, None, case.bias, 16)
    b_ = asp.asp_linear(case.x, case.W, case.s, None, case.bias, 16, variant="shared")
    assert np.array_equal(a, b_)


def test_shared_weight_codes_are_the_quantised_rotated_weight():
    case = workloads.custom(8, 256, 32, 32, 16, seed=102, n_outliers=2)
    wp = asp.prepare_weight_shared(case.W, case.s, case.V, 16)
    c, sc, g = nvfp4.quantize(asp.rotate_weight(case.W, case.s, 16).astype(np.float32))
    assert np.array_equal(wp["codes"], c) and np.array_equal(wp["scales"], sc) and wp["g"] == g
    dp = asp.prepare_weight(case.W, case.s, case.V, 16)
    assert not np.array_equal(dp["codes"], wp["codes"])      # the deflated arm quantises W_d


def test_shared_input_in_span_uses_the_quantised_weight_columns():
    # exact construction as for the deflated arm (b = 1, 2^k smoothing,
    # identity-column V): z == 0, and the branch weight is the picked columns of
    # the dequantised stored weight, so y is an explicit product of those
    rng = np.random.default_rng(103)
    M, K, N, r = 16, 64, 32, 8
    cols = rng.choice(K, r, replace=False)
    V = np.zeros((K, r))
    V[cols, np.arange(r)] = 1.0
    s = 2.0 ** rng.integers(-3, 4, K)
    xt = np.zeros((M, K))
    xt[:, cols] = rng.standard_normal((M, r))
    x = xt * s
    W = rng.standard_normal((N, K)) * 0.02
    bias = rng.standard_normal(N) * 0.01
    y, parts = asp.asp_linear(x, W, s, V, bias, 1, parts=True, variant="shared")
    assert np.all(parts["act"]["z"] == 0) and np.array_equal(parts["y_fp4"], np.zeros((M, N)))
    c, sc, g = nvfp4.quantize((W * s).astype(np.float32))
    deq = nvfp4.dequantize(c, sc, g)
    want = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            want[m, n] = sum(xt[m, cols[j]] * deq[n, cols[j]] for j in range(r)) + bias[n]
    assert np.allclose(y, want, rtol=1e-14, atol=1e-15)
    # the deflated arm's branch uses the exact W~V instead
    yd = asp.asp_linear(x, W, s, V, bias, 1, variant="deflated")
    assert np.allclose(yd, xt[:, cols] @ (W * s)[:, cols].T + bias, rtol=1e-14, atol=1e-15)
