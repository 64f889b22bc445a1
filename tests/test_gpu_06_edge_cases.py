"""The method's degenerate cases on the device, through the C-ABI, against the
float64 oracle.

The deflated ASP layer ("FastWAM UR3 3-task — 4-bit quantisations", section
"What ASP is, and what the deflated form means") sends only the part of x~
outside span(V) through the 4-bit path.  Three inputs make that exact:

1. x~ in span(V): with b = 1 (H = I), power-of-two s and identity-column V
   every step of the prologue is exact, so z is zero everywhere, the
   per-tensor amax is 0 (g_x = 1), every block scale is 0, every code carries
   only a sign, and y is the low-rank product u (W~V)^T + bias, up to the
   bf16 rounding of the branch operands and of y.
2. x = 0: z = 0 and u = 0, so y is the bias, bit for bit.
3. r = 0, s = 1, b = 1: the layer is the textbook NVFP4 GEMM: quantise x and W
   (both bit-exact against the oracle quantiser fed x and W themselves),
   dequantise, multiply; y is checked element by element against explicit
   sums within the fp32 summation bound plus one bf16 rounding.

Each case runs through both prologue forms: the one-launch form (<= 128 rows)
and the two-launch form (Stats / Quantise, more rows).
"""
import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads
from gpu_util import bf16_to_np, codes_of, prepare, scales_of
from oracle import asp, nvfp4

pytestmark = pytest.mark.gpu


def span_case(M, K, N, r, seed):
    """x~ in span(V) with every step exact (the construction of the oracle's
    own span pin, on device shapes): identity-column V, s = 2^k, b = 1, and
    x~ bf16-exact so x = x~ * s is bf16-exact too."""
    rng = np.random.default_rng(seed)
    cols = rng.choice(K, r, replace=False)
    V = np.zeros((K, r), dtype=np.float32)
    V[cols, np.arange(r)] = 1.0
    s = (2.0 ** rng.integers(-3, 4, K)).astype(np.float32)
    xt = np.zeros((M, K), dtype=np.float32)
    xt[:, cols] = workloads.bf16_round(rng.standard_normal((M, r)).astype(np.float32))
    x = (xt * s).astype(np.float32)
    W = workloads.bf16_round((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    bias = workloads.bf16_round((rng.standard_normal(N) * 0.01).astype(np.float32))
    return workloads.LayerCase(f"span_{M}x{K}x{N}_r{r}", M, K, N, r, 1, x, W, s, V, bias), xt, cols


@pytest.mark.parametrize("M", [16, 300])
def test_input_in_span_gives_the_low_rank_product(M):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    K, N, r = 256, 64, 32
    case, xt, cols = span_case(M, K, N, r, seed=40 + M)
    h, x, _ = prepare(case)
    d = qw.debug_prologue(x, h)
    y = qw.linear(x, h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0

    z = d["z"].cpu().numpy()
    assert np.all(z == 0.0)                                   # either sign of zero
    assert d["g_x"].item() == 1.0
    assert np.all(scales_of(d["scales"], M, K) == 0)
    assert np.all((codes_of(d["codes"]) & 7) == 0)            # sign-only codes
    # u = x~ V exactly: the identity columns pick x~'s nonzero columns
    assert np.array_equal(d["u"].cpu().numpy(), xt[:, cols])

    yref, parts = asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, 1, parts=True)
    assert np.all(parts["act"]["z"] == 0) and np.all(parts["y_fp4"] == 0)
    # branch: u' = bf16(u / g_w) and L = bf16(W~V) each round once (bf16 unit
    # roundoff 2^-8: 7 stored mantissa bits), the fp32 accumulate is exact
    # enough, y rounds once to bf16
    L = parts["wt"]["L"]
    bound = 2.0 ** -7 * (np.abs(parts["act"]["u"]) @ np.abs(L).T) + 2.0 ** -8 * np.abs(yref) + 1e-30
    got = bf16_to_np(y)
    assert np.all(np.abs(got - yref) <= bound), np.max(np.abs(got - yref) / bound)


@pytest.mark.parametrize("M,r", [(16, 32), (16, 0), (300, 32), (300, 0)])
def test_zero_input_gives_the_bias(M, r):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.custom(M, 512, 144, r, 128, seed=50 + M + r, n_outliers=4)
    case.x = np.zeros_like(case.x)
    h, x, _ = prepare(case)
    d = qw.debug_prologue(x, h)
    y = qw.linear(x, h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    assert np.all(d["z"].cpu().numpy() == 0.0)
    assert d["g_x"].item() == 1.0
    assert np.all(scales_of(d["scales"], M, case.K) == 0)
    assert np.all(codes_of(d["codes"]) == 0)
    if r:
        assert np.all(d["u"].cpu().numpy() == 0.0)
    want = np.broadcast_to(workloads.bf16_bits(case.bias), (M, case.N))
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want)
    assert np.array_equal(bf16_to_np(y), asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, 128))


@pytest.mark.parametrize("M", [6, 200])
def test_rank0_unit_smoothing_no_rotation_is_textbook_nvfp4(M):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    K, N = 256, 48
    rng = np.random.default_rng(60 + M)
    x = workloads.bf16_round(rng.standard_normal((M, K)).astype(np.float32))
    W = workloads.bf16_round((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    bias = workloads.bf16_round((rng.standard_normal(N) * 0.01).astype(np.float32))
    case = workloads.LayerCase(f"textbook_{M}", M, K, N, 0, 1, x, W, np.ones(K, np.float32),
                               np.zeros((K, 0), np.float32), bias)
    h, xd, _ = prepare(case)
    d = qw.debug_prologue(xd, h)
    w = qw.export_weight(h)
    y = qw.linear(xd, h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0

    # quantiser inputs are x and W themselves: codes, scales and g bit-exact
    ca, sa, ga = nvfp4.quantize(x)
    cb, sb, gb = nvfp4.quantize(W)
    assert np.array_equal(d["z"].cpu().numpy(), x)
    assert np.array_equal(codes_of(d["codes"]), ca)
    assert np.array_equal(scales_of(d["scales"], M, K), sa)
    assert np.float32(d["g_x"].item()) == ga
    assert np.array_equal(codes_of(w["codes"]), cb)
    assert np.array_equal(scales_of(w["scales"], N, K), sb)
    assert np.float32(h.g_w) == gb

    # explicit sums: every product e2m1 * e4m3 * e2m1 * e4m3 is exact in f64
    sign = lambda c: np.where(c >> 3, -1.0, 1.0)
    va = sign(ca) * nvfp4.E2M1_MAGNITUDES[ca & 7] * nvfp4.E4M3_MAGNITUDES[np.repeat(sa, 16, axis=1)]
    vb = sign(cb) * nvfp4.E2M1_MAGNITUDES[cb & 7] * nvfp4.E4M3_MAGNITUDES[np.repeat(sb, 16, axis=1)]
    g = float(np.float32(ga) * np.float32(gb))
    exact = np.zeros((M, N))
    mag = np.zeros((M, N))
    for k in range(K):
        exact += np.outer(va[:, k], vb[:, k])
        mag += np.outer(np.abs(va[:, k]), np.abs(vb[:, k]))
    want = exact * g + bias.astype(np.float64)[None, :]
    # fp32 accumulation of K terms (K * 2^-24 of the magnitude sum, doubled),
    # the fp32 scale multiply and bias add, then one bf16 rounding (unit
    # roundoff 2^-8)
    bound = 2.0 ** -8 * np.abs(want) + (K * 2.0 ** -23) * mag * g + 2.0 ** -22 * np.abs(want) + 1e-30
    got = bf16_to_np(y)
    assert np.all(np.abs(got - want) <= bound), np.max(np.abs(got - want) / bound)
    # the oracle itself is these sums with the per-tensor scales multiplied in
    # float64 (the device's epilogue takes their fp32 product)
    ref = asp.asp_linear(x, W, np.ones(K), None, bias, 1)
    want64 = exact * (float(ga) * float(gb)) + bias.astype(np.float64)[None, :]
    assert np.all(np.abs(ref - want64) <= 1e-12 * (np.abs(want64) + 1))
