"""The SVDQuant INT4 arm on the device (qwam_prepare_weight_int4, the Local
prologue, the group GEMM) against the float64 oracle (oracle.int4,
asp.svdquant_linear).

Checks, through the C-ABI:
1. the quantiser input x^ is x * RN(1 / s) in fp32, and the activation and
   weight levels and fp16 group scales are bit-exact against oracle.int4 fed
   the device's own fp32 inputs (x^ and the residual R); >= 99.9 % of the
   levels equal to the oracle's own, all of the weight levels at r = 0 (where
   R = RN(W s) on both sides);
2. the bare group GEMM (qwam_int4_gemm) on random levels and fp16 scales
   equals the fp32 chain acc = fma(P_g, sa sb, acc) over the exact integer
   group sums P_g, to the last bit on >= 99.99 % of the outputs and within
   one ulp everywhere (a group sum off by one would move an output by
   thousands of ulps), including a ragged M and N;
3. y within TOL relative Frobenius of the oracle's arm, and within LOCAL_TOL
   per row and per 128-column block of the float64 product of the device's
   own operands (levels, scales, u' and L);
4. edge cases: an all-zero x gives y == bias exactly; one row; r = 0.
The cases cover split K (few output tiles) and the one-pass bf16 epilogue
(many tiles), one row tile, several row tiles with a ragged tail, a ragged
column tile, r in {0, 16, 32}.
"""
import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads
from gpu_util import bf16_to_np, local_rel_errors, to_device
from oracle import asp, fp8, int4

pytestmark = pytest.mark.gpu

TOL, LOCAL_TOL = 3e-3, 4e-3

CASES = {
    "c1": lambda: workloads.custom(16, 256, 64, 16, 1, seed=111, n_outliers=2),
    "m32_k1024_n1024_r32": lambda: workloads.custom(32, 1024, 1024, 32, 1, seed=112, n_outliers=10),
    "m300_k512_n256_r16": lambda: workloads.custom(300, 512, 256, 16, 1, seed=113, n_outliers=5),
    "m200_k1024_n144_r0": lambda: workloads.custom(200, 1024, 144, 0, 1, seed=114, n_outliers=10),
    "m1000_k768_n640_r32": lambda: workloads.custom(1000, 768, 640, 32, 1, seed=115, n_outliers=8),
    "m1200_k256_n1024_r16": lambda: workloads.custom(1200, 256, 1024, 16, 1, seed=118, n_outliers=4),
}


def levels_of(dev_bytes) -> np.ndarray:
    """E4M3 bytes of INT4 levels -> int8 levels."""
    v = fp8.decode(np.asarray(dev_bytes))
    assert np.all(v == np.rint(v)) and np.all(np.abs(v) <= 8)
    return v.astype(np.int8)


def prepare_int4(case, wd=True, bias=True):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    x, W, s, V, b = to_device(case)
    wd_t = torch.empty((case.N, case.K), dtype=torch.float32, device="cuda") if wd else None
    h = qw.prepare_weight(W, s, V, b if bias else None, 1, wd_out=wd_t, variant="svdquant", fmt="int4")
    return h, x, wd_t


def act_scales(d, M, K):
    """Device activation scales fp32 [K/64][round_up(M, 128)] -> [M, K/64]."""
    import torch
    Mp = -(-M // 128) * 128
    return d["scales"].cpu().view(torch.float32).numpy().reshape(K // 64, Mp)[:, :M].T


def weight_scales(w, N, K):
    """Device weight scales fp32 [K/64][N] (the first N K / 16 bytes) -> [N, K/64]."""
    import torch
    return w["scales"].cpu().view(torch.float32).numpy()[: K // 64 * N].reshape(K // 64, N).T


def device_reference(case, d, w):
    """float64 y from the device's own operands."""
    y = int4.group_gemm(levels_of(d["codes"].cpu().numpy()), act_scales(d, case.M, case.K),
                        levels_of(w["codes"].cpu().numpy()), weight_scales(w, case.N, case.K))
    if case.r:
        y = y + bf16_to_np(d["ub"]) @ bf16_to_np(w["L"]).T
    return y + np.asarray(case.bias, dtype=np.float64)[None, :]


@pytest.mark.parametrize("name", sorted(CASES))
def test_int4_arm_matches_oracle(name):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = CASES[name]()
    h, x, wd = prepare_int4(case)
    assert (h.fmt, h.variant, h.b, h.g_w) == ("int4", "svdquant", 1, 1.0)
    y = qw.linear(x, h)
    d = qw.debug_prologue(x, h)
    w = qw.export_weight(h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    assert float(d["g_x"].item()) == 1.0

    # 1. quantiser input and bit-exact quantisers on the device's own inputs
    z = d["z"].cpu().numpy()
    inv_s = np.float32(1.0) / case.s.astype(np.float32)
    xb = torch.from_numpy(case.x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(z, xb * inv_s[None, :])
    ca, sa = int4.quantize(z)
    assert np.array_equal(levels_of(d["codes"].cpu().numpy()), ca)
    assert np.array_equal(act_scales(d, case.M, case.K), sa.astype(np.float32))
    cb, sb = int4.quantize(wd.cpu().numpy())
    assert np.array_equal(levels_of(w["codes"].cpu().numpy()), cb)
    assert np.array_equal(weight_scales(w, case.N, case.K), sb.astype(np.float32))

    # ... and against the oracle's own levels
    ref, parts = asp.svdquant_linear(case.x, case.W, case.s, case.V, case.bias, parts=True)
    assert np.mean(ca == parts["act"]["codes"]) >= 0.999
    assert np.mean(cb == parts["wt"]["codes"]) >= 0.999
    if case.r == 0:  # R = RN(W s) exactly on both sides: every weight level equal
        assert np.array_equal(cb, parts["wt"]["codes"])

    # 3. the layer
    got = bf16_to_np(y)
    rel = asp.rel_fro(got, ref)
    row, col = local_rel_errors(got, device_reference(case, d, w))
    print(f"{name}: rel {rel:.3e}, local row {row:.3e} block {col:.3e}")
    assert rel <= TOL, rel
    assert row <= LOCAL_TOL and col <= LOCAL_TOL, (row, col)


def random_levels(rng, rows, K):
    lv = rng.integers(-8, 8, size=(rows, K))
    lv[rng.random((rows, K)) < 0.1] = 0
    return lv


def e4m3_bytes(levels) -> np.ndarray:
    """E4M3 byte of each level, written out from the format (sign, exponent
    bias 7, three mantissa bits): |v| = 2^e (1 + m / 8)."""
    out = np.zeros(levels.shape, dtype=np.uint8)
    for v in range(-8, 8):
        if v == 0:
            continue
        a = abs(v)
        e = int(np.floor(np.log2(a)))
        m = int(round((a / 2 ** e - 1) * 8))
        out[levels == v] = (0x80 if v < 0 else 0) | ((e + 7) << 3) | m
    return out


def fp32_chain(la, sa, lb, sb):
    """acc = RN32(P_g * RN32(sa sb) + acc) in group order, the sum formed in
    80-bit extended precision (P_g * w is exact there) before one rounding to
    fp32."""
    P = int4.group_products(la, lb).astype(np.longdouble)        # [G, M, N]
    w = (sa.astype(np.float32).T[:, :, None] * sb.astype(np.float32).T[:, None, :]).astype(np.float32)  # exact
    acc = np.zeros(P.shape[1:], dtype=np.float32)
    for g in range(P.shape[0]):
        acc = (P[g] * w[g].astype(np.longdouble) + acc.astype(np.longdouble)).astype(np.float32)
    return acc


@pytest.mark.parametrize("M,N,K", [(256, 384, 512), (100, 144, 1024), (4, 16, 128)])
def test_group_gemm_integer_sums_are_exact(M, N, K):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    rng = np.random.default_rng(M + N + K)
    la, lb = random_levels(rng, M, K), random_levels(rng, N, K)
    sa = np.exp(rng.uniform(-6, 2, (M, K // 64))).astype(np.float16)
    sb = np.exp(rng.uniform(-6, 2, (N, K // 64))).astype(np.float16)
    sa[0, 0] = 0  # a zero scale
    dev = torch.device("cuda")
    out = qw.int4_gemm(torch.from_numpy(e4m3_bytes(la)).to(dev),
                       torch.from_numpy(np.ascontiguousarray(sa.astype(np.float32).T)).to(dev),
                       torch.from_numpy(e4m3_bytes(lb)).to(dev),
                       torch.from_numpy(np.ascontiguousarray(sb.astype(np.float32).T)).to(dev))
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    got = out.cpu().numpy()
    want = fp32_chain(la, sa, lb, sb)
    exact = np.mean(got == want)
    ulp = np.spacing(np.abs(want).astype(np.float32))
    assert exact >= 0.9999, exact
    assert np.all(np.abs(got.astype(np.float64) - want) <= ulp), np.max(np.abs(got - want) / ulp)
    # the e4m3 bytes written out above agree with the oracle's decoder
    assert np.array_equal(levels_of(e4m3_bytes(la)), la)


def test_zero_input_gives_the_bias():
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.custom(40, 512, 128, 32, 1, seed=116, n_outliers=2)
    h, x, _ = prepare_int4(case, wd=False)
    y = qw.linear(torch.zeros_like(x), h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    bias = torch.from_numpy(case.bias).to(torch.bfloat16).cuda()
    assert torch.equal(y, bias[None, :].expand_as(y))


@pytest.mark.parametrize("M", [1, 129])
def test_ragged_rows_without_bias(M):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.custom(M, 384, 96, 16, 1, seed=117 + M, n_outliers=3)
    h, x, _ = prepare_int4(case, wd=False, bias=False)
    y = qw.linear(x, h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    ref = asp.svdquant_linear(case.x, case.W, case.s, case.V, None)
    assert asp.rel_fro(bf16_to_np(y), ref) <= TOL


def test_int4_full_size_on_sampled_rows():
    """The SVDQuant arm on the 4096 x 3072 -> 3072 layer with r = 32, as the
    benchmark runs it (Local prologue over 32 row tiles, group GEMM on 768
    output tiles).  Its activation scales are local to a row's group, so the
    oracle runs on the sampled rows alone; levels and scales are checked
    bit-exact on the device's own full inputs."""
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    from gpu_util import sample_rows
    case = workloads.c3_video_attn_int4()
    h, x, wd = prepare_int4(case)
    y = qw.linear(x, h)
    d = qw.debug_prologue(x, h)
    w = qw.export_weight(h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0

    z = d["z"].cpu().numpy()
    ca, sa = int4.quantize(z)
    assert np.array_equal(levels_of(d["codes"].cpu().numpy()), ca)
    assert np.array_equal(act_scales(d, case.M, case.K), sa.astype(np.float32))
    cb, sb = int4.quantize(wd.cpu().numpy())
    assert np.array_equal(levels_of(w["codes"].cpu().numpy()), cb)
    assert np.array_equal(weight_scales(w, case.N, case.K), sb.astype(np.float32))

    rows = sample_rows(case.M)
    ref, parts = asp.svdquant_linear(case.x[rows], case.W, case.s, case.V, case.bias, parts=True)
    assert np.mean(ca[rows] == parts["act"]["codes"]) >= 0.999
    got = bf16_to_np(y)[rows]
    assert asp.rel_fro(got, ref) <= TOL
    own = int4.group_gemm(ca[rows], sa[rows], cb, sb)
    own = own + bf16_to_np(d["ub"])[rows] @ bf16_to_np(w["L"]).T + case.bias.astype(np.float64)[None, :]
    row_err, blk_err = local_rel_errors(got, own)
    assert row_err <= LOCAL_TOL and blk_err <= LOCAL_TOL, (row_err, blk_err)
