"""The FP8 W8A8 arm on the device (qwam_prepare_weight_fp8) against the float64
oracle's FP8 arm (oracle.asp with fmt="fp8", oracle.fp8).

The arm is the QuantWAMs report's FP8 W8A8 for upgraded Linears ("During
inference"), read as E4M3 elements with one fp32 scale per tensor (readings in
oracle/fp8.py).  Checks, through the C-ABI:
1. activation and weight codes and per-tensor scales bit-exact against the
   oracle quantiser fed the device's own fp32 quantiser inputs (z, W_d);
2. >= 99.9 % of the codes equal to the oracle's own;
3. y within 2e-3 relative Frobenius of the oracle's FP8 arm (the bf16 output
   cast is ~1.7e-3 of it), and within 4e-3 per row and per 128-column block of
   the float64 product of the device's own quantised operands.
The cases cover the one-launch prologue, the two-launch prologue (r > 0) and
the tensor-core rotation form (r = 0), split-K, one-CTA and CTA-pair GEMM tiles.
"""
import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads
from gpu_util import bf16_to_np, local_rel_errors, prepare
from oracle import asp, fp8

pytestmark = pytest.mark.gpu

TOL, LOCAL_TOL = 2e-3, 4e-3

CASES = {
    "c1": lambda: workloads.c1_tiny(),
    "c2": lambda: workloads.c2_action_attn(),
    "m48_k4096_n512_r32_b128": lambda: workloads.custom(48, 4096, 512, 32, 128, seed=91, n_outliers=40),
    "m300_k512_n256_r16_b64": lambda: workloads.custom(300, 512, 256, 16, 64, seed=92, n_outliers=5),
    "m200_k1024_n512_r0_b128": lambda: workloads.custom(200, 1024, 512, 0, 128, seed=93, n_outliers=10),
    "m1000_k1024_n2560_r32_b128": lambda: workloads.custom(1000, 1024, 2560, 32, 128, seed=94, n_outliers=10),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_arm_matches_oracle(name):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = CASES[name]()
    h, x, wd = prepare(case, wd_out=True, fmt="fp8")
    assert h.fmt == "fp8"
    y = qw.linear(x, h)
    d = qw.debug_prologue(x, h)
    w = qw.export_weight(h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0

    # 1. bit-exact quantisers on the device's own inputs
    z = d["z"].cpu().numpy()
    ca, ga = fp8.quantize(z)
    assert np.float32(d["g_x"].item()) == ga
    assert np.array_equal(d["codes"].cpu().numpy(), ca)
    cb, gb = fp8.quantize(wd.cpu().numpy())
    assert np.float32(h.g_w) == gb
    assert np.array_equal(w["codes"].cpu().numpy(), cb)

    # 2. against the oracle's own codes
    ref, parts = asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, case.b, fmt="fp8", parts=True)
    assert np.mean(ca == parts["act"]["codes"]) >= 0.999
    assert np.mean(cb == parts["wt"]["codes"]) >= 0.999

    # 3. the layer
    got = bf16_to_np(y)
    assert asp.rel_fro(got, ref) <= TOL
    own = fp8.dequantize(ca, ga) @ fp8.dequantize(cb, gb).T + parts["act"]["u"] @ parts["wt"]["L"].T
    own = own + case.bias.astype(np.float64)[None, :]
    row_err, blk_err = local_rel_errors(got, own)
    assert row_err <= LOCAL_TOL and blk_err <= LOCAL_TOL, (row_err, blk_err)


def test_fp8_full_size_on_sampled_rows():
    """The FP8 arm on the 4096 x 3072 -> 3072 rank-0 layer, as the benchmark
    runs it (one-launch rank-0 prologue, CTA-pair FP8 tiles): quantisers
    bit-exact on the device's own full inputs, the per-tensor scales from the
    whole input, the output on sampled rows against the oracle."""
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    from gpu_util import sample_rows
    case = workloads.c3_video_attn(0)
    h, x, wd = prepare(case, wd_out=True, fmt="fp8")
    y = qw.linear(x, h)
    d = qw.debug_prologue(x, h)
    w = qw.export_weight(h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0

    z = d["z"].cpu().numpy()
    ca, ga = fp8.quantize(z)
    assert np.float32(d["g_x"].item()) == ga
    assert np.array_equal(d["codes"].cpu().numpy(), ca)
    cb, gb = fp8.quantize(wd.cpu().numpy())
    assert np.float32(h.g_w) == gb
    assert np.array_equal(w["codes"].cpu().numpy(), cb)

    rows = sample_rows(case.M)
    wp = asp.prepare_weight(case.W, case.s, case.V, case.b, fmt="fp8")
    ap = asp.activation_prologue(case.x, case.s, case.V, case.b, fmt="fp8")
    assert np.mean(ca[rows] == ap["codes"][rows]) >= 0.999
    bias = case.bias.astype(np.float64)[None, :]
    ref = asp.nvfp4_gemm(ap["deq"][rows], wp["deq"]) + bias
    got = bf16_to_np(y)[rows]
    assert asp.rel_fro(got, ref) <= TOL
    own = fp8.dequantize(ca[rows], ga) @ fp8.dequantize(cb, gb).T + bias
    row_err, blk_err = local_rel_errors(got, own)
    assert row_err <= LOCAL_TOL and blk_err <= LOCAL_TOL, (row_err, blk_err)
