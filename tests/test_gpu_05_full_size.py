"""Full-size layers, run exactly as the benchmark runs them (one qwam_linear
call through the C ABI, the same launch plan), checked on sampled output rows
against the float64 oracle.

The per-tensor activation scale depends on every row, so the oracle prologue
runs on the whole input; the FP4 product and the branch are then formed only
for the sampled rows.  Criterion as for the small cases: relative Frobenius
error <= 2e-3 over the sampled rows ("FastWAM UR3 3-task — 4-bit
quantisations", section "Verification — NVFP4 deflated ASP"), and >= 99.9 %
of the sampled rows' activation codes equal to the oracle's.
"""
import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads
from gpu_util import bf16_to_np, codes_of, device_operand_reference, local_rel_errors, prepare, sample_rows
from oracle import asp, nvfp4

pytestmark = pytest.mark.gpu

TOL = 2e-3
# per sampled row and per 128-column block of the sampled rows, against the
# float64 product of the device's own quantised operands (see test_gpu_04)
LOCAL_TOL = 4e-3

CASES = {
    "c3_r0": lambda: workloads.c3_video_attn(0),
    "c3_r32": lambda: workloads.c3_video_attn(32),
    "c4_up": lambda: workloads.c4_video_ffn_up(),
    "c4_down": lambda: workloads.c4_video_ffn_down(),
    # the video FFN pair as the denoising step holds it (r = 0): FFN up through
    # the one-launch rank-0 prologue, FFN down (K = 14336, 32 row tiles per CTA)
    # through the two-launch rank-0 form, both into CTA-pair tiles without a branch
    "c5_video_ffn0_r0": lambda: workloads.c5_layer(8),
    "c5_video_ffn2_r0": lambda: workloads.c5_layer(9),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_full_size_layer_on_sampled_rows(name):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = CASES[name]()
    h, x, _ = prepare(case)
    y = qw.linear(x, h)
    d = qw.debug_prologue(x, h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    rows = sample_rows(case.M)

    wp = asp.prepare_weight(case.W, case.s, case.V, case.b)
    ap = asp.activation_prologue(case.x, case.s, case.V, case.b, fp4=False)
    codes, scales, g = nvfp4.quantize(ap["z"].astype(np.float32))
    deq_rows = nvfp4.dequantize(codes[rows], scales[rows], g)
    ref = asp.nvfp4_gemm(deq_rows, wp["deq"]) + ap["u"][rows] @ wp["L"].T
    ref = ref + np.asarray(case.bias, dtype=np.float64)[None, :]

    got = bf16_to_np(y)[rows]
    err = asp.rel_fro(got, ref)
    assert err <= TOL, err
    row_err, blk_err = local_rel_errors(got, device_operand_reference(case, h, x, rows))
    assert row_err <= LOCAL_TOL and blk_err <= LOCAL_TOL, (row_err, blk_err)
    same = np.mean(codes_of(d["codes"])[rows] == codes[rows])
    assert same >= 0.999, same
