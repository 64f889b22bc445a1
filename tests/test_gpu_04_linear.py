"""End-to-end ASP NVFP4 linear on the device vs the float64 oracle.

Criterion (the contract's own): ||y - y_oracle||_F / ||y_oracle||_F <= 2e-3,
the bf16 output cast plus the bf16 branch operands being the expected residual
("FastWAM UR3 3-task — 4-bit quantisations", section "Verification — NVFP4
deflated ASP": worst per-layer recompute error 1.7e-3, attributed to the bf16
output cast).
"""
import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads
from gpu_util import bf16_to_np, device_operand_reference, local_rel_errors, prepare
from oracle import asp

pytestmark = pytest.mark.gpu

TOL = 2e-3
# Per row and per 128-column block, against the float64 product of the
# device's own quantised operands (device_operand_reference): what is left is
# the bf16 output rounding (unit roundoff 2^-8 per element, about 1.1e-3 rms),
# the bf16 branch operands (2^-8 each, on the branch's share) and fp32
# accumulation.  Against
# the float64 oracle itself a single FP4 code flip in a row (the contract
# allows 0.1 % of codes to differ) already moves that row by ~8e-3, so local
# bounds are taken on the device's operands.
LOCAL_TOL = 4e-3

CASES = {
    "c1": lambda: workloads.c1_tiny(),
    "c2": lambda: workloads.c2_action_attn(),
    "m1_k256_n16_r32_b16": lambda: workloads.custom(1, 256, 16, 32, 16, seed=11, n_outliers=2),
    "m33_k384_n144_r16_b64": lambda: workloads.custom(33, 384, 144, 16, 64, seed=12, n_outliers=3),
    "m100_k1024_n1024_r0_b128": lambda: workloads.custom(100, 1024, 1024, 0, 128, seed=13, n_outliers=10),
    "m200_k512_n272_r32_b1": lambda: workloads.custom(200, 512, 272, 32, 1, seed=14, n_outliers=5),
    "m129_k768_n512_r32_b32": lambda: workloads.custom(129, 768, 512, 32, 32, seed=15, n_outliers=6),
    "m384_k1024_n768_r32_b128": lambda: workloads.custom(384, 1024, 768, 32, 128, seed=16, n_outliers=10),
    "m64_k4096_n1024_r32_b128": lambda: workloads.custom(64, 4096, 1024, 32, 128, seed=17, n_outliers=40),
    # split-K with several scale-ring slots per split, the last one partial
    "m48_k6144_n128_r32_b128": lambda: workloads.custom(48, 6144, 128, 32, 128, seed=18, n_outliers=60),
    # persistent tiles with a partial last 256-K stage
    "m260_k1408_n640_r16_b64": lambda: workloads.custom(260, 1408, 640, 16, 64, seed=19, n_outliers=14),
    # 256 x 256 tiles on CTA pairs (no split-K): ragged M, then ragged M and N
    "m1000_k1024_n2560_r32_b128": lambda: workloads.custom(1000, 1024, 2560, 32, 128, seed=23, n_outliers=10),
    "m1000_k768_n2320_r16_b64": lambda: workloads.custom(1000, 768, 2320, 16, 64, seed=24, n_outliers=8),
    # rank 0 above 128 rows: the rotation folded into the tensor-core operand
    # (ragged last tile of one row, several tiles per CTA, b = 16 / 32 / 128;
    # b = 1 is in the prologue tests, whose criterion is the code identity: with
    # no rotation a few ulp-level code flips in the x20 outlier channels move
    # this small a layer's error past 2e-3, as a float64 study reproduces)
    "m129_k640_n256_r0_b16": lambda: workloads.custom(129, 640, 256, 0, 16, seed=27, n_outliers=6),
    "m1000_k1024_n2560_r0_b32": lambda: workloads.custom(1000, 1024, 2560, 0, 32, seed=28, n_outliers=10),
    "m4100_k384_n160_r0_b128": lambda: workloads.custom(4100, 384, 160, 0, 128, seed=29, n_outliers=4),
    # the one-launch form with 3 and 4 row tiles per CTA (ragged last tiles), and
    # a layer with 8 tiles per CTA that keeps the two-launch form
    "m1100_k6272_n256_r0_b128": lambda: workloads.custom(1100, 6272, 256, 0, 128, seed=30, n_outliers=31),
    "m1950_k4736_n256_r0_b64": lambda: workloads.custom(1950, 4736, 256, 0, 64, seed=31, n_outliers=24),
    "m1000_k12800_n128_r0_b128": lambda: workloads.custom(1000, 12800, 128, 0, 128, seed=32, n_outliers=64),
    # 32 rows with two and four prologue chunks per CTA (action-expert FFN shapes)
    "m32_k2048_n512_r16_b64": lambda: workloads.custom(32, 2048, 512, 16, 64, seed=25, n_outliers=20),
    "m32_k4096_n1024_r32_b128": lambda: workloads.custom(32, 4096, 1024, 32, 128, seed=26, n_outliers=41),
}


def run_linear(case):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    h, x, _ = prepare(case)
    y = qw.linear(x, h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    return h, x, y


@pytest.mark.parametrize("name", sorted(CASES))
def test_linear_matches_oracle(name):
    case = CASES[name]()
    h, x, y = run_linear(case)
    ref = asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, case.b)
    got = bf16_to_np(y)
    err = asp.rel_fro(got, ref)
    assert err <= TOL, err
    row_err, blk_err = local_rel_errors(got, device_operand_reference(case, h, x))
    assert row_err <= LOCAL_TOL and blk_err <= LOCAL_TOL, (row_err, blk_err)


def test_two_calls_bit_identical():
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.custom(300, 1024, 512, 32, 128, seed=21, n_outliers=10)
    h, x, y1 = run_linear(case)
    y2 = qw.linear(x, h)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_small_and_large_paths_agree_on_shared_rows():
    # M = 64 goes through the one-launch prologue + split-K GEMM; M = 256 through
    # the two-launch prologue + full-tile GEMM.  Rows are independent given the
    # per-tensor scale, so feed the same 64 rows twice as a 128-row input
    # (same amax) and compare against the 64-row call.
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.custom(64, 1024, 512, 32, 128, seed=22, n_outliers=10)
    h, x, y_small = run_linear(case)
    x2 = torch.cat([x, x, x, x], 0).contiguous()
    y_big = qw.linear(x2, h)
    torch.cuda.synchronize()
    for i in range(4):
        d = (y_big[64 * i:64 * (i + 1)].float() - y_small.float()).abs().max().item()
        assert d <= 2 ** -7 * y_small.float().abs().max().item()


def test_empty_input_is_a_noop():
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.c1_tiny()
    h, x, _ = prepare(case)
    y = torch.full((0, case.N), 7.0, dtype=torch.bfloat16, device="cuda")
    qw.linear(x[:0], h, y)
    torch.cuda.synchronize()


def test_argument_errors():
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    dev = "cuda"
    W = torch.zeros((64, 200), dtype=torch.bfloat16, device=dev)
    s = torch.ones(200, device=dev)
    with pytest.raises(qw.QwamError) as e:
        qw.prepare_weight(W, s, None, None, 16)
    assert e.value.status == 2                     # K % 128
    W = torch.zeros((64, 256), dtype=torch.bfloat16, device=dev)
    s = torch.ones(256, device=dev)
    with pytest.raises(qw.QwamError) as e:
        qw.prepare_weight(W, s, None, None, 48)    # not a power of two
    assert e.value.status == 2
    with pytest.raises(qw.QwamError) as e:
        qw.prepare_weight(W, s, torch.zeros((256, 8), device=dev), None, 16)
    assert e.value.status == 2                     # r = 8
    s_bad = s.clone()
    s_bad[3] = -1.0
    with pytest.raises(qw.QwamError) as e:
        qw.prepare_weight(W, s_bad, None, None, 16)
    assert e.value.status == 1                     # s <= 0
    h = qw.prepare_weight(W, s, None, None, 16)
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device=dev)
    y = torch.zeros((4, 64), dtype=torch.bfloat16, device=dev)
    lib = qw.load()
    assert lib.qwam_linear(x.data_ptr() + 2, 4, h.raw, y.data_ptr(), None) == 3   # misaligned
    assert lib.qwam_linear(x.data_ptr(), -1, h.raw, y.data_ptr(), None) == 2
    assert lib.qwam_linear(x.data_ptr(), 4, h.raw, x.data_ptr(), None) in (1, 2)
    h.destroy()
    with pytest.raises(ValueError):
        qw.linear(x, h)
