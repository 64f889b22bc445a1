"""Activation prologue and weight prepare on the device vs the oracle.

1. Bit-exact: the device's FP4 codes, E4M3 scales and per-tensor scale equal
   the oracle quantiser applied to the device's own fp32 quantiser input
   (z for activations, W_d for weights), exported by the debug entry points.
2. Close: the device's z, u, W_d and L match the float64 oracle within the
   precision of fp32 FWHT + bf16x3 tensor-core products, and >= 99.9 % of the
   activation codes equal the oracle's own codes.
"""
import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads
from gpu_util import codes_of, prepare, scales_of
from oracle import asp, nvfp4

pytestmark = pytest.mark.gpu

CASES = {
    "c1": lambda: workloads.c1_tiny(),
    "c2": lambda: workloads.c2_action_attn(),
    "m300_r32_b128": lambda: workloads.custom(300, 512, 256, 32, 128, seed=1, n_outliers=5),
    "m96_r16_b64": lambda: workloads.custom(96, 384, 160, 16, 64, seed=2, n_outliers=3),
    "m200_r0_b16": lambda: workloads.custom(200, 256, 128, 0, 16, seed=3, n_outliers=2),
    "m17_r32_b1": lambda: workloads.custom(17, 256, 64, 32, 1, seed=4, n_outliers=2),
    "m64_r32_b2": lambda: workloads.custom(64, 1024, 128, 32, 2, seed=5, n_outliers=4),
    "m1_r32_b128": lambda: workloads.custom(1, 4096, 64, 32, 128, seed=6, n_outliers=8),
    # the one-launch prologue at <= 32 rows: two chunks per CTA at r = 16,
    # r = 0 with b = 16, eight chunks per CTA
    "m32_k2048_r16_b64": lambda: workloads.custom(32, 2048, 96, 16, 64, seed=7, n_outliers=20),
    "m24_k512_r0_b16": lambda: workloads.custom(24, 512, 64, 0, 16, seed=8, n_outliers=5),
    "m9_k8192_r32_b128": lambda: workloads.custom(9, 8192, 64, 32, 128, seed=9, n_outliers=40),
    # rank 0 above 128 rows: the tensor-core rotation against diag(chan) H_b
    "m257_k1024_r0_b128": lambda: workloads.custom(257, 1024, 128, 0, 128, seed=10, n_outliers=10),
    "m600_k512_r0_b2": lambda: workloads.custom(600, 512, 64, 0, 2, seed=11, n_outliers=5),
    "m129_k640_r0_b1": lambda: workloads.custom(129, 640, 64, 0, 1, seed=12, n_outliers=6),
    # one launch with a grid-wide barrier, 4 row tiles per CTA
    "m1950_k4736_r0_b64": lambda: workloads.custom(1950, 4736, 64, 0, 64, seed=13, n_outliers=24),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def run(request):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = CASES[request.param]()
    h, x, wd = prepare(case, wd_out=True)
    d = qw.debug_prologue(x, h)
    w = qw.export_weight(h)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    ora = asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, case.b, parts=True)[1]
    return case, h, d, w, wd.cpu().numpy(), ora


def test_activation_codes_bit_exact(run):
    case, h, d, _, _, _ = run
    z = d["z"].cpu().numpy()
    oc, osf, og = nvfp4.quantize(z)
    assert np.float32(d["g_x"].item()) == og
    assert np.array_equal(scales_of(d["scales"], case.M, case.K), osf)
    assert np.array_equal(codes_of(d["codes"]), oc)


def test_weight_codes_bit_exact(run):
    case, h, _, w, wd, _ = run
    oc, osf, og = nvfp4.quantize(wd)
    assert np.float32(h.g_w) == og
    assert np.array_equal(scales_of(w["scales"], case.N, case.K), osf)
    assert np.array_equal(codes_of(w["codes"]), oc)


def test_prologue_close_to_float64(run):
    case, h, d, _, _, ora = run
    act = ora["act"]
    xt_max = np.abs(act["xt"]).max()
    z = d["z"].cpu().numpy().astype(np.float64)
    assert np.abs(z - act["z"]).max() <= 2e-5 * xt_max
    if case.r:
        u = d["u"].cpu().numpy().astype(np.float64)
        assert asp.rel_fro(u, act["u"]) <= 1e-4
    same = np.mean(codes_of(d["codes"]) == act["codes"])
    assert same >= 0.999, same


def test_weight_prepare_close_to_float64(run):
    import torch
    case, h, _, w, wd, ora = run
    wt = ora["wt"]
    assert np.abs(wd - wt["Wd"]).max() <= 2e-5 * np.abs(wt["Wt"]).max()
    if case.r:
        L = w["L"].to(torch.float32).cpu().numpy()
        assert asp.rel_fro(L, wt["L"]) <= 2 ** -8
    assert np.mean(codes_of(w["codes"]) == wt["codes"]) >= 0.999


def test_branch_operand_is_scaled_u(run):
    import torch
    case, h, d, _, _, _ = run
    if not case.r:
        pytest.skip("no branch at r = 0")
    gs = np.float64(np.float32(d["g_x"].item()) * np.float32(h.g_w))
    ub = d["ub"].to(torch.float32).cpu().numpy().astype(np.float64)
    u = d["u"].cpu().numpy().astype(np.float64)
    assert np.allclose(ub * gs, u, rtol=2 ** -8, atol=1e-30)
