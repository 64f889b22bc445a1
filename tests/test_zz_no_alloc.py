"""qwam_linear_noalloc (the layer with all scratch in the library's fixed
static array) against qwam_linear, through the C-ABI, two calls in a row.

Both run the same kernels with the same GEMM plan, so the outputs must agree
within the end-to-end tolerance of the parity tests (2e-3 relative Frobenius)
and, the kernels being deterministic, bit for bit.  This file is collected
last so that it also runs after the other GPU tests have grown the ordinary
workspace.
"""
import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads
from gpu_util import bf16_to_np, prepare
from oracle import asp

pytestmark = pytest.mark.gpu

TOL = 2e-3

CASES = {
    "c2_m32_k1024_n1024_r32_b128": lambda: workloads.c2_action_attn(),
    "m1_k256_n16_r32_b16": lambda: workloads.custom(1, 256, 16, 32, 16, seed=31, n_outliers=2),
    "m100_k1024_n1024_r0_b128": lambda: workloads.custom(100, 1024, 1024, 0, 128, seed=32, n_outliers=10),
    "m77_k768_n272_r16_b64": lambda: workloads.custom(77, 768, 272, 16, 64, seed=33, n_outliers=6),
    "m128_k3072_n3072_r32_b128": lambda: workloads.custom(128, 3072, 3072, 32, 128, seed=34, n_outliers=30),
    # the largest scratch layout the limits admit (M = 128, K = 16384)
    "m128_k16384_n2688_r32_b128": lambda: workloads.custom(128, 16384, 2688, 32, 128, seed=35, n_outliers=80),
}


def _rel(a, b):
    return asp.rel_fro(bf16_to_np(a), bf16_to_np(b))


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_linear_two_calls(name):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = CASES[name]()
    h, x, _ = prepare(case)
    y_ref = qw.linear(x, h)
    y1 = torch.full_like(y_ref, float("nan"))
    y2 = torch.full_like(y_ref, float("nan"))
    qw.linear_noalloc(x, h, y1)
    qw.linear_noalloc(x, h, y2)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    for y in (y1, y2):
        assert torch.isfinite(y.float()).all()
        assert _rel(y, y_ref) <= TOL
        assert torch.equal(y, y_ref)


def test_noalloc_matches_oracle():
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.c2_action_attn(layer=3)
    h, x, _ = prepare(case)
    y = torch.empty((case.M, case.N), dtype=torch.bfloat16, device="cuda")
    qw.linear_noalloc(x, h, y)
    torch.cuda.synchronize()
    ref = asp.asp_linear(case.x, case.W, case.s, case.V, case.bias, case.b)
    assert asp.rel_fro(bf16_to_np(y), ref) <= TOL


def test_noalloc_leaves_free_memory_unchanged():
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.custom(64, 2048, 1536, 32, 128, seed=36, n_outliers=20)
    h, x, _ = prepare(case)
    ys = [torch.empty((case.M, case.N), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    qw.linear_noalloc(x, h, ys[0])  # set-up happens on the first call of the process at the latest
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    qw.linear_noalloc(x, h, ys[1])
    qw.linear_noalloc(x, h, ys[2])
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


def test_noalloc_rejects_sizes_beyond_its_limits():
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.custom(129, 256, 32, 32, 16, seed=37, n_outliers=2)
    h, x, _ = prepare(case)
    y = torch.empty((129, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qw.QwamError) as e:
        qw.linear_noalloc(x, h, y)
    assert e.value.status == 2 and "128 rows" in str(e.value)
    # 128 rows of the same layer are accepted
    qw.linear_noalloc(x[:128], h, y[:128])

    wide = workloads.custom(4, 16384 + 128, 16, 0, 128, seed=38, n_outliers=2)
    hw, xw, _ = prepare(wide)
    yw = torch.empty((4, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qw.QwamError) as e:
        qw.linear_noalloc(xw, hw, yw)
    assert e.value.status == 2 and "16384" in str(e.value)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    assert np.isfinite(bf16_to_np(y[:128])).all()
