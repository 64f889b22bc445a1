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


_FRESH_PROCESS_CHECK = r"""
import json, sys
import torch
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
from bit_w4a4_quantised_b200 import binding as qw, workloads
from gpu_util import prepare
# the largest scratch layout the limits admit
case = workloads.custom(128, 16384, 256, 32, 128, seed=36, n_outliers=80)
h, x, _ = prepare(case)
ys = [torch.empty((case.M, case.N), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info()[0]
qw.linear_noalloc(x, h, ys[0])          # first call of the process: the set-up
qw.linear_noalloc(x, h, ys[1])
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
qw.linear(x, h, ys[2])                  # the growable workspace: allocates
torch.cuda.synchronize()
free2 = torch.cuda.mem_get_info()[0]
print(json.dumps({"free0": free0, "free1": free1, "free2": free2, "err": qw.device_error(),
                  "same": bool(torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2]))}))
"""


def test_noalloc_leaves_free_memory_unchanged():
    # A fresh process, so no earlier call has set up the static scratch or
    # grown the ordinary workspace; every kernel is loaded when the library
    # is (CUDA_MODULE_LOADING=EAGER), so only the calls themselves could move
    # device memory.  The ordinary call at the same shape must move it: that
    # is what shows the measurement can see an allocation.
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER")
    out = subprocess.run([sys.executable, "-c", _FRESH_PROCESS_CHECK, root], env=env, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    r = json.loads(out.stdout.strip().splitlines()[-1])
    assert r["err"] == 0 and r["same"]
    assert r["free1"] == r["free0"], r
    assert r["free2"] < r["free1"], r


_FRESH_PROCESS_CAPTURE = r"""
import json, sys
import torch
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
from bit_w4a4_quantised_b200 import binding as qw, workloads
from gpu_util import prepare
case = workloads.custom(32, 1024, 256, 32, 128, seed=39, n_outliers=10)
h, x, _ = prepare(case)
y_ref = qw.linear(x, h)
y = torch.empty_like(y_ref)
torch.cuda.synchronize()
status = None
side = torch.cuda.Stream()
g = torch.cuda.CUDAGraph()
try:
    with torch.cuda.graph(g, stream=side):
        qw.linear_noalloc(x, h, y)      # first call of the process, inside a capture
except qw.QwamError as e:
    status = e.status
torch.cuda.synchronize()
qw.linear_noalloc(x, h, y)              # outside the capture the set-up goes ahead
torch.cuda.synchronize()
print(json.dumps({"status": status, "err": qw.device_error(), "same": bool(torch.equal(y, y_ref))}))
"""


def test_noalloc_first_call_under_capture_is_refused():
    # The set-up synchronises the device, which a stream capture cannot hold:
    # the library refuses it with QWAM_ERR_INVALID_ARG and a later uncaptured
    # call sets up and computes as usual.
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", _FRESH_PROCESS_CAPTURE, root], capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    r = json.loads(out.stdout.strip().splitlines()[-1])
    assert r["status"] == 1 and r["err"] == 0 and r["same"], r


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
