"""Failure detection without a GPU fault: a bounded device wait that runs out.

qwam_debug_fp4_gemm_withheld runs the bare FP4 GEMM with the first pipeline
stage's barrier expecting 16 bytes more than its TMA boxes carry, so that
stage never completes, and with every wait limited to 1 ms.  Each role behind
that barrier (MMA issue, scale copies, epilogue, and with a single stage the
producer's drain) must give up, set its bit in the device error word and
return.  The host then reads QWAM_ERR_TIMEOUT, and the same context still
runs the GEMM correctly.
"""
import numpy as np
import pytest

from oracle import nvfp4

pytestmark = pytest.mark.gpu

MMA_WAIT, EPILOGUE_WAIT, DRAIN_WAIT, SCALE_WAIT = 1 << 1, 1 << 2, 1 << 3, 1 << 5


def _operands(M, N, K, seed):
    import torch
    rng = np.random.default_rng(seed)
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    sa = rng.integers(0x28, 0x49, (M, K // 16), dtype=np.uint8)
    sb = rng.integers(0x28, 0x49, (N, K // 16), dtype=np.uint8)
    pad = lambda S, rows: nvfp4.swizzle_scales(np.pad(S, ((0, rows - S.shape[0]), (0, 0))))
    dev = [torch.from_numpy(a).cuda() for a in (nvfp4.pack_nibbles(ca), pad(sa, -(-M // 128) * 128),
                                                nvfp4.pack_nibbles(cb), pad(sb, -(-N // 128) * 128))]
    return dev, nvfp4.dequantize(ca, sa, 1.0), nvfp4.dequantize(cb, sb, 1.0)


@pytest.mark.parametrize("M,N,K,one_stage", [(200, 128, 256, True), (64, 128, 512, False)])
def test_withheld_stage_expires_every_wait_and_the_context_survives(M, N, K, one_stage):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    assert qw.device_error() == 0
    (a, sa, b, sb), da, db = _operands(M, N, K, seed=M + K)
    qw.debug_fp4_gemm_withheld(a, sa, b, sb, M, N, K, wait_ns=1_000_000)
    code = qw.device_error()           # synchronises the device
    assert code & MMA_WAIT and code & EPILOGUE_WAIT and code & SCALE_WAIT, hex(code)
    if one_stage:
        assert code & DRAIN_WAIT, hex(code)
    # the context is intact: the same operands without the withheld bytes
    out = qw.fp4_gemm(a, sa, b, sb, M, N, K, 1.0)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    ref = da @ db.T
    bound = (np.abs(da) @ np.abs(db).T) * K * 2.0 ** -23 + 1e-30
    assert np.all(np.abs(out.cpu().numpy().astype(np.float64) - ref) <= bound)
