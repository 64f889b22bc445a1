"""Bare tcgen05 block-scaled FP4 GEMM vs dequantise-then-multiply in float64.

Every product e2m1 * e4m3 * e2m1 * e4m3 is exact; only the fp32 accumulation
rounds, so each output must sit within K * 2^-23 of the exact sum measured
against sum |terms| (a loose bound on fp32 summation error).  These cases pin
the operand layouts: packed nibble order, the 128B-swizzled K-major tiles, the
128 x 4 scale tiles and their TMEM placement, ragged M / N / K tails.
"""
import numpy as np
import pytest

from oracle import nvfp4

pytestmark = pytest.mark.gpu


def operands(M, N, K, seed):
    rng = np.random.default_rng(seed)
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    sa = rng.integers(0x28, 0x49, (M, K // 16), dtype=np.uint8)   # 0.25 .. 4.5
    sb = rng.integers(0x28, 0x49, (N, K // 16), dtype=np.uint8)
    return ca, cb, sa, sb


def tiled(S, rows_pad):
    rows, nb = S.shape
    buf = nvfp4.swizzle_scales(np.pad(S, ((0, rows_pad - rows), (0, 0))))
    return buf


@pytest.mark.parametrize("M,N,K", [
    (128, 128, 128), (128, 256, 256), (256, 384, 1024), (200, 144, 384),
    (1, 16, 128), (64, 256, 3072), (130, 272, 640), (300, 512, 2176), (129, 128, 1408)])
def test_fp4_gemm_matches_f64(M, N, K):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    ca, cb, sa, sb = operands(M, N, K, seed=M * 7 + N + K)
    bn = 256 if N > 128 else 128
    a_codes = torch.from_numpy(nvfp4.pack_nibbles(ca)).cuda()
    b_codes = torch.from_numpy(nvfp4.pack_nibbles(cb)).cuda()
    a_sf = torch.from_numpy(tiled(sa, -(-M // 128) * 128)).cuda()
    b_sf = torch.from_numpy(tiled(sb, -(-N // bn) * bn)).cuda()
    alpha = 0.75
    out = qw.fp4_gemm(a_codes, a_sf, b_codes, b_sf, M, N, K, alpha)
    torch.cuda.synchronize()
    assert qw.device_error() == 0
    da = nvfp4.dequantize(ca, sa, 1.0)
    db = nvfp4.dequantize(cb, sb, 1.0)
    ref = alpha * (da @ db.T)
    bound = alpha * (np.abs(da) @ np.abs(db).T) * K * 2.0 ** -23 + 1e-30
    got = out.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= bound), (np.argwhere(err > bound)[:5], float((err / bound).max()))
