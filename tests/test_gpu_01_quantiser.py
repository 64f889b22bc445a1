"""Device NVFP4 quantiser vs the oracle quantiser, bit for bit.

The quantiser's fp32 operation order is fixed (oracle/nvfp4.py and
csrc/quant.cuh describe the same steps), so codes, scales and the per-tensor
scale are a unique function of the fp32 input: any mismatch is a bug.
"""
import numpy as np
import pytest

from gpu_util import codes_of, scales_of
from oracle import nvfp4

pytestmark = pytest.mark.gpu


def run_both(T):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    Td = torch.from_numpy(T).cuda()
    codes, sf, g = qw.quantize_fp32(Td)
    torch.cuda.synchronize()
    rows, K = T.shape
    oc, osf, og = nvfp4.quantize(T)
    return (codes_of(codes), scales_of(sf, rows, K), np.float32(g.item())), (oc, osf, og)


def assert_same(gpu, ora):
    (gc, gs, gg), (oc, os_, og) = gpu, ora
    assert gg == og, (gg, og)
    assert np.array_equal(gs, os_), np.argwhere(gs != os_)[:10]
    bad = np.argwhere(gc != oc)
    assert bad.size == 0, [(tuple(i), gc[tuple(i)], oc[tuple(i)]) for i in bad[:10]]


@pytest.mark.parametrize("rows,K,seed", [(1, 64, 0), (7, 128, 1), (130, 256, 2), (300, 1024, 3), (64, 3072, 4)])
def test_random_tensors(rows, K, seed):
    rng = np.random.default_rng(seed)
    T = (rng.standard_normal((rows, K)) * np.exp(rng.uniform(-3, 3, (rows, 1)))).astype(np.float32)
    T[:, rng.choice(K, max(1, K // 100), replace=False)] *= 30
    assert_same(*run_both(T))


def test_decision_points_of_both_encoders():
    # g = 1 exactly (a block holds 2688); blocks whose max is 6 * S for a power
    # of two S give e = S and an exact reciprocal, so q hits E2M1 ties exactly;
    # further blocks put t = a/6 on E4M3 ties and saturation points
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    rows = []
    head = np.zeros(16, np.float32)
    head[0] = 2688.0
    rows.append(head)
    for S in (1.0, 2.0, 0.5, 2.0 ** -6, 64.0):
        for sign in (1.0, -1.0):
            blk = [6.0 * S]
            for t in ties:
                blk += [sign * t * S, sign * np.nextafter(np.float32(t), np.float32(9)) * S]
            blk.append(sign * 0.0)
            assert len(blk) == 16
            rows.append(np.array(blk, np.float32))
    for t in (2.0 ** -10, 3 * 2.0 ** -10, 1.0625, 1.1875, 248.0, 432.0, 400.0, 448.0):
        blk = np.linspace(-1, 1, 16).astype(np.float32) * np.float32(6 * t)
        blk[3] = np.float32(6 * t)
        rows.append(blk)
    blk = np.array([-0.0, 0.0, -1e-30, 1e-30] * 4, np.float32)
    rows.append(blk)
    T = np.concatenate(rows)[None, :]
    pad = (-T.shape[1]) % 64
    T = np.pad(T, ((0, 0), (0, pad)))
    assert_same(*run_both(T.astype(np.float32)))


def test_e2m1_conversion_sweep():
    # every value v in [-8, 8] quantised with S = 1 and g = 1 is encoded directly:
    # compare the device encoder with the oracle's nearest-even table search
    rng = np.random.default_rng(5)
    vals = np.concatenate([rng.uniform(-8, 8, 60000), np.linspace(-7, 7, 1401)]).astype(np.float32)
    n = len(vals) // 15 * 15
    blocks = np.empty((n // 15, 16), np.float32)
    blocks[:, 0] = 6.0
    blocks[:, 1:] = np.clip(vals[:n].reshape(-1, 15), -6.0, 6.0)   # keep block max at 6
    T = blocks.reshape(1, -1)
    T = np.concatenate([np.full((1, 16), 0, np.float32), T], axis=1)
    T[0, 0] = 2688.0
    T = np.pad(T, ((0, 0), (0, (-T.shape[1]) % 64)))
    assert_same(*run_both(T.astype(np.float32)))


def test_all_zero_tensor():
    T = np.zeros((3, 128), np.float32)
    T[1, :40] = -0.0
    gpu, ora = run_both(T)
    assert_same(gpu, ora)
    assert ora[2] == 1.0


def test_fma_quotients_match_ieee_ops():
    # the quantiser's a / 6 and 1 / e (FMA-corrected) must equal the IEEE fp32
    # division / reciprocal for every positive fp32 input, and the E4M3 code of
    # its u / g the code of the IEEE quotient (every u at four divisors, 2^28
    # random pairs)
    from bit_w4a4_quantised_b200 import binding as qw
    assert qw.selfcheck_rounding(1 << 28) == [0, 0, 0]
