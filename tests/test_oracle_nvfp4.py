"""Pins for the oracle's NVFP4 encoding (CPU only).

Each test ties ``oracle.nvfp4`` to something other than itself: hand-worked
values (tests/golden), an independent library cast, exhaustive search, a
closed-form error bound, or figures printed on the model card.
"""
import itertools

import numpy as np
import pytest

from conftest import read_golden
from oracle import nvfp4

F32 = np.float32


def test_e2m1_golden():
    rows = read_golden("e2m1_rounding.txt")
    assert len(rows) > 20
    x = np.array([float(r[0]) for r in rows], dtype=np.float32)
    want = np.array([int(r[1], 16) for r in rows], dtype=np.uint8)
    got = nvfp4.encode_e2m1(x)
    assert np.array_equal(got, want), list(zip(x, got, want))


def test_e4m3_golden():
    rows = read_golden("e4m3_rounding.txt")
    t = np.array([float(r[0]) for r in rows], dtype=np.float32)
    want = np.array([int(r[1], 16) for r in rows], dtype=np.uint8)
    got = nvfp4.encode_e4m3_satfinite(t)
    assert np.array_equal(got, want), list(zip(t, got, want))


def test_e2m1_decode_grid():
    # the hand-worked grid {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}
    got = nvfp4.decode_e2m1(np.arange(16))
    want = [0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6]
    assert np.array_equal(got, want)


def test_e4m3_table_matches_torch_float8():
    # library pin: decode every finite non-negative code through torch's e4m3fn
    torch = pytest.importorskip("torch")
    codes = torch.arange(127, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(lib, nvfp4.E4M3_MAGNITUDES)
    assert nvfp4.E4M3_MAGNITUDES[-1] == 448.0


def test_e4m3_encoder_matches_torch_cast():
    # library pin on the rounding rule: torch's fp32 -> e4m3fn cast is RNE;
    # compare on [0, 448] where saturation does not enter
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    t = np.concatenate([
        rng.uniform(0, 448, 20000), 2.0 ** rng.uniform(-12, 8.8, 20000),
        (nvfp4.E4M3_MAGNITUDES[:-1] + nvfp4.E4M3_MAGNITUDES[1:]) / 2,  # every tie
    ]).astype(np.float32)
    t = t[t <= 448]
    lib = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nvfp4.encode_e4m3_satfinite(t), lib)


def test_e2m1_encoder_exhaustive_nearest():
    # brute force: for many fp32 values, the chosen code is a nearest grid point,
    # and on ties the even one
    rng = np.random.default_rng(3)
    q = np.concatenate([rng.uniform(-7, 7, 50000),
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])]).astype(np.float32)
    codes = nvfp4.encode_e2m1(q)
    mags = np.minimum(np.abs(q.astype(np.float64)), 6.0)
    for qi, mi, c in zip(q[:3000], mags[:3000], codes[:3000]):
        d = np.abs(nvfp4.E2M1_MAGNITUDES - mi)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert (c & 7) == want and (c >> 3) == int(np.signbit(qi))


def test_quantizer_worked_example():
    rows = read_golden("quantizer_worked_example.txt")
    g = float(rows[0][0])
    scales = [int(v, 16) for v in rows[1]]
    vals = np.array([float(v) for v in rows[2] + rows[4]], dtype=np.float32)[None, :]
    want = np.array([int(v, 16) for v in rows[3] + rows[5]], dtype=np.uint8)
    codes, S, gq = nvfp4.quantize(vals)
    assert gq == np.float32(g)
    assert list(S[0]) == scales
    assert np.array_equal(codes[0], want), list(zip(vals[0], codes[0], want))


def test_global_scale_closed_form():
    rng = np.random.default_rng(11)
    T = rng.standard_normal((8, 64)).astype(np.float32) * F32(3.7)
    _, S, g = nvfp4.quantize(T)
    assert g == np.abs(T).max() / F32(2688.0)
    # the block holding the tensor maximum gets a scale at (or rounded to) 448
    i = np.unravel_index(np.argmax(np.abs(T)), T.shape)
    assert S[i[0], i[1] // 16] == 0x7E


def test_zero_tensor_and_zero_block():
    T = np.zeros((2, 32), dtype=np.float32)
    T[1, :16] = -0.0
    codes, S, g = nvfp4.quantize(T)
    assert g == 1.0 and np.all(S == 0)
    assert np.all(codes[0] == 0) and np.all(codes[1, :16] == 8) and np.all(codes[1, 16:] == 0)
    T2 = np.zeros((1, 32), dtype=np.float32)
    T2[0, 16:] = np.linspace(-3, 3, 16, dtype=np.float32)
    codes2, S2, _ = nvfp4.quantize(T2)
    assert S2[0, 0] == 0 and np.all(codes2[0, :16] == 0) and S2[0, 1] != 0


def test_tiny_block_underflows_to_zero_scale():
    # a block whose amax is below half the smallest E4M3 step relative to g
    T = np.zeros((1, 32), dtype=np.float32)
    T[0, 0] = 2688.0
    T[0, 16] = -1e-4       # t = 1e-4 / 6 < 2**-10 -> S = 0 -> codes keep only the sign
    codes, S, g = nvfp4.quantize(T)
    assert g == 1.0 and S[0, 1] == 0 and codes[0, 16] == 0x8


def _grid_step(m):
    return np.where(m < 2, 0.5, np.where(m < 4, 1.0, 2.0))


def test_roundtrip_error_bound():
    # closed-form bound: |deq - T| <= half a grid step * e, plus the excess
    # above 6e when the rounded block scale undershoots
    rng = np.random.default_rng(5)
    T = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-4, 4, (64, 1)))).astype(np.float32)
    T[:, 7] *= 40
    codes, S, g = nvfp4.quantize(T)
    deq = nvfp4.dequantize(codes, S, g)
    e = (nvfp4.decode_e4m3(S) * float(g)).repeat(16, axis=1)
    m = np.abs(T.astype(np.float64)) / e
    bound = 0.5 * _grid_step(np.minimum(m, 6.0)) * e * (1 + 1e-6) + np.maximum(0, np.abs(T) - 6 * e)
    assert np.all(np.abs(deq - T) <= bound + 1e-30)


def test_quantizer_brute_force_code_search():
    # independent restatement: for each element try all 16 codes and keep the
    # nearest (ties to even magnitude), with q formed by the same fp32 ops
    rng = np.random.default_rng(9)
    T = rng.standard_normal((3, 48)).astype(np.float32)
    codes, S, g = nvfp4.quantize(T)
    allvals = nvfp4.decode_e2m1(np.arange(16))
    for r, j in itertools.product(range(3), range(48)):
        e = np.float32(nvfp4.decode_e4m3(S[r, j // 16])) * g
        q = T[r, j] * (np.float32(1.0) / e)
        qc = np.float64(np.clip(q, -6, 6))
        d = np.abs(allvals - qc)
        cands = [c for c in range(16) if d[c] == d.min() and (c >> 3) == int(np.signbit(q))]
        best = [c for c in cands if (c & 7) % 2 == 0] if len(cands) > 1 else cands
        assert codes[r, j] == best[0]


def test_pack_nibbles_low_is_even():
    codes = np.array([[1, 2, 3, 4, 0xF, 0x8]], dtype=np.uint8)
    p = nvfp4.pack_nibbles(codes)
    assert list(p[0]) == [0x21, 0x43, 0x8F]
    assert np.array_equal(nvfp4.unpack_nibbles(p), codes)


def test_scale_tile_layout_hand_offsets():
    K = 256  # 4 tiles of 64 columns per 128-row band
    cases = {(0, 0): 0, (1, 0): 16, (31, 0): 496, (32, 0): 4, (64, 0): 8, (96, 0): 12,
             (0, 1): 1, (0, 3): 3, (0, 4): 512, (0, 15): 3 * 512 + 3,
             (128, 0): 4 * 512, (33, 5): 512 + 16 + 4 + 1}
    for (m, kb), off in cases.items():
        assert nvfp4.scale_tile_offset(m, kb, K) == off, (m, kb)


def test_scale_tile_layout_is_a_bijection():
    rows, K = 256, 512
    m, kb = np.meshgrid(np.arange(rows), np.arange(K // 16), indexing="ij")
    off = nvfp4.scale_tile_offset(m, kb, K).ravel()
    assert np.array_equal(np.sort(off), np.arange(rows * K // 16))
    S = np.random.default_rng(0).integers(0, 127, (200, 32)).astype(np.uint8)
    buf = nvfp4.swizzle_scales(S)
    assert buf.size == 256 * 32 and np.all(buf[nvfp4.scale_tile_offset(
        np.arange(200, 256)[:, None], np.arange(32)[None, :], 512).ravel()] == 0)
    assert np.array_equal(nvfp4.unswizzle_scales(buf, 200, 512), S)


def test_storage_figures_printed_on_the_card():
    (n, codes_mib, scales_mib), = [tuple(map(float, r)) for r in read_golden("storage_figures.txt")]
    cb, sb = nvfp4.storage_bytes(int(n))
    assert abs(cb / 2 ** 20 - codes_mib) / codes_mib < 1e-3
    assert abs(sb / 2 ** 20 - scales_mib) / scales_mib < 1e-3
    assert cb * 8 / n == 4.0
