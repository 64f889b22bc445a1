"""Layer images on the device: a handle saved with qwam_save_image and loaded
with qwam_load_image computes exactly what the saved handle computes.

Checks, through the C-ABI, for the deflated arm (r = 32 with bias, r = 0
without), the shared-weight arm, the FP8 arm and the SVDQuant INT4 arm (its
levels stored 4-bit and its scales fp16 in the image):
1. the image parsed by the documented layout holds the handle's exported
   codes, scales and L byte for byte, and g_w in its header;
2. the loaded handle reports the same shape, format and g_w, exports the same
   bytes, and its y is bit-identical to the saved handle's at a small M (one
   CTA row tile) and a large M (split plans, several row tiles), through both
   qwam_linear and qwam_linear_noalloc;
3. saving the loaded handle gives the same image byte for byte;
4. its codes agree with the float64 oracle's (>= 99.9 %), as for any prepared
   handle, so the image carries a parity-checked layer;
5. a damaged image is refused with QWAM_ERR_FORMAT and allocates nothing.
"""
import struct

import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads
from gpu_util import codes_of, prepare
from oracle import asp, fp8


def levels_of(dev_bytes):
    """E4M3 bytes of INT4 levels -> int8 levels."""
    return fp8.decode(np.asarray(dev_bytes)).astype(np.int8)

pytestmark = pytest.mark.gpu

CASES = {
    "deflated_r32_bias": (lambda: workloads.custom(300, 1024, 512, 32, 128, seed=101, n_outliers=10), "deflated", "nvfp4"),
    "deflated_r0": (lambda: workloads.custom(200, 512, 256, 0, 16, seed=102, n_outliers=5), "deflated", "nvfp4"),
    "shared_r16": (lambda: workloads.custom(260, 768, 384, 16, 64, seed=103, n_outliers=8), "shared", "nvfp4"),
    "fp8_r32": (lambda: workloads.custom(300, 1024, 512, 32, 128, seed=104, n_outliers=10), "deflated", "fp8"),
    "int4_r32": (lambda: workloads.custom(300, 1024, 512, 32, 1, seed=106, n_outliers=10), "svdquant", "int4"),
}


def pad16(n):
    return (n + 15) // 16 * 16


def parse_image(img: bytes):
    magic, ver, hb, N, K, r, b, fmt, var, flags, g_w, total, _ = struct.unpack_from("<8sII6iIfQQ", img, 0)
    assert magic == b"QWAMIMG\0" and ver == 1 and hb == 64 and total == len(img)
    off, out = 64, {"N": N, "K": K, "r": r, "b": b, "fmt": fmt, "variant": var, "g_w": g_w}

    def take(name, n):
        nonlocal off
        out[name] = np.frombuffer(img, np.uint8, n, off)
        off += pad16(n)

    take("codes", N * (K if fmt == 1 else K // 2))
    if fmt == 0:
        take("scales", (N + 255) // 256 * 256 * K // 16)
    if fmt == 2:
        take("scales", K // 64 * N * 2)
    if r:
        take("L", N * r * 2)
        for name in ("v_hi", "v_lo", "px_hi", "px_lo"):
            take(name, K * r * 2)
    take("inv_s", K * 4)
    if flags & 1:
        take("bias", N * 2)
    assert off == total
    return out


@pytest.mark.parametrize("name", sorted(CASES))
def test_image_round_trip(name):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    make, variant, fmt = CASES[name]
    case = make()
    with_bias = name != "deflated_r0"
    h, x, _ = prepare(case, variant=variant, fmt=fmt)
    if not with_bias:  # same layer without a bias
        _, W, s, V, _ = __import__("gpu_util").to_device(case)
        h = qw.prepare_weight(W, s, V, None, case.b, variant=variant, fmt=fmt)
    img = h.save_image()

    # 1. the documented layout
    p = parse_image(img)
    assert (p["N"], p["K"], p["r"], p["b"]) == (case.N, case.K, case.r, case.b)
    assert p["fmt"] == {"nvfp4": 0, "fp8": 1, "int4": 2}[fmt]
    assert p["variant"] == {"deflated": 0, "shared": 1, "svdquant": 2}[variant]
    assert np.float32(p["g_w"]) == np.float32(h.g_w)
    w = qw.export_weight(h)
    if fmt == "int4":
        # 4-bit two's complement, even element in the low nibble; fp16 scales
        lo = (p["codes"] & 15).astype(np.int8)
        hi = (p["codes"] >> 4).astype(np.int8)
        lv = np.stack([np.where(lo >= 8, lo - 16, lo), np.where(hi >= 8, hi - 16, hi)], axis=1).reshape(case.N, case.K)
        assert np.array_equal(lv, levels_of(w["codes"].cpu().numpy()))
        sc = np.frombuffer(p["scales"].tobytes(), np.float16).astype(np.float32)
        ws = w["scales"].cpu().view(torch.float32).numpy()[: sc.size]
        assert np.array_equal(sc, ws)
    else:
        assert np.array_equal(p["codes"], w["codes"].cpu().numpy().reshape(-1))
    if fmt == "nvfp4":  # the image keeps the device's 256-row padding of the tiles
        ws = w["scales"].cpu().numpy().reshape(-1)
        assert np.array_equal(p["scales"][:ws.size], ws)
    if case.r:
        assert np.array_equal(p["L"], w["L"].cpu().view(torch.uint8).numpy().reshape(-1))
    inv_s = np.frombuffer(p["inv_s"].tobytes(), np.float32)
    assert np.array_equal(inv_s, (np.float32(1.0) / case.s.astype(np.float32)))
    if with_bias:
        b16 = torch.from_numpy(case.bias).to(torch.bfloat16).view(torch.int16).numpy()
        assert np.array_equal(np.frombuffer(p["bias"].tobytes(), np.int16), b16)

    # 2. the loaded handle
    h2 = qw.load_image(img)
    assert (h2.N, h2.K, h2.r, h2.b, h2.fmt, h2.variant) == (h.N, h.K, h.r, h.b, h.fmt, h.variant)
    assert np.float32(h2.g_w) == np.float32(h.g_w)
    w2 = qw.export_weight(h2)
    keys = ["codes", "L"] + (["scales"] if fmt == "nvfp4" else [])
    for k in keys:
        assert torch.equal(w[k], w2[k]), k
    if fmt == "int4":  # the first N K / 16 scale bytes are the weight scales
        nb = case.N * case.K // 16
        assert torch.equal(w["scales"][:nb], w2["scales"][:nb])
    for rows in (min(37, case.M), case.M):
        xr = x[:rows].contiguous()
        y1, y2 = qw.linear(xr, h), qw.linear(xr, h2)
        assert torch.equal(y1, y2), rows
        if rows <= 128:
            y3 = torch.empty_like(y1)
            qw.linear_noalloc(xr, h2, y3)
            assert torch.equal(y1, y3)
    torch.cuda.synchronize()
    assert qw.device_error() == 0

    # 3. image of the image
    assert h2.save_image() == img

    # 4. the image's codes against the oracle's own
    if variant == "shared":
        ref = asp.prepare_weight_shared(case.W, case.s, case.V, case.b)
    else:
        ref = asp.prepare_weight(case.W, case.s, case.V, case.b, fmt=fmt)
    if fmt == "fp8":
        got = p["codes"].reshape(case.N, case.K)
    elif fmt == "int4":
        got = lv
    else:
        got = codes_of(torch.from_numpy(p["codes"].reshape(case.N, case.K // 2).copy()))
    assert np.mean(got == ref["codes"]) >= 0.999
    h.destroy()
    h2.destroy()


def test_damaged_image_is_refused():
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    case = workloads.custom(64, 256, 128, 16, 16, seed=105, n_outliers=2)
    h, _, _ = prepare(case)
    img = bytearray(h.save_image())
    free0 = torch.cuda.mem_get_info()[0]
    for off in (70, len(img) // 2, len(img) - 1):
        bad = bytearray(img)
        bad[off] ^= 0x01
        with pytest.raises(qw.QwamError) as e:
            qw.load_image(bytes(bad))
        assert e.value.status == 8
    assert torch.cuda.mem_get_info()[0] == free0
    h.destroy()
