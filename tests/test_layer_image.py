"""Layer images (qwam_image_size / qwam_save_image / qwam_load_image): the
host-side checks of qwam_load_image, which run before any device call.

Images are built here from the layout the header documents (a 64-byte
header, 16-byte-padded arrays, FNV-1a 64 checksum), so a valid image must get
past every host check and stop only at the device (no GPU here), and any
damaged one must be refused with QWAM_ERR_FORMAT."""
import ctypes
import struct

import pytest

FORMAT, INVALID = 8, 1


def fnv1a64(data: bytes, h: int = 0xCBF29CE484222325) -> int:
    for c in data:
        h ^= c
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def pad16(n):
    return (n + 15) // 16 * 16


def image_len(N, K, r, fmt, bias):
    n = 64 + pad16(N * (K if fmt == 1 else K // 2))   # INT4: 4-bit levels, two per byte
    if fmt == 0:
        n += pad16((N + 255) // 256 * 256 * K // 16)
    if fmt == 2:
        n += pad16(K // 64 * N * 2)                   # fp16 group scales
    if r:
        n += pad16(N * r * 2) + 4 * pad16(K * r * 2)
    n += pad16(K * 4)
    if bias:
        n += pad16(N * 2)
    return n


def make_image(N=16, K=128, r=0, b=1, fmt=0, variant=0, bias=False, g_w=1.0, total=None, magic=b"QWAMIMG\0",
               version=1, fix_checksum=True):
    n = image_len(N, K, r, fmt, bias)
    total = n if total is None else total
    hdr = struct.pack("<8sII6iIfQQ", magic, version, 64, N, K, r, b, fmt, variant, 1 if bias else 0, g_w, total, 0)
    img = bytearray(hdr + bytes(range(256)) * ((n - 64) // 256) + bytes((n - 64) % 256))
    if fix_checksum:
        img[56:64] = struct.pack("<Q", fnv1a64(bytes(img)))
    return bytes(img)


@pytest.fixture(scope="module")
def lib():
    import os
    from bit_w4a4_quantised_b200 import binding
    if not os.path.exists(binding.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    return binding.load()


def load(lib, img, n=None):
    out = ctypes.c_void_p()
    st = lib.qwam_load_image(img, len(img) if n is None else n, None, ctypes.byref(out))
    return st, lib.qwam_last_error().decode(), out.value


def test_fnv1a64_published_vectors():
    # the FNV-1a 64 test vectors of its authors: "", "a", "foobar"
    assert fnv1a64(b"") == 0xCBF29CE484222325
    assert fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a64(b"foobar") == 0x85944171F73967E8


def test_header_is_64_bytes():
    assert struct.calcsize("<8sII6iIfQQ") == 64


@pytest.mark.parametrize("kw", [dict(), dict(r=32, b=128, K=256, N=48, bias=True), dict(fmt=1, r=16, K=384, b=64),
                                dict(variant=1, r=16, N=64), dict(fmt=2, variant=2, r=32, K=256, N=32, bias=True)])
def test_valid_image_passes_every_host_check(lib, kw):
    st, msg, h = load(lib, make_image(**kw))
    # no GPU here: the first device call fails, after the format checks
    assert st not in (FORMAT, INVALID), msg
    assert h is None


def test_longer_buffer_is_accepted(lib):
    img = make_image()
    st, msg, _ = load(lib, img + bytes(100))
    assert st != FORMAT, msg


@pytest.mark.parametrize("offset", [0, 8, 16, 44, 64, 1000, -1])
def test_any_flipped_byte_is_refused(lib, offset):
    img = bytearray(make_image(r=16, N=32, K=256, b=16, bias=True))
    img[offset] ^= 0x10
    st, msg, h = load(lib, bytes(img))
    assert st == FORMAT and h is None, msg


@pytest.mark.parametrize("kw,word", [
    (dict(magic=b"QWAMIMX\0"), "magic"),
    (dict(version=2), "version"),
    (dict(K=100), "shape"),
    (dict(r=8), "shape"),
    (dict(b=3), "shape"),
    (dict(fmt=2), "out of range"),
    (dict(fmt=1, variant=1), "out of range"),
    (dict(fmt=2, variant=0), "out of range"),
    (dict(fmt=0, variant=2), "out of range"),
    (dict(fmt=2, variant=2, b=16), "out of range"),
    (dict(g_w=0.0), "out of range"),
    (dict(g_w=float("nan")), "out of range"),
    (dict(total=3000), "bytes"),
])
def test_bad_header_is_refused(lib, kw, word):
    st, msg, h = load(lib, make_image(**kw))
    assert st == FORMAT and h is None
    assert word in msg


def test_short_buffer_is_refused(lib):
    img = make_image()
    assert load(lib, img, len(img) - 16)[0] == FORMAT
    assert load(lib, img[:40])[0] == FORMAT


def test_null_arguments(lib):
    out = ctypes.c_void_p()
    assert lib.qwam_load_image(None, 100, None, ctypes.byref(out)) == INVALID
    assert lib.qwam_load_image(make_image(), 100, None, None) == INVALID
    n = ctypes.c_size_t()
    assert lib.qwam_image_size(None, ctypes.byref(n)) == INVALID
    assert lib.qwam_save_image(None, None, 0, None) == INVALID
