"""NVFP4 encoding in plain NumPy — test infrastructure (see ``oracle/__init__``).

What the pages fix ("FastWAM UR3 3-task — 4-bit quantisations", top table,
row "numeric format"; section "Files", row for the NVFP4 checkpoint):

* elements are E2M1 (1 sign, 2 exponent, 1 mantissa bit), stored two per byte
  (the ``float4_e2m1fn_x2`` packing, 4.00 bits per weight — "Verification —
  NVFP4 deflated ASP", first table);
* blocks of 16 consecutive elements share one E4M3 scale (1 byte per 16
  elements — same table, "E4M3 block scales" row);
* scales are stored pre-swizzled into the 128-row x 4-column tile layout that
  FP4 tensor cores consume ("SWIZZLE_32_4_4", section "Files").

What the pages leave open and this oracle fixes (one reading each):

* a fp32 per-tensor scale ``g = amax / (6 * 448)`` over the whole tensor;
* the quantiser's fp32 operation order (below), with correctly rounded fp32
  divides / reciprocal / multiplies and round-to-nearest-even encoders;
* sign-preserving zero codes and the all-zero tensor convention ``g = 1``.

Quantiser Q on a fp32 tensor T[rows, K], blocks of 16 along K::

    A = max|T|                                  exact
    g = 1 if A == 0 else fp32(A / 2688)
    per block:  a = max|T_block|
                t = fp32(fp32(a / 6) / g)
                S = E4M3_RNE_satfinite(t)
                e = fp32(S * g)
                code_i = sign(T_i)<<3 | 0                         if e == 0
                code_i = sign(T_i)<<3 | E2M1_RNE(min(|q_i|, 6))   otherwise,
                         q_i = fp32(T_i * fp32(1 / e))
    dequant:    e2m1(code) * S * g

Both encoders are brute-force nearest-value searches over the full table of
representable magnitudes, ties to the even code, so nothing here depends on a
library's float8/float4 cast.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32

#: E2M1 magnitudes for the 3-bit magnitude code 0..7 (exponent bias 1,
#: exponent 0 is subnormal: 0, 0.5; then 1, 1.5, 2, 3, 4, 6).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)

#: Largest finite E4M3 magnitude (exponent 15, mantissa 6: 1.75 * 2**8).
E4M3_MAX = 448.0
#: Largest E2M1 magnitude.
E2M1_MAX = 6.0
#: Global-scale divisor 6 * 448.
GLOBAL_DIV = 2688.0
#: Elements per scale block.
BLOCK = 16


def e4m3_magnitudes() -> np.ndarray:
    """Value of every non-negative finite E4M3 code 0x00..0x7E (0x7F is NaN).

    E4M3 (the "fn" variant): 4 exponent bits with bias 7, 3 mantissa bits,
    exponent field 0 holds subnormals m * 2**-9, no infinities.
    """
    vals = np.empty(127, dtype=np.float64)
    for code in range(127):
        e, m = code >> 3, code & 7
        if e == 0:
            vals[code] = m * 2.0 ** -9
        else:
            vals[code] = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


E4M3_MAGNITUDES = e4m3_magnitudes()


def _nearest_even(table: np.ndarray, x: np.ndarray) -> np.ndarray:
    """Index of the table value nearest to each x (table ascending, x >= 0,
    x <= table[-1]); on an exact tie the even index wins."""
    x = np.asarray(x, dtype=np.float64)
    hi = np.searchsorted(table, x, side="left")
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    d_lo = x - table[lo]
    d_hi = table[hi] - x
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    return np.where(pick_hi, hi, lo).astype(np.int64)


def encode_e4m3_satfinite(t) -> np.ndarray:
    """E4M3 code of non-negative fp32 t: round to nearest, ties to even,
    values above 448 saturate to 448 (code 0x7E)."""
    t = np.asarray(t, dtype=np.float32).astype(np.float64)
    if np.any(t < 0) or np.any(~np.isfinite(t)):
        raise ValueError("E4M3 block scale input must be finite and >= 0")
    t = np.minimum(t, E4M3_MAX)
    return _nearest_even(E4M3_MAGNITUDES, t).astype(np.uint8)


def decode_e4m3(code) -> np.ndarray:
    """Value of an unsigned E4M3 scale code (0..126)."""
    code = np.asarray(code, dtype=np.int64)
    if np.any(code > 126) or np.any(code < 0):
        raise ValueError("scale code out of the finite non-negative range")
    return E4M3_MAGNITUDES[code]


def encode_e2m1(q) -> np.ndarray:
    """4-bit E2M1 code of fp32 q: sign bit from q's sign bit (so -0.0 and small
    negatives give 0x8), magnitude by round-to-nearest-even of min(|q|, 6)."""
    q = np.asarray(q, dtype=np.float32)
    sign = np.signbit(q).astype(np.uint8) << 3
    mag = np.minimum(np.abs(q).astype(np.float64), E2M1_MAX)
    return (sign | _nearest_even(E2M1_MAGNITUDES, mag).astype(np.uint8)).astype(np.uint8)


def decode_e2m1(code) -> np.ndarray:
    """Signed value of a 4-bit E2M1 code."""
    code = np.asarray(code, dtype=np.int64)
    mag = E2M1_MAGNITUDES[code & 7]
    return np.where(code & 8, -mag, mag)


def quantize(T) -> tuple[np.ndarray, np.ndarray, np.float32]:
    """Two-level NVFP4 quantiser Q on a fp32 tensor T[rows, K] (K % 16 == 0).

    Returns ``(codes, scales, g)``: codes uint8 [rows, K] holding one 4-bit
    code per element (unpacked), scales uint8 [rows, K/16] E4M3 codes, and the
    fp32 per-tensor scale g.  Every arithmetic step is a single correctly
    rounded fp32 operation in the order given in the module docstring.
    """
    T = np.asarray(T)
    if T.dtype != np.float32:
        raise TypeError("the quantiser input is fp32 by definition")
    rows, K = T.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    absT = np.abs(T)
    A = absT.max() if T.size else F32(0)
    g = F32(1.0) if A == 0 else F32(A) / F32(GLOBAL_DIV)
    blocks = T.reshape(rows, K // BLOCK, BLOCK)
    a = np.abs(blocks).max(axis=2)                       # exact, fp32
    t = (a / F32(6.0)) / g                               # two RN divisions
    assert t.dtype == np.float32
    S = encode_e4m3_satfinite(t)
    e = decode_e4m3(S).astype(np.float32) * g            # exact decode, RN multiply
    assert e.dtype == np.float32
    nz = e != 0
    safe_e = np.where(nz, e, F32(1.0))
    rc = F32(1.0) / safe_e                               # RN reciprocal
    q = blocks * rc[:, :, None]                          # RN multiply, no FMA
    assert q.dtype == np.float32
    codes = encode_e2m1(q)
    zero_codes = (np.signbit(blocks).astype(np.uint8) << 3)
    codes = np.where(nz[:, :, None], codes, zero_codes).astype(np.uint8)
    return codes.reshape(rows, K), S, F32(g)


def dequantize(codes, scales, g) -> np.ndarray:
    """float64 value of every element: e2m1(code) * e4m3(S) * g (exact in f64)."""
    codes = np.asarray(codes)
    rows, K = codes.shape
    s = decode_e4m3(scales)
    out = decode_e2m1(codes).reshape(rows, K // BLOCK, BLOCK) * s[:, :, None] * float(g)
    return out.reshape(rows, K)


def pack_nibbles(codes) -> np.ndarray:
    """Two codes per byte, element 2j in the low nibble (float4_e2m1fn_x2)."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_nibbles(packed) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    out = np.empty((rows, 2 * half), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def scale_tile_offset(m, kb, K: int):
    """Byte offset of the scale of row m, 16-element block kb, in the 128x4
    tiled layout for a tensor with K columns.

    Tiles cover 128 rows x 4 blocks (512 bytes) and are stored row-major over
    (row tile, block tile) with the block-tile index fastest.  Inside a tile,
    row m sits at (m % 32) * 16 + ((m // 32) % 4) * 4 and block kb at kb % 4.
    """
    m = np.asarray(m, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    kt = K // 64
    tile = (m // 128) * kt + kb // 4
    return tile * 512 + (m % 32) * 16 + ((m // 32) % 4) * 4 + kb % 4


def padded_rows(rows: int) -> int:
    return -(-rows // 128) * 128


def swizzle_scales(scales) -> np.ndarray:
    """Scale codes [rows, K/16] -> flat tiled buffer of padded_rows(rows)*K/16
    bytes; padding rows hold code 0."""
    scales = np.asarray(scales, dtype=np.uint8)
    rows, nb = scales.shape
    K = nb * BLOCK
    if K % 64:
        raise ValueError("the tiled scale layout needs K % 64 == 0")
    out = np.zeros(padded_rows(rows) * nb, dtype=np.uint8)
    m, kb = np.meshgrid(np.arange(rows), np.arange(nb), indexing="ij")
    out[scale_tile_offset(m, kb, K)] = scales
    return out


def unswizzle_scales(buf, rows: int, K: int) -> np.ndarray:
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    m, kb = np.meshgrid(np.arange(rows), np.arange(K // BLOCK), indexing="ij")
    return buf[scale_tile_offset(m, kb, K)]


def storage_bytes(n_weights: int) -> tuple[int, int]:
    """Bytes of packed E2M1 codes and of E4M3 block scales for n weights."""
    return n_weights // 2, n_weights // BLOCK
