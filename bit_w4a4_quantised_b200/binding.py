"""ctypes binding of libqwam.so (declared in include/qwam.h).

Argument marshalling only: tensors are passed as raw device pointers, streams
as cudaStream_t handles, and every step of the layer runs in the library's
CUDA kernels.  There is no fallback: if the shared library is missing or a call
fails, this module raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqwam.so")

#: Every entry point declared in include/qwam.h, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
SIGNATURES = {
    "qwam_prepare_weight": (_I, [_P, _I, _I, _P, _P, _I, _P, _I, _P, ctypes.POINTER(_P)]),
    "qwam_destroy": (_I, [_P]),
    "qwam_linear": (_I, [_P, _I, _P, _P, _P]),
    "qwam_linear_noalloc": (_I, [_P, _I, _P, _P, _P]),
    "qwam_prologue": (_I, [_P, _I, _P, _P]),
    "qwam_gemm": (_I, [_I, _P, _P, _P]),
    "qwam_handle_info": (_I, [_P, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I),
                              ctypes.POINTER(_I), ctypes.POINTER(_F)]),
    "qwam_export_weight": (_I, [_P, _P, _P, _P, _P]),
    "qwam_debug_prepare_weight": (_I, [_P, _I, _I, _P, _P, _I, _P, _I, _P, _P, ctypes.POINTER(_P)]),
    "qwam_prepare_weight_shared": (_I, [_P, _I, _I, _P, _P, _I, _P, _I, _P, _P, ctypes.POINTER(_P)]),
    "qwam_prepare_weight_fp8": (_I, [_P, _I, _I, _P, _P, _I, _P, _I, _P, _P, ctypes.POINTER(_P)]),
    "qwam_prepare_weight_int4": (_I, [_P, _I, _I, _P, _P, _I, _P, _P, _P, ctypes.POINTER(_P)]),
    "qwam_int4_gemm": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "qwam_handle_format": (_I, [_P, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "qwam_image_size": (_I, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "qwam_save_image": (_I, [_P, _P, ctypes.c_size_t, _P]),
    "qwam_load_image": (_I, [_P, ctypes.c_size_t, _P, ctypes.POINTER(_P)]),
    "qwam_debug_prologue": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "qwam_quantize_fp32": (_I, [_P, _I, _I, _P, _P, _P, _P]),
    "qwam_fp4_gemm": (_I, [_P, _P, _P, _P, _I, _I, _I, _F, _P, _P]),
    "qwam_debug_fp4_gemm_withheld": (_I, [_P, _P, _P, _P, _I, _I, _I, ctypes.c_uint64, _P, _P]),
    "qwam_plan_info": (_I, [_I, _P, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I),
                            ctypes.POINTER(_I)]),
    "qwam_device_error": (_I, [ctypes.POINTER(ctypes.c_uint32)]),
    "qwam_selfcheck_rounding": (_I, [ctypes.POINTER(ctypes.c_uint64), ctypes.c_uint64, ctypes.c_void_p]),
    "qwam_last_error": (ctypes.c_char_p, []),
    "qwam_status_string": (ctypes.c_char_p, [_I]),
    "qwam_version": (_I, []),
}

STATUS = {0: "QWAM_OK", 1: "QWAM_ERR_INVALID_ARG", 2: "QWAM_ERR_SHAPE", 3: "QWAM_ERR_ALIGN",
          4: "QWAM_ERR_ARCH", 5: "QWAM_ERR_OOM", 6: "QWAM_ERR_CUDA", 7: "QWAM_ERR_TIMEOUT",
          8: "QWAM_ERR_FORMAT"}


class QwamError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libqwam.so once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m bit_w4a4_quantised_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        raise QwamError(status, load().qwam_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t, dtype, shape, name):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class Handle:
    """A prepared layer (owns device memory inside the library)."""

    def __init__(self, raw: int):
        self._raw = raw
        N, K, r, b, gw = _I(), _I(), _I(), _I(), _F()
        _check(load().qwam_handle_info(raw, ctypes.byref(N), ctypes.byref(K), ctypes.byref(r),
                                       ctypes.byref(b), ctypes.byref(gw)))
        self.N, self.K, self.r, self.b, self.g_w = N.value, K.value, r.value, b.value, gw.value
        fmt, var = _I(), _I()
        _check(load().qwam_handle_format(raw, ctypes.byref(fmt), ctypes.byref(var)))
        self.fmt = {0: "nvfp4", 1: "fp8", 2: "int4"}[fmt.value]
        self.variant = {0: "deflated", 1: "shared", 2: "svdquant"}[var.value]

    @property
    def code_bytes(self) -> int:
        """Bytes of one row of codes: K / 2 (NVFP4) or K (FP8; INT4 levels as E4M3 bytes)."""
        return self.K // 2 if self.fmt == "nvfp4" else self.K

    @property
    def raw(self) -> int:
        if not self._raw:
            raise ValueError("handle already destroyed")
        return self._raw

    def save_image(self, stream=None) -> bytes:
        """The layer image (qwam_save_image): header, operands, checksum."""
        n = ctypes.c_size_t()
        _check(load().qwam_image_size(self.raw, ctypes.byref(n)))
        buf = ctypes.create_string_buffer(n.value)
        _check(load().qwam_save_image(self.raw, buf, n.value, _stream(stream)))
        return buf.raw

    def destroy(self) -> None:
        if self._raw:
            _check(load().qwam_destroy(self._raw))
            self._raw = None

    def __del__(self):
        try:
            if self._raw and _lib is not None:
                _lib.qwam_destroy(self._raw)
        except Exception:
            pass


def prepare_weight(W, s, V, bias, hadamard_block: int, stream=None, wd_out=None, variant: str = "deflated",
                   fmt: str = "nvfp4") -> Handle:
    """W bf16 [N, K], s fp32 [K], V fp32 [K, r] or None, bias bf16 [N] or None.
    variant "deflated" (qwam_prepare_weight) or "shared" (the shared-weight
    arm, qwam_prepare_weight_shared); fmt "nvfp4" or "fp8" (the W8A8 arm,
    qwam_prepare_weight_fp8, deflated only); fmt "int4" with variant
    "svdquant" (the SVDQuant arm, qwam_prepare_weight_int4, hadamard_block 1).
    wd_out (fp32 [N, K]) receives the exact quantiser input: W_d for the
    deflated arm, W~ for the shared one, the residual R for SVDQuant."""
    import torch
    lib = load()
    N, K = W.shape
    _need(W, torch.bfloat16, (N, K), "W")
    _need(s, torch.float32, (K,), "s")
    r = 0 if V is None else V.shape[1]
    if V is not None:
        _need(V, torch.float32, (K, r), "V")
    if bias is not None:
        _need(bias, torch.bfloat16, (N,), "bias")
    out = _P()
    if variant not in ("deflated", "shared", "svdquant"):
        raise ValueError(f"variant must be 'deflated', 'shared' or 'svdquant', got {variant!r}")
    if (fmt not in ("nvfp4", "fp8", "int4") or (fmt == "fp8" and variant != "deflated")
            or ((fmt == "int4") != (variant == "svdquant")) or (fmt == "int4" and hadamard_block != 1)):
        raise ValueError(f"format {fmt!r} with variant {variant!r} and block {hadamard_block}")
    if wd_out is not None:
        _need(wd_out, torch.float32, (N, K), "wd_out")
    if fmt == "int4":
        _check(lib.qwam_prepare_weight_int4(_ptr(W), N, K, _ptr(s), _ptr(V), r, _ptr(bias), _ptr(wd_out),
                                            _stream(stream), ctypes.byref(out)))
    elif fmt == "fp8":
        _check(lib.qwam_prepare_weight_fp8(_ptr(W), N, K, _ptr(s), _ptr(V), r, _ptr(bias), hadamard_block,
                                           _ptr(wd_out), _stream(stream), ctypes.byref(out)))
    elif variant == "shared":
        _check(lib.qwam_prepare_weight_shared(_ptr(W), N, K, _ptr(s), _ptr(V), r, _ptr(bias), hadamard_block,
                                              _ptr(wd_out), _stream(stream), ctypes.byref(out)))
    elif wd_out is None:
        _check(lib.qwam_prepare_weight(_ptr(W), N, K, _ptr(s), _ptr(V), r, _ptr(bias), hadamard_block,
                                       _stream(stream), ctypes.byref(out)))
    else:
        _check(lib.qwam_debug_prepare_weight(_ptr(W), N, K, _ptr(s), _ptr(V), r, _ptr(bias), hadamard_block,
                                             _ptr(wd_out), _stream(stream), ctypes.byref(out)))
    return Handle(out.value)


def load_image(image: bytes, stream=None) -> Handle:
    """A handle on the current device from a layer image (qwam_load_image)."""
    out = _P()
    _check(load().qwam_load_image(image, len(image), _stream(stream), ctypes.byref(out)))
    return Handle(out.value)


def linear(x, h: Handle, y=None, stream=None):
    """y = the ASP NVFP4 layer applied to x (bf16 [M, K]) -> bf16 [M, N]."""
    import torch
    M = x.shape[0]
    _need(x, torch.bfloat16, (M, h.K), "x")
    if y is None:
        y = torch.empty((M, h.N), dtype=torch.bfloat16, device=x.device)
    _need(y, torch.bfloat16, (M, h.N), "y")
    _check(load().qwam_linear(_ptr(x), M, h.raw, _ptr(y), _stream(stream)))
    return y


def linear_noalloc(x, h: Handle, y, stream=None):
    """qwam_linear_noalloc: the layer with all scratch in the library's fixed
    static array (M <= 128, K <= 16384).  y (bf16 [M, N]) must be given, so the
    call itself allocates nothing."""
    import torch
    M = x.shape[0]
    _need(x, torch.bfloat16, (M, h.K), "x")
    _need(y, torch.bfloat16, (M, h.N), "y")
    _check(load().qwam_linear_noalloc(_ptr(x), M, h.raw, _ptr(y), _stream(stream)))
    return y


def prologue(x, h: Handle, stream=None) -> None:
    import torch
    _need(x, torch.bfloat16, (x.shape[0], h.K), "x")
    _check(load().qwam_prologue(_ptr(x), x.shape[0], h.raw, _stream(stream)))


def gemm(M: int, h: Handle, y, stream=None):
    import torch
    _need(y, torch.bfloat16, (M, h.N), "y")
    _check(load().qwam_gemm(M, h.raw, _ptr(y), _stream(stream)))
    return y


def export_weight(h: Handle, stream=None) -> dict:
    import torch
    dev = torch.device("cuda")
    codes = torch.empty((h.N, h.code_bytes), dtype=torch.uint8, device=dev)
    sf = torch.empty((-(-h.N // 128) * 128 * h.K // 16,), dtype=torch.uint8, device=dev)
    L = torch.empty((h.N, max(h.r, 1)), dtype=torch.bfloat16, device=dev)
    _check(load().qwam_export_weight(h.raw, _ptr(codes), _ptr(sf), _ptr(L) if h.r else None, _stream(stream)))
    return {"codes": codes, "scales": sf, "L": L[:, :h.r], "g_w": h.g_w}


def debug_prologue(x, h: Handle, stream=None) -> dict:
    import torch
    M = x.shape[0]
    _need(x, torch.bfloat16, (M, h.K), "x")
    dev = x.device
    z = torch.empty((M, h.K), dtype=torch.float32, device=dev)
    u = torch.empty((M, max(h.r, 1)), dtype=torch.float32, device=dev)
    codes = torch.empty((M, h.code_bytes), dtype=torch.uint8, device=dev)
    sf = torch.empty((-(-M // 128) * 128 * h.K // 16,), dtype=torch.uint8, device=dev)
    ub = torch.empty((M, max(h.r, 1)), dtype=torch.bfloat16, device=dev)
    gx = torch.empty((1,), dtype=torch.float32, device=dev)
    _check(load().qwam_debug_prologue(_ptr(x), M, h.raw, _ptr(z), _ptr(u) if h.r else None, _ptr(codes),
                                      _ptr(sf), _ptr(ub) if h.r else None, _ptr(gx), _stream(stream)))
    return {"z": z, "u": u[:, :h.r], "codes": codes, "scales": sf, "ub": ub[:, :h.r], "g_x": gx}


def int4_gemm(a_levels, a_scales, b_levels, b_scales, stream=None):
    """qwam_int4_gemm: a_levels u8 [M, K], a_scales fp32 [K/64, M], b_levels
    u8 [N, K], b_scales fp32 [K/64, N] (device) -> fp32 [M, N]."""
    import torch
    M, K = a_levels.shape
    N = b_levels.shape[0]
    _need(a_levels, torch.uint8, (M, K), "a_levels")
    _need(b_levels, torch.uint8, (N, K), "b_levels")
    _need(a_scales, torch.float32, (K // 64, M), "a_scales")
    _need(b_scales, torch.float32, (K // 64, N), "b_scales")
    out = torch.empty((M, N), dtype=torch.float32, device=a_levels.device)
    _check(load().qwam_int4_gemm(_ptr(a_levels), _ptr(a_scales), _ptr(b_levels), _ptr(b_scales), M, N, K, _ptr(out),
                                 _stream(stream)))
    return out


def quantize_fp32(T, stream=None):
    """Bare NVFP4 quantiser: T fp32 [rows, K] -> (codes [rows, K/2], tiled scales, g)."""
    import torch
    rows, K = T.shape
    _need(T, torch.float32, (rows, K), "T")
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=T.device)
    sf = torch.zeros((-(-rows // 128) * 128 * K // 16,), dtype=torch.uint8, device=T.device)
    g = torch.empty((1,), dtype=torch.float32, device=T.device)
    _check(load().qwam_quantize_fp32(_ptr(T), rows, K, _ptr(codes), _ptr(sf), _ptr(g), _stream(stream)))
    return codes, sf, g


def fp4_gemm(a_codes, a_scales, b_codes, b_scales, M: int, N: int, K: int, alpha: float = 1.0, stream=None):
    """Bare block-scaled FP4 GEMM -> fp32 [M, N] (scales tiled; B rows padded to 256)."""
    import torch
    out = torch.empty((M, N), dtype=torch.float32, device=a_codes.device)
    _check(load().qwam_fp4_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K,
                                float(alpha), _ptr(out), _stream(stream)))
    return out


def debug_fp4_gemm_withheld(a_codes, a_scales, b_codes, b_scales, M: int, N: int, K: int, wait_ns: int,
                            stream=None) -> None:
    """qwam_debug_fp4_gemm_withheld: the bare GEMM with a pipeline barrier that
    never completes and every bounded wait limited to wait_ns; the caller then
    reads the expired waits with device_error()."""
    import torch
    out = torch.empty((M, N), dtype=torch.float32, device=a_codes.device)
    _check(load().qwam_debug_fp4_gemm_withheld(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K,
                                               int(wait_ns), _ptr(out), _stream(stream)))


def plan_info(M: int, h: Handle) -> dict:
    """How qwam_linear runs M rows of this layer: kernel launches per call,
    single-launch prologue or not, GEMM K splits and tile width."""
    k, f, sp, bn = _I(), _I(), _I(), _I()
    _check(load().qwam_plan_info(M, h.raw, ctypes.byref(k), ctypes.byref(f), ctypes.byref(sp), ctypes.byref(bn)))
    return {"kernels": k.value, "fused": bool(f.value), "splits": sp.value, "bn": bn.value}


def device_error() -> int:
    code = ctypes.c_uint32(0)
    st = load().qwam_device_error(ctypes.byref(code))
    if st not in (0, 7):
        _check(st)
    return code.value


def selfcheck_rounding(random_pairs: int = 1 << 26) -> list:
    """Mismatch counts [a / 6, 1 / e, E4M3 code of u / g] of the quantiser's
    FMA-based arithmetic against the IEEE fp32 operations (qwam_selfcheck_rounding)."""
    out = (ctypes.c_uint64 * 3)()
    _check(load().qwam_selfcheck_rounding(out, random_pairs, None))
    return [int(v) for v in out]


def version() -> int:
    return load().qwam_version()
