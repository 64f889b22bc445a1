"""The C-ABI library loads and exports every entry point the header declares
(CPU only: argument checks that return before any device work)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "qwam.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qwam_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from bit_w4a4_quantised_b200 import binding
    if not os.path.exists(binding.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    return binding.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("qwam_prepare_weight", "qwam_linear", "qwam_destroy", "qwam_last_error"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_the_header(lib):
    from bit_w4a4_quantised_b200 import binding
    assert sorted(binding.SIGNATURES) == declared_functions()


def test_status_strings_and_version(lib):
    assert lib.qwam_status_string(0) == b"QWAM_OK"
    assert lib.qwam_status_string(7) == b"QWAM_ERR_TIMEOUT"
    assert lib.qwam_version() >= 100


def test_argument_errors_need_no_device(lib):
    # rejected before any CUDA call: NULL out pointer, NULL handle
    assert lib.qwam_prepare_weight(None, 16, 128, None, None, 0, None, 1, None, None) == 1
    assert b"NULL" in lib.qwam_last_error()
    assert lib.qwam_handle_info(None, None, None, None, None, None) == 1
    assert lib.qwam_destroy(None) == 1
    assert lib.qwam_device_error(None) == 1


def test_built_for_sm100a_only():
    src = open(os.path.join(ROOT, "bit_w4a4_quantised_b200", "build.py")).read()
    assert "arch=compute_100a,code=sm_100a" in src


def test_int4_and_image_entry_points_check_arguments_first(lib):
    import ctypes
    assert lib.qwam_status_string(8) == b"QWAM_ERR_FORMAT"
    out = ctypes.c_void_p()
    # NULL out pointer / NULL weight: refused before any device call
    assert lib.qwam_prepare_weight_int4(None, 16, 128, None, None, 0, None, None, None, None) == 1
    assert lib.qwam_prepare_weight_int4(None, 16, 128, None, None, 0, None, None, None, ctypes.byref(out)) == 1
    # the bare group GEMM: NULL buffers, then shapes, before any device call
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks stop first
    assert lib.qwam_int4_gemm(None, fake, fake, fake, 4, 16, 128, fake, None) == 1
    assert lib.qwam_int4_gemm(fake, fake, fake, fake, 3, 16, 128, fake, None) == 2   # M % 4
    assert lib.qwam_int4_gemm(fake, fake, fake, fake, 4, 24, 128, fake, None) == 2   # N % 16
    assert lib.qwam_int4_gemm(fake, fake, fake, fake, 4, 16, 192, fake, None) == 2   # K % 128
    assert b"multiple" in lib.qwam_last_error()
