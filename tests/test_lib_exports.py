"""The C-ABI library loads and exports every entry point include/averis.h
declares; host-side validation needs no GPU (no compute calls here)."""

import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "averis.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^(?:size_t|avr_status|const char\s*\*)\s*(\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from quantized_gemm_column_b200 import build, api
    build.build()
    return api.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["averis_split_quant", "averis_linear_fwd", "averis_linear_dgrad", "nvfp4_quant",
              "nvfp4_linear_fwd", "nvfp4_linear_dgrad", "nvfp4_gemm", "averis_quant_weight",
              "averis_workspace_size", "averis_check_status"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_the_header():
    from quantized_gemm_column_b200 import api
    for n in declared_functions():
        assert hasattr(api, n), n


def test_host_side_sizes(lib):
    from quantized_gemm_column_b200 import api
    assert api.avr_nvfp4_scales_bytes(1, 1024) == 128 * 64
    assert api.avr_nvfp4_scales_bytes(300, 64) == 384 * 4
    assert api.averis_workspace_size(8192, 4096, 4096) > 8192 * 4096 // 2
    assert api.status_string(api.AVR_ERR_NONFINITE).startswith("non-finite")


def test_validation_rejects_before_any_launch(lib):
    """Bad arguments return their codes without touching a device."""
    from quantized_gemm_column_b200 import api
    q = api.avr_nvfp4(16, 16, 16, 256, 100)
    ws = ctypes.c_void_p(256)
    # null input
    assert lib.averis_split_quant(None, 1, 256, 128, 0, 0, 0, 0, None, None, ctypes.byref(q), None,
                                  ws, 1 << 30, None) == api.AVR_ERR_INVALID_ARG
    # K not a multiple of 64
    assert lib.averis_split_quant(ctypes.c_void_p(16), 1, 256, 100, 0, 0, 0, 0, None, None,
                                  ctypes.byref(q), None, ws, 1 << 30, None) == api.AVR_ERR_UNSUPPORTED_SHAPE
    # descriptor shape disagrees with the call
    assert lib.averis_split_quant(ctypes.c_void_p(16), 1, 256, 128, 0, 0, 0, 0, None, None,
                                  ctypes.byref(q), None, ws, 1 << 30, None) == api.AVR_ERR_INVALID_ARG
    q2 = api.avr_nvfp4(16, 16, 16, 256, 128)
    # misaligned input
    assert lib.averis_split_quant(ctypes.c_void_p(18), 1, 256, 128, 0, 0, 0, 0, None, None,
                                  ctypes.byref(q2), None, ws, 1 << 30, None) == api.AVR_ERR_MISALIGNED
    # workspace too small
    assert lib.averis_split_quant(ctypes.c_void_p(16), 1, 256, 128, 0, 0, 0, 0, None, None,
                                  ctypes.byref(q2), None, ws, 64, None) == api.AVR_ERR_WORKSPACE_TOO_SMALL
    # bad enum
    assert lib.averis_split_quant(ctypes.c_void_p(16), 7, 256, 128, 0, 0, 0, 0, None, None,
                                  ctypes.byref(q2), None, ws, 1 << 30, None) == api.AVR_ERR_INVALID_ARG
    # l = 0 is a no-op that needs no device
    q0 = api.avr_nvfp4(16, 16, 16, 0, 128)
    assert lib.averis_split_quant(ctypes.c_void_p(16), 1, 0, 128, 0, 0, 0, 0, None, None,
                                  ctypes.byref(q0), None, ws, 1 << 30, None) == api.AVR_OK
    # GEMM: N not a multiple of 64
    a = api.avr_nvfp4(16, 16, 16, 128, 128)
    b = api.avr_nvfp4(16, 16, 16, 100, 128)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), None, ctypes.c_void_p(16), 1, ws, 1 << 30,
                          None) == api.AVR_ERR_UNSUPPORTED_SHAPE


def test_mean_energy_ratio_validation(lib):
    """The R monitor rejects bad arguments, and l = 0 (R is 0/0), before any launch."""
    from quantized_gemm_column_b200 import api
    ws = ctypes.c_void_p(256)
    R = ctypes.c_void_p(16)
    f = lib.averis_mean_energy_ratio
    assert f(None, 1, 256, 128, None, R, ws, 1 << 30, None) == api.AVR_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(16), 1, 256, 128, None, None, ws, 1 << 30, None) == api.AVR_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(16), 1, 0, 128, None, R, ws, 1 << 30, None) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert f(ctypes.c_void_p(16), 1, 256, 96, None, R, ws, 1 << 30, None) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert f(ctypes.c_void_p(24), 1, 256, 128, None, R, ws, 1 << 30, None) == api.AVR_ERR_MISALIGNED
    assert f(ctypes.c_void_p(16), 1, 256, 128, None, R, ws, 64, None) == api.AVR_ERR_WORKSPACE_TOO_SMALL
    assert f(ctypes.c_void_p(16), 9, 256, 128, None, R, ws, 1 << 30, None) == api.AVR_ERR_INVALID_ARG
