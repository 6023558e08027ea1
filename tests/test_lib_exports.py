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


def test_wgrad_validation(lib):
    """Weight-gradient entry points reject bad arguments before any launch."""
    from quantized_gemm_column_b200 import api
    ws = ctypes.c_void_p(256)
    a = api.avr_nvfp4(16, 16, 16, 128, 320)     # [m = 128, L = 320]
    b = api.avr_nvfp4(16, 16, 16, 192, 320)
    mx = api.avr_nvfp4(16, 16, 16, 1, 128)
    md = api.avr_nvfp4(16, 16, 16, 1, 192)
    f = lib.averis_wgrad_gemm
    Y = ctypes.c_void_p(16)
    # one mean without the other
    assert f(ctypes.byref(a), ctypes.byref(b), ctypes.byref(mx), None, 300, Y, 0, ws, 1 << 30,
             None) == api.AVR_ERR_INVALID_ARG
    # L must be l rounded up to 64
    assert f(ctypes.byref(a), ctypes.byref(b), ctypes.byref(mx), ctypes.byref(md), 250, Y, 0, ws,
             1 << 30, None) == api.AVR_ERR_UNSUPPORTED_SHAPE
    # operands of different token lengths
    b2 = api.avr_nvfp4(16, 16, 16, 192, 384)
    assert f(ctypes.byref(a), ctypes.byref(b2), None, None, 300, Y, 0, ws, 1 << 30,
             None) == api.AVR_ERR_INVALID_ARG
    # workspace too small
    assert f(ctypes.byref(a), ctypes.byref(b), ctypes.byref(mx), ctypes.byref(md), 300, Y, 0, ws, 64,
             None) == api.AVR_ERR_WORKSPACE_TOO_SMALL
    # whole wgrad: n not a multiple of 64, bad dtype
    g = lib.averis_linear_wgrad
    assert g(Y, 1, Y, 1, 300, 128, 100, 1, 0, 0, Y, 0, ws, 1 << 30, None) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert g(Y, 5, Y, 1, 300, 128, 128, 1, 0, 0, Y, 0, ws, 1 << 30, None) == api.AVR_ERR_INVALID_ARG
    # token-axis quantizer: descriptor must be [K, L]
    q = api.avr_nvfp4(16, 16, 16, 128, 300)
    assert lib.averis_split_quant_t(Y, 1, 300, 128, 0, 0, 0, 0, None, None, ctypes.byref(q), ws,
                                    1 << 30, None) == api.AVR_ERR_INVALID_ARG
    assert api.averis_wgrad_workspace_size(8192, 1024, 4096) > (1024 + 4096) * 8192 // 2
