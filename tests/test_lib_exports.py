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


def test_moe_validation(lib):
    """The MoE entry points reject bad arguments before any launch: the
    buffer's row count, the expert-count and tile limits, null or misaligned
    pointers, descriptors that disagree with the call, a short workspace."""
    from quantized_gemm_column_b200 import api
    ws = ctypes.c_void_p(256)
    X = ctypes.c_void_p(16)
    cnt = ctypes.c_void_p(64)
    E, l_cap, K = 4, 512, 256
    xr = api.avr_nvfp4(16, 16, 16, l_cap, K)
    f = lib.averis_moe_split_quant
    args = lambda **kw: [kw.get("X", X), kw.get("xt", 1), kw.get("l_cap", l_cap), kw.get("cnt", cnt),
                         kw.get("E", E), kw.get("K", K), 0, 0, 0, 0, None, None, ctypes.byref(kw.get("xr", xr)),
                         ws, kw.get("ws_bytes", 1 << 40), None]
    assert f(*args(xt=7)) == api.AVR_ERR_INVALID_ARG
    assert f(*args(l_cap=300, xr=api.avr_nvfp4(16, 16, 16, 300, K))) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert f(*args(E=0)) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert f(*args(E=1025)) == api.AVR_ERR_UNSUPPORTED_SHAPE
    # E x ceil(K / 128) column tiles above the 4096 slots
    assert f(*args(E=1024, K=640, xr=api.avr_nvfp4(16, 16, 16, l_cap, 640))) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert f(*args(K=96, xr=api.avr_nvfp4(16, 16, 16, l_cap, 96))) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert f(*args(cnt=None)) == api.AVR_ERR_INVALID_ARG
    assert f(*args(xr=api.avr_nvfp4(16, 16, 16, 384, K))) == api.AVR_ERR_INVALID_ARG
    assert f(*args(X=ctypes.c_void_p(24))) == api.AVR_ERR_MISALIGNED
    assert f(*args(cnt=ctypes.c_void_p(66))) == api.AVR_ERR_MISALIGNED
    assert f(*args(ws_bytes=64)) == api.AVR_ERR_WORKSPACE_TOO_SMALL
    # linear: N must be a multiple of 128, the stacked weights [E n, m]
    m, n = 256, 384
    w = api.avr_nvfp4(16, 16, 16, E * n, m)
    g = lib.averis_moe_linear_fwd
    Y = ctypes.c_void_p(16)
    assert g(X, 1, l_cap, cnt, E, m, 320, ctypes.byref(api.avr_nvfp4(16, 16, 16, E * 320, m)), 1, 0, 0, Y, 1,
             ws, 1 << 40, None) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert g(X, 1, l_cap, cnt, E, m, n, ctypes.byref(api.avr_nvfp4(16, 16, 16, n, m)), 1, 0, 0, Y, 1, ws,
             1 << 40, None) == api.AVR_ERR_INVALID_ARG
    assert g(X, 1, l_cap, cnt, E, m, n, ctypes.byref(w), 1, 0, 0, None, 1, ws, 1 << 40,
             None) == api.AVR_ERR_INVALID_ARG
    assert g(X, 1, l_cap, cnt, E, m, n, ctypes.byref(w), 1, 0, 0, Y, 1, ws, 64,
             None) == api.AVR_ERR_WORKSPACE_TOO_SMALL
    # the workspace grows with the experts and the buffer
    assert api.averis_moe_workspace_size(l_cap, K, 0, 8) > api.averis_moe_workspace_size(l_cap, K, 0, 4)
    assert api.averis_moe_workspace_size(2 * l_cap, K, 0, 4) > api.averis_moe_workspace_size(l_cap, K, 0, 4)


def test_linear_and_weight_validation(lib):
    """The linear, weight, one-kernel-split and rank-one-row entry points
    reject bad arguments before any launch; l = 0 is a no-op."""
    from quantized_gemm_column_b200 import api
    ws = ctypes.c_void_p(256)
    X, Y = ctypes.c_void_p(16), ctypes.c_void_p(32)
    l, m, n = 256, 128, 192
    wf = api.avr_nvfp4(16, 16, 16, n, m)          # w_fwd [n, m]
    wd = api.avr_nvfp4(16, 16, 16, m, n)          # w_dgrad [m, n]
    fwd = lambda **kw: lib.averis_linear_fwd(kw.get("X", X), kw.get("xt", 1), kw.get("l", l), kw.get("m", m),
                                             kw.get("n", n), ctypes.byref(kw.get("w", wf)), 1, 0, 0,
                                             kw.get("Y", Y), kw.get("yt", 1), kw.get("save_xr"), None, ws,
                                             kw.get("ws_bytes", 1 << 40), None)
    assert fwd(xt=3) == api.AVR_ERR_INVALID_ARG
    assert fwd(yt=3) == api.AVR_ERR_INVALID_ARG
    assert fwd(m=96, w=api.avr_nvfp4(16, 16, 16, n, 96)) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert fwd(n=100, w=api.avr_nvfp4(16, 16, 16, 100, m)) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert fwd(w=wd) == api.AVR_ERR_INVALID_ARG                      # [m, n] given for [n, m]
    assert fwd(save_xr=ctypes.byref(api.avr_nvfp4(16, 16, 16, l, n))) == api.AVR_ERR_INVALID_ARG
    assert fwd(Y=ctypes.c_void_p(40)) == api.AVR_ERR_MISALIGNED
    assert fwd(ws_bytes=64) == api.AVR_ERR_WORKSPACE_TOO_SMALL
    assert fwd(l=0) == api.AVR_OK
    assert lib.averis_linear_dgrad(X, 1, l, m, n, ctypes.byref(wf), 1, 0, 0, Y, 1, ws, 1 << 40,
                                   None) == api.AVR_ERR_INVALID_ARG       # w_fwd given for w_dgrad
    # weights: both dimensions multiples of 64, descriptors [n, m] and [m, n]
    qw = lib.averis_quant_weight
    assert qw(X, 1, m, 100, ctypes.byref(wf), ctypes.byref(wd), ws, 1 << 40, None) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert qw(X, 1, m, n, ctypes.byref(wd), ctypes.byref(wf), ws, 1 << 40, None) == api.AVR_ERR_INVALID_ARG
    assert qw(ctypes.c_void_p(24), 1, m, n, ctypes.byref(wf), ctypes.byref(wd), ws, 1 << 40,
              None) == api.AVR_ERR_MISALIGNED
    # one-kernel split
    xr = api.avr_nvfp4(16, 16, 16, l, m)
    fu = lib.averis_split_quant_fused
    assert fu(X, 1, l, 100, 0, 0, 0, 0, None, None, ctypes.byref(xr), ws, 1 << 40, None) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert fu(X, 1, l, m, 0, 0, 0, 0, None, None, ctypes.byref(wf), ws, 1 << 40, None) == api.AVR_ERR_INVALID_ARG
    assert fu(X, 1, 0, m, 0, 0, 0, 0, None, None, ctypes.byref(xr), ws, 1 << 40, None) == api.AVR_OK
    # rank-one row: mu_bar [1, K] against W_bar [N, K]
    mq = api.avr_nvfp4(16, 16, 16, 1, m)
    assert lib.averis_bias_row(None, ctypes.byref(wf), Y, ws, 1 << 40, None) == api.AVR_ERR_INVALID_ARG
    assert lib.averis_bias_row(ctypes.byref(mq), ctypes.byref(wd), Y, ws, 1 << 40, None) == api.AVR_ERR_INVALID_ARG


def test_valid_call_without_a_device_fails_loudly(lib):
    """A call that passes every host check returns AVR_ERR_NO_DEVICE when no
    sm_100 device is current: there is no CPU path to fall back to.  (Skipped
    where a GPU is visible: the pointers here are not device memory.)"""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible; this check is for a host without one")
    from quantized_gemm_column_b200 import api
    wf = api.avr_nvfp4(16, 16, 16, 192, 128)
    st = lib.averis_linear_fwd(ctypes.c_void_p(16), 1, 256, 128, 192, ctypes.byref(wf), 1, 0, 0,
                               ctypes.c_void_p(32), 1, None, None, ctypes.c_void_p(256), 1 << 40, None)
    assert st == api.AVR_ERR_NO_DEVICE


def test_noalloc_validation_matches_the_workspace_entry_point(lib):
    """averis_split_quant_noalloc rejects what averis_split_quant rejects, with
    the same codes, before it touches a device: null and mis-shaped
    descriptors, misaligned codes, scales and decode scales, a misaligned
    status word, sizes beyond its fixed scratch."""
    from quantized_gemm_column_b200 import api
    f = lib.averis_split_quant_noalloc
    X = ctypes.c_void_p(16)

    def call(xr, muq=None, x=X, l=256, K=128, status=None, xt=1, rm=0):
        return f(x, xt, l, K, rm, 0, 0, 0, None, None if muq is None else ctypes.byref(muq),
                 None if xr is None else ctypes.byref(xr), None, status, None)

    good = api.avr_nvfp4(16, 16, 16, 256, 128)
    assert call(None) == api.AVR_ERR_INVALID_ARG                                   # no X_bar_R descriptor
    assert call(good, x=None) == api.AVR_ERR_INVALID_ARG                           # no input
    assert call(api.avr_nvfp4(0, 16, 16, 256, 128)) == api.AVR_ERR_INVALID_ARG     # null codes
    assert call(api.avr_nvfp4(16, 0, 16, 256, 128)) == api.AVR_ERR_INVALID_ARG     # null scales
    assert call(api.avr_nvfp4(16, 16, 0, 256, 128)) == api.AVR_ERR_INVALID_ARG     # null g_dec
    assert call(api.avr_nvfp4(16, 16, 16, 255, 128)) == api.AVR_ERR_INVALID_ARG   # rows != l
    assert call(api.avr_nvfp4(16, 16, 16, 256, 192)) == api.AVR_ERR_INVALID_ARG   # K disagrees
    assert call(good, api.avr_nvfp4(16, 16, 16, 2, 128)) == api.AVR_ERR_INVALID_ARG   # mu_bar rows != 1
    assert call(good, api.avr_nvfp4(0, 16, 16, 1, 128)) == api.AVR_ERR_INVALID_ARG    # mu_bar null codes
    assert call(api.avr_nvfp4(24, 16, 16, 256, 128)) == api.AVR_ERR_MISALIGNED    # codes
    assert call(api.avr_nvfp4(16, 24, 16, 256, 128)) == api.AVR_ERR_MISALIGNED    # scales
    assert call(api.avr_nvfp4(16, 16, 18, 256, 128)) == api.AVR_ERR_MISALIGNED    # g_dec
    assert call(good, api.avr_nvfp4(16, 16, 18, 1, 128)) == api.AVR_ERR_MISALIGNED   # mu_bar g_dec
    assert call(good, x=ctypes.c_void_p(24)) == api.AVR_ERR_MISALIGNED           # input
    assert call(good, status=ctypes.c_void_p(18)) == api.AVR_ERR_MISALIGNED      # status word
    assert call(good, K=100) == api.AVR_ERR_UNSUPPORTED_SHAPE
    assert call(good, xt=5) == api.AVR_ERR_INVALID_ARG
    assert call(good, rm=3) == api.AVR_ERR_INVALID_ARG
    assert call(api.avr_nvfp4(16, 16, 16, 0, 128), l=0) == api.AVR_OK             # no tokens: no-op
    # beyond the fixed scratch: 3 ceil(l/256) K 4 bytes of partials alone exceed 4 MiB
    big = api.avr_nvfp4(16, 16, 16, 32768, 4096)
    assert call(big, l=32768, K=4096) == api.AVR_ERR_WORKSPACE_TOO_SMALL
    # the workspace entry point gives the same codes for the same arguments
    ws = ctypes.c_void_p(256)
    for xr, muq in ((api.avr_nvfp4(16, 16, 18, 256, 128), None), (api.avr_nvfp4(16, 16, 16, 255, 128), None),
                    (good, api.avr_nvfp4(16, 16, 16, 2, 128))):
        ws_code = lib.averis_split_quant(X, 1, 256, 128, 0, 0, 0, 0, None,
                                         None if muq is None else ctypes.byref(muq), ctypes.byref(xr), None,
                                         ws, 1 << 40, None)
        assert call(xr, muq) == ws_code


def test_noalloc_without_a_device_fails_loudly(lib):
    """A valid no-alloc call returns AVR_ERR_NO_DEVICE on a host without an
    sm_100 device (skipped where a GPU is visible)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible; this check is for a host without one")
    from quantized_gemm_column_b200 import api
    xr = api.avr_nvfp4(16, 16, 16, 256, 128)
    st = lib.averis_split_quant_noalloc(ctypes.c_void_p(16), 1, 256, 128, 1, 0, 0, 0, None, None,
                                        ctypes.byref(xr), None, None, None)
    assert st == api.AVR_ERR_NO_DEVICE


def test_set_wait_limit_validation_on_the_host(lib):
    from quantized_gemm_column_b200 import api
    f = lib.averis_set_wait_limit
    assert f(None, 1 << 20, 5, None) == api.AVR_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(272), 1 << 20, 5, None) == api.AVR_ERR_MISALIGNED
    assert f(ctypes.c_void_p(256), 128, 5, None) == api.AVR_ERR_WORKSPACE_TOO_SMALL
    import torch
    if not torch.cuda.is_available():
        assert f(ctypes.c_void_p(256), 1 << 20, 5, None) == api.AVR_ERR_NO_DEVICE


def _prototypes():
    """{name: (return type, [parameter types])} of every entry point in the
    header, comments removed, parameter names dropped."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    out = {}
    for ret, name, params in re.findall(
            r"^(size_t|avr_status|const char\s*\*)\s*(\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M | re.S):
        types = []
        for p in params.split(","):
            p = " ".join(p.split())
            if not p or p == "void":
                continue
            m = re.match(r"^(.*?[\s*])(\w+)$", p)        # type, then the parameter's name
            types.append(m.group(1).replace(" ", "") if m else p.replace(" ", ""))
        out[name] = (ret.replace(" ", ""), types)
    return out


def _c_class(t):
    """The ctypes class a C parameter or return type must be marshalled as."""
    if t.endswith("*") or t == "avr_stream":
        return "ptr"
    # size_t and uint64_t are one ctypes type (c_ulong) on this ABI
    return {"int64_t": "i64", "uint64_t": "u64", "uint32_t": "u32", "size_t": "u64", "int": "int",
            "avr_dtype": "int", "avr_round": "int", "avr_status": "int"}[t]


def _ctypes_class(ct):
    if ct is ctypes.c_void_p or ct is ctypes.c_char_p or (isinstance(ct, type) and issubclass(ct, ctypes._Pointer)):
        return "ptr"
    assert ctypes.c_size_t is ctypes.c_uint64
    return {ctypes.c_int64: "i64", ctypes.c_uint64: "u64", ctypes.c_uint32: "u32", ctypes.c_int: "int"}[ct]


def test_binding_signatures_match_the_header():
    """Every entry point's ctypes signature has the header's arity and, per
    argument, the same class (pointer, int, int64, uint64 or size_t, uint32):
    a slip in the argument list would otherwise pass garbage silently."""
    from quantized_gemm_column_b200 import api
    protos = _prototypes()
    assert set(protos) == set(declared_functions())
    for name, (ret, params) in protos.items():
        assert name in api._SIGS, name
        res, args = api._SIGS[name]
        assert len(args) == len(params), (name, len(args), params)
        got = [_ctypes_class(a) for a in args]
        want = [_c_class(p) for p in params]
        assert got == want, (name, got, want)
        assert _ctypes_class(res) == ("ptr" if ret == "constchar*" else _c_class(ret)), name


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """Without the built library the binding raises: nothing falls back to a
    CPU path or to the oracle."""
    from quantized_gemm_column_b200 import api
    monkeypatch.setattr(api, "_LIB", None)
    monkeypatch.setattr(api._build, "LIB", str(tmp_path / "libaveris.so"))
    with pytest.raises(api.AverisError) as e:
        api.load()
    assert e.value.status == api.AVR_ERR_NO_DEVICE
    with pytest.raises(api.AverisError):
        api.averis_workspace_size(256, 128)


def test_product_path_never_imports_the_oracle():
    """The package's sources name no oracle module: only the tests, the smoke
    check and the benchmark's CPU legs use it."""
    pkg = os.path.join(ROOT, "quantized_gemm_column_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
                assert "import oracle" not in text, f


def test_oracle_imports_nothing_of_the_cuda_path():
    """The oracle is independent of the CUDA path: it imports only numpy and
    the standard library, never the package or its library."""
    allowed = {"numpy", "math", "dataclasses"}
    odir = os.path.join(ROOT, "oracle")
    for f in os.listdir(odir):
        if not f.endswith(".py"):
            continue
        text = open(os.path.join(odir, f), encoding="utf-8").read()
        for mod in re.findall(r"^\s*(?:import|from)\s+([\w.]+)", text, flags=re.M):
            assert mod.startswith(".") or mod.split(".")[0] in allowed, (f, mod)
        assert "quantized_gemm_column_b200" not in text and "libaveris" not in text, f
