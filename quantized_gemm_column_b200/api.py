"""ctypes binding of libaveris (include/averis.h), argument marshalling only.

Every function here has the name of the C entry point it calls.  Tensors are
torch CUDA tensors (PyTorch only provides device memory and streams); all
arithmetic happens in the library's CUDA kernels.  A missing library raises
``AverisError``: there is no CPU path.
"""

import ctypes
import os

import torch

from . import build as _build

_LIB = None

AVR_OK = 0
AVR_ERR_INVALID_ARG = 1
AVR_ERR_UNSUPPORTED_SHAPE = 2
AVR_ERR_MISALIGNED = 3
AVR_ERR_WORKSPACE_TOO_SMALL = 4
AVR_ERR_CUDA = 5
AVR_ERR_DEVICE_TIMEOUT = 6
AVR_ERR_NONFINITE = 7
AVR_ERR_NO_DEVICE = 8

AVR_F32 = 0
AVR_BF16 = 1
AVR_RNE = 0
AVR_SR = 1

_c_i64 = ctypes.c_int64
_c_u64 = ctypes.c_uint64
_c_u32 = ctypes.c_uint32
_c_size = ctypes.c_size_t
_c_int = ctypes.c_int
_c_ptr = ctypes.c_void_p


class AverisError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = int(status)
        msg = status_string(self.status) if _LIB is not None else str(status)
        super().__init__(f"{where}: {msg} (status {self.status})")


class avr_nvfp4(ctypes.Structure):
    _fields_ = [("codes", _c_ptr), ("scales", _c_ptr), ("g_dec", _c_ptr),
                ("rows", _c_i64), ("K", _c_i64)]


_SIGS = {
    "avr_nvfp4_scales_bytes": (_c_size, [_c_i64, _c_i64]),
    "averis_workspace_size": (_c_size, [_c_i64, _c_i64, _c_i64]),
    "averis_workspace_init": (_c_int, [_c_ptr, _c_size, _c_ptr]),
    "averis_check_status": (_c_int, [_c_ptr, _c_ptr]),
    "averis_set_wait_limit": (_c_int, [_c_ptr, _c_size, _c_u64, _c_ptr]),
    "averis_probe_mma_rate": (_c_int, [_c_int, _c_int, _c_ptr, _c_ptr, _c_size, _c_ptr]),
    "averis_status_string": (ctypes.c_char_p, [_c_int]),
    "averis_split_quant": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_int, _c_u64, _c_u64, _c_int,
                                    _c_ptr, ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4),
                                    _c_ptr, _c_ptr, _c_size, _c_ptr]),
    "averis_moe_workspace_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "averis_moe_quant_weights": (_c_int, [_c_ptr, _c_int, _c_int, _c_i64, _c_i64, ctypes.POINTER(avr_nvfp4),
                                          ctypes.POINTER(avr_nvfp4), _c_ptr, _c_size, _c_ptr]),
    "averis_moe_split_quant": (_c_int, [_c_ptr, _c_int, _c_i64, _c_ptr, _c_int, _c_i64, _c_int, _c_u64, _c_u64,
                                        _c_int, _c_ptr, ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4),
                                        _c_ptr, _c_size, _c_ptr]),
    "averis_moe_linear_fwd": (_c_int, [_c_ptr, _c_int, _c_i64, _c_ptr, _c_int, _c_i64, _c_i64,
                                       ctypes.POINTER(avr_nvfp4), _c_int, _c_u64, _c_u64, _c_ptr, _c_int, _c_ptr,
                                       _c_size, _c_ptr]),
    "averis_moe_linear_dgrad": (_c_int, [_c_ptr, _c_int, _c_i64, _c_ptr, _c_int, _c_i64, _c_i64,
                                         ctypes.POINTER(avr_nvfp4), _c_int, _c_u64, _c_u64, _c_ptr, _c_int,
                                         _c_ptr, _c_size, _c_ptr]),
    "averis_split_quant_fused": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_int, _c_u64, _c_u64, _c_int,
                                          _c_ptr, ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4),
                                          _c_ptr, _c_size, _c_ptr]),
    "averis_split_quant_t": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_int, _c_u64, _c_u64, _c_int,
                                      _c_ptr, ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4),
                                      _c_ptr, _c_size, _c_ptr]),
    "nvfp4_quant_t": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_int, _c_u64, _c_u64, _c_int,
                               ctypes.POINTER(avr_nvfp4), _c_ptr, _c_size, _c_ptr]),
    "averis_wgrad_workspace_size": (_c_size, [_c_i64, _c_i64, _c_i64]),
    "averis_wgrad_gemm": (_c_int, [ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4),
                                   ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4), _c_i64,
                                   _c_ptr, _c_int, _c_ptr, _c_size, _c_ptr]),
    "averis_linear_wgrad": (_c_int, [_c_ptr, _c_int, _c_ptr, _c_int, _c_i64, _c_i64, _c_i64, _c_int,
                                     _c_u64, _c_u64, _c_ptr, _c_int, _c_ptr, _c_size, _c_ptr]),
    "nvfp4_linear_wgrad": (_c_int, [_c_ptr, _c_int, _c_ptr, _c_int, _c_i64, _c_i64, _c_i64, _c_int,
                                    _c_u64, _c_u64, _c_ptr, _c_int, _c_ptr, _c_size, _c_ptr]),
    "averis_mean_energy_ratio": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_ptr, _c_ptr, _c_ptr,
                                          _c_size, _c_ptr]),
    "nvfp4_quant": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_int, _c_u64, _c_u64, _c_int,
                             ctypes.POINTER(avr_nvfp4), _c_ptr, _c_size, _c_ptr]),
    "averis_quant_weight": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, ctypes.POINTER(avr_nvfp4),
                                     ctypes.POINTER(avr_nvfp4), _c_ptr, _c_size, _c_ptr]),
    "averis_bias_row": (_c_int, [ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4), _c_ptr,
                                 _c_ptr, _c_size, _c_ptr]),
    "nvfp4_gemm": (_c_int, [ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4), _c_ptr, _c_ptr,
                            _c_int, _c_ptr, _c_size, _c_ptr]),
    "averis_linear_fwd": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_i64, ctypes.POINTER(avr_nvfp4),
                                   _c_int, _c_u64, _c_u64, _c_ptr, _c_int, ctypes.POINTER(avr_nvfp4),
                                   ctypes.POINTER(avr_nvfp4), _c_ptr, _c_size, _c_ptr]),
    "averis_linear_dgrad": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_i64, ctypes.POINTER(avr_nvfp4),
                                     _c_int, _c_u64, _c_u64, _c_ptr, _c_int, _c_ptr, _c_size, _c_ptr]),
    "nvfp4_linear_fwd": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_i64, ctypes.POINTER(avr_nvfp4),
                                  _c_int, _c_u64, _c_u64, _c_ptr, _c_int, _c_ptr, _c_size, _c_ptr]),
    "nvfp4_linear_dgrad": (_c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_i64, ctypes.POINTER(avr_nvfp4),
                                    _c_int, _c_u64, _c_u64, _c_ptr, _c_int, _c_ptr, _c_size, _c_ptr]),
    "averis_probe_convert": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_i64, _c_ptr]),
    "averis_probe_philox": (_c_int, [_c_u64, _c_u64, _c_u32, _c_i64, _c_ptr, _c_ptr]),
    "averis_probe_convert_sr": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_i64, _c_ptr]),
}


def library_path():
    return _build.LIB


def load():
    """Load libaveris.so (built in-tree); raise if it is missing."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise AverisError(AVR_ERR_NO_DEVICE,
                          f"{path} is missing; build it with python -m quantized_gemm_column_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def _check(st, where):
    if st != AVR_OK:
        raise AverisError(st, where)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return AVR_BF16
    if t.dtype == torch.float32:
        return AVR_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _round(rm):
    return {"rne": AVR_RNE, "sr": AVR_SR, AVR_RNE: AVR_RNE, AVR_SR: AVR_SR}[rm]


class NVFP4Tensor:
    """Device storage of an NVFP4 tensor [rows, K]: packed codes, E4M3 scales
    in the tcgen05 atom layout and the fp32 decode scale."""

    def __init__(self, rows, K, device="cuda"):
        self.rows, self.K = int(rows), int(K)
        self.codes = torch.empty((self.rows, self.K // 2), dtype=torch.uint8, device=device)
        nbytes = ((self.rows + 127) // 128 * 128) * (self.K // 16)
        self.scales = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.g_dec = torch.empty(1, dtype=torch.float32, device=device)

    def struct(self):
        return avr_nvfp4(self.codes.data_ptr(), self.scales.data_ptr(), self.g_dec.data_ptr(),
                         self.rows, self.K)


def _s(t):
    return None if t is None else ctypes.byref(t.struct())


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------
def avr_nvfp4_scales_bytes(rows, K):
    return int(load().avr_nvfp4_scales_bytes(rows, K))


def averis_workspace_size(l, K, N=0):
    return int(load().averis_workspace_size(l, K, N))


def status_string(st):
    return load().averis_status_string(int(st)).decode()


averis_status_string = status_string


def workspace(l, K, N=0, device="cuda", stream=None):
    """Allocate and zero-fill a workspace for the given sizes."""
    n = averis_workspace_size(l, K, N)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    averis_workspace_init(ws, stream)
    return ws


def averis_workspace_init(ws, stream=None):
    _check(load().averis_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "averis_workspace_init")


def averis_check_status(ws, stream=None):
    """Synchronize and return the latched device status (0 = ok)."""
    return int(load().averis_check_status(_ptr(ws), _stream(stream)))


def averis_probe_mma_rate(iters, ns, ws, stream=None):
    """MMA-only tcgen05 FP4 loop on ns.numel() CTAs; ns (int64, device) gets
    each CTA's elapsed nanoseconds."""
    _check(load().averis_probe_mma_rate(int(iters), ns.numel(), _ptr(ns), _ptr(ws), ws.numel(), _stream(stream)),
           "averis_probe_mma_rate")


def averis_set_wait_limit(ws, limit_ns, stream=None):
    """Bound (ns) of the waits on other CTAs; 0 restores the default 2 s."""
    _check(load().averis_set_wait_limit(_ptr(ws), ws.numel(), int(limit_ns), _stream(stream)),
           "averis_set_wait_limit")


def averis_split_quant(X, rm, seed, offset, grad, mu, mu_q, xr_q, xr_debug, ws, stream=None):
    l, K = X.shape
    _check(load().averis_split_quant(_ptr(X), _dtype(X), l, K, _round(rm), seed, offset, int(grad),
                                     _ptr(mu), _s(mu_q), _s(xr_q), _ptr(xr_debug), _ptr(ws),
                                     ws.numel(), _stream(stream)), "averis_split_quant")


def padded_tokens(l):
    """The token axis of the weight-gradient operands: l rounded up to 64."""
    return (int(l) + 63) // 64 * 64


def averis_wgrad_workspace_size(l, m, n):
    return int(load().averis_wgrad_workspace_size(l, m, n))


def wgrad_workspace(l, m, n, device="cuda"):
    """A zero-initialised workspace for the weight-gradient calls."""
    return torch.zeros(averis_wgrad_workspace_size(l, m, n), dtype=torch.uint8, device=device)


def averis_split_quant_t(X, rm, seed, offset, grad, mu, mu_q, xrt_q, ws, stream=None):
    l, K = X.shape
    _check(load().averis_split_quant_t(_ptr(X), _dtype(X), l, K, _round(rm), seed, offset, int(grad),
                                       _ptr(mu), _s(mu_q), _s(xrt_q), _ptr(ws), ws.numel(),
                                       _stream(stream)), "averis_split_quant_t")


def nvfp4_quant_t(X, rm, seed, offset, grad, out, ws, stream=None):
    l, K = X.shape
    _check(load().nvfp4_quant_t(_ptr(X), _dtype(X), l, K, _round(rm), seed, offset, int(grad),
                                _s(out), _ptr(ws), ws.numel(), _stream(stream)), "nvfp4_quant_t")


def averis_wgrad_gemm(xrt_q, drt_q, mu_x_q, mu_d_q, l, dW, ws, stream=None):
    _check(load().averis_wgrad_gemm(_s(xrt_q), _s(drt_q), _s(mu_x_q), _s(mu_d_q), l, _ptr(dW),
                                    _dtype(dW), _ptr(ws), ws.numel(), _stream(stream)),
           "averis_wgrad_gemm")


def averis_linear_wgrad(X, D, rm, seed, offset, dW, ws, stream=None):
    l, m = X.shape
    n = D.shape[1]
    _check(load().averis_linear_wgrad(_ptr(X), _dtype(X), _ptr(D), _dtype(D), l, m, n, _round(rm),
                                      seed, offset, _ptr(dW), _dtype(dW), _ptr(ws), ws.numel(),
                                      _stream(stream)), "averis_linear_wgrad")


def nvfp4_linear_wgrad(X, D, rm, seed, offset, dW, ws, stream=None):
    l, m = X.shape
    n = D.shape[1]
    _check(load().nvfp4_linear_wgrad(_ptr(X), _dtype(X), _ptr(D), _dtype(D), l, m, n, _round(rm),
                                     seed, offset, _ptr(dW), _dtype(dW), _ptr(ws), ws.numel(),
                                     _stream(stream)), "nvfp4_linear_wgrad")


def averis_mean_energy_ratio(X, mu, R, ws, stream=None):
    """R = ||mu_X|| / sqrt(E||x||^2 / m) into the 1-element fp32 device tensor R."""
    l, K = X.shape
    _check(load().averis_mean_energy_ratio(_ptr(X), _dtype(X), l, K, _ptr(mu), _ptr(R), _ptr(ws),
                                           ws.numel(), _stream(stream)), "averis_mean_energy_ratio")


class NVFP4Group(NVFP4Tensor):
    """An NVFP4 tensor [rows, K] with one decode scale per expert (MoE calls)."""

    def __init__(self, rows, K, groups, device="cuda"):
        super().__init__(rows, K, device)
        self.g_dec = torch.empty(groups, dtype=torch.float32, device=device)


def moe_padded_rows(counts):
    """Rows the permuted buffer needs: every expert's count rounded up to 128."""
    return sum((int(c) + 127) // 128 * 128 for c in counts)


def averis_moe_workspace_size(l_cap, K, N, E):
    return int(load().averis_moe_workspace_size(l_cap, K, N, E))


def moe_workspace(l_cap, K, N, E, device="cuda", stream=None):
    ws = torch.empty(averis_moe_workspace_size(l_cap, K, N, E), dtype=torch.uint8, device=device)
    averis_workspace_init(ws, stream)
    return ws


def averis_moe_quant_weights(W, w_fwd, w_dgrad, ws, stream=None):
    E, m, n = W.shape
    _check(load().averis_moe_quant_weights(_ptr(W), _dtype(W), E, m, n, _s(w_fwd), _s(w_dgrad), _ptr(ws),
                                           ws.numel(), _stream(stream)), "averis_moe_quant_weights")


def averis_moe_split_quant(X, counts, rm, seed, offset, grad, mu, mu_q, xr_q, ws, stream=None):
    l_cap, K = X.shape
    _check(load().averis_moe_split_quant(_ptr(X), _dtype(X), l_cap, _ptr(counts), counts.numel(), K, _round(rm),
                                         seed, offset, int(grad), _ptr(mu), _s(mu_q), _s(xr_q), _ptr(ws),
                                         ws.numel(), _stream(stream)), "averis_moe_split_quant")


def averis_moe_linear_fwd(X, counts, w_fwd, rm, seed, offset, Y, ws, stream=None):
    l_cap, m = X.shape
    n = Y.shape[1]
    _check(load().averis_moe_linear_fwd(_ptr(X), _dtype(X), l_cap, _ptr(counts), counts.numel(), m, n,
                                        _s(w_fwd), _round(rm), seed, offset, _ptr(Y), _dtype(Y), _ptr(ws),
                                        ws.numel(), _stream(stream)), "averis_moe_linear_fwd")


def averis_moe_linear_dgrad(D, counts, w_dgrad, rm, seed, offset, dX, ws, stream=None):
    l_cap, n = D.shape
    m = dX.shape[1]
    _check(load().averis_moe_linear_dgrad(_ptr(D), _dtype(D), l_cap, _ptr(counts), counts.numel(), m, n,
                                          _s(w_dgrad), _round(rm), seed, offset, _ptr(dX), _dtype(dX), _ptr(ws),
                                          ws.numel(), _stream(stream)), "averis_moe_linear_dgrad")


def averis_split_quant_fused(X, rm, seed, offset, grad, mu, mu_q, xr_q, ws, stream=None):
    l, K = X.shape
    _check(load().averis_split_quant_fused(_ptr(X), _dtype(X), l, K, _round(rm), seed, offset, int(grad),
                                           _ptr(mu), _s(mu_q), _s(xr_q), _ptr(ws), ws.numel(),
                                           _stream(stream)), "averis_split_quant_fused")


def nvfp4_quant(X, rm, seed, offset, grad, out, ws, stream=None):
    rows, K = X.shape
    _check(load().nvfp4_quant(_ptr(X), _dtype(X), rows, K, _round(rm), seed, offset, int(grad),
                              _s(out), _ptr(ws), ws.numel(), _stream(stream)), "nvfp4_quant")


def averis_quant_weight(W, w_fwd, w_dgrad, ws, stream=None):
    m, n = W.shape
    _check(load().averis_quant_weight(_ptr(W), _dtype(W), m, n, _s(w_fwd), _s(w_dgrad), _ptr(ws),
                                      ws.numel(), _stream(stream)), "averis_quant_weight")


def averis_bias_row(mu_q, w_q, bias, ws, stream=None):
    _check(load().averis_bias_row(_s(mu_q), _s(w_q), _ptr(bias), _ptr(ws), ws.numel(),
                                  _stream(stream)), "averis_bias_row")


def nvfp4_gemm(a, b, bias, Y, ws, stream=None):
    _check(load().nvfp4_gemm(_s(a), _s(b), _ptr(bias), _ptr(Y), _dtype(Y), _ptr(ws), ws.numel(),
                             _stream(stream)), "nvfp4_gemm")


def averis_linear_fwd(X, w_fwd, rm, seed, offset, Y, ws, save_xr=None, save_mu=None, stream=None):
    l, m = X.shape
    n = w_fwd.rows
    _check(load().averis_linear_fwd(_ptr(X), _dtype(X), l, m, n, _s(w_fwd), _round(rm), seed, offset,
                                    _ptr(Y), _dtype(Y), _s(save_xr), _s(save_mu), _ptr(ws),
                                    ws.numel(), _stream(stream)), "averis_linear_fwd")


def averis_linear_dgrad(D, w_dgrad, rm, seed, offset, dX, ws, stream=None):
    l, n = D.shape
    m = w_dgrad.rows
    _check(load().averis_linear_dgrad(_ptr(D), _dtype(D), l, m, n, _s(w_dgrad), _round(rm), seed,
                                      offset, _ptr(dX), _dtype(dX), _ptr(ws), ws.numel(),
                                      _stream(stream)), "averis_linear_dgrad")


def nvfp4_linear_fwd(X, w_fwd, rm, seed, offset, Y, ws, stream=None):
    l, m = X.shape
    n = w_fwd.rows
    _check(load().nvfp4_linear_fwd(_ptr(X), _dtype(X), l, m, n, _s(w_fwd), _round(rm), seed, offset,
                                   _ptr(Y), _dtype(Y), _ptr(ws), ws.numel(), _stream(stream)),
           "nvfp4_linear_fwd")


def nvfp4_linear_dgrad(D, w_dgrad, rm, seed, offset, dX, ws, stream=None):
    l, n = D.shape
    m = w_dgrad.rows
    _check(load().nvfp4_linear_dgrad(_ptr(D), _dtype(D), l, m, n, _s(w_dgrad), _round(rm), seed,
                                     offset, _ptr(dX), _dtype(dX), _ptr(ws), ws.numel(),
                                     _stream(stream)), "nvfp4_linear_dgrad")


def averis_probe_convert(x, e4m3, e2m1, stream=None):
    _check(load().averis_probe_convert(_ptr(x), _ptr(e4m3), _ptr(e2m1), x.numel(), _stream(stream)),
           "averis_probe_convert")


def averis_probe_convert_sr(x, rbits, out, stream=None):
    _check(load().averis_probe_convert_sr(_ptr(x), _ptr(rbits), _ptr(out), rbits.numel(), _stream(stream)),
           "averis_probe_convert_sr")


def averis_probe_philox(seed, offset, tag, n, out, stream=None):
    _check(load().averis_probe_philox(seed, offset, tag, n, _ptr(out), _stream(stream)),
           "averis_probe_philox")


# ---------------------------------------------------------------------------
# split quantization without a caller workspace
# ---------------------------------------------------------------------------
_SIGS["averis_split_quant_noalloc"] = (
    _c_int, [_c_ptr, _c_int, _c_i64, _c_i64, _c_int, _c_u64, _c_u64, _c_int, _c_ptr,
             ctypes.POINTER(avr_nvfp4), ctypes.POINTER(avr_nvfp4), _c_ptr, _c_ptr, _c_ptr])


def averis_split_quant_noalloc(X, rm, seed, offset, grad, mu, mu_q, xr_q, xr_debug,
                               device_status=None, stream=None):
    """averis_split_quant without a workspace, for callers that cannot
    allocate device memory; its scratch is a fixed 4 MiB array inside the
    library (see include/averis.h for the size limit and the rules)."""
    l, K = X.shape
    _check(load().averis_split_quant_noalloc(_ptr(X), _dtype(X), l, K, _round(rm), seed, offset,
                                             int(grad), _ptr(mu), _s(mu_q), _s(xr_q), _ptr(xr_debug),
                                             _ptr(device_status), _stream(stream)),
           "averis_split_quant_noalloc")
