"""Moving NVFP4 tensors between the CUDA library and the oracle, and the
GEMM tolerance.  Used by the GPU tests, smoke() and bench.py."""

import numpy as np
import torch

import oracle
from oracle import nvfp4 as F


def to_oracle(t):
    """quantized_gemm_column_b200.api.NVFP4Tensor -> oracle.NVFP4 (host copy)."""
    codes = t.codes.cpu().numpy()
    flat = t.scales.cpu().numpy()
    lin = F.unswizzle_scales(flat, t.rows, t.K) if t.rows else np.zeros((0, t.K // 16), np.uint8)
    return oracle.NVFP4(codes, lin, np.float32(t.g_dec.cpu().item()), t.rows, t.K)


def from_oracle(q, api, device="cuda"):
    """oracle.NVFP4 -> a device NVFP4Tensor with the same bytes."""
    t = api.NVFP4Tensor(q.rows, q.K, device)
    t.codes.copy_(torch.from_numpy(np.ascontiguousarray(q.codes)))
    t.scales.copy_(torch.from_numpy(F.swizzle_scales(q.scales, q.rows, q.K)))
    t.g_dec.fill_(float(q.g_dec))
    return t


def assert_nvfp4_equal(gpu, ref, what=""):
    """Bit-exact comparison: packed codes, every scale byte (padding rows
    included) and the decode scale."""
    codes = gpu.codes.cpu().numpy()
    flat = gpu.scales.cpu().numpy()
    assert codes.shape == ref.codes.shape, what
    bad = np.argwhere(codes != ref.codes)
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ, first {bad[:5].tolist()}"
    want = F.swizzle_scales(ref.scales, ref.rows, ref.K)
    bad = np.flatnonzero(flat != want)
    assert bad.size == 0, f"{what}: {len(bad)} scale bytes differ, first {bad[:5].tolist()}"
    g = np.float32(gpu.g_dec.cpu().item())
    assert g.view(np.uint32) == np.float32(ref.g_dec).view(np.uint32), f"{what}: g_dec {g} vs {ref.g_dec}"


def bf16_ulp(y):
    """Spacing of bf16 numbers at |y| (8 significant bits)."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def gemm_tolerance(a_q, b_q, bias, K, rows=None):
    """Per-element bound for an fp32-accumulated product of these operands:
    K 2^-24 (|A| |B|^T + |bias|), the worst-case recursive-sum error of fp32
    accumulation (it matters only where the sum cancels)."""
    A = np.abs(oracle.nvfp4_dequantize(a_q))
    if rows is not None:
        A = A[np.asarray(rows)]
    E = A @ np.abs(oracle.nvfp4_dequantize(b_q)).T
    if bias is not None:
        E = E + np.abs(np.asarray(bias, dtype=np.float64))[None, :]
    return K * 2.0 ** -24 * E


def check_bf16_output(Y, Yref, acc_bound):
    """|Y - Yref| <= 1 bf16 ulp of Yref, or within the fp32 accumulation bound
    plus half an ulp where cancellation makes that larger.  Returns the
    number of elements that needed the accumulation bound."""
    Y = np.asarray(Y, dtype=np.float64)
    err = np.abs(Y - Yref)
    ulp = bf16_ulp(Yref)
    ok1 = err <= ulp
    ok2 = err <= 0.5 * ulp + acc_bound
    bad = ~(ok1 | ok2)
    assert not bad.any(), (f"{bad.sum()} elements out of tolerance; worst err "
                           f"{err[bad].max():.3e} at ref {Yref[bad][np.argmax(err[bad])]:.4e}")
    return int((~ok1).sum())
