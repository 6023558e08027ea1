"""Averis mean-residual split, its quantized operands and the reference
products.  TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

From "The Curse and Blessing of Mean Bias in FP4-Quantized LLM Training":

  * column mean over the l tokens, mu_X = (1/l) 1^T X, X in R^{l x m}
    (Lighthouse review, section 二 2.1 "核心 Insight");
  * forward:  Y_hat = 1 (mu_bar_X W_bar) + X_bar_R W_bar,
              mu_bar_X = Q_4(mu_X),  X_bar_R = Q_4(X - 1 mu_X)
    (Lighthouse review, section 二 "Averis 方法", forward equation;
    gist.science technical summary, section 2 "Il Metodo Proposto: Averis",
    which writes the same residual as X - 1 mu_X^T in column convention);
  * backward (dgrad): dL/dX_hat = 1 (mu_bar_D W_bar^T) + D_bar_R W_bar^T,
    the same split of the output gradient D (same section, backward
    equation);
  * cost: only reductions and elementwise subtractions (same section,
    "计算开销"; arXiv abstract).

Readings where the pages are silent:
  * fixed fp32 order of the mean: rows cut into 256-token chunks; each chunk
    partial starts at +0.0 and adds its rows in ascending order; the column
    sum starts at +0.0 and adds the chunk partials in ascending chunk order;
    mu = fl(S / l) (IEEE division);
  * W_bar in the two equations is one symbol but two quantizations, one per
    contraction axis: along m for the forward (stored [n, m/2]) and along n
    for dgrad (stored [m, n/2]); weights are always rounded to nearest even;
  * stochastic rounding (when selected) applies to the split operands X_R,
    mu_X, D_R, mu_D and to the vanilla operands, each with its own stream tag.
  * weight gradient (the pages name W4A4G4 but give no Averis equation for
    it): dW = X^T D = X_R^T D_R + l mu_X^T mu_D, since 1^T X_R = 0 removes both
    cross terms.  The two residuals are quantized along the tokens (the
    contraction axis), as [m, L] and [n, L] tensors with L = l rounded up to
    a multiple of 64 and zero padding; their tensor scales are those of the
    row-wise residuals (same amax); the rank-one term uses the same
    quantized means mu_bar_X, mu_bar_D as the forward and dgrad.
"""

import numpy as np

from .nvfp4 import NVFP4, nvfp4_quantize, nvfp4_dequantize

CHUNK = 256

# Philox stream tags (third counter word) per quantized operand.
TAGS = {
    "x_r": 1, "mu_x": 2, "d_r": 3, "mu_d": 4,
    "w_fwd": 5, "w_dgrad": 6, "vanilla_x": 7, "vanilla_d": 8,
    "x_r_t": 9, "d_r_t": 10, "vanilla_x_t": 11, "vanilla_d_t": 12,
}

TOKEN_ALIGN = 64     # the token axis of the weight-gradient operands is padded to this


def _as_f32(X):
    """Widen the input (fp32, or bf16 held as torch/uint16/float) to fp32
    exactly."""
    X = np.asarray(X)
    if X.dtype == np.float32:
        return X
    if X.dtype == np.uint16:           # raw bf16 bit patterns
        return (X.astype(np.uint32) << 16).view(np.float32)
    return X.astype(np.float32)


def column_mean(X):
    """mu_j in the fixed order (256-row chunks, then chunks in order)."""
    X = _as_f32(X)
    l, m = X.shape
    S = np.zeros(m, dtype=np.float32)
    for c0 in range(0, l, CHUNK):
        p = np.zeros(m, dtype=np.float32)
        for i in range(c0, min(c0 + CHUNK, l)):
            p = p + X[i]                # one fp32 add per column, row by row
        S = S + p
    return (S / np.float32(l)).astype(np.float32)


def mean_residual_split(X, mu):
    """X_R = fl(X - 1 mu), elementwise."""
    return (_as_f32(X) - np.asarray(mu, dtype=np.float32)[None, :]).astype(np.float32)


def column_mean_and_residual_amax(X):
    """(mu, X_R, max|X_R|) with the amax taken directly from X_R."""
    mu = column_mean(X)
    XR = mean_residual_split(X, mu)
    A = np.float32(np.max(np.abs(XR))) if XR.size else np.float32(0.0)
    return mu, XR, A


def _check_finite(X):
    if not np.all(np.isfinite(X)):
        raise ValueError("non-finite input")


def averis_split_quant(X, rounding="sr", seed=0, offset=0, grad=False):
    """(mu, X_R, mu_bar, X_bar_R) for activations (grad=False) or output
    gradients (grad=True, which only changes the stream tags)."""
    X = _as_f32(X)
    _check_finite(X)
    mu, XR, A = column_mean_and_residual_amax(X)
    _check_finite(mu)
    t_r, t_mu = (TAGS["d_r"], TAGS["mu_d"]) if grad else (TAGS["x_r"], TAGS["mu_x"])
    xr_q = nvfp4_quantize(XR, rounding, seed, offset, t_r, amax=A)
    mu_q = nvfp4_quantize(mu[None, :], rounding, seed, offset, t_mu)
    return mu, XR, mu_q, xr_q


def vanilla_quant(X, rounding="sr", seed=0, offset=0, grad=False):
    """Q_4(X) with no split (the comparison path)."""
    X = _as_f32(X)
    _check_finite(X)
    tag = TAGS["vanilla_d"] if grad else TAGS["vanilla_x"]
    return nvfp4_quantize(X, rounding, seed, offset, tag)


def quant_weight(W):
    """(W_bar_fwd [n, m/2], W_bar_dgrad [m, n/2]) from W [m, n], RNE."""
    W = _as_f32(W)
    _check_finite(W)
    w_fwd = nvfp4_quantize(np.ascontiguousarray(W.T), "rne", tag=TAGS["w_fwd"])
    w_dgrad = nvfp4_quantize(W, "rne", tag=TAGS["w_dgrad"])
    return w_fwd, w_dgrad


def bias_row(mu_q: NVFP4, w_q: NVFP4):
    """The rank-one row mu_bar W_bar (fp64), one value per output column."""
    return (nvfp4_dequantize(mu_q) @ nvfp4_dequantize(w_q).T)[0]


def gemm_reference(a_q: NVFP4, b_q: NVFP4, bias=None, rows=None):
    """fp64 product deq(A) deq(B)^T (+ bias broadcast to every row).

    ``rows`` restricts the product to a subset of output rows."""
    A = nvfp4_dequantize(a_q)
    if rows is not None:
        A = A[np.asarray(rows)]
    Y = A @ nvfp4_dequantize(b_q).T
    if bias is not None:
        Y = Y + np.asarray(bias, dtype=np.float64)[None, :]
    return Y


def averis_linear_reference(X, w_q: NVFP4, rounding="sr", seed=0, offset=0, grad=False):
    """Forward (grad=False, w_q = W_bar_fwd) or dgrad (grad=True,
    w_q = W_bar_dgrad) of the Averis linear: fp64 Y_hat plus the operands."""
    mu, XR, mu_q, xr_q = averis_split_quant(X, rounding, seed, offset, grad)
    b = bias_row(mu_q, w_q)
    return gemm_reference(xr_q, w_q, b), dict(mu=mu, xr=XR, mu_q=mu_q, xr_q=xr_q, bias=b)


def vanilla_linear_reference(X, w_q: NVFP4, rounding="sr", seed=0, offset=0, grad=False):
    x_q = vanilla_quant(X, rounding, seed, offset, grad)
    return gemm_reference(x_q, w_q), dict(x_q=x_q)


# ---------------------------------------------------------------------------
# weight gradient: operands quantized along the tokens
# ---------------------------------------------------------------------------

def padded_tokens(l):
    """L = l rounded up to a multiple of 64 (the contraction length of dW)."""
    return (int(l) + TOKEN_ALIGN - 1) // TOKEN_ALIGN * TOKEN_ALIGN


def transpose_padded(T):
    """[l, K] -> [K, L]: T^T with zero columns l .. L-1."""
    T = np.asarray(T, dtype=np.float32)
    l, K = T.shape
    out = np.zeros((K, padded_tokens(l)), dtype=np.float32)
    out[:, :l] = T.T
    return out


def averis_split_quant_t(X, rounding="sr", seed=0, offset=0, grad=False):
    """(mu, mu_bar, X_bar_R^T): the split of X (grad=False) or D (grad=True)
    with the residual quantized along the tokens, [K, L].  mu_bar is the same
    tensor averis_split_quant gives (same stream tag)."""
    X = _as_f32(X)
    _check_finite(X)
    mu, XR, A = column_mean_and_residual_amax(X)
    _check_finite(mu)
    t_rt, t_mu = (TAGS["d_r_t"], TAGS["mu_d"]) if grad else (TAGS["x_r_t"], TAGS["mu_x"])
    xrt_q = nvfp4_quantize(transpose_padded(XR), rounding, seed, offset, t_rt, amax=A)
    mu_q = nvfp4_quantize(mu[None, :], rounding, seed, offset, t_mu)
    return mu, mu_q, xrt_q


def vanilla_quant_t(X, rounding="sr", seed=0, offset=0, grad=False):
    """Q_4(X^T) along the tokens with no split, [K, L]."""
    X = _as_f32(X)
    _check_finite(X)
    tag = TAGS["vanilla_d_t"] if grad else TAGS["vanilla_x_t"]
    return nvfp4_quantize(transpose_padded(X), rounding, seed, offset, tag)


def wgrad_reference(xt_q: NVFP4, dt_q: NVFP4, mu_x_q=None, mu_d_q=None, l=0):
    """fp64 dW = deq(A^T) deq(B^T)^T (+ l deq(mu_bar_X)^T deq(mu_bar_D)), [m, n]."""
    dW = nvfp4_dequantize(xt_q) @ nvfp4_dequantize(dt_q).T
    if mu_x_q is not None:
        dW = dW + float(l) * np.outer(nvfp4_dequantize(mu_x_q)[0], nvfp4_dequantize(mu_d_q)[0])
    return dW


def averis_wgrad_reference(X, D, rounding="sr", seed=0, offset=0):
    """Weight gradient of the Averis linear from X [l, m] and D [l, n]: fp64 dW
    [m, n] plus the operands."""
    l = np.asarray(X).shape[0]
    mu_x, mu_x_q, xrt_q = averis_split_quant_t(X, rounding, seed, offset, grad=False)
    mu_d, mu_d_q, drt_q = averis_split_quant_t(D, rounding, seed, offset, grad=True)
    dW = wgrad_reference(xrt_q, drt_q, mu_x_q, mu_d_q, l)
    return dW, dict(mu_x=mu_x, mu_d=mu_d, mu_x_q=mu_x_q, mu_d_q=mu_d_q, xrt_q=xrt_q, drt_q=drt_q)


def vanilla_wgrad_reference(X, D, rounding="sr", seed=0, offset=0):
    xt_q = vanilla_quant_t(X, rounding, seed, offset, grad=False)
    dt_q = vanilla_quant_t(D, rounding, seed, offset, grad=True)
    return wgrad_reference(xt_q, dt_q), dict(xt_q=xt_q, dt_q=dt_q)


# ---------------------------------------------------------------------------
# MoE: one Averis linear per expert over a token buffer permuted by expert
# ---------------------------------------------------------------------------
# Readings (the pages name the Qwen3 7B-A1.5B MoE model and nothing more):
#  * each expert is its own linear layer, so each gets its own split: mu_e is
#    the mean of the tokens routed to expert e (the same fixed order, chunks
#    counted from the first token of the segment), with its own tensor scales
#    for X_bar_R,e and mu_bar_e;
#  * the tokens of expert e are rows [o_e, o_e + n_e) of the permuted buffer,
#    o_0 = 0 and o_{e+1} = o_e + n_e rounded up to 128; rows in between are
#    padding that no statistic sees and whose outputs are undefined;
#  * random streams: element (r, j) of the buffer counts from offset +
#    (r K + j) / 16 as in the dense layer; mu_bar_e counts as row e of an
#    [E, K] tensor (offset + (e K + j) / 16), with the dense layer's tags.

MOE_ALIGN = 128


def moe_offsets(counts):
    """Row offsets o_e of the expert segments and the buffer's padded length."""
    o, r = [], 0
    for n in counts:
        o.append(r)
        r += (int(n) + MOE_ALIGN - 1) // MOE_ALIGN * MOE_ALIGN
    return o, r


def moe_split_quant(X, counts, rounding="sr", seed=0, offset=0, grad=False, experts=None):
    """Per-expert split of the permuted buffer X [L, K]: lists (per expert) of
    mu_e, X_R,e, mu_bar_e, X_bar_R,e (the latter quantized as rows o_e .. of
    the buffer).  `experts` restricts the work to those experts (the others
    are None)."""
    X = _as_f32(X)
    K = X.shape[1]
    offs, L = moe_offsets(counts)
    assert X.shape[0] >= L
    t_r, t_mu = (TAGS["d_r"], TAGS["mu_d"]) if grad else (TAGS["x_r"], TAGS["mu_x"])
    out = []
    for e, (o, n) in enumerate(zip(offs, counts)):
        if n == 0 or (experts is not None and e not in experts):
            out.append(None)
            continue
        Xe = X[o:o + n]
        _check_finite(Xe)
        mu, XR, A = column_mean_and_residual_amax(Xe)
        xr_q = nvfp4_quantize(XR, rounding, seed, offset + (o * K) // 16, t_r, amax=A)
        mu_q = nvfp4_quantize(mu[None, :], rounding, seed, offset + (e * K) // 16, t_mu)
        out.append(dict(mu=mu, xr=XR, mu_q=mu_q, xr_q=xr_q, row0=o, rows=n))
    return out


def moe_quant_weights(Ws):
    """Per-expert (W_bar_fwd, W_bar_dgrad), each with its own tensor scale."""
    return [quant_weight(W) for W in Ws]


def moe_linear_reference(X, counts, w_qs, rounding="sr", seed=0, offset=0, grad=False, experts=None):
    """fp64 output rows of every expert's segment: Y[o_e + i] for i < n_e, the
    Averis product of expert e (w_qs[e] = W_bar_fwd,e, or W_bar_dgrad,e for
    grad=True).  Returns (dict row -> output row block, the split)."""
    split = moe_split_quant(X, counts, rounding, seed, offset, grad, experts)
    Y = {}
    for e, s in enumerate(split):
        if s is None:
            continue
        b = bias_row(s["mu_q"], w_qs[e])
        Y[e] = gemm_reference(s["xr_q"], w_qs[e], b)
    return Y, split
