"""Pins of the oracle's mean, split and reference products (no GPU)."""

import numpy as np
import pytest

import oracle
from oracle import nvfp4 as F
from quantized_gemm_column_b200 import inputs


# --------------------------------------------------------------------------
# the fixed reduction order
# --------------------------------------------------------------------------
def test_within_chunk_order_is_sequential():
    """Column [2^24, 1, 1, ..., 1] (256 rows): adding row by row in fp32 keeps
    2^24 (each +1 is a tie that rounds to even), so the mean is 2^24 / 256 =
    65536 exactly.  Any other order that groups the ones first would give
    (2^24 + 254 or so) / 256."""
    X = np.ones((256, 2), dtype=np.float32)
    X[0, 0] = 2.0 ** 24
    X[:, 1] = 1.0
    mu = oracle.column_mean(X)
    assert mu[0] == np.float32(65536.0)
    assert mu[1] == 1.0
    # the ones first (reverse order) would have given the exact sum
    assert np.float32((np.float32(255.0) + np.float32(2.0 ** 24)) / 256) != mu[0]


def test_chunk_partials_are_summed_in_chunk_order():
    """Chunk 0 sums to 2^24 and each later chunk to exactly 1 (one row of 1,
    255 rows of 0): adding the partials in chunk order keeps 2^24."""
    l = 256 * 4
    X = np.zeros((l, 1), dtype=np.float32)
    X[0, 0] = 2.0 ** 24
    X[256, 0] = X[512, 0] = X[768, 0] = 1.0
    mu = oracle.column_mean(X)
    assert mu[0] == np.float32(2.0 ** 24 / l)


def test_ragged_last_chunk():
    X = np.zeros((300, 1), dtype=np.float32)
    X[0, 0] = 2.0 ** 24
    X[256:, 0] = 1.0             # 44 ones in the short chunk: partial 44, exact
    mu = oracle.column_mean(X)
    assert mu[0] == np.float32(np.float32(2.0 ** 24 + 44) / 300)


def test_constant_columns_give_exact_mean_and_zero_residual():
    """X = 1 c^T with bf16-representable c and power-of-two l: every partial
    sum is exact, so mu = c and X_R = 0 exactly."""
    rng = np.random.default_rng(1)
    c = inputs.bf16_as_f32(inputs.to_bf16(rng.standard_normal(64) * 10))
    X = np.repeat(c[None, :], 1024, axis=0)
    mu, XR, A = oracle.column_mean_and_residual_amax(X)
    assert np.array_equal(mu, c)
    assert not XR.any() and A == 0


def test_mean_is_close_to_exact_mean():
    """|fl mean - exact mean| <= (256 + C) u mean|x| (recursive summation
    bound, u = 2^-24) for every column."""
    rng = np.random.default_rng(2)
    X = (rng.standard_normal((2048, 32)) + rng.normal(0, 3, 32)).astype(np.float32)
    mu = oracle.column_mean(X).astype(np.float64)
    exact = X.astype(np.float64).mean(axis=0)
    bound = (256 + 8 + 1) * 2.0 ** -24 * np.abs(X).astype(np.float64).mean(axis=0)
    assert np.all(np.abs(mu - exact) <= bound)


# --------------------------------------------------------------------------
# the split
# --------------------------------------------------------------------------
def test_split_reconstruction_and_zero_column_mean():
    """X_R is the correctly rounded x - mu: 1 mu + X_R = X within half an
    ulp of X_R (exactly where the subtraction is exact), and the columns of
    X_R sum to ~0 (1^T X_R = 0 in exact arithmetic)."""
    X, _ = inputs.workload0()
    mu, XR, _ = oracle.column_mean_and_residual_amax(X)
    recon = mu.astype(np.float64)[None, :] + XR.astype(np.float64)
    half_ulp = np.spacing(np.abs(XR)).astype(np.float64) / 2
    assert np.all(np.abs(recon - X) <= half_ulp)
    l = X.shape[0]
    col = XR.astype(np.float64).sum(axis=0)
    bound = l * (256 + 2) * 2.0 ** -24 * np.abs(X).astype(np.float64).mean(axis=0) + half_ulp.sum(axis=0)
    assert np.all(np.abs(col) <= bound)


def test_residual_amax_from_column_extremes():
    """max_i |fl(x_ij - mu_j)| = max(fl(colmax - mu), fl(mu - colmin)), by
    monotonicity of rounded subtraction: the shortcut a one-pass reduction
    can use gives the same amax as the direct scan."""
    rng = np.random.default_rng(3)
    for _ in range(20):
        X = (rng.standard_normal((512, 16)) * rng.uniform(0.1, 50) + rng.normal(0, 20, 16)).astype(np.float32)
        mu, XR, A = oracle.column_mean_and_residual_amax(X)
        short = np.maximum(X.max(0) - mu, mu - X.min(0)).astype(np.float32).max()
        assert short == A


def test_gemm_identity_brute_force():
    """1 (mu W) + X_R W = X W in exact arithmetic (fp64 triple loops on a
    tiny case, unquantized operands; the only error is the rounding of X_R)."""
    rng = np.random.default_rng(4)
    l, m, n = 24, 16, 8
    X = (rng.standard_normal((l, m)) + 3).astype(np.float32)
    W = rng.standard_normal((m, n))
    mu = oracle.column_mean(X).astype(np.float64)
    XR32 = oracle.mean_residual_split(X, mu.astype(np.float32))
    XR = XR32.astype(np.float64)
    lhs = np.zeros((l, n))
    rhs = np.zeros((l, n))
    for i in range(l):
        for j in range(n):
            for k in range(m):
                lhs[i, j] += mu[k] * W[k, j] + XR[i, k] * W[k, j]
                rhs[i, j] += float(X[i, k]) * W[k, j]
    err_bound = np.abs(W).sum(axis=0)[None, :] * np.max(np.spacing(np.abs(XR32))) / 2 + 1e-12
    assert np.all(np.abs(lhs - rhs) <= err_bound)


def test_gemm_reference_brute_force_and_orientation():
    """gemm_reference = sum_k deq(A)_ik deq(B)_jk (+ b_j), checked with
    explicit loops on a non-square case (a transposed operand would fail)."""
    rng = np.random.default_rng(5)
    A = oracle.nvfp4_quantize(rng.standard_normal((5, 64)).astype(np.float32), "rne")
    B = oracle.nvfp4_quantize(rng.standard_normal((3, 64)).astype(np.float32), "rne")
    b = rng.standard_normal(3)
    Y = oracle.gemm_reference(A, B, b)
    dA, dB = oracle.nvfp4_dequantize(A), oracle.nvfp4_dequantize(B)
    assert Y.shape == (5, 3)
    for i in range(5):
        for j in range(3):
            s = b[j]
            for k in range(64):
                s += dA[i, k] * dB[j, k]
            assert abs(Y[i, j] - s) <= 1e-12 * (1 + abs(s))


def test_bias_row_brute_force():
    rng = np.random.default_rng(6)
    mu_q = oracle.nvfp4_quantize(rng.standard_normal((1, 64)).astype(np.float32), "rne")
    w_q = oracle.nvfp4_quantize(rng.standard_normal((7, 64)).astype(np.float32), "rne")
    b = oracle.bias_row(mu_q, w_q)
    dm, dw = oracle.nvfp4_dequantize(mu_q)[0], oracle.nvfp4_dequantize(w_q)
    for j in range(7):
        assert abs(b[j] - sum(dm[k] * dw[j, k] for k in range(64))) < 1e-12


def test_weight_quant_orientations():
    rng = np.random.default_rng(7)
    W = rng.standard_normal((64, 128)).astype(np.float32)
    w_fwd, w_dgrad = oracle.quant_weight(W)
    assert (w_fwd.rows, w_fwd.K) == (128, 64) and (w_dgrad.rows, w_dgrad.K) == (64, 128)
    assert w_fwd.g_dec == w_dgrad.g_dec                 # same tensor amax
    assert np.linalg.norm(oracle.nvfp4_dequantize(w_fwd) - W.T) / np.linalg.norm(W) < 0.2
    assert np.linalg.norm(oracle.nvfp4_dequantize(w_dgrad) - W) / np.linalg.norm(W) < 0.2


def test_averis_equals_vanilla_when_mean_is_zero():
    """Rows in +-pairs make every column sum exactly zero in the fixed order,
    so mu = 0, X_R = X and (with RNE) Q_4(X_R) = Q_4(X) bit for bit, and the
    rank-one row is zero."""
    rng = np.random.default_rng(8)
    half = rng.standard_normal((128, 64)).astype(np.float32)
    X = np.empty((256, 64), np.float32)
    X[0::2], X[1::2] = half, -half
    mu, XR, mu_q, xr_q = oracle.averis_split_quant(X, "rne")
    v = oracle.vanilla_quant(X, "rne")
    assert not mu.any()
    assert np.array_equal(xr_q.codes, v.codes) and np.array_equal(xr_q.scales, v.scales)
    assert xr_q.g_dec == v.g_dec
    w_fwd, _ = oracle.quant_weight(rng.standard_normal((64, 32)).astype(np.float32))
    assert not oracle.bias_row(mu_q, w_fwd).any()


def test_averis_reduces_error_with_strong_mean():
    """On data with a strong column mean the split operand quantizes with a
    smaller error than the plain one (the point of the method; section 二 of
    the review), and Y_hat approaches X W."""
    X, W = inputs.workload0()
    w_fwd, _ = oracle.quant_weight(W)
    Ya, _ = oracle.averis_linear_reference(X, w_fwd, "rne")
    Yv, _ = oracle.vanilla_linear_reference(X, w_fwd, "rne")
    Y = X.astype(np.float64) @ oracle.nvfp4_dequantize(w_fwd).T
    ea = np.linalg.norm(Ya - Y) / np.linalg.norm(Y)
    ev = np.linalg.norm(Yv - Y) / np.linalg.norm(Y)
    assert ea < ev


def test_nonfinite_rejected():
    X = np.ones((4, 16), np.float32)
    X[1, 1] = np.inf
    with pytest.raises(ValueError):
        oracle.averis_split_quant(X)


# --------------------------------------------------------------------------
# separate random streams for the split's operands
# --------------------------------------------------------------------------
def _twin_rows(K=256):
    """X = [2a; 0] with a on the grid of 1.25 steps and a 6 in every block:
    mu = a and X_R = [a; -a] exactly, and mu and X_R share the tensor amax
    (6), so mu and row 0 of X_R have the same scales and the same scaled
    values, each 1.25 (round-up probability 1/2) except the block maxima."""
    a = np.full(K, 1.25, dtype=np.float32)
    a[::16] = 6.0
    return np.stack([2 * a, np.zeros(K, np.float32)]), a


def test_mean_and_residual_draw_separate_streams():
    """With one stream for both, mu_bar and row 0 of X_bar_R would round every
    element the same way; with separate streams about half of the 1.25s
    round differently (the stochastic rounding of the two operands must be
    independent)."""
    X, a = _twin_rows()
    mu, XR, mu_q, xr_q = oracle.averis_split_quant(X, "sr", seed=11, offset=3)
    assert np.array_equal(mu, a) and np.array_equal(XR[0], a)
    assert np.array_equal(mu_q.scales[0], xr_q.scales[0]) and mu_q.g_dec == xr_q.g_dec
    c_mu, c_r = F.unpack_codes(mu_q.codes)[0], F.unpack_codes(xr_q.codes)[0]
    free = a != 6.0
    assert set(np.unique(c_mu[free])) <= {2, 3} and set(np.unique(c_r[free])) <= {2, 3}
    differ = np.mean(c_mu[free] != c_r[free])
    assert 0.35 < differ < 0.65, differ


def test_activation_and_gradient_splits_draw_separate_streams():
    """The forward's and the dgrad's split of the same tensor (same seed and
    offset) round independently."""
    X, a = _twin_rows()
    _, _, _, q_x = oracle.averis_split_quant(X, "sr", seed=11, offset=3, grad=False)
    _, _, _, q_d = oracle.averis_split_quant(X, "sr", seed=11, offset=3, grad=True)
    free = np.tile(a != 6.0, (2, 1))
    differ = np.mean(F.unpack_codes(q_x.codes)[free] != F.unpack_codes(q_d.codes)[free])
    assert 0.35 < differ < 0.65, differ
