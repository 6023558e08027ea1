"""Pins of the oracle's MoE variant (one Averis linear per expert over a
token buffer permuted by expert): it reduces to the dense layer for one
expert, keeps experts apart, ignores padding rows, and is exact on inputs
whose every operand quantizes exactly."""

import numpy as np
import pytest

import oracle

E2M1_POS = np.array([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _buffer(rng, counts, K, mean_scale=1.0):
    offs, L = oracle.moe_offsets(counts)
    X = np.zeros((L, K), np.float32)
    for e, (o, n) in enumerate(zip(offs, counts)):
        mu = rng.standard_normal(K) * mean_scale * (e + 1)
        X[o:o + n] = (mu + rng.standard_normal((n, K))).astype(np.float32)
    return X, offs


def test_offsets_are_aligned_segments():
    offs, L = oracle.moe_offsets([5, 0, 300, 128, 1])
    assert offs == [0, 128, 128, 512, 640] and L == 768
    assert all(o % 128 == 0 for o in offs)


@pytest.mark.parametrize("rounding", ["rne", "sr"])
def test_one_expert_is_the_dense_layer(rounding):
    rng = np.random.default_rng(1)
    X = rng.standard_normal((300, 128)).astype(np.float32) + 2.0
    s = oracle.moe_split_quant(np.vstack([X, np.zeros((84, 128), np.float32)]), [300], rounding, seed=4,
                               offset=9)[0]
    mu, XR, mu_q, xr_q = oracle.averis_split_quant(X, rounding, seed=4, offset=9)
    assert np.array_equal(s["mu"], mu) and np.array_equal(s["xr"], XR)
    assert np.array_equal(s["xr_q"].codes, xr_q.codes) and np.array_equal(s["xr_q"].scales, xr_q.scales)
    assert np.array_equal(s["mu_q"].codes, mu_q.codes)


def test_each_expert_is_its_own_dense_layer():
    """With RNE (no stream) expert e's outputs are the dense Averis linear of
    its own rows and its own weights, bit for bit."""
    rng = np.random.default_rng(2)
    counts, K, n = [200, 0, 129, 64], 128, 192
    X, offs = _buffer(rng, counts, K)
    Ws = [rng.standard_normal((K, n)).astype(np.float32) / 8 for _ in counts]
    wq = [w[0] for w in oracle.moe_quant_weights(Ws)]
    Y, _ = oracle.moe_linear_reference(X, counts, wq, "rne")
    assert set(Y) == {0, 2, 3}
    for e in Y:
        ref, _ = oracle.averis_linear_reference(X[offs[e]:offs[e] + counts[e]], wq[e], "rne")
        assert np.array_equal(Y[e], ref)


def test_experts_and_padding_do_not_leak():
    """Shifting expert 1's tokens by a constant, or filling the padding rows
    with huge values, leaves expert 0's operands and outputs unchanged."""
    rng = np.random.default_rng(3)
    counts, K = [100, 150], 64
    X, offs = _buffer(rng, counts, K)
    Ws = [rng.standard_normal((K, 128)).astype(np.float32) / 8 for _ in counts]
    wq = [w[0] for w in oracle.moe_quant_weights(Ws)]
    Y0, s0 = oracle.moe_linear_reference(X, counts, wq, "sr", seed=5)
    X2 = X.copy()
    X2[offs[1]:offs[1] + counts[1]] += np.float32(7.0)
    X2[counts[0]:offs[1]] = np.float32(1e30)          # padding of expert 0
    Y2, s2 = oracle.moe_linear_reference(X2, counts, wq, "sr", seed=5)
    assert np.array_equal(Y0[0], Y2[0])
    assert np.array_equal(s0[0]["xr_q"].codes, s2[0]["xr_q"].codes)
    assert not np.array_equal(s0[1]["mu"], s2[1]["mu"])


def _exact_expert(rng, n, K):
    """x_i = mu + r_i with mu and r on the E2M1 grid: each 16-block of mu holds
    a +/-6, each row's 16-blocks hold a +/-6, and rows come in +/- pairs, so
    the mean is exact and every operand quantizes exactly."""
    mu = rng.choice(E2M1_POS, K) * rng.choice([-1.0, 1.0], K)
    mu[::16] = 6.0
    R = np.zeros((n, K))
    half = rng.choice(E2M1_POS, (n // 2, K)) * rng.choice([-1.0, 1.0], (n // 2, K))
    half[:, ::16] = 6.0
    R[0::2], R[1::2] = half, -half
    return (mu[None, :] + R).astype(np.float32)


@pytest.mark.parametrize("rounding", ["rne", "sr"])
def test_moe_chain_is_exact_on_representable_inputs(rounding):
    """Every expert's output equals brute-force X_e W_e (fp64) up to the fp32
    decode scales, with the weights on the E2M1 grid too (a +/-6 in every
    16-block along m)."""
    rng = np.random.default_rng(4)
    counts, K, n = [64, 130, 32], 64, 128
    offs, L = oracle.moe_offsets(counts)
    X = np.zeros((L, K), np.float32)
    Ws = []
    for e, (o, c) in enumerate(zip(offs, counts)):
        X[o:o + c] = _exact_expert(rng, c, K)
        W = rng.choice(E2M1_POS, (K, n)) * rng.choice([-1.0, 1.0], (K, n))
        W[::16, :] = 6.0
        Ws.append(W.astype(np.float32))
    wq = [w[0] for w in oracle.moe_quant_weights(Ws)]
    Y, _ = oracle.moe_linear_reference(X, counts, wq, rounding, seed=6)
    for e in Y:
        Xe = X[offs[e]:offs[e] + counts[e]].astype(np.float64)
        ref = np.zeros((counts[e], n))
        for i in range(counts[e]):
            for k in range(K):
                ref[i] += Xe[i, k] * Ws[e][k].astype(np.float64)
        assert np.allclose(Y[e], ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_experts_draw_separate_streams():
    """Two experts holding the same tokens round them independently: each
    buffer row has its own place in the stream, so their stochastic codes
    differ in about half of the elements whose round-up probability is 1/2."""
    K, n = 128, 64
    a = np.full((n, K), 1.25, np.float32)
    a[:, ::16] = 6.0
    a[1::2] *= -1                                     # +/- row pairs: mu = 0, X_R = X
    offs, L = oracle.moe_offsets([n, n])
    X = np.zeros((L, K), np.float32)
    X[offs[0]:offs[0] + n] = a
    X[offs[1]:offs[1] + n] = a
    s = oracle.moe_split_quant(X, [n, n], "sr", seed=2, offset=5)
    c0, c1 = (oracle.unpack_codes(s[e]["xr_q"].codes)[:n] & 7 for e in (0, 1))
    assert np.array_equal(s[0]["xr_q"].scales[:n], s[1]["xr_q"].scales[:n])
    free = np.abs(a) != 6.0
    differ = np.mean(c0[free] != c1[free])
    assert 0.35 < differ < 0.65, differ
