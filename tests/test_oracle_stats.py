"""The pages' statistical statements, checked on seeded synthetic data (no
GPU): Theorem 1, Theorem 2, cos(mu, v_1) ~ 0.99, and stage II of the mean's
origin (E[SwiGLU] > 0)."""

import math

import numpy as np
import pytest

from oracle import stats
from quantized_gemm_column_b200 import inputs


@pytest.mark.parametrize("t", [3.0, 4.0])
def test_theorem1_constant_rate(t):
    """Columns with planted |mu_j| = t + k sigma, k = 1.5..4: the fraction of
    entries over t is at least the bound minus 3 binomial standard errors."""
    l = 16384
    ks = (1.5, 2.0, 3.0, 4.0)          # the bound is vacuous below |mu| - t = sqrt(2 ln 2)
    mus = np.array([t + k for k in ks] + [-(t + k) for k in ks])
    X = inputs.planted_mean_columns(inputs.rng_for(9, int(t)), l, mus)
    frac = stats.over_threshold_fraction(X, t)
    for j, mu in enumerate(mus):
        b = stats.theorem1_bound(abs(mu), t)
        assert b > 0.2
        assert frac[j] >= b - 3 * math.sqrt(max(b * (1 - b), 1e-12) / l)


def test_theorem2_linear_count_vs_exponential_tail():
    """Over-threshold counts grow like Theta(l) in planted-mean columns (the
    rate count / l stays put as l grows 64x) while zero-mean columns stay at
    the Gaussian tail rate 2 Phi(-t)."""
    t = 3.0
    rates = []
    for l in (256, 1024, 4096, 16384):
        X = inputs.planted_mean_columns(inputs.rng_for(9, 10 + l % 97), l, [t + 1.0, 0.0])
        frac = stats.over_threshold_fraction(X, t)
        rates.append(frac)
    rates = np.array(rates)
    p_mean = 1 - 0.5 * math.erfc(1.0 / math.sqrt(2))       # P(N(1,1) > 0)
    for (l, r) in zip((256, 1024, 4096, 16384), rates):
        assert abs(r[0] - p_mean) <= 4 * math.sqrt(p_mean * (1 - p_mean) / l) + 1e-3
    tail = stats.gaussian_two_sided_tail(t)
    assert abs(rates[-1][1] - tail) <= 4 * math.sqrt(tail / 16384)
    assert rates[-1][0] > 100 * rates[-1][1]


def test_cos_mean_top_singular_vector():
    """Brute-force SVD on the tiny forward case and a 2048-token slice of
    the QKV case: the column mean is the leading right singular direction."""
    X0, _ = inputs.workload0()
    assert stats.cos_mean_top_singular(X0) >= 0.99
    X1, _, _ = inputs.workload1(l=2048)
    assert stats.cos_mean_top_singular(inputs.bf16_as_f32(X1)) >= 0.99


def test_swiglu_input_has_positive_mean():
    """E[silu(a) b] = E[silu(a)] E[b] with a, b ~ N(0.2, 1): about 0.07 > 0."""
    X = inputs.swiglu_input(inputs.rng_for(2, 99), 16384, 64)
    assert 0.04 < X.mean() < 0.12
    assert np.mean(X.mean(axis=0) > 0) > 0.95


def test_mean_energy_ratio_grows_with_mean_scale():
    r = [stats.mean_energy_ratio(inputs.bf16_as_f32(inputs.workload3(c, l=1024, m=256)[0]))
         for c in (0.0, 2.0, 8.0)]
    assert r[0] < r[1] < r[2]


def test_mean_energy_ratio_closed_forms():
    """Constant rows x_i = c give mu = c and ||x_i||^2 = ||c||^2, so R = sqrt(m)
    exactly; rows in +/- pairs give mu = 0, so R = 0."""
    rng = np.random.default_rng(3)
    m = 96
    c = rng.standard_normal(m)
    X = np.tile(c, (40, 1))
    assert stats.mean_energy_ratio(X) == pytest.approx(math.sqrt(m), rel=1e-12)
    Y = rng.standard_normal((20, m))
    pairs = np.stack([Y, -Y], axis=1).reshape(40, m)     # y1, -y1, y2, -y2, ...
    assert stats.mean_energy_ratio(pairs) < 1e-12
    # scaling X leaves R unchanged
    Z = rng.standard_normal((64, m)) + 0.5
    assert stats.mean_energy_ratio(3.0 * Z) == pytest.approx(stats.mean_energy_ratio(Z), rel=1e-12)
