"""Statistical statements of the pages, as checks on generated data.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

  * Theorem 1 (single-element dominance), Lighthouse review section 二 2.2
    "理论分析": if |mu_j| > t then
        P(|X_ij| > t) >= 1 - 2 exp(-(|mu_j| - t)^2 / (2 sigma^2))
    for sub-Gaussian noise of scale sigma -- a constant-order probability.
  * Theorem 2 (dense amplification), same section: a mean shift gives
    Theta(l) over-threshold entries, while the variance-driven count decays
    like exp(-t^2 / (2 sigma^2)).
  * cos(mu_X, v_1) close to 0.99, v_1 the first right singular vector of X
    (section 二 2.1; section 三 3.2).

The threshold t is not defined on the pages; the checks take t = 3 sigma
and t = 4 sigma of the unit Gaussian tail.
"""

import math

import numpy as np


def theorem1_bound(mu_abs, t, sigma=1.0):
    """Lower bound of P(|X_ij| > t) for a column with mean magnitude mu_abs."""
    if mu_abs <= t:
        return 0.0
    return 1.0 - 2.0 * math.exp(-((mu_abs - t) ** 2) / (2.0 * sigma ** 2))


def over_threshold_fraction(X, t):
    """Per-column fraction of entries with |X_ij| > t (fp64)."""
    X = np.asarray(X, dtype=np.float64)
    return np.mean(np.abs(X) > t, axis=0)


def gaussian_two_sided_tail(t, sigma=1.0):
    """P(|N(0, sigma^2)| > t) = erfc(t / (sigma sqrt 2))."""
    return math.erfc(t / (sigma * math.sqrt(2.0)))


def cos_mean_top_singular(X):
    """|cos| between the column mean and the first right singular vector,
    by a brute-force fp64 SVD."""
    X = np.asarray(X, dtype=np.float64)
    mu = X.mean(axis=0)
    _, _, vt = np.linalg.svd(X, full_matrices=False)
    v1 = vt[0]
    return abs(float(mu @ v1)) / (np.linalg.norm(mu) * np.linalg.norm(v1))


def mean_energy_ratio(X):
    """R = ||mu||_2 / sqrt(E||x||^2 / N) with N read as the feature count m
    (Lighthouse review, section 七 practice advice 2; N is undefined there)."""
    X = np.asarray(X, dtype=np.float64)
    mu = X.mean(axis=0)
    m = X.shape[1]
    return float(np.linalg.norm(mu) / math.sqrt(np.mean(np.sum(X * X, axis=1)) / m))
