"""Pins of the oracle's Philox4x32-10 and of its random-bit stream mapping
(no GPU)."""

import math

import numpy as np

import oracle
from oracle.philox import philox4x32_10, random_bits16
from conftest import read_golden


def test_known_answer_vectors():
    for row in read_golden("philox4x32_10_kat.txt"):
        v = [int(x, 16) for x in row]
        out = philox4x32_10(*[np.uint64(x) for x in v[:6]])
        assert [int(o) for o in out] == v[6:], row


def test_uniformity_chi_square():
    """2^20 outputs of 16-bit halves binned into 256 bins: chi^2 with 255
    degrees of freedom stays below its 1e-6 upper quantile (~370)."""
    r = random_bits16(seed=12345, offset=0, tag=1, n_elements=1 << 20)
    counts = np.bincount(r >> 8, minlength=256)
    expect = r.size / 256
    chi2 = float(np.sum((counts - expect) ** 2 / expect))
    assert chi2 < 370, chi2


def test_stream_mapping_properties():
    seed, tag = 0xDEADBEEF12345678, 3
    a = random_bits16(seed, 100, tag, 4096)
    # advancing the counter offset by one equals skipping 16 elements
    b = random_bits16(seed, 101, tag, 4096 - 16)
    assert np.array_equal(a[16:], b)
    # starting inside the stream gives the same bits as slicing it
    c = random_bits16(seed, 100, tag, 100, start=36)
    assert np.array_equal(a[36:136], c)
    # the 16 elements of one call: each group of 4 rebuilds its output word
    # from W (elements 0, 1 = W and its bit reversal) and V (elements 2, 3)
    w = philox4x32_10(np.uint64(100), np.uint64(0), np.uint64(tag), np.uint64(0),
                      np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32))
    for k in range(4):
        W, Wr, V, Vr = (int(x) for x in a[4 * k:4 * k + 4])
        assert int(w[k]) == ((V >> 8) << 24) | ((W >> 8) << 16) | ((V & 0xFF) << 8) | (W & 0xFF)
        assert Wr == int(f"{W:016b}"[::-1], 2) and Vr == int(f"{V:016b}"[::-1], 2)
    # tag, seed and offset each select a different stream
    assert not np.array_equal(a, random_bits16(seed, 100, tag + 1, 4096))
    assert not np.array_equal(a, random_bits16(seed + 1, 100, tag, 4096))
    assert not np.array_equal(a[:16], a[16:32])
    # 64-bit counter: the high word of the offset is used
    hi = random_bits16(seed, 100 + (1 << 32), tag, 16)
    assert not np.array_equal(a[:16], hi)


def test_sr_is_unbiased_over_seeds():
    """Quantize one tensor under 2048 seeds: the mean dequantized value of
    each element approaches the input within 5 binomial standard errors
    (two-point law with p = (a - lo) / (h - lo)) plus the 2^-16 resolution of
    the random bits."""
    rng = np.random.default_rng(0)
    T = rng.standard_normal((4, 64)).astype(np.float32)
    S = 2048
    acc = np.zeros(T.shape)
    for s in range(S):
        acc += oracle.nvfp4_dequantize(oracle.nvfp4_quantize(T, "sr", seed=s, tag=1))
    mean = acc / S
    q = oracle.nvfp4_quantize(T, "rne")                # same scales as SR
    scale = np.repeat(oracle.e4m3_value(q.scales).astype(np.float64), 16, axis=1) * float(q.g_dec)
    a = np.abs(T / scale)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    inside = a < 6
    idx = np.clip(np.searchsorted(grid, a, side="right") - 1, 0, 6)
    step = grid[idx + 1] - grid[idx]
    p = np.clip((a - grid[idx]) / step, 0, 1)
    sd = step * np.sqrt(p * (1 - p)) * scale
    tol = 5 * sd / math.sqrt(S) + 2.0 * step * scale / 65536 + 1e-12
    assert np.all(np.abs(mean - T)[inside] <= tol[inside])
    assert inside.sum() > 200


def test_group_values_uniform_and_round_ups_uncorrelated():
    """Pin of the random-value-to-element map (``group_values16``): it does
    not come from the pages, and a mistake in it (two elements of a group
    drawing the same bits, a byte lost or repeated) would leave every
    bit-exact test of the oracle against itself green.  So check what any
    correct map must give, on 2^20 groups of four elements:

    - each of the four 16-bit values is uniform: chi^2 of its high byte and
      of its low byte over 256 bins below the 1e-6 quantile of chi^2(255);
    - the round-up decisions of ``e2m1_sr`` for every pair of elements in a
      group are uncorrelated (|corr| < 5 standard errors, 5 / sqrt(2^20)) and
      each happens with the probability the rounding rule fixes, at p = 0.5
      (y = 1.25, halfway between 1 and 1.5) and p = 0.3 (y = 1.15).

    A group draws 32 random bits for its four elements, so the values of a
    pair are not independent as a whole; what stochastic rounding needs is
    that the decisions are, and enumerating all 2^16 values of a pair sharing
    one half-word gives |corr| < 5e-4 at every p tried -- well inside the
    bound -- while a pair reading the same bits gives corr = 1."""
    n = 1 << 20
    r = random_bits16(seed=0x5EED0001, offset=7, tag=3, n_elements=4 * n).reshape(n, 4)
    for k in range(4):
        for part in (r[:, k] >> 8, r[:, k] & 0xFF):
            counts = np.bincount(part, minlength=256)
            chi2 = float(np.sum((counts - n / 256) ** 2 / (n / 256)))
            assert chi2 < 370, (k, chi2)
    bound = 5.0 / math.sqrt(n)
    for y in (1.25, 1.15):
        codes = oracle.e2m1_sr(np.full((n, 4), y, dtype=np.float32), r)
        assert set(np.unique(codes)) <= {2, 3}            # 1.0 or 1.5
        up = (codes == 3).astype(np.float64)
        F = math.floor((np.float32(y) - np.float32(1.0)) / np.float32(0.5) * 65536.0)
        p = F / 65536.0
        se = math.sqrt(p * (1 - p) / n)
        for k in range(4):
            assert abs(up[:, k].mean() - p) < 5 * se, (y, k, up[:, k].mean(), p)
        for i in range(4):
            for j in range(i + 1, 4):
                corr = np.corrcoef(up[:, i], up[:, j])[0, 1]
                assert abs(corr) < bound, (y, i, j, corr)
