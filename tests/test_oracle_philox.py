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
