"""Pins of the oracle's number-format code against definitions, brute force
and hand-worked cases (no GPU)."""

import numpy as np
import pytest

import oracle
from oracle import nvfp4 as F
from conftest import read_golden


# --------------------------------------------------------------------------
# E2M1
# --------------------------------------------------------------------------
def _e2m1_brute(y):
    """Nearest of the 16 signed E2M1 values, ties to the even code (mantissa
    bit 0), saturating; independent of the threshold form in the oracle."""
    vals = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    out = []
    for v in np.asarray(y, dtype=np.float64).ravel():
        a = min(abs(v), 6.0)
        d = np.abs(vals - a)
        best = np.flatnonzero(d == d.min())
        code = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        out.append(code | (8 if np.signbit(v) else 0))
    return np.array(out, dtype=np.uint8)


def test_e2m1_tie_table():
    for val, code in read_golden("e2m1_rne_ties.txt"):
        got = oracle.e2m1_rne(np.array([float(val)], dtype=np.float32))[0]
        assert got == int(code, 16), (val, got, code)


def test_e2m1_rne_matches_brute_force():
    rng = np.random.default_rng(5)
    y = np.concatenate([
        rng.uniform(-7, 7, 20000),
        np.array([m for m in [0.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0]]),
        np.nextafter(np.float32([0.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0]), 0),
        np.nextafter(np.float32([0.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0]), 10),
        -np.array([0.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0]),
    ]).astype(np.float32)
    assert np.array_equal(oracle.e2m1_rne(y), _e2m1_brute(y))


def test_e2m1_decode_roundtrip():
    codes = np.arange(16, dtype=np.uint8)
    v = oracle.e2m1_value(codes)
    assert np.array_equal(oracle.e2m1_rne(v)[1:], codes[1:])   # -0 -> 0x8, +0 -> 0x0
    assert v[7] == 6.0 and v[15] == -6.0 and v[9] == -0.5


def test_e2m1_sr_takes_a_neighbour_and_is_unbiased_over_all_bits():
    """Over all 2^16 random draws the rounded value's mean is within one
    2^-16 step of the input: the rounding is unbiased up to the resolution
    of the random bits, and it only ever returns the two grid neighbours."""
    r = np.arange(65536, dtype=np.uint32)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    for y in [0.1, 0.3, 0.74, 0.9, 1.1, 1.3, 1.9, 2.2, 2.9, 3.3, 4.5, 5.9, -0.3, -4.7,
              0.5, 3.0, 6.0, 7.5]:
        yy = np.full(65536, y, dtype=np.float32)
        q = oracle.e2m1_value(oracle.e2m1_sr(yy, r)).astype(np.float64)
        a = min(abs(float(np.float32(y))), 6.0)
        lo = grid[grid <= a].max()
        hi = grid[grid >= a].min()
        assert set(np.unique(np.abs(q))) <= {lo, hi}
        step = max(hi - lo, 1e-30)
        assert abs(np.mean(np.abs(q)) - a) <= step / 65536 + 1e-12, y
        assert np.all(np.sign(q[q != 0]) == np.sign(y))


# --------------------------------------------------------------------------
# E4M3
# --------------------------------------------------------------------------
def _e4m3_table():
    codes = np.arange(0x7F)                         # 0x7F is NaN
    return codes, oracle.e4m3_value(codes).astype(np.float64)


def _e4m3_brute(s):
    codes, vals = _e4m3_table()
    out = []
    for v in np.asarray(s, dtype=np.float64).ravel():
        if v > 448.0:
            out.append(0x7E)
            continue
        d = np.abs(vals - v)
        best = np.flatnonzero(d == d.min())
        out.append(best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0])
    return np.array(out, dtype=np.uint8)


def test_e4m3_known_values():
    for code, val in read_golden("e4m3_values.txt"):
        assert oracle.e4m3_value(np.array([int(code, 16)]))[0] == np.float32(val)
        assert oracle.e4m3_rne_satfinite(np.array([float(val)], np.float32))[0] == int(code, 16)


def test_e4m3_rne_matches_brute_force():
    rng = np.random.default_rng(7)
    _, vals = _e4m3_table()
    mids = (vals[1:] + vals[:-1]) / 2
    s = np.concatenate([
        np.exp2(rng.uniform(-12, 9.5, 30000)),
        mids, np.nextafter(mids.astype(np.float32), 0), np.nextafter(mids.astype(np.float32), 1e9),
        vals, [0.0, 2.0 ** -10, 3 * 2.0 ** -11, 464.0, 500.0, 1e30],
    ]).astype(np.float32)
    assert np.array_equal(oracle.e4m3_rne_satfinite(s), _e4m3_brute(s))


# --------------------------------------------------------------------------
# scale layout and packing
# --------------------------------------------------------------------------
def test_scale_layout_hand_examples():
    # K = 256 -> 16 scale columns -> 4 atoms per 128-row group.
    assert F.scale_offset(0, 0, 4) == 0
    assert F.scale_offset(0, 3, 4) == 3
    assert F.scale_offset(1, 0, 4) == 16
    assert F.scale_offset(32, 0, 4) == 4
    assert F.scale_offset(33, 5, 4) == 512 + 16 + 4 + 1
    assert F.scale_offset(127, 15, 4) == 3 * 512 + 31 * 16 + 3 * 4 + 3
    assert F.scale_offset(128, 0, 4) == 4 * 512
    assert F.scale_offset(200, 6, 4) == (4 + 1) * 512 + 8 * 16 + 2 * 4 + 2


def test_scale_layout_is_a_bijection_with_padding():
    rows, K = 300, 192
    lin = np.random.default_rng(1).integers(1, 255, (rows, K // 16)).astype(np.uint8)
    flat = F.swizzle_scales(lin, rows, K)
    assert flat.size == 384 * K // 16
    assert np.array_equal(F.unswizzle_scales(flat, rows, K), lin)
    assert np.count_nonzero(flat) == lin.size          # padding rows are zero


def test_nibble_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    assert F.pack_codes(codes).tolist() == [[0x21, 0x43]]
    assert np.array_equal(F.unpack_codes(F.pack_codes(codes)), codes)


# --------------------------------------------------------------------------
# the block quantizer
# --------------------------------------------------------------------------
def test_tensor_scale_closed_forms():
    g_enc, g_dec = F.tensor_scales(np.float32(6.0))
    assert g_enc == 448.0 and g_dec == np.float32(6.0 / 2688.0)
    assert F.tensor_scales(np.float32(2688.0)) == (1.0, 1.0)
    assert F.tensor_scales(np.float32(0.0)) == (1.0, 1.0)


def test_quantize_worked_block_on_grid():
    """A = 6: g_enc = 448, the block max 6 gives s = 448 -> scale code 0x7E,
    r = 1, so grid values come out as their own codes."""
    row = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6],
                   dtype=np.float32)[None, :]
    T = np.concatenate([row, row * 0.5], axis=1)   # second block: max 3
    T = np.concatenate([T, T, T, T], axis=1)        # K = 128
    q = oracle.nvfp4_quantize(T, "rne")
    codes = F.unpack_codes(q.codes)[0]
    assert codes[:16].tolist() == list(range(16))
    # block 2: a = 3 -> s = 0.5 * 448 = 224 (code 0x76) -> r = 2 -> y = T
    assert q.scales[0, 0] == 0x7E and q.scales[0, 1] == 0x76
    assert codes[16:32].tolist() == list(range(16))
    assert q.g_dec == np.float32(6.0 / 2688.0)
    D = oracle.nvfp4_dequantize(q)
    assert np.allclose(D * 2688.0 / 6.0 / 448.0, T, rtol=1e-6, atol=0)


def test_quantize_worked_block_off_grid():
    """A = 6 in block 0; block 1 = [1.2, 0.3, -0.9, 0.1, 0...]: a = 1.2,
    s = fl(0.2) * 448 = 89.6 -> E4M3 binade [64, 128) quantum 8 -> 88 (0x6B),
    r = fl(448 / 88) = 5.0909..., y = [6.109, 1.527, -4.582, 0.509],
    RNE codes [7 (sat), 3 (1.5), 0xE (-4... 4.58 < 5 -> 4), 1 (0.5)]."""
    T = np.zeros((1, 64), dtype=np.float32)
    T[0, 0] = 6.0
    T[0, 16:20] = [1.2, 0.3, -0.9, 0.1]
    q = oracle.nvfp4_quantize(T, "rne")
    assert q.scales[0, 1] == 0x6B
    assert oracle.e4m3_value(np.array([0x6B]))[0] == 88.0
    assert F.unpack_codes(q.codes)[0, 16:20].tolist() == [7, 3, 0xE, 1]


def test_quantize_underflowing_block_is_zero_with_sign():
    T = np.zeros((1, 64), dtype=np.float32)
    T[0, 0] = 1000.0
    T[0, 16:18] = [1e-6, -1e-6]
    q = oracle.nvfp4_quantize(T, "rne")
    assert q.scales[0, 1] == 0
    assert F.unpack_codes(q.codes)[0, 16:18].tolist() == [0, 8]


def test_quantize_idempotent_on_representable_tensor():
    rng = np.random.default_rng(3)
    R, K = 64, 256
    codes = rng.integers(0, 16, (R, K)).astype(np.uint8)
    codes[:, ::16] = 7                                 # every block reaches 6
    sc = rng.integers(0x30, 0x50, (R, K // 16))
    sc[0, 0] = 0x7E                                    # tensor max 6 * 448 * g_dec
    q0 = F.NVFP4(F.pack_codes(codes), sc.astype(np.uint8), np.float32(1.0), R, K)
    T = oracle.nvfp4_dequantize(q0).astype(np.float32)
    q = oracle.nvfp4_quantize(T, "rne")
    assert np.array_equal(oracle.nvfp4_dequantize(q), T.astype(np.float64))


def test_quantize_error_bound_rne():
    """Each element lands within half a grid step (scaled) of the input, or
    at +-6 scaled when the E4M3 rounding of the scale pushed it past 6."""
    rng = np.random.default_rng(4)
    T = (rng.standard_normal((128, 256)) * np.exp(rng.uniform(-3, 3, (128, 1)))).astype(np.float32)
    q = oracle.nvfp4_quantize(T, "rne")
    D = oracle.nvfp4_dequantize(q)
    scale = np.repeat(oracle.e4m3_value(q.scales).astype(np.float64), 16, axis=1) * float(q.g_dec)
    y = T / scale
    codes = F.unpack_codes(q.codes)
    a = np.abs(y)
    spacing = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    ok = (np.abs(D / scale - y) <= spacing / 2 * (1 + 1e-6)) | ((codes & 7) == 7)
    assert ok.all()
    # relative reconstruction error of Gaussian data is FP4-sized
    rel = np.linalg.norm(D - T) / np.linalg.norm(T)
    assert 0.02 < rel < 0.2


def test_quantize_block_max_maps_near_six():
    rng = np.random.default_rng(8)
    T = rng.standard_normal((32, 128)).astype(np.float32)
    q = oracle.nvfp4_quantize(T, "rne")
    codes = F.unpack_codes(q.codes).reshape(32, 8, 16) & 7
    assert np.all(codes.max(axis=2) >= 6)              # |y_max| in [4.9, 6.x]


def test_nonfinite_input_rejected():
    T = np.ones((1, 16), np.float32)
    T[0, 3] = np.nan
    with pytest.raises(ValueError):
        oracle.nvfp4_quantize(T)
