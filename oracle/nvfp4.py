"""NVFP4 number format: E2M1 codes, E4M3 block scales, FP32 tensor scale.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The pages name the format "E2M1 NVFP4" with stochastic rounding as the
default (Lighthouse review of "The Curse and Blessing of Mean Bias in
FP4-Quantized LLM Training", section 三 3.1 "实验设置") and call the
quantizer Q_4 (section 二 "Averis 方法": mu_bar = Q_4(mu_X),
X_bar_R = Q_4(X - 1 mu_X)).  Nothing finer is printed.  The readings below
follow the public NVFP4 definition (16-element blocks along the contraction
axis, one unsigned E4M3 scale per block, one FP32 per-tensor scale):

  A      = max |T|                       (exact, order free)
  g_enc  = min(fl(2688 / A), FLT_MAX),  g_dec = fl(A / 2688)   (A > 0)
  g_enc  = g_dec = 1                                            (A = 0)
           2688 = 6 * 448 = E2M1 max * E4M3 max; g_dec is the stored
           per-tensor (decode) scale.
  s_b    = fl(fl(a_b / 6) * g_enc),  S_b = E4M3_RNE_SATFINITE(s_b)
  r_b    = 0 if S_b == 0 else fl(g_enc / value(S_b))
  y      = fl(T * r_b)
  code   = E2M1_RNE(y)  or  E2M1_SR(y, r16)
  deq    = value(code) * value(S_b) * g_dec

All fl() are single IEEE fp32 operations with round to nearest even.
"""

from dataclasses import dataclass

import numpy as np

from .philox import random_bits16

# E2M1 magnitudes of codes 0..7 (sign is bit 3).
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)
E2M1_MAX = np.float32(6.0)
E4M3_MAX = np.float32(448.0)
FP4_FP8_PRODUCT = np.float32(2688.0)   # 6 * 448
FLT_MAX = np.float32(np.finfo(np.float32).max)

BLOCK = 16          # elements per E4M3 scale, along the contraction axis
ATOM_ROWS = 128     # rows per scale-layout atom
ATOM_COLS = 4       # scales per atom row (64 elements)
ATOM_BYTES = 512


def _f32(x):
    return np.asarray(x, dtype=np.float32)


# --------------------------------------------------------------------------
# E2M1
# --------------------------------------------------------------------------
def e2m1_value(codes):
    """Decode 4-bit E2M1 codes (uint8, low nibble) to float32 values."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_GRID[c & 7]
    return np.where(c & 8, -mag, mag).astype(np.float32)


def e2m1_rne(y):
    """Round fp32 values to E2M1 codes, nearest with ties to the even code,
    saturating at +-6; the sign bit is kept for values that round to zero.

    Tie points of the magnitude grid {0, .5, 1, 1.5, 2, 3, 4, 6} and the even
    code each one goes to: .25 -> 0, .75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2.0,
    2.5 -> 2.0, 3.5 -> 4.0, 5 -> 4.0.  So the magnitude code counts the
    thresholds passed, with '>' where the lower neighbour is even and '>='
    where the upper one is.
    """
    y = _f32(y)
    a = np.abs(y)
    code = ((a > 0.25).astype(np.uint8) + (a >= 0.75) + (a > 1.25) + (a >= 1.75)
            + (a > 2.5) + (a >= 3.5) + (a > 5.0)).astype(np.uint8)
    sign = np.signbit(y).astype(np.uint8) << 3
    return (code | sign).astype(np.uint8)


def e2m1_sr(y, r16):
    """Stochastic rounding of fp32 values to E2M1 with a 16-bit random value
    each (add-and-carry):

    a = min(|y|, 6); lo <= a < h are its grid neighbours; F = floor of the
    position of a in [lo, h) scaled to 16 bits, floor((a - lo) / (h - lo) *
    65536) (exact in fp32: a - lo is exact because lo = 0 or lo <= a < 2 lo,
    h - lo and 65536 are powers of two); round up iff F + r16 >= 65536, i.e.
    the random value added to the 16 bits below the kept precision carries.
    The sign is kept, also on zero.  P(up) = F / 65536, so the rounding is
    unbiased to within 2^-16 of a grid step.
    """
    y = _f32(y)
    a = np.minimum(np.abs(y), E2M1_MAX)
    idx = (np.searchsorted(E2M1_GRID, a, side="right") - 1).astype(np.int64)
    lo = E2M1_GRID[idx]
    hi = E2M1_GRID[np.minimum(idx + 1, 7)]
    step = np.where(idx == 7, np.float32(1.0), hi - lo).astype(np.float32)
    F = np.floor(((a - lo) / step).astype(np.float32) * np.float32(65536.0)).astype(np.int64)
    up = (F + np.asarray(r16, dtype=np.int64)) >= 65536
    code = (idx + (up & (idx < 7))).astype(np.uint8)
    sign = np.signbit(y).astype(np.uint8) << 3
    return (code | sign).astype(np.uint8)


# --------------------------------------------------------------------------
# E4M3 (OCP FP8 E4M3FN: bias 7, no infinities, max 448, 0x7F = NaN)
# --------------------------------------------------------------------------
def e4m3_value(codes):
    """Decode unsigned E4M3 codes (0..0x7E) to float32."""
    c = np.asarray(codes, dtype=np.int64)
    e = (c >> 3) & 0xF
    m = c & 7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return np.where(c & 0x80, -val, val).astype(np.float32)


def e4m3_rne_satfinite(s):
    """Round non-negative fp32 values to unsigned E4M3 codes, nearest with
    ties to even, saturating to 448 (code 0x7E) above the largest finite.

    Below 2^-6 the quantum is 2^-9 (subnormals); in the binade [2^E, 2^E+1)
    it is 2^(E-3).  n = s / quantum is exact in fp64 and is rounded half to
    even; the code is then n itself in the lowest two binades and
    ((E + 7) << 3) + (n - 8) above, which carries into the exponent when n
    rounds up to 16.
    """
    s = np.asarray(s, dtype=np.float32).astype(np.float64)
    out = np.zeros(s.shape, dtype=np.uint8)
    pos = s > 0
    sat = s > 448.0
    sp = np.where(pos & ~sat, s, 1.0)
    E = np.maximum(np.floor(np.log2(sp)), -6.0)
    # log2 is only used to pick the binade; correct it where it is off by one.
    E = np.where(sp < np.exp2(E), E - 1, E)
    E = np.where(sp >= np.exp2(E + 1), E + 1, E)
    E = np.maximum(E, -6.0)
    q = np.exp2(E - 3.0)
    n = np.rint(sp / q)                      # rint = round half to even
    code = np.where(E <= -6.0, n, (E + 7.0) * 8.0 + (n - 8.0))
    code = np.where(pos & ~sat, code, 0.0)
    code = np.where(sat, 0x7E, code)
    out[...] = code.astype(np.uint8)
    return out


# --------------------------------------------------------------------------
# Scale layout (tcgen05 block-scaled MMA, 4 scales per 64 elements)
# --------------------------------------------------------------------------
def scale_offset(r, c, n_kb64):
    """Byte offset of the scale of (row r, block column c) in the atom layout.

    The rows are cut into 128-row groups and the block columns into groups of
    4; each (row group, column group) pair is a 512-byte atom, atoms ordered
    row group major.  Inside an atom, row r sits at 16 * (r % 32) +
    4 * ((r % 128) // 32), and the 4 scales of that row are consecutive bytes.
    ``n_kb64`` = number of 64-element column groups = K / 64.
    """
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    atom = (r // ATOM_ROWS) * n_kb64 + c // ATOM_COLS
    return atom * ATOM_BYTES + (r % 32) * 16 + ((r % ATOM_ROWS) // 32) * 4 + c % ATOM_COLS


def scales_nbytes(rows, K):
    rows_pad = -(-rows // ATOM_ROWS) * ATOM_ROWS
    return rows_pad * (K // BLOCK)


def swizzle_scales(linear, rows, K):
    """[rows, K/16] scale codes -> flat atom-layout bytes, zero padded."""
    assert K % 64 == 0
    out = np.zeros(scales_nbytes(rows, K), dtype=np.uint8)
    if rows == 0:
        return out
    r, c = np.meshgrid(np.arange(rows), np.arange(K // BLOCK), indexing="ij")
    out[scale_offset(r, c, K // 64)] = linear
    return out


def unswizzle_scales(flat, rows, K):
    r, c = np.meshgrid(np.arange(rows), np.arange(K // BLOCK), indexing="ij")
    return np.asarray(flat, dtype=np.uint8)[scale_offset(r, c, K // 64)]


def pack_codes(codes):
    """[R, K] 4-bit codes -> [R, K/2] bytes, element 2k in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


# --------------------------------------------------------------------------
# The block quantizer Q_4
# --------------------------------------------------------------------------
@dataclass
class NVFP4:
    codes: np.ndarray      # uint8 [R, K/2] packed
    scales: np.ndarray     # uint8 [R, K/16] linear E4M3 codes
    g_dec: np.float32      # per-tensor decode scale
    rows: int
    K: int

    @property
    def scales_swizzled(self):
        return swizzle_scales(self.scales, self.rows, self.K)


def tensor_scales(A):
    """(g_enc, g_dec) for a tensor whose max magnitude is A (fp32)."""
    A = np.float32(A)
    if A == 0:
        return np.float32(1.0), np.float32(1.0)
    with np.errstate(over="ignore", divide="ignore"):
        g_enc = np.minimum(np.float32(FP4_FP8_PRODUCT / A), FLT_MAX)
    g_dec = np.float32(A / FP4_FP8_PRODUCT)
    return np.float32(g_enc), g_dec


def nvfp4_quantize(T, rounding="rne", seed=0, offset=0, tag=0, amax=None):
    """Q_4 of an fp32 tensor T [R, K] along K.  ``rounding`` is "rne" or "sr".

    ``amax`` may be given when the caller already holds max |T| (it is exact
    and order free, so any correct computation gives the same value).
    """
    T = np.ascontiguousarray(_f32(T))
    R, K = T.shape
    assert K % BLOCK == 0
    if not np.all(np.isfinite(T)):
        raise ValueError("non-finite input to the NVFP4 quantizer")
    A = np.float32(np.max(np.abs(T))) if (amax is None and T.size) else np.float32(amax or 0.0)
    g_enc, g_dec = tensor_scales(A)
    blocks = T.reshape(R, K // BLOCK, BLOCK)
    a_b = np.max(np.abs(blocks), axis=2) if T.size else np.zeros((R, K // BLOCK), np.float32)
    with np.errstate(over="ignore"):
        s_b = ((a_b / np.float32(6.0)).astype(np.float32) * g_enc).astype(np.float32)
    S = e4m3_rne_satfinite(s_b)
    Sv = e4m3_value(S)
    with np.errstate(divide="ignore"):
        r_b = np.where(S == 0, np.float32(0.0), (g_enc / np.where(S == 0, 1.0, Sv)).astype(np.float32))
    r_b = r_b.astype(np.float32)
    y = (blocks * r_b[:, :, None]).astype(np.float32).reshape(R, K)
    if rounding == "rne":
        codes = e2m1_rne(y)
    elif rounding == "sr":
        r16 = random_bits16(seed, offset, tag, R * K).reshape(R, K)
        codes = e2m1_sr(y, r16)
    else:
        raise ValueError(rounding)
    return NVFP4(pack_codes(codes), S, g_dec, R, K)


def nvfp4_dequantize(q: NVFP4):
    """fp64 values value(code) * value(S_b) * g_dec."""
    codes = unpack_codes(q.codes)
    v = e2m1_value(codes).astype(np.float64)
    s = np.repeat(e4m3_value(q.scales).astype(np.float64), BLOCK, axis=1)
    return v * s * np.float64(q.g_dec)
