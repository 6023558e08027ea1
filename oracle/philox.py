"""Philox4x32-10 counter-based generator and the random-bit stream of the
stochastic rounder.  TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The pages say stochastic rounding is the default for the E2M1 NVFP4 format
(Lighthouse review, section 三 3.1 "实验设置": "默认使用随机舍入") and say
nothing about the generator.  The reading taken here: Philox4x32 with 10
rounds, from Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy
as 1, 2, 3" (SC'11), written from the paper's definition:

  one round:  (c0, c1, c2, c3) -> (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2),
                                   hi(M0*c0) ^ c3 ^ k1, lo(M0*c0))
  key bump:   (k0, k1) -> (k0 + W0, k1 + W1)  (mod 2^32), after every round

with the paper's multipliers M0 = 0xD2511F53, M1 = 0xCD9E8D57 and Weyl
constants W0 = 0x9E3779B9 (golden ratio), W1 = 0xBB67AE85 (sqrt(3) - 1).

Stream mapping (a reading; the pages are silent):
  key     = (lo32(seed), hi32(seed))
  counter = (lo32(g), hi32(g), tag, 0) with g = offset + floor(e / 8),
            e = i*K + j the row-major index of the element in its tensor
  element e takes the 16-bit half (e mod 2) (0 = low) of output word
  floor((e mod 8) / 2).
"""

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint64(0x9E3779B9)
W1 = np.uint64(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)
SHIFT32 = np.uint64(32)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32-10 on arrays of 32-bit words (held in uint64).

    Returns the four output words as uint64 arrays with values < 2^32.
    The 32x32 -> 64-bit products never exceed 2^64, so uint64 is exact.
    """
    c0 = np.asarray(c0, dtype=np.uint64)
    c1 = np.asarray(c1, dtype=np.uint64)
    c2 = np.asarray(c2, dtype=np.uint64)
    c3 = np.asarray(c3, dtype=np.uint64)
    k0 = np.asarray(k0, dtype=np.uint64)
    k1 = np.asarray(k1, dtype=np.uint64)
    for _ in range(10):
        p0 = M0 * c0
        p1 = M1 * c2
        c0, c1, c2, c3 = ((p1 >> SHIFT32) ^ c1 ^ k0, p1 & MASK32,
                          (p0 >> SHIFT32) ^ c3 ^ k1, p0 & MASK32)
        k0 = (k0 + W0) & MASK32
        k1 = (k1 + W1) & MASK32
    return c0, c1, c2, c3


def random_bits16(seed, offset, tag, n_elements, start=0):
    """The 16 random bits of elements e = start .. start+n_elements-1.

    Returns a uint32 array of values in [0, 65535].
    """
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    if n_elements == 0:
        return np.zeros(0, dtype=np.uint32)
    e = np.arange(start, start + n_elements, dtype=np.uint64)
    # One generator call serves the 8 elements that share floor(e / 8).
    first_blk, last_blk = start // 8, (start + n_elements - 1) // 8
    blk = np.arange(first_blk, last_blk + 1, dtype=np.uint64)
    g = np.uint64(offset) + blk            # wraps mod 2^64 like the 64-bit counter
    words = philox4x32_10(g & MASK32, g >> SHIFT32,
                          np.full_like(g, np.uint64(tag)), np.zeros_like(g),
                          np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32))
    w = np.stack(words, axis=0)                       # [4, n_blocks]
    sub = e % np.uint64(8)
    col = (e // np.uint64(8) - np.uint64(first_blk)).astype(np.int64)
    word = w[(sub // np.uint64(2)).astype(np.int64), col]
    half = (sub % np.uint64(2)) * np.uint64(16)
    return ((word >> half) & np.uint64(0xFFFF)).astype(np.uint32)
