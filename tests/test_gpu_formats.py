"""The device's number conversions and Philox against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from oracle.philox import philox4x32_10

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _class_sweep():
    """fp32 values covering every (sign, exponent, top 12 mantissa bits) with
    low mantissa bits 0, 1 and a random pattern: E4M3 (3 mantissa bits) and
    E2M1 (1 mantissa bit) rounding depends only on these plus a sticky bit."""
    rng = np.random.default_rng(11)
    sign = np.arange(2, dtype=np.uint32)[:, None, None]
    exp = np.arange(255, dtype=np.uint32)[None, :, None]          # no Inf/NaN
    top = np.arange(4096, dtype=np.uint32)[None, None, :]
    base = (sign << 31) | (exp << 23) | (top << 11)
    lows = [np.zeros_like(base), np.ones_like(base),
            rng.integers(0, 2048, base.shape, dtype=np.uint32)]
    bits = np.concatenate([(base | lo).ravel() for lo in lows])
    return bits.view(np.float32)


def test_conversions_match_oracle(api):
    x = _class_sweep()
    xd = torch.from_numpy(x).cuda()
    e4 = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    e2 = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    api.averis_probe_convert(xd, e4, e2)
    torch.cuda.synchronize()
    g4, g2 = e4.cpu().numpy(), e2.cpu().numpy()
    r4 = oracle.e4m3_rne_satfinite(np.abs(x))
    r2 = oracle.e2m1_rne(x)
    bad4 = np.flatnonzero(g4 != r4)
    assert bad4.size == 0, f"E4M3: {bad4.size} differ, e.g. x={x[bad4[:4]]} gpu={g4[bad4[:4]]} ref={r4[bad4[:4]]}"
    bad2 = np.flatnonzero(g2 != r2)
    assert bad2.size == 0, f"E2M1: {bad2.size} differ, e.g. x={x[bad2[:4]]} gpu={g2[bad2[:4]]} ref={r2[bad2[:4]]}"


def test_stochastic_conversion_matches_oracle(api):
    """Every (sign, exponent, top-12-mantissa-bit) class in [2^-20, 8) x 3
    random words (zero, all ones, random), four values per word: the device's
    stochastic rounding gives the oracle's codes."""
    from oracle.philox import group_values16
    rng = np.random.default_rng(12)
    sign = np.arange(2, dtype=np.uint32)[:, None, None]
    exp = np.arange(107, 130, dtype=np.uint32)[None, :, None]          # 2^-20 .. 8
    top = np.arange(4096, dtype=np.uint32)[None, None, :]
    base = ((sign << 31) | (exp << 23) | (top << 11)).ravel()
    vals = np.concatenate([base | 0, base | 1, base | rng.integers(0, 2048, base.size, dtype=np.uint32)])
    vals = rng.permutation(vals).view(np.float32)
    vals = vals[: vals.size // 4 * 4].reshape(-1, 4)
    for words in (np.zeros(len(vals), np.uint32), np.full(len(vals), 0xFFFFFFFF, np.uint32),
                  rng.integers(0, 2 ** 32, len(vals), dtype=np.uint64).astype(np.uint32)):
        xd = torch.from_numpy(np.ascontiguousarray(vals)).cuda()
        wd = torch.from_numpy(words.view(np.int32)).cuda()
        out = torch.empty(len(vals), dtype=torch.int16, device="cuda")
        api.averis_probe_convert_sr(xd, wd, out)
        got = out.cpu().numpy().view(np.uint16).astype(np.uint32)
        got = np.stack([(got >> (4 * k)) & 0xF for k in range(4)], axis=1)
        ref = oracle.e2m1_sr(vals, group_values16(words))
        bad = np.argwhere(got != ref)
        assert bad.size == 0, f"{len(bad)} codes differ, e.g. x={vals[tuple(bad[0])]} got={got[tuple(bad[0])]} ref={ref[tuple(bad[0])]}"


@pytest.mark.parametrize("seed,offset,tag", [(0, 0, 1), (0xDEADBEEF12345678, (1 << 32) - 5, 4)])
def test_philox_matches_oracle(api, seed, offset, tag):
    n = 1 << 18
    out = torch.empty(4 * n, dtype=torch.int32, device="cuda")
    api.averis_probe_philox(seed, offset, tag, n, out)
    got = out.cpu().numpy().view(np.uint32).reshape(n, 4).astype(np.uint64)
    g = (np.uint64(offset) + np.arange(n, dtype=np.uint64))
    ref = philox4x32_10(g & np.uint64(0xFFFFFFFF), g >> np.uint64(32), np.full(n, tag, np.uint64),
                        np.zeros(n, np.uint64), np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32))
    assert np.array_equal(got, np.stack(ref, axis=1))
