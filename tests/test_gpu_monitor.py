"""The mean-energy ratio monitor R = ||mu|| / sqrt(E||x||^2 / m) on the GPU
(Lighthouse review, section 七, practice advice item 2), against the oracle's
fp64 definition and against closed forms.

Tolerance: the kernel's column sums of squares are fp32 (fma within a
256-row chunk, chunk partials in order), so for l <= 2^14 their relative
error is at most about (256 + l/256) u <= 2e-5 (u = 2^-24, positive terms);
mu is the split's fp32 mean, bit-exact with the oracle's fixed order, whose
error relative to ||mu|| is of the same order for inputs whose mean is not
cancelled; the norms are fp64 and R is rounded once to fp32.  rel 1e-4
bounds all of it with margin."""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import stats
from quantized_gemm_column_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _ratio(api, Xd):
    l, K = Xd.shape
    mu = torch.empty(K, dtype=torch.float32, device="cuda")
    R = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    ws = api.workspace(l, K)
    api.averis_mean_energy_ratio(Xd, mu, R, ws)
    assert api.averis_check_status(ws) == 0
    return float(R.item()), mu.cpu().numpy()


def _dev(X, dt):
    if dt == "bf16":
        t = inputs.to_bf16(X)
        return t.cuda(), inputs.bf16_as_f32(t)
    x = inputs.to_f32(X)
    return torch.from_numpy(x).cuda(), x


@pytest.mark.parametrize("l,K,dt,mean_scale", [
    (256, 128, "f32", 1.0), (300, 192, "bf16", 1.0), (4133, 640, "bf16", 2.0),
    (8192, 1024, "bf16", 1.0), (1024, 4096, "bf16", 0.25), (77, 8256, "bf16", 1.0),
    (5000, 2112, "bf16", 0.5)])     # ragged column tile and chunk
def test_ratio_matches_oracle(api, l, K, dt, mean_scale):
    rng = inputs.rng_for(61, l + K)
    X = inputs.spiked_activations(rng, l, K, rank=2, s=(8.0, 4.0), n_hot=max(1, K // 100),
                                  mean_scale=mean_scale)
    Xd, x = _dev(X, dt)
    R, mu = _ratio(api, Xd)
    # the mean is the split's, bit for bit
    rmu = oracle.column_mean(x)
    assert np.array_equal(mu.view(np.uint32), rmu.view(np.uint32))
    assert R == pytest.approx(stats.mean_energy_ratio(x), rel=1e-4)


def test_ratio_tracks_mean_scale(api):
    """R rises with the strength of the mean, as the oracle's does."""
    got = []
    for c in (0.0, 2.0, 8.0):
        X, _ = inputs.workload3(c, l=1024, m=256)
        R, _ = _ratio(api, X.cuda())
        got.append(R)
        assert R == pytest.approx(stats.mean_energy_ratio(inputs.bf16_as_f32(X)), rel=1e-4)
    assert got[0] < got[1] < got[2]


@pytest.mark.parametrize("l", [1, 256, 2048])
def test_ratio_constant_rows_is_sqrt_m(api, l):
    """Every row equal to c: mu = c exactly (the fp32 sums of bf16 values are
    exact here), so R = sqrt(m)."""
    m = 512
    rng = inputs.rng_for(62, l)
    c = inputs.to_bf16(rng.standard_normal((1, m)))
    Xd = c.repeat(l, 1).cuda()
    R, mu = _ratio(api, Xd)
    assert np.array_equal(mu, inputs.bf16_as_f32(c)[0])
    assert R == pytest.approx(math.sqrt(m), rel=1e-6)


def test_ratio_zero_mean_pairs_is_zero(api):
    """Rows in +/- pairs (both rows of a pair in one 256-row chunk): every
    column sum cancels exactly, mu = 0 and R = 0."""
    rng = inputs.rng_for(63, 0)
    Y = inputs.to_f32(rng.standard_normal((300, 256)))
    pairs = np.stack([Y, -Y], axis=1).reshape(600, 256)
    R, mu = _ratio(api, torch.from_numpy(np.ascontiguousarray(pairs)).cuda())
    assert not mu.any()
    assert R == 0.0


def test_ratio_nonfinite_latches(api):
    X = torch.randn(512, 128, dtype=torch.float32, device="cuda")
    X[37, 5] = float("inf")
    ws = api.workspace(512, 128)
    R = torch.empty(1, dtype=torch.float32, device="cuda")
    api.averis_mean_energy_ratio(X, None, R, ws)
    assert api.averis_check_status(ws) == api.AVR_ERR_NONFINITE
