"""Column reduce and split quantizer on the GPU, bit-exact against the
oracle (mu, X_R, codes, scales, decode scales)."""

import numpy as np
import pytest
import torch

import oracle
from quantized_gemm_column_b200 import inputs
from nvfp4_io import assert_nvfp4_equal

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _x(l, K, dtype, seed=0, mean_scale=1.0):
    rng = inputs.rng_for(50, seed)
    X = inputs.spiked_activations(rng, l, K, rank=2, s=(8.0, 4.0), n_hot=max(1, K // 100),
                                  mean_scale=mean_scale)
    if dtype == "bf16":
        t = inputs.to_bf16(X)
        return t.cuda(), inputs.bf16_as_f32(t)
    x = inputs.to_f32(X)
    return torch.from_numpy(x).cuda(), x


def _split(api, Xd, rm, seed=7, offset=0, grad=False, debug=True, fused=False):
    """The two-kernel split, with X_R as well when debug; fused=True runs the
    one-kernel variant (no X_R)."""
    l, K = Xd.shape
    mu = torch.empty(K, dtype=torch.float32, device="cuda")
    mu_q = api.NVFP4Tensor(1, K)
    xr_q = api.NVFP4Tensor(l, K)
    xr = torch.empty((l, K), dtype=torch.float32, device="cuda") if debug and not fused else None
    ws = api.workspace(l, K)
    if fused:
        api.averis_split_quant_fused(Xd, rm, seed, offset, grad, mu, mu_q, xr_q, ws)
    else:
        api.averis_split_quant(Xd, rm, seed, offset, grad, mu, mu_q, xr_q, xr, ws)
    assert api.averis_check_status(ws) == 0
    return mu, mu_q, xr_q, xr


SHAPES = [(256, 128, "f32"), (300, 192, "bf16"), (1024, 1024, "bf16"), (4133, 640, "bf16"),
          (512, 6144, "bf16"), (64, 64, "f32"), (1, 256, "bf16"),
          (40, 8256, "bf16"),     # K above the 8192-column window of the mean quantizer
          (5000, 2112, "bf16")]   # 17 x 20 reduce units, a ragged column tile and a ragged chunk


@pytest.mark.parametrize("l,K,dt", SHAPES)
@pytest.mark.parametrize("rm", ["rne", "sr"])
@pytest.mark.parametrize("path", ["two-kernel", "two-kernel-no-debug", "fused"])
def test_split_quant_bit_exact(api, l, K, dt, rm, path):
    Xd, x = _x(l, K, dt, seed=l + K)
    debug = path == "two-kernel"
    mu, mu_q, xr_q, xr = _split(api, Xd, rm, seed=1234 + l, offset=99, debug=debug, fused=path == "fused")
    rmu, rxr, rmu_q, rxr_q = oracle.averis_split_quant(x, rm, seed=1234 + l, offset=99)
    assert np.array_equal(mu.cpu().numpy().view(np.uint32), rmu.view(np.uint32))
    if debug:
        assert np.array_equal(xr.cpu().numpy().view(np.uint32), rxr.view(np.uint32))
    assert_nvfp4_equal(xr_q, rxr_q, "X_bar_R")
    assert_nvfp4_equal(mu_q, rmu_q, "mu_bar")


def test_grad_tags(api):
    Xd, x = _x(512, 256, "bf16", seed=3)
    _, mu_q, xr_q, _ = _split(api, Xd, "sr", seed=5, grad=True)
    _, _, rmu_q, rxr_q = oracle.averis_split_quant(x, "sr", seed=5, grad=True)
    assert_nvfp4_equal(xr_q, rxr_q, "D_bar_R")
    assert_nvfp4_equal(mu_q, rmu_q, "mu_bar_D")


def test_order_pins_on_device(api):
    """The oracle's order pins hold on the device: [2^24, 1, ..., 1] keeps
    2^24 inside a chunk and across chunks."""
    X = np.zeros((1024, 64), dtype=np.float32)
    X[0, 0] = 2.0 ** 24
    X[1:256, 0] = 1.0
    X[0, 1] = 2.0 ** 24
    X[256, 1] = X[512, 1] = X[768, 1] = 1.0
    mu, _, _, _ = _split(api, torch.from_numpy(X).cuda(), "rne")
    m = mu.cpu().numpy()
    assert m[0] == np.float32(2.0 ** 24 / 1024) and m[1] == np.float32(2.0 ** 24 / 1024)


def test_constant_columns(api):
    rng = np.random.default_rng(1)
    c = inputs.bf16_as_f32(inputs.to_bf16(rng.standard_normal(128) * 10))
    X = np.repeat(c[None, :], 2048, axis=0)
    mu, _, xr_q, xr = _split(api, torch.from_numpy(X).to(torch.bfloat16).cuda(), "sr")
    assert np.array_equal(mu.cpu().numpy(), c)
    assert not xr.cpu().numpy().any()
    assert not xr_q.codes.cpu().numpy().any() and xr_q.g_dec.item() == 1.0


@pytest.mark.parametrize("rm", ["rne", "sr"])
def test_vanilla_quant_bit_exact(api, rm):
    Xd, x = _x(700, 384, "bf16", seed=9)
    q = api.NVFP4Tensor(700, 384)
    ws = api.workspace(700, 384)
    api.nvfp4_quant(Xd, rm, 77, 3, False, q, ws)
    assert api.averis_check_status(ws) == 0
    assert_nvfp4_equal(q, oracle.vanilla_quant(x, rm, 77, 3), "Q_4(X)")


@pytest.mark.parametrize("m,n,dt", [(128, 256, "f32"), (1024, 4096, "bf16"), (192, 320, "bf16")])
def test_weight_quant_bit_exact(api, m, n, dt):
    rng = inputs.rng_for(51, m + n)
    W = inputs.weight(rng, m, n)
    if dt == "bf16":
        Wt = inputs.to_bf16(W)
        w = inputs.bf16_as_f32(Wt)
        Wd = Wt.cuda()
    else:
        w = inputs.to_f32(W)
        Wd = torch.from_numpy(w).cuda()
    w_fwd, w_dgrad = api.NVFP4Tensor(n, m), api.NVFP4Tensor(m, n)
    ws = api.workspace(m, n)
    api.averis_quant_weight(Wd, w_fwd, w_dgrad, ws)
    assert api.averis_check_status(ws) == 0
    r_fwd, r_dgrad = oracle.quant_weight(w)
    assert_nvfp4_equal(w_fwd, r_fwd, "W_bar fwd")
    assert_nvfp4_equal(w_dgrad, r_dgrad, "W_bar dgrad")


def test_nonfinite_input_sets_status(api):
    X = torch.ones((256, 64), dtype=torch.bfloat16, device="cuda")
    X[17, 5] = float("nan")
    mu = torch.empty(64, dtype=torch.float32, device="cuda")
    xr_q = api.NVFP4Tensor(256, 64)
    ws = api.workspace(256, 64)
    api.averis_split_quant(X, "rne", 0, 0, False, mu, None, xr_q, None, ws)
    assert api.averis_check_status(ws) == api.AVR_ERR_NONFINITE
    assert api.averis_check_status(ws) == 0       # cleared by the read


def test_empty_input_is_a_no_op(api):
    X = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    mu = torch.full((128,), 3.0, device="cuda")
    xr_q = api.NVFP4Tensor(0, 128)
    ws = api.workspace(0, 128)
    api.averis_split_quant(X, "sr", 0, 0, False, mu, None, xr_q, None, ws)
    assert api.averis_check_status(ws) == 0
    assert torch.all(mu == 3.0)


def test_repeat_calls_reuse_workspace(api):
    """Tickets wrap back to zero, so one workspace serves many calls and
    shapes in a row with identical results."""
    ws = api.workspace(4096, 1024)
    Xd, x = _x(1024, 512, "bf16", seed=21)
    outs = []
    for _ in range(3):
        mu = torch.empty(512, device="cuda")
        q = api.NVFP4Tensor(1024, 512)
        api.averis_split_quant(Xd, "sr", 1, 0, False, mu, None, q, None, ws)
        outs.append((mu.cpu().numpy(), q.codes.cpu().numpy()))
        Yd, _ = _x(4096, 1024, "bf16", seed=22)
        api.averis_split_quant(Yd, "rne", 1, 0, False, torch.empty(1024, device="cuda"), None,
                               api.NVFP4Tensor(4096, 1024), None, ws)
    assert api.averis_check_status(ws) == 0
    for o in outs[1:]:
        assert np.array_equal(o[0], outs[0][0]) and np.array_equal(o[1], outs[0][1])


def test_alternating_shapes_share_tickets(api):
    """Reduces of different grids (4 x 4 and 17 x 20 units) count on the same
    tickets; alternating them on one workspace gives the same bytes every time."""
    ws = api.workspace(5000, 2112)
    Xd, _ = _x(1024, 512, "bf16", seed=23)
    Yd, _ = _x(5000, 2112, "bf16", seed=24)
    outs = []
    for _ in range(3):
        got = []
        for src, (l, K) in ((Xd, (1024, 512)), (Yd, (5000, 2112)), (Xd, (1024, 512))):
            mu = torch.empty(K, device="cuda")
            q = api.NVFP4Tensor(l, K)
            api.averis_split_quant(src, "sr", 2, 0, False, mu, None, q, None, ws)
            got.append((mu.cpu().numpy(), q.codes.cpu().numpy(), q.g_dec.item()))
        outs.append(got)
    assert api.averis_check_status(ws) == 0
    for o in outs[1:]:
        for (m0, c0, g0), (m1, c1, g1) in zip(o, outs[0]):
            assert np.array_equal(m0, m1) and np.array_equal(c0, c1) and g0 == g1
    assert np.array_equal(outs[0][0][0], outs[0][2][0]) and np.array_equal(outs[0][0][1], outs[0][2][1])


@pytest.mark.parametrize("l,K,dt", [(8192, 1024, "bf16"), (16384, 3072, "bf16"), (32768, 4096, "bf16"),
                                    (2000, 384, "f32"), (257, 4160, "bf16")])
def test_fused_split_matches_two_kernel_split(api, l, K, dt):
    """The persistent one-kernel split (the unit resident in shared memory,
    the others copied in again) gives the two-kernel chain's bytes, also where
    every CTA has several units."""
    Xd, _ = _x(l, K, dt, seed=l + 3 * K)
    a = _split(api, Xd, "sr", seed=99, offset=5, debug=True)
    b = _split(api, Xd, "sr", seed=99, offset=5, fused=True)
    assert torch.equal(a[0], b[0])
    for qa, qb in ((a[1], b[1]), (a[2], b[2])):
        assert torch.equal(qa.codes, qb.codes) and torch.equal(qa.scales, qb.scales)
        assert torch.equal(qa.g_dec, qb.g_dec)


def test_fused_split_reuses_workspace_and_reports_nonfinite(api):
    """The one-kernel split's grid barriers leave the workspace reusable across
    calls and shapes; a NaN input latches AVR_ERR_NONFINITE, and after the
    status is read the next call runs clean."""
    ws = api.workspace(4096, 1024)
    Xd, x = _x(1024, 512, "bf16", seed=31)
    Yd, _ = _x(4096, 1024, "bf16", seed=32)
    ref = oracle.averis_split_quant(x, "sr", seed=3, offset=1)
    for _ in range(3):
        q, m = api.NVFP4Tensor(1024, 512), api.NVFP4Tensor(1, 512)
        api.averis_split_quant_fused(Xd, "sr", 3, 1, False, None, m, q, ws)
        api.averis_split_quant_fused(Yd, "rne", 3, 1, False, None, None, api.NVFP4Tensor(4096, 1024), ws)
        assert api.averis_check_status(ws) == 0
        assert_nvfp4_equal(q, ref[3], "X_bar_R (fused, repeated)")
    bad = Xd.clone()
    bad[5, 7] = float("nan")
    api.averis_split_quant_fused(bad, "rne", 0, 0, False, None, None, api.NVFP4Tensor(1024, 512), ws)
    assert api.averis_check_status(ws) == api.AVR_ERR_NONFINITE
    q = api.NVFP4Tensor(1024, 512)
    api.averis_split_quant_fused(Xd, "sr", 3, 1, False, None, None, q, ws)
    assert api.averis_check_status(ws) == 0
    assert_nvfp4_equal(q, ref[3], "X_bar_R (fused, after an error)")
