"""Weight gradient dW = X^T D of the Averis linear on the GPU: the token-axis
split quantizer bit-exact against the oracle, the rank-one GEMM epilogue and
the whole chain against the oracle's fp64 product."""

import numpy as np
import pytest
import torch

import oracle
from quantized_gemm_column_b200 import inputs
from nvfp4_io import assert_nvfp4_equal, bf16_ulp, check_bf16_output, to_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _dev(X, dt):
    if dt == "bf16":
        t = inputs.to_bf16(X)
        return t.cuda(), inputs.bf16_as_f32(t)
    x = inputs.to_f32(X)
    return torch.from_numpy(x).cuda(), x


def _acts(l, K, seed, mean_scale=1.0):
    rng = inputs.rng_for(70, seed)
    return inputs.spiked_activations(rng, l, K, rank=2, s=(8.0, 4.0), n_hot=max(1, K // 100),
                                     mean_scale=mean_scale)


def wgrad_tolerance(xt_q, dt_q, mu_x_q, mu_d_q, l, ref, rows=None):
    """Per element: the fp32 accumulation bound over the L-long contraction,
    plus a few fp32 roundings of the epilogue (alpha acc, u v, their sum)."""
    A = np.abs(oracle.nvfp4_dequantize(xt_q))
    if rows is not None:
        A = A[np.asarray(rows)]
    tol = xt_q.K * 2.0 ** -24 * (A @ np.abs(oracle.nvfp4_dequantize(dt_q)).T)
    extra = np.abs(ref)
    if mu_x_q is not None:
        u = np.abs(oracle.nvfp4_dequantize(mu_x_q)[0])
        if rows is not None:
            u = u[np.asarray(rows)]
        extra = extra + l * np.outer(u, np.abs(oracle.nvfp4_dequantize(mu_d_q)[0]))
    return tol + 2.0 ** -22 * extra


SHAPES = [(256, 128, "f32"), (300, 192, "bf16"), (1024, 1024, "bf16"), (4133, 640, "bf16"),
          (1, 256, "bf16"), (40, 8256, "bf16")]


@pytest.mark.parametrize("l,K,dt", SHAPES)
@pytest.mark.parametrize("rm", ["rne", "sr"])
def test_split_quant_t_bit_exact(api, l, K, dt, rm):
    Xd, x = _dev(_acts(l, K, l + K), dt)
    for grad in (False, True):
        L = api.padded_tokens(l)
        mu = torch.empty(K, dtype=torch.float32, device="cuda")
        mu_q, xrt_q = api.NVFP4Tensor(1, K), api.NVFP4Tensor(K, L)
        ws = api.workspace(l, K)
        api.averis_split_quant_t(Xd, rm, 77 + l, 5, grad, mu, mu_q, xrt_q, ws)
        assert api.averis_check_status(ws) == 0
        rmu, rmu_q, rxrt = oracle.averis_split_quant_t(x, rm, seed=77 + l, offset=5, grad=grad)
        assert np.array_equal(mu.cpu().numpy().view(np.uint32), rmu.view(np.uint32))
        assert_nvfp4_equal(xrt_q, rxrt, f"X_bar_R^T grad={grad}")
        assert_nvfp4_equal(mu_q, rmu_q, f"mu_bar grad={grad}")


@pytest.mark.parametrize("l,K,dt", [(256, 128, "f32"), (300, 192, "bf16"), (40, 8256, "bf16")])
def test_vanilla_quant_t_bit_exact(api, l, K, dt):
    Xd, x = _dev(_acts(l, K, 3 * l + K), dt)
    q = api.NVFP4Tensor(K, api.padded_tokens(l))
    ws = api.workspace(l, K)
    api.nvfp4_quant_t(Xd, "sr", 8, 1, True, q, ws)
    assert api.averis_check_status(ws) == 0
    assert_nvfp4_equal(q, oracle.vanilla_quant_t(x, "sr", seed=8, offset=1, grad=True), "Q4(X^T)")


def test_token_quant_mean_matches_rowwise_split(api):
    """mu_bar from the token-axis split is the row-wise split's, bit for bit."""
    l, K = 700, 320
    Xd, _ = _dev(_acts(l, K, 9), "bf16")
    ws = api.workspace(l, K)
    a, b = api.NVFP4Tensor(1, K), api.NVFP4Tensor(1, K)
    api.averis_split_quant(Xd, "sr", 4, 2, False, None, a, api.NVFP4Tensor(l, K), None, ws)
    api.averis_split_quant_t(Xd, "sr", 4, 2, False, None, b, api.NVFP4Tensor(K, api.padded_tokens(l)), ws)
    assert api.averis_check_status(ws) == 0
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales) and torch.equal(a.g_dec, b.g_dec)


@pytest.mark.parametrize("l,m,n,wt", [(256, 128, 192, "f32"), (300, 192, 256, "f32"),
                                      (1000, 256, 384, "bf16"), (40, 64, 128, "f32")])
@pytest.mark.parametrize("rm", ["rne", "sr"])
def test_linear_wgrad_matches_oracle(api, l, m, n, wt, rm):
    Xd, x = _dev(_acts(l, m, l + m, mean_scale=2.0), "bf16")
    rng = inputs.rng_for(71, l + n)
    Dd, d = _dev(inputs.output_gradient(rng, l, n), "bf16")
    dtype = torch.float32 if wt == "f32" else torch.bfloat16
    dW = torch.empty((m, n), dtype=dtype, device="cuda")
    ws = api.wgrad_workspace(l, m, n)
    api.averis_linear_wgrad(Xd, Dd, rm, 31, 7, dW, ws)
    assert api.averis_check_status(ws) == 0
    ref, ops = oracle.averis_wgrad_reference(x, d, rm, seed=31, offset=7)
    tol = wgrad_tolerance(ops["xrt_q"], ops["drt_q"], ops["mu_x_q"], ops["mu_d_q"], l, ref)
    got = dW.float().cpu().numpy().astype(np.float64)
    if wt == "f32":
        err = np.abs(got - ref)
        assert np.all(err <= tol), f"worst {np.max(err - tol):.3e} over the bound"
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-5
    else:
        check_bf16_output(got, ref, tol)


@pytest.mark.parametrize("rm", ["rne", "sr"])
def test_vanilla_wgrad_matches_oracle(api, rm):
    l, m, n = 520, 192, 320
    Xd, x = _dev(_acts(l, m, 5), "bf16")
    Dd, d = _dev(inputs.output_gradient(inputs.rng_for(72, 0), l, n), "bf16")
    dW = torch.empty((m, n), dtype=torch.float32, device="cuda")
    ws = api.wgrad_workspace(l, m, n)
    api.nvfp4_linear_wgrad(Xd, Dd, rm, 3, 0, dW, ws)
    assert api.averis_check_status(ws) == 0
    ref, ops = oracle.vanilla_wgrad_reference(x, d, rm, seed=3, offset=0)
    tol = wgrad_tolerance(ops["xt_q"], ops["dt_q"], None, None, l, ref)
    assert np.all(np.abs(dW.cpu().numpy() - ref) <= tol)


def test_wgrad_gemm_entry_point_from_oracle_operands(api):
    """averis_wgrad_gemm on operands the oracle quantized (no GPU quantizer
    involved): the rank-one epilogue u_i v_j with u = l deq(mu_bar_X)."""
    from nvfp4_io import from_oracle
    rng = np.random.default_rng(12)
    l, m, n = 200, 256, 320
    x = (rng.standard_normal((l, m)) + rng.standard_normal(m) * 2).astype(np.float32)
    d = (rng.standard_normal((l, n)) - 0.5).astype(np.float32)
    ref, ops = oracle.averis_wgrad_reference(x, d, "rne")
    dW = torch.empty((m, n), dtype=torch.float32, device="cuda")
    ws = api.wgrad_workspace(l, m, n)
    api.averis_wgrad_gemm(from_oracle(ops["xrt_q"], api), from_oracle(ops["drt_q"], api),
                          from_oracle(ops["mu_x_q"], api), from_oracle(ops["mu_d_q"], api), l, dW, ws)
    assert api.averis_check_status(ws) == 0
    tol = wgrad_tolerance(ops["xrt_q"], ops["drt_q"], ops["mu_x_q"], ops["mu_d_q"], l, ref)
    assert np.all(np.abs(dW.cpu().numpy() - ref) <= tol)
    # without the means: the plain product
    api.averis_wgrad_gemm(from_oracle(ops["xrt_q"], api), from_oracle(ops["drt_q"], api), None, None, l, dW, ws)
    plain = oracle.wgrad_reference(ops["xrt_q"], ops["drt_q"])
    assert np.all(np.abs(dW.cpu().numpy() - plain) <= wgrad_tolerance(ops["xrt_q"], ops["drt_q"], None, None, l, plain))


def _grid_inputs(rng, l, K):
    """X = 1 mu + R with mu and R on the E2M1 grid, every 16-block of mu and
    every 16-token block of each residual column holding a +/-6 and the
    residual columns summing to 0 in +/- pairs: every operand of the split
    quantizes exactly."""
    pos = np.array([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mu = rng.choice(pos, K) * rng.choice([-1.0, 1.0], K)
    mu[::16] = 6.0
    R = np.zeros((l, K))
    for j in range(K):
        for b0 in range(0, l, 16):
            nb = min(16, l - b0)
            v = rng.choice(pos, nb // 2)
            v[0] = 6.0
            v = v * rng.choice([-1.0, 1.0], nb // 2)
            R[b0:b0 + nb:2, j], R[b0 + 1:b0 + nb:2, j] = v, -v
    return (mu[None, :] + R).astype(np.float32)


@pytest.mark.parametrize("rm", ["rne", "sr"])
def test_wgrad_exact_on_representable_inputs(api, rm):
    """On inputs whose split quantizes exactly, dW is X^T D (fp64 product of
    the fp32 inputs) up to fp32 accumulation and the decode scales: a check
    that needs no quantizer at all on the reference side."""
    rng = np.random.default_rng(21)
    l, m, n = 40, 128, 192
    x, d = _grid_inputs(rng, l, m), _grid_inputs(rng, l, n)
    dW = torch.empty((m, n), dtype=torch.float32, device="cuda")
    ws = api.wgrad_workspace(l, m, n)
    api.averis_linear_wgrad(torch.from_numpy(x).cuda(), torch.from_numpy(d).cuda(), rm, 1, 0, dW, ws)
    assert api.averis_check_status(ws) == 0
    ref = x.astype(np.float64).T @ d.astype(np.float64)
    assert np.allclose(dW.cpu().numpy(), ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_wgrad_empty_tokens_is_zero(api):
    dW = torch.full((64, 128), 7.0, dtype=torch.float32, device="cuda")
    ws = api.wgrad_workspace(0, 64, 128)
    X = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    D = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    api.averis_linear_wgrad(X, D, "sr", 0, 0, dW, ws)
    assert not dW.any()


def test_qkv_wgrad_full_size_sampled(api):
    """The fused-QKV workload's weight gradient at full size (X [8192, 1024],
    dY [8192, 4096], SR): both token-axis operands and both means bit-exact,
    dW [1024, 4096] (fp32) checked on 128 sampled rows."""
    X, _, D = inputs.workload1()
    l, m, n = 8192, 1024, 4096
    dW = torch.empty((m, n), dtype=torch.float32, device="cuda")
    ws = api.wgrad_workspace(l, m, n)
    api.averis_linear_wgrad(X.cuda(), D.cuda(), "sr", 2026, 0, dW, ws)
    assert api.averis_check_status(ws) == 0
    x, d = inputs.bf16_as_f32(X), inputs.bf16_as_f32(D)
    # the operands, recomputed through the token-axis entry point with the same streams
    ws1 = api.workspace(l, n)
    xq, mxq = api.NVFP4Tensor(m, l), api.NVFP4Tensor(1, m)
    dq, mdq = api.NVFP4Tensor(n, l), api.NVFP4Tensor(1, n)
    api.averis_split_quant_t(X.cuda(), "sr", 2026, 0, False, None, mxq, xq, ws1)
    api.averis_split_quant_t(D.cuda(), "sr", 2026, 0, True, None, mdq, dq, ws1)
    assert api.averis_check_status(ws1) == 0
    _, rmx, rxq = oracle.averis_split_quant_t(x, "sr", 2026, 0, grad=False)
    _, rmd, rdq = oracle.averis_split_quant_t(d, "sr", 2026, 0, grad=True)
    assert_nvfp4_equal(xq, rxq, "X_bar_R^T (QKV)")
    assert_nvfp4_equal(mxq, rmx, "mu_bar_X (QKV)")
    assert_nvfp4_equal(dq, rdq, "D_bar_R^T (QKV)")
    assert_nvfp4_equal(mdq, rmd, "mu_bar_D (QKV)")
    rows = np.sort(np.random.default_rng(1).choice(m, 128, replace=False))
    A = oracle.nvfp4_dequantize(rxq)[rows]
    ref = A @ oracle.nvfp4_dequantize(rdq).T + l * np.outer(oracle.nvfp4_dequantize(rmx)[0][rows],
                                                             oracle.nvfp4_dequantize(rmd)[0])
    tol = wgrad_tolerance(rxq, rdq, rmx, rmd, l, ref, rows=rows)
    got = dW.cpu().numpy()[rows]
    assert np.all(np.abs(got - ref) <= tol)
