"""The Averis and vanilla NVFP4 linear layers end to end on the GPU against
the oracle: operands bit-exact, outputs within the GEMM tolerance."""

import numpy as np
import pytest
import torch

import oracle
from quantized_gemm_column_b200 import inputs
from nvfp4_io import (assert_nvfp4_equal, check_bf16_output, from_oracle, gemm_tolerance,
                      to_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _weights(api, Wd):
    m, n = Wd.shape
    w_fwd, w_dgrad = api.NVFP4Tensor(n, m), api.NVFP4Tensor(m, n)
    ws = api.workspace(m, n)
    api.averis_quant_weight(Wd, w_fwd, w_dgrad, ws)
    assert api.averis_check_status(ws) == 0
    return w_fwd, w_dgrad


@pytest.mark.parametrize("rm", ["rne", "sr"])
def test_tiny_forward_fp32(api, rm):
    """The tiny forward-only case: X fp32 [256, 128], W fp32 [128, 256],
    Y fp32 [256, 256]; relative Frobenius error <= 1e-5 against the fp64
    product of the same quantized operands."""
    X, W = inputs.workload0()
    w_fwd, _ = _weights(api, torch.from_numpy(W).cuda())
    Y = torch.empty((256, 256), dtype=torch.float32, device="cuda")
    xr, mu = api.NVFP4Tensor(256, 128), api.NVFP4Tensor(1, 128)
    ws = api.workspace(256, 128, 256)
    api.averis_linear_fwd(torch.from_numpy(X).cuda(), w_fwd, rm, 0, 0, Y, ws, save_xr=xr, save_mu=mu)
    assert api.averis_check_status(ws) == 0
    Yref, ops = oracle.averis_linear_reference(X, to_oracle(w_fwd), rm, seed=0, offset=0)
    assert_nvfp4_equal(xr, ops["xr_q"], "X_bar_R")
    assert_nvfp4_equal(mu, ops["mu_q"], "mu_bar")
    Yg = Y.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(Yg - Yref) / np.linalg.norm(Yref) <= 1e-5


@pytest.mark.parametrize("l,m,n", [(300, 192, 320), (1024, 512, 768),
                                   (256, 8320, 192)])   # forward K above the mean window
def test_forward_and_dgrad_bf16(api, l, m, n):
    rng = inputs.rng_for(60, l)
    X = inputs.to_bf16(inputs.spiked_activations(rng, l, m, 2, (8.0, 4.0), n_hot=3))
    W = inputs.to_bf16(inputs.weight(rng, m, n))
    D = inputs.to_bf16(inputs.output_gradient(rng, l, n))
    x, d = inputs.bf16_as_f32(X), inputs.bf16_as_f32(D)
    w_fwd, w_dgrad = _weights(api, W.cuda())
    ws = api.workspace(l, max(m, n), max(m, n))
    Y = torch.empty((l, n), dtype=torch.bfloat16, device="cuda")
    api.averis_linear_fwd(X.cuda(), w_fwd, "sr", 11, 5, Y, ws)
    dX = torch.empty((l, m), dtype=torch.bfloat16, device="cuda")
    api.averis_linear_dgrad(D.cuda(), w_dgrad, "sr", 12, 6, dX, ws)
    assert api.averis_check_status(ws) == 0
    wf, wd = to_oracle(w_fwd), to_oracle(w_dgrad)
    Yref, ops = oracle.averis_linear_reference(x, wf, "sr", seed=11, offset=5)
    check_bf16_output(Y.float().cpu().numpy(), Yref, gemm_tolerance(ops["xr_q"], wf, ops["bias"], m))
    dref, dops = oracle.averis_linear_reference(d, wd, "sr", seed=12, offset=6, grad=True)
    check_bf16_output(dX.float().cpu().numpy(), dref, gemm_tolerance(dops["xr_q"], wd, dops["bias"], n))


def test_vanilla_forward_and_dgrad(api):
    l, m, n = 512, 256, 384
    rng = inputs.rng_for(61, 0)
    X = inputs.to_bf16(inputs.spiked_activations(rng, l, m, 2, (8.0, 4.0), n_hot=3))
    W = inputs.to_bf16(inputs.weight(rng, m, n))
    D = inputs.to_bf16(inputs.output_gradient(rng, l, n))
    w_fwd, w_dgrad = _weights(api, W.cuda())
    ws = api.workspace(l, max(m, n), max(m, n))
    Y = torch.empty((l, n), dtype=torch.float32, device="cuda")
    api.nvfp4_linear_fwd(X.cuda(), w_fwd, "sr", 3, 0, Y, ws)
    dX = torch.empty((l, m), dtype=torch.float32, device="cuda")
    api.nvfp4_linear_dgrad(D.cuda(), w_dgrad, "rne", 0, 0, dX, ws)
    assert api.averis_check_status(ws) == 0
    Yref, _ = oracle.vanilla_linear_reference(inputs.bf16_as_f32(X), to_oracle(w_fwd), "sr", 3, 0)
    dref, _ = oracle.vanilla_linear_reference(inputs.bf16_as_f32(D), to_oracle(w_dgrad), "rne",
                                              grad=True)
    for g, r in ((Y, Yref), (dX, dref)):
        g = g.cpu().numpy().astype(np.float64)
        assert np.linalg.norm(g - r) / np.linalg.norm(r) <= 1e-5


@pytest.mark.parametrize("K", [512, 8384])   # one and two windows of K
def test_bias_row_entry_point(api, K):
    rng = np.random.default_rng(5)
    mu_q = oracle.nvfp4_quantize(rng.standard_normal((1, K)).astype(np.float32), "rne")
    w_q = oracle.nvfp4_quantize(rng.standard_normal((320, K)).astype(np.float32), "rne")
    bias = torch.empty(320, dtype=torch.float32, device="cuda")
    ws = api.workspace(0, K)
    api.averis_bias_row(from_oracle(mu_q, api), from_oracle(w_q, api), bias, ws)
    ref = oracle.bias_row(mu_q, w_q)
    tol = K * 2.0 ** -24 * (np.abs(oracle.nvfp4_dequantize(mu_q)) @
                            np.abs(oracle.nvfp4_dequantize(w_q)).T)[0] + 1e-30
    assert np.all(np.abs(bias.cpu().numpy() - ref) <= tol)


def test_qkv_shape_full_size_sampled(api):
    """The fused-QKV workload at full size (X [8192, 1024], W [1024, 4096],
    dY [8192, 4096], SR), in the launch configuration the benchmark times:
    every quantized operand bit-exact, outputs checked on 256 sampled rows."""
    X, W, D = inputs.workload1()
    l, m, n = 8192, 1024, 4096
    w_fwd, w_dgrad = _weights(api, W.cuda())
    ws = api.workspace(l, n, n)
    xr, muq = api.NVFP4Tensor(l, m), api.NVFP4Tensor(1, m)
    Y = torch.empty((l, n), dtype=torch.bfloat16, device="cuda")
    api.averis_linear_fwd(X.cuda(), w_fwd, "sr", 2024, 0, Y, ws, save_xr=xr, save_mu=muq)
    dX = torch.empty((l, m), dtype=torch.bfloat16, device="cuda")
    api.averis_linear_dgrad(D.cuda(), w_dgrad, "sr", 2025, 0, dX, ws)
    # the dgrad operand, recomputed through the split entry point with the same stream
    dr, dmu = api.NVFP4Tensor(l, n), api.NVFP4Tensor(1, n)
    api.averis_split_quant(D.cuda(), "sr", 2025, 0, True, None, dmu, dr, None, ws)
    assert api.averis_check_status(ws) == 0
    x, d = inputs.bf16_as_f32(X), inputs.bf16_as_f32(D)
    wf, wd = to_oracle(w_fwd), to_oracle(w_dgrad)
    _, _, rmu, rxr = oracle.averis_split_quant(x, "sr", 2024, 0)
    assert_nvfp4_equal(xr, rxr, "X_bar_R (QKV)")
    assert_nvfp4_equal(muq, rmu, "mu_bar (QKV)")
    _, _, rdmu, rdr = oracle.averis_split_quant(d, "sr", 2025, 0, grad=True)
    assert_nvfp4_equal(dr, rdr, "D_bar_R (QKV)")
    assert_nvfp4_equal(dmu, rdmu, "mu_bar_D (QKV)")
    rows = np.sort(np.random.default_rng(0).choice(l, 256, replace=False))
    for out, a_q, mq, w_q, K in ((Y, rxr, rmu, wf, m), (dX, rdr, rdmu, wd, n)):
        b = oracle.bias_row(mq, w_q)
        ref = oracle.gemm_reference(a_q, w_q, b, rows=rows)
        got = out.float().cpu().numpy()[rows]
        check_bf16_output(got, ref, gemm_tolerance(a_q, w_q, b, K, rows=rows))
