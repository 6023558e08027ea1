"""Parity at the full sizes of the larger workloads (the FFN projections, the
mean-strength sweep, the 32768-token layer shapes), in the launch
configuration the benchmark uses: the fp32 mean bit-exact over every column,
the quantized mean (codes, every scale byte and its decode scale) bit-exact,
the residual's decode scale bit-exact, the quantized residual bit-exact on
sampled rows, outputs within the R19 bound on the same rows.

The oracle quantizes only the sampled rows.  Row r of an [l, K] tensor is the
1 x K tensor at stream offset offset + r K / 16 with the full tensor's amax:
the oracle's stream counts from offset + e / 16 for element e (pinned by the
generator tests), and the tensor scale depends on the amax alone."""

import numpy as np
import pytest
import torch

import oracle
from oracle import nvfp4 as F
from quantized_gemm_column_b200 import inputs
from nvfp4_io import assert_nvfp4_equal, check_bf16_output, gemm_tolerance, to_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _weights(api, W):
    m, n = W.shape
    w_fwd, w_dgrad = api.NVFP4Tensor(n, m), api.NVFP4Tensor(m, n)
    ws = api.workspace(m, n, n)
    api.averis_quant_weight(W.cuda(), w_fwd, w_dgrad, ws)
    assert api.averis_check_status(ws) == 0
    return w_fwd, w_dgrad


def _rows_of(q, rows):
    """Codes and linear scales of some rows of a device NVFP4 tensor."""
    codes = q.codes.cpu().numpy()[rows]
    lin = F.unswizzle_scales(q.scales.cpu().numpy(), q.rows, q.K)[rows]
    return codes, lin


def _check_split_rows(xq, muq, mu_dev, x, rows, rm, seed, offset, grad):
    """The split of x: the fp32 mean over every column, the whole of mu_bar
    (codes, scale bytes, decode scale), X_bar_R's decode scale, and X_bar_R's
    codes and scales on `rows`."""
    t_r, t_mu = (oracle.TAGS["d_r"], oracle.TAGS["mu_d"]) if grad else (oracle.TAGS["x_r"], oracle.TAGS["mu_x"])
    mu, XR, A = oracle.column_mean_and_residual_amax(x)
    K = x.shape[1]
    got = mu_dev.cpu().numpy()
    bad = np.flatnonzero(got.view(np.uint32) != mu.astype(np.float32).view(np.uint32))
    assert bad.size == 0, f"{bad.size} of {K} mean columns differ, first {bad[:5].tolist()}"
    g_enc, g_dec = F.tensor_scales(A)
    assert np.float32(xq.g_dec.item()).view(np.uint32) == np.float32(g_dec).view(np.uint32)
    codes, lin = _rows_of(xq, rows)
    for i, r in enumerate(rows):
        ref = oracle.nvfp4_quantize(XR[r:r + 1], rm, seed, offset + (int(r) * K) // 16, t_r, amax=A)
        assert np.array_equal(codes[i], ref.codes[0]), f"codes of row {r}"
        assert np.array_equal(lin[i], ref.scales[0]), f"scales of row {r}"
    assert_nvfp4_equal(muq, oracle.nvfp4_quantize(mu[None, :], rm, seed, offset, t_mu), "mu_bar")
    return mu


def _linear_rows(api, X, W, D, rm, seed, n_rows=48):
    """Forward and dgrad of one Averis linear at full size; checks on sampled rows."""
    l, m = X.shape
    n = W.shape[1]
    w_fwd, w_dgrad = _weights(api, W)
    wf, wd = to_oracle(w_fwd), to_oracle(w_dgrad)
    ws = api.workspace(l, max(m, n), max(m, n))
    xr, muq = api.NVFP4Tensor(l, m), api.NVFP4Tensor(1, m)
    Y = torch.empty((l, n), dtype=torch.bfloat16, device="cuda")
    api.averis_linear_fwd(X.cuda(), w_fwd, rm, seed, 0, Y, ws, save_xr=xr, save_mu=muq)
    # the same split once more with the fp32 mean requested: it must repeat
    # the forward's saved operands byte for byte
    mu_x = torch.empty(m, dtype=torch.float32, device="cuda")
    xr2, muq2 = api.NVFP4Tensor(l, m), api.NVFP4Tensor(1, m)
    api.averis_split_quant(X.cuda(), rm, seed, 0, False, mu_x, muq2, xr2, None, ws)
    dr, dmu = api.NVFP4Tensor(l, n), api.NVFP4Tensor(1, n)
    mu_d = torch.empty(n, dtype=torch.float32, device="cuda")
    api.averis_split_quant(D.cuda(), rm, seed + 1, 0, True, mu_d, dmu, dr, None, ws)
    dX = torch.empty((l, m), dtype=torch.bfloat16, device="cuda")
    api.averis_linear_dgrad(D.cuda(), w_dgrad, rm, seed + 1, 0, dX, ws)
    assert api.averis_check_status(ws) == 0
    for a, b in ((xr, xr2), (muq, muq2)):
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales) and torch.equal(a.g_dec, b.g_dec)
    rows = np.sort(np.random.default_rng(seed).choice(l, n_rows, replace=False))
    x, d = inputs.bf16_as_f32(X), inputs.bf16_as_f32(D)
    for q, mq, mu_dev, src, w_q, out, K, s, grad in ((xr, muq, mu_x, x, wf, Y, m, seed, False),
                                                    (dr, dmu, mu_d, d, wd, dX, n, seed + 1, True)):
        _check_split_rows(q, mq, mu_dev, src, rows, rm, s, 0, grad)
        a_rows = to_oracle(q)
        a_rows = oracle.NVFP4(a_rows.codes[rows], a_rows.scales[rows], a_rows.g_dec, len(rows), K)
        b = oracle.bias_row(to_oracle(mq), w_q)
        ref = oracle.gemm_reference(a_rows, w_q, b)
        check_bf16_output(out.float().cpu().numpy()[rows], ref, gemm_tolerance(a_rows, w_q, b, K))


def test_ffn_gate_up_full_size(api):
    """FFN gate/up: X [16384, 1024] -> W [1024, 6144], dY [16384, 6144], SR."""
    l, m, n = 16384, 1024, 6144
    X = inputs.to_bf16(inputs.spiked_activations(inputs.rng_for(2, 1), l, m, rank=4, s=(16.0, 8.0, 6.0, 4.0),
                                                 n_hot=m // 100))
    W = inputs.to_bf16(inputs.weight(inputs.rng_for(2, 2), m, n))
    D = inputs.to_bf16(inputs.output_gradient(inputs.rng_for(2, 3), l, n))
    _linear_rows(api, X, W, D, "sr", 41)


def test_ffn_down_full_size(api):
    """FFN down projection: the SwiGLU input [16384, 3072] -> W [3072, 1024], SR."""
    X, W, D = inputs.workload2_down()
    _linear_rows(api, X, W, D, "sr", 43)


@pytest.mark.parametrize("c", [0.0, 0.5, 2.0, 8.0, 32.0])
def test_mean_sweep_full_size(api, c):
    """The mean-strength sweep X [16384, 2048] -> W [2048, 2048] at every c, RNE
    (forward and dgrad)."""
    X, W = inputs.workload3(c)
    D = inputs.to_bf16(inputs.output_gradient(inputs.rng_for(3, 9), 16384, 2048))
    _linear_rows(api, X, W, D, "rne", 47, n_rows=32)


def test_stack_layer_shapes_at_32768_tokens(api):
    """The 28-layer stack's four linear shapes at l = 32768 tokens (QKV 1024 ->
    4096, o-proj 2048 -> 1024, gate/up 1024 -> 6144, down 3072 -> 1024): one
    forward + dgrad of each, checked on sampled rows."""
    l = 32768
    for k, (m, n) in enumerate(((1024, 4096), (2048, 1024), (1024, 6144), (3072, 1024))):
        rng = inputs.rng_for(6, k)
        X = inputs.to_bf16(inputs.swiglu_input(rng, l, m) if m == 3072 else
                           inputs.spiked_activations(rng, l, m, rank=4, s=(16.0, 8.0, 6.0, 4.0), n_hot=m // 100))
        W = inputs.to_bf16(inputs.weight(rng, m, n))
        D = inputs.to_bf16(inputs.output_gradient(rng, l, n))
        _linear_rows(api, X, W, D, "sr", 50 + k, n_rows=24)
