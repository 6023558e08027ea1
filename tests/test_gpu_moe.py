"""The MoE variant on the GPU: per-expert split operands bit-exact against the
oracle, the grouped GEMM's outputs within the fp32 accumulation bound, the
segment table's edge cases (empty experts, one-row experts, a buffer too
small for the counts)."""

import numpy as np
import pytest
import torch

import oracle
from oracle import nvfp4 as F
from quantized_gemm_column_b200 import inputs
from nvfp4_io import check_bf16_output, gemm_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _buffer(counts, K, seed, mean_scale=1.0, l_cap=None):
    """bf16 [l_cap, K]: expert e's rows carry their own planted mean; padding
    rows hold large values no statistic may see."""
    offs, L = oracle.moe_offsets(counts)
    l_cap = L if l_cap is None else l_cap
    rng = inputs.rng_for(90, seed)
    X = np.full((l_cap, K), 300.0)
    for e, (o, n) in enumerate(zip(offs, counts)):
        if n:
            X[o:o + n] = inputs.spiked_activations(rng, n, K, rank=2, s=(6.0, 3.0), n_hot=max(1, K // 100),
                                                   mean_scale=mean_scale * (1 + e % 3))
    t = inputs.to_bf16(X)
    return t, inputs.bf16_as_f32(t), offs


def _codes(q, rows):
    return q.codes.cpu().numpy()[rows]


def _seg_scales(q, o, n, K):
    """The scale bytes of rows o .. o + n rounded up to 128 (whole atoms)."""
    per_row = K // 16
    b0, b1 = o * per_row, (o + (n + 127) // 128 * 128) * per_row
    return q.scales.cpu().numpy()[b0:b1]


def _check_split(api, counts, K, rm, grad, seed=0):
    E = len(counts)
    Xt, x, offs = _buffer(counts, K, seed=len(counts) + K + seed)
    l_cap = Xt.shape[0]
    cnt = torch.tensor(counts, dtype=torch.int32, device="cuda")
    mu = torch.full((E, K), -7.0, dtype=torch.float32, device="cuda")
    mu_q, xr_q = api.NVFP4Group(E, K, E), api.NVFP4Group(l_cap, K, E)
    ws = api.moe_workspace(l_cap, K, 0, E)
    api.averis_moe_split_quant(Xt.cuda(), cnt, rm, 21 + seed, 5, grad, mu, mu_q, xr_q, ws)
    assert api.averis_check_status(ws) == 0
    ref = oracle.moe_split_quant(x, counts, rm, seed=21 + seed, offset=5, grad=grad)
    mu_h = mu.cpu().numpy()
    mu_lin = F.unswizzle_scales(mu_q.scales.cpu().numpy(), E, K)
    for e, (o, n) in enumerate(zip(offs, counts)):
        if n == 0:
            continue
        r = ref[e]
        assert np.array_equal(mu_h[e].view(np.uint32), r["mu"].view(np.uint32)), f"mu of expert {e}"
        assert np.array_equal(_codes(xr_q, slice(o, o + n)), r["xr_q"].codes), f"codes of expert {e}"
        assert np.array_equal(_seg_scales(xr_q, o, n, K), F.swizzle_scales(r["xr_q"].scales, n, K)), \
            f"scales of expert {e}"
        assert np.float32(xr_q.g_dec[e].item()).view(np.uint32) == np.float32(r["xr_q"].g_dec).view(np.uint32)
        assert np.array_equal(mu_q.codes.cpu().numpy()[e], r["mu_q"].codes[0]), f"mu_bar codes of expert {e}"
        assert np.array_equal(mu_lin[e], r["mu_q"].scales[0]), f"mu_bar scales of expert {e}"
        assert np.float32(mu_q.g_dec[e].item()).view(np.uint32) == np.float32(r["mu_q"].g_dec).view(np.uint32)
        # padding rows of the segment: zero codes
        pad = slice(o + n, o + (n + 127) // 128 * 128)
        assert not _codes(xr_q, pad).any()


@pytest.mark.parametrize("counts,K", [([300, 0, 129, 1, 512], 256), ([128], 192), ([5, 700, 0, 0, 33], 640),
                                      ([2100, 17], 128)])
@pytest.mark.parametrize("rm", ["rne", "sr"])
def test_moe_split_bit_exact(api, counts, K, rm):
    _check_split(api, counts, K, rm, grad=False)


def test_moe_split_grad_tags(api):
    _check_split(api, [260, 40, 0, 129], 256, "sr", grad=True, seed=3)


def _weights(api, E, m, n, seed):
    rng = inputs.rng_for(91, seed)
    W = np.stack([inputs.weight(rng, m, n) for _ in range(E)])
    Wt = inputs.to_bf16(W)
    w_fwd, w_dgrad = api.NVFP4Group(E * n, m, E), api.NVFP4Group(E * m, n, E)
    ws = api.workspace(m, n, n)
    api.averis_moe_quant_weights(Wt.cuda(), w_fwd, w_dgrad, ws)
    assert api.averis_check_status(ws) == 0
    w = inputs.bf16_as_f32(Wt)
    refs = oracle.moe_quant_weights([w[e] for e in range(E)])
    return w_fwd, w_dgrad, refs


def _slice_nvfp4(t, e, rows, K):
    """Expert e's [rows, K] slice of a stacked NVFP4 group, as an oracle tensor."""
    codes = t.codes.cpu().numpy()[e * rows:(e + 1) * rows]
    per = (rows + 127) // 128 * 128 * (K // 16)
    flat = t.scales.cpu().numpy()[e * per:(e + 1) * per]
    return oracle.NVFP4(codes, F.unswizzle_scales(flat, rows, K), np.float32(t.g_dec[e].item()), rows, K)


def test_moe_weight_quant_bit_exact(api):
    E, m, n = 3, 256, 384
    w_fwd, w_dgrad, refs = _weights(api, E, m, n, 0)
    for e in range(E):
        for got, want in ((_slice_nvfp4(w_fwd, e, n, m), refs[e][0]), (_slice_nvfp4(w_dgrad, e, m, n), refs[e][1])):
            assert np.array_equal(got.codes, want.codes) and np.array_equal(got.scales, want.scales)
            assert np.float32(got.g_dec) == np.float32(want.g_dec)


@pytest.mark.parametrize("counts", [[200, 0, 129, 64], [1, 300]])
def test_moe_forward_and_dgrad_match_oracle(api, counts):
    E, m, n = len(counts), 256, 384
    w_fwd, w_dgrad, refs = _weights(api, E, m, n, 1)
    Xt, x, offs = _buffer(counts, m, seed=11)
    l_cap = Xt.shape[0]
    cnt = torch.tensor(counts, dtype=torch.int32, device="cuda")
    ws = api.moe_workspace(l_cap, max(m, n), max(m, n), E)
    Y = torch.empty((l_cap, n), dtype=torch.bfloat16, device="cuda")
    api.averis_moe_linear_fwd(Xt.cuda(), cnt, w_fwd, "sr", 8, 2, Y, ws)
    assert api.averis_check_status(ws) == 0
    Yref, split = oracle.moe_linear_reference(x, counts, [r[0] for r in refs], "sr", seed=8, offset=2)
    Yh = Y.float().cpu().numpy()
    for e, (o, c) in enumerate(zip(offs, counts)):
        if c == 0:
            continue
        b = oracle.bias_row(split[e]["mu_q"], refs[e][0])
        check_bf16_output(Yh[o:o + c], Yref[e], gemm_tolerance(split[e]["xr_q"], refs[e][0], b, m))
    # dgrad: D [l_cap, n] in the same segments
    rng = inputs.rng_for(92, 0)
    Dn = np.zeros((l_cap, n))
    for o, c in zip(offs, counts):
        Dn[o:o + c] = inputs.output_gradient(rng, c, n) if c else 0.0
    Dt = inputs.to_bf16(Dn)
    dX = torch.empty((l_cap, m), dtype=torch.float32, device="cuda")
    api.averis_moe_linear_dgrad(Dt.cuda(), cnt, w_dgrad, "sr", 9, 3, dX, ws)
    assert api.averis_check_status(ws) == 0
    dref, dsplit = oracle.moe_linear_reference(inputs.bf16_as_f32(Dt), counts, [r[1] for r in refs], "sr", seed=9,
                                               offset=3, grad=True)
    dh = dX.cpu().numpy()
    for e, (o, c) in enumerate(zip(offs, counts)):
        if c == 0:
            continue
        b = oracle.bias_row(dsplit[e]["mu_q"], refs[e][1])
        tol = gemm_tolerance(dsplit[e]["xr_q"], refs[e][1], b, n)
        assert np.all(np.abs(dh[o:o + c] - dref[e]) <= tol + 2.0 ** -22 * np.abs(dref[e]))


def test_moe_counts_beyond_the_buffer_latch_an_error(api):
    counts, K = [200, 300], 128
    l_cap = 384                                  # needs 256 + 384 = 640 rows
    X = torch.zeros((l_cap, K), dtype=torch.bfloat16, device="cuda")
    cnt = torch.tensor(counts, dtype=torch.int32, device="cuda")
    xr_q = api.NVFP4Group(l_cap, K, 2)
    ws = api.moe_workspace(l_cap, K, 0, 2)
    api.averis_moe_split_quant(X, cnt, "rne", 0, 0, False, None, None, xr_q, ws)
    assert api.averis_check_status(ws) == api.AVR_ERR_INVALID_ARG
    # the workspace is usable again once the status is read
    ok = torch.tensor([200, 100], dtype=torch.int32, device="cuda")
    api.averis_moe_split_quant(X, ok, "rne", 0, 0, False, None, None, xr_q, ws)
    assert api.averis_check_status(ws) == 0


def test_moe_layer_size_sampled(api):
    """64 experts, hidden 2048 -> 1024 per expert, 4096 tokens routed to 8
    experts each (32768 rows, skewed counts): every expert's operands are
    produced; three experts (the largest, a small one, a middle one) are
    checked bit for bit and on 64 sampled output rows each."""
    E, m, n = 64, 2048, 1024
    counts = inputs.moe_counts(E, tokens=4096, top_k=8, seed=0)
    Xt, x, offs = _buffer(counts, m, seed=5)
    l_cap = Xt.shape[0]
    w_fwd, _, refs = _weights(api, E, m, n, 2)
    cnt = torch.tensor(counts, dtype=torch.int32, device="cuda")
    ws = api.moe_workspace(l_cap, m, n, E)
    Y = torch.empty((l_cap, n), dtype=torch.bfloat16, device="cuda")
    api.averis_moe_linear_fwd(Xt.cuda(), cnt, w_fwd, "sr", 31, 0, Y, ws)
    assert api.averis_check_status(ws) == 0
    nz = [e for e in range(E) if counts[e] > 0]
    picks = sorted({max(nz, key=lambda e: counts[e]), min(nz, key=lambda e: counts[e]), nz[len(nz) // 2]})
    Yref, split = oracle.moe_linear_reference(x, counts, [r[0] for r in refs], "sr", seed=31, offset=0,
                                              experts=picks)
    Yh = Y.float().cpu().numpy()
    rng = np.random.default_rng(0)
    for e in picks:
        o, c = offs[e], counts[e]
        rows = np.sort(rng.choice(c, min(c, 64), replace=False))
        b = oracle.bias_row(split[e]["mu_q"], refs[e][0])
        check_bf16_output(Yh[o + rows], Yref[e][rows], gemm_tolerance(split[e]["xr_q"], refs[e][0], b, m)[rows])
