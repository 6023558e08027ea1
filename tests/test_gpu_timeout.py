"""Failure detection on the device, without a fault: a wait that runs out
records AVR_ERR_DEVICE_TIMEOUT in the workspace status word, its kernel
returns with no copy in flight, the host reads the code, and the next call on
the same workspace is clean.

The wait made to run out is the one-kernel split's grid barrier, where a CTA
waits for the other CTAs (not for its own copies).  A 1 ns bound makes every
CTA that reaches a barrier before the last one give up at its first poll;
the input is cut so that CTAs hold 3 or 4 units of work, so the early ones
always wait."""

import pytest
import torch

from quantized_gemm_column_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _operands(api, l, K):
    return (torch.empty(K, dtype=torch.float32, device="cuda"), api.NVFP4Tensor(1, K), api.NVFP4Tensor(l, K))


def _same(a, b):
    return all(torch.equal(x, y) for x, y in ((a.codes, b.codes), (a.scales, b.scales), (a.g_dec, b.g_dec)))


def test_grid_barrier_timeout_is_reported_and_the_workspace_recovers(api):
    l, K = 8192 + 256, 4096            # 33 chunks x 32 column tiles = 1056 units over the resident CTAs
    rng = inputs.rng_for(80, 0)
    X = inputs.to_bf16(inputs.spiked_activations(rng, l, K, 2, (8.0, 4.0), n_hot=4)).cuda()
    ws = api.workspace(l, K)
    mu, muq, xr = _operands(api, l, K)
    api.averis_set_wait_limit(ws, 1)
    api.averis_split_quant_fused(X, "sr", 3, 0, False, mu, muq, xr, ws)
    assert api.averis_check_status(ws) == api.AVR_ERR_DEVICE_TIMEOUT
    # check_status cleared the status block (barrier words, and the bound back
    # to its default): the same workspace gives a clean call, bit for bit the
    # two-kernel split's result
    api.averis_split_quant_fused(X, "sr", 3, 0, False, mu, muq, xr, ws)
    assert api.averis_check_status(ws) == 0
    mu2, muq2, xr2 = _operands(api, l, K)
    ws2 = api.workspace(l, K)
    api.averis_split_quant(X, "sr", 3, 0, False, mu2, muq2, xr2, None, ws2)
    assert api.averis_check_status(ws2) == 0
    assert torch.equal(mu.view(torch.int32), mu2.view(torch.int32))
    assert _same(muq, muq2) and _same(xr, xr2)


def test_a_generous_bound_changes_nothing(api):
    """A 10 s bound, then the default restored with 0: both calls are clean and
    equal the two-kernel split."""
    l, K = 4096, 1024
    rng = inputs.rng_for(80, 1)
    X = inputs.to_bf16(inputs.spiked_activations(rng, l, K, 2, (8.0, 4.0), n_hot=4)).cuda()
    ws = api.workspace(l, K)
    ref = _operands(api, l, K)
    api.averis_split_quant(X, "rne", 0, 0, True, ref[0], ref[1], ref[2], None, api.workspace(l, K))
    for limit in (10_000_000_000, 0):
        api.averis_set_wait_limit(ws, limit)
        out = _operands(api, l, K)
        api.averis_split_quant_fused(X, "rne", 0, 0, True, *out, ws)
        assert api.averis_check_status(ws) == 0
        assert torch.equal(out[0].view(torch.int32), ref[0].view(torch.int32))
        assert _same(out[1], ref[1]) and _same(out[2], ref[2])


def test_set_wait_limit_validation(api):
    ws = api.workspace(256, 128)
    with pytest.raises(api.AverisError):
        api.averis_set_wait_limit(ws[:64], 5)          # smaller than the status block
    with pytest.raises(api.AverisError):
        api.averis_set_wait_limit(ws[8:], 5)           # not 256-byte aligned
