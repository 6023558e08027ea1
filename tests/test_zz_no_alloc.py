"""averis_split_quant_noalloc: the split quantizer for callers that cannot
allocate device memory (a plugin handed only its input and output pointers,
or latency-critical code that must not call cudaMalloc, which synchronizes
the device).  Its scratch is a fixed array inside the library.

The test calls it through the C ABI twice in a row and checks both results
against the workspace entry point averis_split_quant, bit for bit (the same
bar as every quantizer test).  This file is collected last, so a run that
stops at the first failure has already run every other test; it also passes
alone in a fresh process."""

import ctypes

import numpy as np
import pytest
import torch

from quantized_gemm_column_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _bytes(q):
    return (q.codes.cpu().numpy().copy(), q.scales.cpu().numpy().copy(),
            q.g_dec.cpu().numpy().view(np.uint32).copy())


@pytest.mark.parametrize("l,K,rm", [(8192, 1024, "sr"), (300, 192, "rne"), (4133, 640, "sr")])
def test_noalloc_matches_workspace_entry_point(api, l, K, rm):
    rng = inputs.rng_for(80, l + K)
    X = inputs.to_bf16(inputs.spiked_activations(rng, l, K, 2, (8.0, 4.0), n_hot=3)).cuda()

    # the existing entry point, with a workspace
    mu_ref = torch.empty(K, dtype=torch.float32, device="cuda")
    q_ref, m_ref = api.NVFP4Tensor(l, K), api.NVFP4Tensor(1, K)
    ws = api.workspace(l, K)
    api.averis_split_quant(X, rm, 42, 7, False, mu_ref, m_ref, q_ref, None, ws)
    assert api.averis_check_status(ws) == 0
    ref = (_bytes(q_ref), _bytes(m_ref), mu_ref.cpu().numpy().view(np.uint32))

    lib = api.load()
    for call in range(2):
        mu = torch.full((K,), -1.0, dtype=torch.float32, device="cuda")
        q, m = api.NVFP4Tensor(l, K), api.NVFP4Tensor(1, K)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = lib.averis_split_quant_noalloc(
            ctypes.c_void_p(X.data_ptr()), api.AVR_BF16, l, K, api._round(rm), 42, 7, 0,
            ctypes.c_void_p(mu.data_ptr()), ctypes.byref(m.struct()), ctypes.byref(q.struct()), None,
            ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == api.AVR_OK, api.status_string(st)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        got = (_bytes(q), _bytes(m), mu.cpu().numpy().view(np.uint32))
        for a, b in zip(got[0] + got[1], ref[0] + ref[1]):
            assert np.array_equal(a, b), f"call {call}: quantized bytes differ"
        assert np.array_equal(got[2], ref[2]), f"call {call}: mean differs"


def test_noalloc_rejects_sizes_beyond_its_scratch(api):
    lib = api.load()
    l, K = 32768, 4096            # partials alone are 6 MiB > 4 MiB
    q = api.avr_nvfp4(16, 16, 16, l, K)
    st = lib.averis_split_quant_noalloc(ctypes.c_void_p(16), api.AVR_BF16, l, K, api.AVR_RNE, 0, 0, 0,
                                        None, None, ctypes.byref(q), None, None, None)
    assert st == api.AVR_ERR_WORKSPACE_TOO_SMALL
