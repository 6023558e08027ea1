"""The tcgen05 block-scaled FP4 GEMM against the oracle's fp64 product."""

import numpy as np
import pytest
import torch

import oracle
from oracle import nvfp4 as F
from nvfp4_io import from_oracle, gemm_tolerance, check_bf16_output

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from quantized_gemm_column_b200 import api as a
    a.load()
    return a


def _rand_q(rng, rows, K, scale_lo=0x28, scale_hi=0x48, g_dec=1.0):
    codes = rng.integers(0, 16, (rows, K), dtype=np.uint8)
    sc = rng.integers(scale_lo, scale_hi, (rows, K // 16)).astype(np.uint8)
    return F.NVFP4(F.pack_codes(codes), sc, np.float32(g_dec), rows, K)


def _gemm(api, a_q, b_q, bias=None, out=torch.float32):
    a, b = from_oracle(a_q, api), from_oracle(b_q, api)
    Y = torch.empty((a_q.rows, b_q.rows), dtype=out, device="cuda")
    ws = api.workspace(0, a_q.K)
    bd = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).cuda()
    api.nvfp4_gemm(a, b, bd, Y, ws)
    assert api.averis_check_status(ws) == 0
    return Y.float().cpu().numpy().astype(np.float64)


# bf16 outputs with K a multiple of 256 run on a CTA-pair kernel (the
# short-contraction one for K <= 1024), the others on the one-CTA kernel: the
# probes run at K = 64 and 256 to cover both.
KERNELS = [(torch.float32, 64), (torch.bfloat16, 64), (torch.bfloat16, 256)]


@pytest.mark.parametrize("out,K", KERNELS)
def test_scale_layout_probe_A(api, out, K):
    """A has every code 1.0 and random E4M3 scales; row j of B is 1.0 on the
    16-block (j mod K/16) of K and 0 elsewhere, with scale 1.  Then
    Y[r, j] = 16 * scale_A[r, j mod K/16] exactly: each output names one scale
    of A, so a wrong tensor-memory scale layout cannot pass."""
    rng = np.random.default_rng(0)
    M, N = 256, 64
    nb = K // 16
    a = F.NVFP4(F.pack_codes(np.full((M, K), 2, np.uint8)),
                rng.integers(0x20, 0x58, (M, K // 16)).astype(np.uint8), np.float32(1.0), M, K)
    bc = np.zeros((N, K), np.uint8)
    for j in range(N):
        bc[j, 16 * (j % nb):16 * (j % nb) + 16] = 2
    b = F.NVFP4(F.pack_codes(bc), np.full((N, K // 16), 0x38, np.uint8), np.float32(1.0), N, K)
    Y = _gemm(api, a, b, out=out)
    want = 16.0 * oracle.e4m3_value(a.scales).astype(np.float64)[:, np.arange(N) % nb]
    assert np.array_equal(Y, want)


@pytest.mark.parametrize("out,K", KERNELS)
def test_scale_layout_probe_B(api, out, K):
    """The same with the roles swapped: Y[i, j] = 16 * scale_B[j, i mod K/16]
    for N = 256 (two 128-row scale atoms of B)."""
    rng = np.random.default_rng(1)
    M, N = 256, 256
    nb = K // 16
    ac = np.zeros((M, K), np.uint8)
    for i in range(M):
        ac[i, 16 * (i % nb):16 * (i % nb) + 16] = 2
    a = F.NVFP4(F.pack_codes(ac), np.full((M, K // 16), 0x38, np.uint8), np.float32(1.0), M, K)
    b = F.NVFP4(F.pack_codes(np.full((N, K), 2, np.uint8)),
                rng.integers(0x20, 0x58, (N, K // 16)).astype(np.uint8), np.float32(1.0), N, K)
    Y = _gemm(api, a, b, out=out)
    want = 16.0 * oracle.e4m3_value(b.scales).astype(np.float64)[:, np.arange(M) % nb].T
    assert np.array_equal(Y, want)


@pytest.mark.parametrize("out,K", KERNELS)
def test_nibble_order_probe(api, out, K):
    """Row j of B is one-hot at element j: Y[r, j] = value of A's element
    (r, j), so a swapped nibble order shows at every odd j."""
    rng = np.random.default_rng(2)
    M = 256
    ac = rng.integers(0, 16, (M, K)).astype(np.uint8)
    a = F.NVFP4(F.pack_codes(ac), np.full((M, K // 16), 0x38, np.uint8), np.float32(1.0), M, K)
    bc = np.zeros((K, K), np.uint8)
    bc[np.arange(K), np.arange(K)] = 2
    b = F.NVFP4(F.pack_codes(bc), np.full((K, K // 16), 0x38, np.uint8), np.float32(1.0), K, K)
    Y = _gemm(api, a, b, out=out)
    assert np.array_equal(Y, oracle.e2m1_value(ac).astype(np.float64))


@pytest.mark.parametrize("out,K", [(torch.float32, 640), (torch.bfloat16, 640), (torch.bfloat16, 1280),
                                   (torch.bfloat16, 2304)])
def test_k_stage_and_kblock_order(api, out, K):
    """Each 64-element k-block of A holds one constant per row and row j of B
    selects k-block j mod K/64, so Y[:, j] = 64 * that constant: a wrong k
    advance inside a stage or across stages changes the products.  K = 640
    leaves the one-CTA kernel a partial last stage; 1280 gives the pair kernel
    a last stage of one 256-deep chunk with all of B's scales resident, 2304
    the same with B's scales streamed.  All values are exact in fp32 and bf16."""
    rng = np.random.default_rng(3)
    M = 256
    nkb = K // 64
    ac = np.zeros((M, K), np.uint8)
    for kb in range(nkb):
        ac[:, 64 * kb:64 * kb + 64] = rng.integers(1, 8, (M, 1))
    a = F.NVFP4(F.pack_codes(ac), np.full((M, K // 16), 0x38, np.uint8), np.float32(1.0), M, K)
    N = 64
    bc = np.zeros((N, K), np.uint8)
    for j in range(N):
        kb = (j * 7) % nkb
        bc[j, 64 * kb:64 * kb + 64] = 2
    b = F.NVFP4(F.pack_codes(bc), np.full((N, K // 16), 0x38, np.uint8), np.float32(1.0), N, K)
    Y = _gemm(api, a, b, out=out)
    assert np.array_equal(Y, oracle.gemm_reference(a, b))


@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (256, 256, 256), (300, 192, 320),
                                   (1024, 512, 1024), (129, 64, 2048)])
def test_random_gemm_fp32_out(api, M, N, K):
    rng = np.random.default_rng(M + N + K)
    a = _rand_q(rng, M, K, g_dec=0.013)
    b = _rand_q(rng, N, K, g_dec=0.002)
    bias = rng.standard_normal(N)
    Y = _gemm(api, a, b, bias)
    ref = oracle.gemm_reference(a, b, bias)
    rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    assert rel <= 1e-5, rel


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (300, 192, 320), (2048, 1024, 4096)])
def test_random_gemm_bf16_out(api, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    a = _rand_q(rng, M, K, g_dec=0.01)
    b = _rand_q(rng, N, K, g_dec=0.003)
    bias = rng.standard_normal(N) * 0.1
    Y = _gemm(api, a, b, bias, out=torch.bfloat16)
    ref = oracle.gemm_reference(a, b, bias)
    check_bf16_output(Y, ref, gemm_tolerance(a, b, bias, K))


@pytest.mark.parametrize("M,N,K", [(1000, 704, 512), (4224, 2112, 768), (8192, 1280, 1024)])
def test_short_pair_kernel_ragged(api, M, N, K):
    """The short-contraction pair kernel (bf16 out, K <= 1024): M and N not
    multiples of the 256 x 256 pair tile (the last row block leaves the second
    CTA of its pair with no rows, the last column block half empty), and runs
    of several tiles per pair that change column block (B's resident rows and
    scales reloaded).  Every output is compared."""
    rng = np.random.default_rng(M + 3 * N + K)
    a = _rand_q(rng, M, K, g_dec=0.01)
    b = _rand_q(rng, N, K, g_dec=0.003)
    bias = rng.standard_normal(N) * 0.1
    Y = _gemm(api, a, b, bias, out=torch.bfloat16)
    ref = oracle.gemm_reference(a, b, bias)
    check_bf16_output(Y, ref, gemm_tolerance(a, b, bias, K))


def test_quantized_operands_from_oracle(api):
    """Operands produced by the oracle's quantizer (realistic scale mix)."""
    rng = np.random.default_rng(4)
    X = (rng.standard_normal((512, 1024)) * 2 + 1).astype(np.float32)
    W = rng.standard_normal((768, 1024)).astype(np.float32)
    a = oracle.nvfp4_quantize(X, "sr", seed=3, tag=1)
    b = oracle.nvfp4_quantize(W, "rne")
    Y = _gemm(api, a, b)
    ref = oracle.gemm_reference(a, b)
    assert np.linalg.norm(Y - ref) / np.linalg.norm(ref) <= 1e-5


def _gemm_sampled(api, a_q, b_q, cols, bias=None, out=torch.float32):
    """Run the GEMM and return its output and the oracle's product on the
    columns `cols` (rows of B) only."""
    Y = _gemm(api, a_q, b_q, bias, out=out)
    b_sub = oracle.NVFP4(b_q.codes[cols], b_q.scales[cols], b_q.g_dec, len(cols), b_q.K)
    ref = oracle.gemm_reference(a_q, b_sub, None if bias is None else np.asarray(bias)[cols])
    return Y[:, cols], ref, b_sub


@pytest.mark.parametrize("K", [256, 1280, 1536, 2112, 2048, 2304])
def test_resident_b_scales_across_column_blocks_bf16(api, K):
    """Many more tiles than CTAs (or CTA pairs), so a run of tiles changes
    column block (B's resident scales are reloaded) and shares it between
    tiles.  K = 256 runs the short-contraction pair kernel (B's rows and
    scales resident per column block); the pair kernel keeps all of B's
    scales resident at K = 1280 and 1536 and streams them beyond (2048, 2304:
    a last stage of one chunk); K = 2112 runs the one-CTA kernel (five of
    nine stages resident, a partial last stage)."""
    rng = np.random.default_rng(K)
    M, N = 512, 256 * 160
    a = _rand_q(rng, M, K, g_dec=0.01)
    b = _rand_q(rng, N, K, g_dec=0.003)
    bias = rng.standard_normal(N) * 0.1
    cols = np.sort(rng.choice(N, 640, replace=False))
    Y, ref, b_sub = _gemm_sampled(api, a, b, cols, bias, out=torch.bfloat16)
    check_bf16_output(Y, ref, gemm_tolerance(a, b_sub, np.asarray(bias)[cols], K))


@pytest.mark.parametrize("K", [3072, 3264])
def test_resident_b_scales_across_column_blocks_fp32(api, K):
    """The fp32-output tiles (128 columns) keep up to twelve stages of B's
    scales resident: K = 3072 is all resident, 3264 leaves a partial
    thirteenth stage streamed."""
    rng = np.random.default_rng(K + 1)
    M, N = 256, 128 * 320
    a = _rand_q(rng, M, K, g_dec=0.013)
    b = _rand_q(rng, N, K, g_dec=0.002)
    cols = np.sort(rng.choice(N, 512, replace=False))
    Y, ref, _ = _gemm_sampled(api, a, b, cols)
    rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    assert rel <= 1e-5, rel
