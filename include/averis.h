/*
 * averis.h -- C ABI of libaveris: the Averis mean-residual split NVFP4
 * linear layer (forward and dgrad) on NVIDIA B200 (sm_100a).
 *
 * Source of the method: "The Curse and Blessing of Mean Bias in
 * FP4-Quantized LLM Training" (Cao, Huang et al.).  Passages cited below:
 *   [R2.1]  Lighthouse review page, section 二 2.1 "核心 Insight": column mean
 *           mu_X = (1/l) 1^T X of X in R^{l x m} (l tokens, m features).
 *   [RAv]   same page, section 二 "Averis 方法": forward
 *           Y_hat = 1 (mu_bar_X W_bar) + X_bar_R W_bar with mu_bar_X = Q_4(mu_X),
 *           X_bar_R = Q_4(X - 1 mu_X); backward
 *           dL/dX_hat = 1 (mu_bar_D W_bar^T) + D_bar_R W_bar^T; cost: two
 *           reductions and two subtractions.
 *   [R3.1]  same page, section 三 3.1: W4A4G4, E2M1 NVFP4, stochastic
 *           rounding by default; vanilla FP4 as the comparison.
 *   [Abs]   arXiv abstract page: mean-residual splitting with reductions and
 *           elementwise subtractions before FP4 quantization; 2.20%
 *           end-to-end overhead over vanilla NVFP4.
 *   [GS2]   gist.science technical summary, section 2 "Il Metodo Proposto:
 *           Averis": X_R = X - 1 mu_X^T, mean and residual quantized
 *           separately, forward and backward recombined.
 *   [R7.2]  Lighthouse review page, section 七 "对我们的启示", under "实践建议",
 *           item 2: monitor the mean-energy ratio
 *           R = ||mu||_2 / sqrt(E||x||^2 / N) as a training-stability signal.
 *
 * Readings where the pages are silent (the same readings the CPU oracle
 * follows): 16-element blocks along the contraction axis with unsigned E4M3
 * block scales and one FP32 per-tensor decode scale g_dec = amax / 2688;
 * the fixed fp32 order of the mean (256-row chunks summed row by row, then
 * chunk partials in chunk order, mu = S / l); Philox4x32-10 random bits,
 * 16 per element, for stochastic rounding; weights always round to nearest
 * even.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers to caller-owned memory; the
 *     library never allocates and never frees.  Row-major, contiguous.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronize, except averis_check_status.
 *   - Validation happens on the host before any launch; a rejected call
 *     launches nothing and returns a non-zero avr_status.  Launch failures
 *     return AVR_ERR_CUDA.
 *   - Conditions found on the device (a bounded wait that expired, a
 *     non-finite mean or amax) are latched in the workspace status word and
 *     returned by averis_check_status.  Outputs of such a call are undefined.
 *   - `ws` is a device workspace of at least averis_workspace_size(l, K, N)
 *     bytes (256-byte aligned).  It must be zero-filled before its first use
 *     (averis_workspace_init); every call that completes leaves it reusable.
 *     One workspace must not be used by two calls that may run concurrently.
 *   - Shape rules: K (the contraction size) > 0 and K % 64 == 0; N % 64 == 0;
 *     l (tokens / rows) >= 0, any value (l = 0 is a no-op returning AVR_OK, and
 *     the tensor pointers may then be NULL);
 *     every pointer 16-byte aligned; l, K, N < 2^31.
 */
#ifndef AVERIS_H_
#define AVERIS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* avr_stream; /* same type as cudaStream_t */

typedef enum {
  AVR_OK = 0,
  AVR_ERR_INVALID_ARG = 1,         /* null pointer, unknown enum value */
  AVR_ERR_UNSUPPORTED_SHAPE = 2,   /* K % 64, N % 64, sizes out of range */
  AVR_ERR_MISALIGNED = 3,          /* a pointer not 16-byte aligned */
  AVR_ERR_WORKSPACE_TOO_SMALL = 4,
  AVR_ERR_CUDA = 5,                /* a CUDA runtime/driver call failed */
  AVR_ERR_DEVICE_TIMEOUT = 6,      /* a device-side bounded wait expired */
  AVR_ERR_NONFINITE = 7,           /* the input held NaN/Inf (mean or amax not finite) */
  AVR_ERR_NO_DEVICE = 8            /* current device is not an sm_100 GPU */
} avr_status;

typedef enum { AVR_F32 = 0, AVR_BF16 = 1 } avr_dtype;
typedef enum { AVR_RNE = 0, AVR_SR = 1 } avr_round;

/* An NVFP4 tensor T [rows, K] quantized along K ([R3.1] "E2M1 NVFP4").
 *   codes  : rows * K/2 bytes; element 2k of a row in the low nibble of
 *            byte k, element 2k+1 in the high nibble; E2M1 code = sign<<3 |
 *            magnitude index into {0, .5, 1, 1.5, 2, 3, 4, 6}.
 *   scales : avr_nvfp4_scales_bytes(rows, K) bytes of unsigned E4M3 block
 *            scales in the tcgen05 block-scaling layout: 512-byte atoms of
 *            128 rows x 4 scales, atom (r/128, c/4) at index
 *            (r/128) * (K/64) + c/4, and inside an atom the scale of (r, c)
 *            at byte 16*(r%32) + 4*((r%128)/32) + c%4.  Rows past `rows` up
 *            to the next multiple of 128 are zero.
 *   g_dec  : one fp32 per-tensor decode scale.
 * value(r, k) = e2m1(code) * e4m3(scale(r, k/16)) * g_dec. */
typedef struct {
  uint8_t* codes;
  uint8_t* scales;
  float* g_dec;
  int64_t rows;
  int64_t K;
} avr_nvfp4;

/* Bytes of the scale array of an NVFP4 tensor [rows, K]. */
size_t avr_nvfp4_scales_bytes(int64_t rows, int64_t K);

/* Workspace bytes that cover every call below for l rows, contraction K and
 * N output columns (N may be 0 for calls without a GEMM). */
size_t averis_workspace_size(int64_t l, int64_t K, int64_t N);

/* Zero-fill a workspace before its first use (stream ordered). */
avr_status averis_workspace_init(void* ws, size_t ws_bytes, avr_stream stream);

/* Synchronize `stream`, return the first device-side error latched in the
 * workspace status word since the last check (AVR_OK if none) and clear it.
 * After an error the whole 256-byte status block is cleared (the status
 * word, the one-kernel split's grid-barrier words, which a kernel that gave
 * up may have left part-counted, and the wait limit below), so the workspace
 * is ready for the next call. */
avr_status averis_check_status(void* ws, avr_stream stream);

/* Bound, in nanoseconds, of the waits in which a CTA waits for other CTAs
 * (the grid-wide barriers of averis_split_quant_fused); 0 restores the
 * default of 2 s.  Written in stream order into the workspace's status block
 * (a zero-filled workspace has the default); averis_check_status resets it
 * to the default after an error.  A wait that runs out records
 * AVR_ERR_DEVICE_TIMEOUT and its kernel returns with no copy in flight; the
 * waits for a CTA's own copies keep the 2 s bound.  This is failure
 * detection (a grid that cannot be co-resident, a stuck CTA), not a tuning
 * knob.  Errors: AVR_ERR_INVALID_ARG (null ws), AVR_ERR_MISALIGNED (ws not
 * 256-byte aligned), AVR_ERR_WORKSPACE_TOO_SMALL (ws_bytes < 256),
 * AVR_ERR_NO_DEVICE. */
avr_status averis_set_wait_limit(void* ws, size_t ws_bytes, uint64_t limit_ns, avr_stream stream);

/* Static description of a status code. */
const char* averis_status_string(avr_status status);

/* -------------------------------------------------------------------------
 * Split quantization [R2.1], [RAv], [GS2]
 * ------------------------------------------------------------------------- */

/* Mean-residual split and quantization of X [l, K] (K = the feature axis).
 *   mu      [K] fp32 out : column mean in the fixed order (nullable).
 *   mu_q    out          : Q_4(mu) as a 1 x K NVFP4 tensor (nullable).
 *   xr_q    out          : Q_4(X - 1 mu), l x K.
 *   xr_debug [l, K] fp32 : X_R itself (nullable; for tests).
 *   grad = 0 for activations X (random-stream tags 1 and 2), 1 for output
 *   gradients D (tags 3 and 4).  rm selects RNE or Philox SR; the stream of
 *   element e (row-major index) is keyed by `seed` and counted from
 *   `offset` + e/16.  Launches 2 kernels (column reduce, split-quantize). */
avr_status averis_split_quant(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                              uint64_t seed, uint64_t offset, int grad, float* mu,
                              const avr_nvfp4* mu_q, const avr_nvfp4* xr_q, float* xr_debug,
                              void* ws, size_t ws_bytes, avr_stream stream);

/* Mean-energy ratio monitor [R7.2]:
 *   R = ||mu_X||_2 / sqrt(E_i ||x_i||^2 / m),
 * mu_X the column mean of X [l, K] (m = K features, l >= 1 tokens), E_i the
 * average over the l rows.  The pages leave N in the formula undefined; it
 * is read as the feature count m, so that R = sqrt(m) when every row equals
 * the mean and R = 0 when the columns average to zero.
 *   mu [K] fp32 out : the column mean in the fixed order of averis_split_quant
 *                     (nullable; the workspace holds it otherwise).
 *   R  fp32 device scalar out.
 * mu in fp32 as the split computes it; column sums of squares in fp32 (fma,
 * rows of a 256-row chunk in order, chunk partials in chunk order); the two
 * norms in fp64.  Non-finite X latches AVR_ERR_NONFINITE.  l == 0 is
 * rejected with AVR_ERR_UNSUPPORTED_SHAPE (R is 0/0).  Launches 2 kernels
 * (column reduce with sums of squares, one-CTA ratio). */
avr_status averis_mean_energy_ratio(const void* X, avr_dtype xt, int64_t l, int64_t K, float* mu,
                                    float* R, void* ws, size_t ws_bytes, avr_stream stream);

/* averis_split_quant as one persistent kernel (the "fewer passes" variant):
 * the input is read from memory once, each CTA keeping its last 256 x 128
 * unit in shared memory, with grid-wide barriers between the reduce, the fold
 * and the quantization instead of a second launch.  Same arguments and the
 * same output bits as averis_split_quant (no X_R debug output).  On B200 the
 * two-kernel chain is faster at the benchmark's sizes (its second read of the
 * input comes from L2), so the linear entry points use that chain.  Every CTA
 * of the grid must be resident at once: the call uses at most two CTAs per SM
 * and no other work may hold the GPU's SMs meanwhile, else its barriers time
 * out (AVR_ERR_DEVICE_TIMEOUT).  Launches 1 kernel (2 when l % 128 != 0). */
avr_status averis_split_quant_fused(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                                    uint64_t seed, uint64_t offset, int grad, float* mu,
                                    const avr_nvfp4* mu_q, const avr_nvfp4* xr_q, void* ws,
                                    size_t ws_bytes, avr_stream stream);

/* averis_split_quant for callers that cannot allocate.  The paper has no
 * counterpart to this entry point; it exists for the library's users.
 *
 * Some callers have no device memory to give the library: a plugin that
 * receives only its input and output pointers from a framework that owns
 * every allocation, or latency-critical code that must not call
 * cudaMalloc/cudaFree (they synchronize the device).  This call takes no
 * workspace: the column reduce's scratch lives in a fixed 4 MiB array inside
 * the library, which every GPU that loads the library holds until the
 * process exits.  It computes exactly what averis_split_quant computes, with
 * the same arguments except `ws`/`ws_bytes`.
 *   Limit: 3 * ceil(l/256) * K * 4 bytes of chunk partials plus K * 4 bytes
 *   for the mean and 48.25 KiB of bookkeeping must fit in 4 MiB, so K can be
 *   at most 10624 for l = 8192 and at most 2688 for l = 32768; larger sizes
 *   return AVR_ERR_WORKSPACE_TOO_SMALL without launching anything.
 *   device_status: nullable device pointer to a uint32 the caller has set to
 *   0; the first device-side error of the call (AVR_ERR_NONFINITE,
 *   AVR_ERR_DEVICE_TIMEOUT) is stored there.
 *   The first call on each device looks up the array's device address (with
 *   that device current) and keeps it for as long as the device's context
 *   lives; make that first call before any stream capture.  A
 *   cudaDeviceReset ends the context, and with it the array: the next call
 *   sees a new context and looks the address up again, so it, too, belongs
 *   before any capture.  Every call shares the array, so calls that may
 *   overlap on the GPU (other streams, other threads) race: issue them in one
 *   stream order.  Each call clears the parts of the array that must start
 *   at zero.  Validation is averis_split_quant's (the same codes for the same
 *   bad arguments), and a host without an sm_100 device gets
 *   AVR_ERR_NO_DEVICE. */
avr_status averis_split_quant_noalloc(const void* X, avr_dtype xt, int64_t l, int64_t K,
                                      avr_round rm, uint64_t seed, uint64_t offset, int grad,
                                      float* mu, const avr_nvfp4* mu_q, const avr_nvfp4* xr_q,
                                      float* xr_debug, uint32_t* device_status, avr_stream stream);

/* Vanilla NVFP4 quantization of X [rows, K] (no split; [R3.1] "Vanilla FP4").
 * grad selects stream tag 7 (0) or 8 (1). */
avr_status nvfp4_quant(const void* X, avr_dtype xt, int64_t rows, int64_t K, avr_round rm,
                       uint64_t seed, uint64_t offset, int grad, const avr_nvfp4* out,
                       void* ws, size_t ws_bytes, avr_stream stream);

/* Both quantizations of a weight W [m, n] (W_bar in both equations of [RAv]):
 *   w_fwd   : Q_4(W^T), n x m (blocks along m, the forward contraction);
 *   w_dgrad : Q_4(W),   m x n (blocks along n, the dgrad contraction).
 * Round to nearest even; one tensor scale (amax of W) for both.  Needs
 * m % 64 == 0 and n % 64 == 0. */
avr_status averis_quant_weight(const void* W, avr_dtype wt, int64_t m, int64_t n,
                               const avr_nvfp4* w_fwd, const avr_nvfp4* w_dgrad, void* ws,
                               size_t ws_bytes, avr_stream stream);

/* The rank-one row mu_bar W_bar of [RAv]: bias[j] = sum_k value(mu_q)[k] *
 * value(w_q)[j, k] in fp32, j < w_q->rows.  mu_q is 1 x K, w_q is N x K. */
avr_status averis_bias_row(const avr_nvfp4* mu_q, const avr_nvfp4* w_q, float* bias, void* ws,
                           size_t ws_bytes, avr_stream stream);

/* Block-scaled FP4 GEMM on the tcgen05 tensor cores:
 *   Y[i, j] = g_dec(a) g_dec(b) sum_k e2m1(a)e4m3(sa) e2m1(b)e4m3(sb) + bias[j]
 * with A = a [M, K], B = b [N, K] (both K-major), bias [N] fp32 nullable,
 * Y [M, N] in yt (row-major). */
avr_status nvfp4_gemm(const avr_nvfp4* a, const avr_nvfp4* b, const float* bias, void* Y,
                      avr_dtype yt, void* ws, size_t ws_bytes, avr_stream stream);

/* -------------------------------------------------------------------------
 * The linear layer [RAv]
 * ------------------------------------------------------------------------- */

/* Forward: Y [l, n] = 1 (Q_4(mu_X) W_bar) + Q_4(X - 1 mu_X) W_bar for
 * X [l, m] and w_fwd = Q_4(W^T) [n, m].  save_xr / save_mu (nullable)
 * receive the quantized operands for a later weight-gradient pass; when
 * NULL they live in the workspace.  Four launches: column reduce, fold,
 * split-quantize (+ mean quantize + rank-one row), GEMM. */
avr_status averis_linear_fwd(const void* X, avr_dtype xt, int64_t l, int64_t m, int64_t n,
                             const avr_nvfp4* w_fwd, avr_round rm, uint64_t seed,
                             uint64_t offset, void* Y, avr_dtype yt, const avr_nvfp4* save_xr,
                             const avr_nvfp4* save_mu, void* ws, size_t ws_bytes,
                             avr_stream stream);

/* Dgrad: dX [l, m] = 1 (Q_4(mu_D) W_bar^T) + Q_4(D - 1 mu_D) W_bar^T for
 * D [l, n] and w_dgrad = Q_4(W) [m, n]. */
avr_status averis_linear_dgrad(const void* D, avr_dtype dt, int64_t l, int64_t m, int64_t n,
                               const avr_nvfp4* w_dgrad, avr_round rm, uint64_t seed,
                               uint64_t offset, void* dX, avr_dtype xt, void* ws,
                               size_t ws_bytes, avr_stream stream);

/* Vanilla NVFP4 forward / dgrad ([R3.1], [Abs] "vanilla NVFP4"): Y = Q_4(X)
 * W_bar, dX = Q_4(D) W_bar^T, the same four launches without the split
 * (the reduce and the fold then give the amax only). */
avr_status nvfp4_linear_fwd(const void* X, avr_dtype xt, int64_t l, int64_t m, int64_t n,
                            const avr_nvfp4* w_fwd, avr_round rm, uint64_t seed, uint64_t offset,
                            void* Y, avr_dtype yt, void* ws, size_t ws_bytes, avr_stream stream);
avr_status nvfp4_linear_dgrad(const void* D, avr_dtype dt, int64_t l, int64_t m, int64_t n,
                              const avr_nvfp4* w_dgrad, avr_round rm, uint64_t seed,
                              uint64_t offset, void* dX, avr_dtype xt, void* ws, size_t ws_bytes,
                              avr_stream stream);

/* -------------------------------------------------------------------------
 * Weight gradient [R3.1], [RAv]
 *
 * The pages train W4A4G4 (all three GEMMs of a linear in FP4) but write the
 * Averis split only for the forward and dgrad.  For dW = X^T D (X [l, m],
 * D [l, n], Y = X W) the same split gives
 *     X^T D = X_R^T D_R + l mu_X^T mu_D
 * (both cross terms vanish because 1^T X_R = 0), so the residual product
 * runs on the tensor cores and the mean part is a rank-one fp32 term.
 * Readings: the residuals are quantized along the tokens (the contraction
 * axis) as [m, L] and [n, L] tensors, L = l rounded up to a multiple of 64,
 * tokens l..L-1 exact zeros; their tensor scales are the row-wise
 * residuals' (same amax); the rank-one term uses the quantized means
 * mu_bar_X, mu_bar_D (the bits averis_split_quant gives for the same seed and
 * offset).  Random-stream tags: 9 (X_R^T), 10 (D_R^T), 11/12 (vanilla X^T,
 * D^T); element (j, i) of the [K, L] tensor counts from offset + (j L + i)/16.
 * ------------------------------------------------------------------------- */

/* Split of X [l, K] (grad = 0) or D (grad = 1) with the residual quantized
 * along the tokens.
 *   mu     [K] fp32 out (nullable), mu_q 1 x K out (nullable): as averis_split_quant.
 *   xrt_q  out: Q_4((X - 1 mu)^T), rows = K, K-field = L.
 * Workspace: averis_workspace_size(l, K, 0).  Launches 2 kernels. */
avr_status averis_split_quant_t(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                                uint64_t seed, uint64_t offset, int grad, float* mu,
                                const avr_nvfp4* mu_q, const avr_nvfp4* xrt_q, void* ws,
                                size_t ws_bytes, avr_stream stream);

/* Q_4(X^T) along the tokens with no split (the vanilla comparison). */
avr_status nvfp4_quant_t(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                         uint64_t seed, uint64_t offset, int grad, const avr_nvfp4* out, void* ws,
                         size_t ws_bytes, avr_stream stream);

/* Workspace bytes of averis_wgrad_gemm and the two *_linear_wgrad calls. */
size_t averis_wgrad_workspace_size(int64_t l, int64_t m, int64_t n);

/* dW [m, n] = g(A) g(B) deq(A) deq(B)^T + l deq(mu_bar_X)^T deq(mu_bar_D)
 * from xrt_q [m, L] and drt_q [n, L] (L = l rounded up to 64); mu_x_q 1 x m
 * and mu_d_q 1 x n are both given (Averis) or both NULL (plain product).
 * wt: fp32 or bf16 output.  Needs m % 64 == 0, n % 64 == 0, l >= 1.
 * Launches 2 kernels (rank-one factors, GEMM) or 1. */
avr_status averis_wgrad_gemm(const avr_nvfp4* xrt_q, const avr_nvfp4* drt_q, const avr_nvfp4* mu_x_q,
                             const avr_nvfp4* mu_d_q, int64_t l, void* dW, avr_dtype wt, void* ws,
                             size_t ws_bytes, avr_stream stream);

/* The whole Averis weight gradient from X [l, m] and D [l, n]: the two
 * token-axis splits into workspace scratch, then averis_wgrad_gemm.
 * l == 0 writes dW = 0.  Launches 6 kernels. */
avr_status averis_linear_wgrad(const void* X, avr_dtype xt, const void* D, avr_dtype dt, int64_t l,
                               int64_t m, int64_t n, avr_round rm, uint64_t seed, uint64_t offset,
                               void* dW, avr_dtype wt, void* ws, size_t ws_bytes, avr_stream stream);

/* Vanilla NVFP4 weight gradient Q_4(X^T) Q_4(D^T)^T.  Launches 5 kernels. */
avr_status nvfp4_linear_wgrad(const void* X, avr_dtype xt, const void* D, avr_dtype dt, int64_t l,
                              int64_t m, int64_t n, avr_round rm, uint64_t seed, uint64_t offset,
                              void* dW, avr_dtype wt, void* ws, size_t ws_bytes, avr_stream stream);

/* -------------------------------------------------------------------------
 * Mixture of experts [Abs], [RAv]
 *
 * The pages train a Qwen3 7B-A1.5B MoE model with Averis and say no more.
 * Reading: every expert is its own linear layer with its own split.  The
 * tokens routed to expert e are rows [o_e, o_e + n_e) of a buffer permuted by
 * expert, o_0 = 0 and o_{e+1} = o_e + n_e rounded up to 128 (rows in between
 * are padding: no statistic sees them and their outputs are undefined).  mu_e
 * is the mean of the expert's rows in the dense layer's fixed order (chunks
 * from o_e); X_bar_R,e and mu_bar_e have per-expert tensor scales.  The counts
 * n_e are a device array (int32 [E]), e.g. from a router; the buffer has
 * l_cap rows (a multiple of 128, at least sum_e n_e rounded up per expert).
 * Random streams: row r of the buffer as in the dense layer; mu_bar_e as row
 * e of an [E, K] tensor.  Limits: E <= 1024, E * ceil(K / 128) <= 4096,
 * N % 128 == 0.  A segment table that does not fit l_cap latches
 * AVR_ERR_INVALID_ARG and nothing is computed.
 * NVFP4 tensors of the MoE calls hold E decode scales (g_dec[E]):
 *   xr_q [l_cap, K]: rows of expert e scaled by g_dec[e];
 *   mu_q [E, K]: row e is mu_bar_e;
 *   w_fwd [E * n, m/2] and w_dgrad [E * m, n/2]: the experts stacked.
 * ------------------------------------------------------------------------- */

/* Workspace bytes of the MoE calls (N = output features per expert; 0 for
 * averis_moe_split_quant). */
size_t averis_moe_workspace_size(int64_t l_cap, int64_t K, int64_t N, int E);

/* Per-expert quantization of W [E][m][n] (each expert's own tensor scale),
 * RNE, into the stacked w_fwd / w_dgrad.  ws: averis_workspace_size(m, n, n).
 * m % 128 == 0 and n % 128 == 0. */
avr_status averis_moe_quant_weights(const void* W, avr_dtype wt, int E, int64_t m, int64_t n,
                                    const avr_nvfp4* w_fwd, const avr_nvfp4* w_dgrad, void* ws,
                                    size_t ws_bytes, avr_stream stream);

/* Per-expert split of X [l_cap, K]: mu [E][K] (nullable), mu_q (nullable),
 * xr_q (padding rows: zero codes and scales).  grad selects the stream tags
 * as in averis_split_quant.  Launches 3 kernels (table, reduce, quantize). */
avr_status averis_moe_split_quant(const void* X, avr_dtype xt, int64_t l_cap, const int32_t* counts, int E,
                                  int64_t K, avr_round rm, uint64_t seed, uint64_t offset, int grad, float* mu,
                                  const avr_nvfp4* mu_q, const avr_nvfp4* xr_q, void* ws, size_t ws_bytes,
                                  avr_stream stream);

/* Forward of the MoE layer: Y[o_e + i] = 1 (mu_bar_e W_bar_e) + X_bar_R,e W_bar_e
 * for every expert, one grouped block-scaled GEMM over all segments.
 * X [l_cap, m], Y [l_cap, n].  Launches 5 kernels (table, reduce, quantize,
 * rank-one rows, grouped GEMM). */
avr_status averis_moe_linear_fwd(const void* X, avr_dtype xt, int64_t l_cap, const int32_t* counts, int E,
                                 int64_t m, int64_t n, const avr_nvfp4* w_fwd, avr_round rm, uint64_t seed,
                                 uint64_t offset, void* Y, avr_dtype yt, void* ws, size_t ws_bytes,
                                 avr_stream stream);

/* Dgrad of the MoE layer: dX[o_e + i] from D [l_cap, n] and w_dgrad, as the
 * forward with the split of D (stream tags 3 and 4). */
avr_status averis_moe_linear_dgrad(const void* D, avr_dtype dt, int64_t l_cap, const int32_t* counts, int E,
                                   int64_t m, int64_t n, const avr_nvfp4* w_dgrad, avr_round rm, uint64_t seed,
                                   uint64_t offset, void* dX, avr_dtype xt, void* ws, size_t ws_bytes,
                                   avr_stream stream);

/* -------------------------------------------------------------------------
 * Diagnostics (used by the tests to pin the number formats on the device)
 * ------------------------------------------------------------------------- */

/* For n fp32 inputs: e4m3[i] = E4M3 RNE-satfinite code of |in[i]| and
 * e2m1[i] = E2M1 RNE-satfinite code of in[i], exactly as the quantizer
 * computes them.  Either output may be NULL. */
avr_status averis_probe_convert(const float* in, uint8_t* e4m3, uint8_t* e2m1, int64_t n,
                                avr_stream stream);

/* For n groups of four fp32 values in[4i .. 4i+3] and one 32-bit random word
 * rbits[i] each: out[i] = the four E2M1 codes (element 4i in bits 0..3) that
 * the quantizer's stochastic rounding gives them. */
avr_status averis_probe_convert_sr(const float* in, const uint32_t* rbits, uint16_t* out, int64_t n,
                                   avr_stream stream);

/* The tensor pipe's block-scaled FP4 rate, measured (for the roofline; not
 * part of the method): `grid` CTAs, one per SM at most, each issue `iters`
 * stages of four tcgen05.mma.kind::mxf4nvf4.block_scale.block16 of M 128 x
 * N 256 x K 64 from constant shared-memory operands, no loads or copies in
 * the loop.  ns [grid] (device, 8-byte aligned) receives each CTA's elapsed
 * nanoseconds; the rate is 2*128*256*256*iters*grid / max(ns) flop/ns.  ws:
 * a workspace for the status word (timeouts).  Errors: AVR_ERR_INVALID_ARG
 * (iters or grid < 1, null ns), AVR_ERR_MISALIGNED, AVR_ERR_NO_DEVICE. */
avr_status averis_probe_mma_rate(int iters, int grid, uint64_t* ns, void* ws, size_t ws_bytes, avr_stream stream);

/* out[4*i .. 4*i+3] = Philox4x32-10 words of counter (lo32(offset+i),
 * hi32(offset+i), tag, 0) under key (lo32(seed), hi32(seed)), i < n. */
avr_status averis_probe_philox(uint64_t seed, uint64_t offset, uint32_t tag, int64_t n,
                               uint32_t* out, avr_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* AVERIS_H_ */
