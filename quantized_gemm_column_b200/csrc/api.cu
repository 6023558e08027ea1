// The C ABI of libaveris (declared in include/averis.h): host-side
// validation, workspace layout, tensor maps and the launch chains.
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <set>
#include <tuple>
#include <utility>

#include "internal.h"

namespace avr {

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t scales_bytes(int64_t rows, int64_t K) {
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  return static_cast<size_t>(rows_pad) * static_cast<size_t>(K / 16);
}

WsLayout ws_layout(int64_t l, int64_t K, int64_t N) {
  WsLayout w;
  size_t off = round_up(w.slots + 2 * sizeof(float) * kMaxColTiles, 256);
  const size_t C = static_cast<size_t>((l + kChunkRows - 1) / kChunkRows);
  w.partials = off;  off = round_up(off + 3 * C * static_cast<size_t>(K) * sizeof(float), 256);
  w.mu = off;        off = round_up(off + static_cast<size_t>(K) * sizeof(float), 256);
  w.mu_codes = off;  off = round_up(off + static_cast<size_t>(K) / 2, 256);
  w.mu_scales = off; off = round_up(off + scales_bytes(1, K), 256);
  w.mu_gdec = off;   off += 256;
  w.xr_gdec = off;   off += 256;
  w.bias = off;      off = round_up(off + static_cast<size_t>(N) * sizeof(float), 256);
  w.xr_codes = off;  off = round_up(off + static_cast<size_t>(l) * static_cast<size_t>(K) / 2, 256);
  w.xr_scales = off; off = round_up(off + scales_bytes(l, K), 256);
  w.energy_partials = off; off = round_up(off + C * static_cast<size_t>(K) * sizeof(float), 256);
  w.energy = off;    off = round_up(off + static_cast<size_t>(K) * sizeof(float), 256);
  w.total = off;
  return w;
}

int64_t padded_tokens(int64_t l) { return (l + 63) / 64 * 64; }

WgLayout wgrad_layout(int64_t l, int64_t m, int64_t n) {
  WgLayout w;
  w.base = ws_layout(l, m > n ? m : n, 0);
  const size_t L = static_cast<size_t>(padded_tokens(l));
  const size_t M = static_cast<size_t>(m), N = static_cast<size_t>(n);
  size_t off = w.base.total;
  w.xt_codes = off;   off = round_up(off + M * L / 2, 256);
  w.xt_scales = off;  off = round_up(off + scales_bytes(m, static_cast<int64_t>(L)), 256);
  w.dt_codes = off;   off = round_up(off + N * L / 2, 256);
  w.dt_scales = off;  off = round_up(off + scales_bytes(n, static_cast<int64_t>(L)), 256);
  w.mux_codes = off;  off = round_up(off + M / 2, 256);
  w.mux_scales = off; off = round_up(off + scales_bytes(1, m), 256);
  w.mud_codes = off;  off = round_up(off + N / 2, 256);
  w.mud_scales = off; off = round_up(off + scales_bytes(1, n), 256);
  w.gdec = off;       off += 256;
  w.u = off;          off = round_up(off + M * sizeof(float), 256);
  w.v = off;          off = round_up(off + N * sizeof(float), 256);
  w.total = off;
  return w;
}

// ---------------------------------------------------------------------------
// driver entry point for tensor maps (no link-time dependency on libcuda)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                        uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                        CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tensor_map_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, const uint64_t dims[3],
                        const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t st[2] = {strides[0], strides[1]};
  cuuint32_t b[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t set_max_dynamic_smem(const void* func, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> done;   // largest size set so far
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  auto it = done.find({dev, func});
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  // every kernel of the library asks for the largest shared-memory carveout,
  // so that back-to-back launches never wait for the SM to re-split L1
  e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done[{dev, func}] = bytes;
  return e;
}

int blocks_per_sm(const void* func, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, int, size_t>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> g(mu);
  auto key = std::make_tuple(dev, func, threads, smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem) != cudaSuccess || n < 1) n = 1;
  cache[key] = n;
  return n;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// ---------------------------------------------------------------------------
// validation helpers
// ---------------------------------------------------------------------------
avr_status device_ok() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AVR_ERR_NO_DEVICE;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return AVR_ERR_NO_DEVICE;
  return major == 10 ? AVR_OK : AVR_ERR_NO_DEVICE;
}

avr_status check_nvfp4(const avr_nvfp4* t, int64_t rows, int64_t K) {
  if (!t || !t->codes || !t->scales || !t->g_dec) return AVR_ERR_INVALID_ARG;
  if (t->rows != rows || t->K != K) return AVR_ERR_INVALID_ARG;
  if (!aligned16(t->codes) || !aligned16(t->scales) || (reinterpret_cast<uintptr_t>(t->g_dec) & 3u))
    return AVR_ERR_MISALIGNED;
  return AVR_OK;
}

static avr_status make_ws(void* ws, size_t ws_bytes, int64_t l, int64_t K, int64_t N, Ws* out) {
  if (!ws) return AVR_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return AVR_ERR_MISALIGNED;
  out->base = static_cast<char*>(ws);
  out->lay = ws_layout(l, K, N);
  if (ws_bytes < out->lay.total) return AVR_ERR_WORKSPACE_TOO_SMALL;
  return AVR_OK;
}

static int n_tiles(int64_t K) { return static_cast<int>((K + kColTile - 1) / kColTile); }

// K1 + K2 (+ mean quantizer and rank-one row when mu_q / w are given)
avr_status split_chain(const void* X, avr_dtype xt, int64_t l, int64_t K, int split, avr_round rm,
                       uint64_t seed, uint64_t offset, uint32_t tag, uint32_t tag_mu, float* mu_buf,
                       const avr_nvfp4* mu_q, const avr_nvfp4* xr_q, float* xr_debug, const avr_nvfp4* w,
                       float* bias, const Ws& ws, cudaStream_t s, bool fused, bool pdl) {
  ColReduceArgs ca;
  ca.X = X;
  ca.xt = xt;
  ca.l = l;
  ca.K = K;
  ca.split = split;
  ca.mu_out = mu_buf;
  ca.energy = 0;
  ca.ws = ws.base;
  ca.lay = &ws.lay;
  QuantArgs qa = {};
  qa.X = X;
  qa.xt = xt;
  qa.rows = l;
  qa.K = K;
  qa.mu = split ? mu_buf : nullptr;
  qa.n_tiles = n_tiles(K);
  qa.slot_xr = ws.slot_xr();
  qa.codes = xr_q->codes;
  qa.scales = xr_q->scales;
  qa.g_dec = xr_q->g_dec;
  qa.xr_debug = xr_debug;
  qa.seed = seed;
  qa.offset = offset;
  qa.tag = tag;
  qa.sr = rm == AVR_SR;
  qa.status = ws.status();
  qa.slot_mu = ws.slot_mu();
  qa.tag_mu = tag_mu;
  if (mu_q) {
    qa.mu_codes = mu_q->codes;
    qa.mu_scales = mu_q->scales;
    qa.mu_gdec = mu_q->g_dec;
  }
  if (w) {
    qa.w_codes = w->codes;
    qa.w_scales = w->scales;
    qa.w_gdec = w->g_dec;
    qa.n_out = w->rows;
    qa.bias = bias;
  }
  if (fused) return cuda_status(launch_split_fused(ca, qa, s, pdl));
  AVR_TRY(cuda_status(launch_colreduce(ca, s, pdl)));
  return cuda_status(launch_quant(qa, s, pdl));
}

// K1 + K2 along the tokens (+ mean quantizer when mu_q is given), for the
// weight gradient
static avr_status split_chain_tokens(const void* X, avr_dtype xt, int64_t l, int64_t K, int split,
                                     avr_round rm, uint64_t seed, uint64_t offset, uint32_t tag,
                                     uint32_t tag_mu, float* mu_buf, const avr_nvfp4* mu_q,
                                     const avr_nvfp4* xt_q, const Ws& ws, cudaStream_t s) {
  ColReduceArgs ca;
  ca.X = X;
  ca.xt = xt;
  ca.l = l;
  ca.K = K;
  ca.split = split;
  ca.mu_out = mu_buf;
  ca.energy = 0;
  ca.ws = ws.base;
  ca.lay = &ws.lay;
  AVR_TRY(cuda_status(launch_colreduce(ca, s, true)));
  QuantArgs qa = {};
  qa.X = X;
  qa.xt = xt;
  qa.rows = l;
  qa.K = K;
  qa.mu = split ? mu_buf : nullptr;
  qa.n_tiles = n_tiles(K);
  qa.slot_xr = ws.slot_xr();
  qa.codes = xt_q->codes;
  qa.scales = xt_q->scales;
  qa.g_dec = xt_q->g_dec;
  qa.seed = seed;
  qa.offset = offset;
  qa.tag = tag;
  qa.sr = rm == AVR_SR;
  qa.status = ws.status();
  qa.slot_mu = ws.slot_mu();
  qa.tag_mu = tag_mu;
  if (mu_q) {
    qa.mu_codes = mu_q->codes;
    qa.mu_scales = mu_q->scales;
    qa.mu_gdec = mu_q->g_dec;
  }
  return cuda_status(launch_quant_tokens(qa, s, true));
}

static avr_status gemm(const avr_nvfp4* a, const avr_nvfp4* b, const float* bias, void* Y,
                       avr_dtype yt, uint32_t* status, cudaStream_t s, const float* row_scale = nullptr) {
  GemmArgs g;
  g.a_codes = a->codes;
  g.a_scales = a->scales;
  g.a_gdec = a->g_dec;
  g.b_codes = b->codes;
  g.b_scales = b->scales;
  g.b_gdec = b->g_dec;
  g.M = a->rows;
  g.N = b->rows;
  g.K = a->K;
  g.bias = bias;
  g.row_scale = row_scale;
  g.Y = Y;
  g.yt = yt;
  g.status = status;
  return cuda_status(launch_gemm(g, s, true));
}

}  // namespace avr

using namespace avr;

// one 64-bit word written in stream order (a launch, so it can be captured)
__global__ void set_word64_kernel(uint64_t* dst, uint64_t value) { *dst = value; }

extern "C" {

size_t avr_nvfp4_scales_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 16) return 0;
  return scales_bytes(rows, K);
}

size_t averis_workspace_size(int64_t l, int64_t K, int64_t N) {
  if (l < 0 || K <= 0 || N < 0) return 0;
  return ws_layout(l, K, N).total;
}

avr_status averis_workspace_init(void* ws, size_t ws_bytes, avr_stream stream) {
  if (!ws) return AVR_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, stream));
}

avr_status averis_set_wait_limit(void* ws, size_t ws_bytes, uint64_t limit_ns, avr_stream stream) {
  if (!ws) return AVR_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return AVR_ERR_MISALIGNED;
  if (ws_bytes < WsLayout{}.tickets) return AVR_ERR_WORKSPACE_TOO_SMALL;
  AVR_TRY(device_ok());
  set_word64_kernel<<<1, 1, 0, stream>>>(reinterpret_cast<uint64_t*>(static_cast<char*>(ws) + kWaitLimitOffset),
                                         limit_ns);
  return cuda_status(cudaGetLastError());
}

avr_status averis_check_status(void* ws, avr_stream stream) {
  if (!ws) return AVR_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return AVR_ERR_CUDA;
  uint32_t st = 0;
  if (cudaMemcpy(&st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return AVR_ERR_CUDA;
  // after an error the 256-byte status block (status word and the grid-barrier
  // words of the fused split) and the reduce's tickets, which a kernel that
  // gave up may have left part-counted, start again from zero
  if (st != 0 && cudaMemset(ws, 0, WsLayout{}.slots) != cudaSuccess) return AVR_ERR_CUDA;
  return static_cast<avr_status>(st);
}

const char* averis_status_string(avr_status s) {
  switch (s) {
    case AVR_OK: return "ok";
    case AVR_ERR_INVALID_ARG: return "invalid argument";
    case AVR_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (need K % 64 == 0, N % 64 == 0, sizes < 2^31)";
    case AVR_ERR_MISALIGNED: return "misaligned pointer (need 16-byte alignment, 256 for the workspace)";
    case AVR_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case AVR_ERR_CUDA: return "CUDA error";
    case AVR_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case AVR_ERR_NONFINITE: return "non-finite input (mean or amax is NaN/Inf)";
    case AVR_ERR_NO_DEVICE: return "no sm_100 device is current";
  }
  return "unknown status";
}

avr_status averis_split_quant(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                              uint64_t seed, uint64_t offset, int grad, float* mu,
                              const avr_nvfp4* mu_q, const avr_nvfp4* xr_q, float* xr_debug,
                              void* ws, size_t ws_bytes, avr_stream stream) {
  if (!dtype_ok(xt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(K) || !l_ok(l)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (l == 0) return AVR_OK;   // no tokens: nothing is read or written
  if (!X) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(xr_q, l, K));
  if (mu_q) AVR_TRY(check_nvfp4(mu_q, 1, K));
  if (!aligned16(X) || !aligned16(mu) || !aligned16(xr_debug)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, l, K, 0, &w));
  AVR_TRY(device_ok());
  float* mu_buf = mu ? mu : w.at<float>(w.lay.mu);
  return split_chain(X, xt, l, K, 1, rm, seed, offset, grad ? 3u : 1u, grad ? 4u : 2u, mu_buf, mu_q,
                     xr_q, xr_debug, nullptr, nullptr, w, stream);
}

avr_status averis_mean_energy_ratio(const void* X, avr_dtype xt, int64_t l, int64_t K, float* mu,
                                    float* R, void* ws, size_t ws_bytes, avr_stream stream) {
  if (!dtype_ok(xt)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(K) || !l_ok(l) || l == 0) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (!X || !R) return AVR_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(mu)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, l, K, 0, &w));
  AVR_TRY(device_ok());
  float* mu_buf = mu ? mu : w.at<float>(w.lay.mu);
  ColReduceArgs ca;
  ca.X = X;
  ca.xt = xt;
  ca.l = l;
  ca.K = K;
  ca.split = 1;
  ca.mu_out = mu_buf;
  ca.energy = 1;
  ca.ws = w.base;
  ca.lay = &w.lay;
  AVR_TRY(cuda_status(launch_colreduce(ca, stream, true)));
  return cuda_status(launch_energy_ratio(mu_buf, w.at<float>(w.lay.energy), K, l, R, w.status(), stream, true));
}

avr_status averis_split_quant_fused(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                                    uint64_t seed, uint64_t offset, int grad, float* mu,
                                    const avr_nvfp4* mu_q, const avr_nvfp4* xr_q, void* ws,
                                    size_t ws_bytes, avr_stream stream) {
  if (!dtype_ok(xt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(K) || !l_ok(l)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (l == 0) return AVR_OK;   // no tokens: nothing is read or written
  if (!X) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(xr_q, l, K));
  if (mu_q) AVR_TRY(check_nvfp4(mu_q, 1, K));
  if (!aligned16(X) || !aligned16(mu)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, l, K, 0, &w));
  AVR_TRY(device_ok());
  float* mu_buf = mu ? mu : w.at<float>(w.lay.mu);
  return split_chain(X, xt, l, K, 1, rm, seed, offset, grad ? 3u : 1u, grad ? 4u : 2u, mu_buf, mu_q,
                     xr_q, nullptr, nullptr, nullptr, w, stream, true);
}

avr_status nvfp4_quant(const void* X, avr_dtype xt, int64_t rows, int64_t K, avr_round rm,
                       uint64_t seed, uint64_t offset, int grad, const avr_nvfp4* out, void* ws,
                       size_t ws_bytes, avr_stream stream) {
  if (!dtype_ok(xt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(K) || !l_ok(rows)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return AVR_OK;
  if (!X) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(out, rows, K));
  if (!aligned16(X)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, rows, K, 0, &w));
  AVR_TRY(device_ok());
  return split_chain(X, xt, rows, K, 0, rm, seed, offset, grad ? 8u : 7u, 0u, nullptr, nullptr, out,
                     nullptr, nullptr, nullptr, w, stream);
}

avr_status averis_quant_weight(const void* W, avr_dtype wt, int64_t m, int64_t n,
                               const avr_nvfp4* w_fwd, const avr_nvfp4* w_dgrad, void* ws,
                               size_t ws_bytes, avr_stream stream) {
  if (!W || !dtype_ok(wt)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(m) || !k_ok(n) || !n_ok(m) || !n_ok(n)) return AVR_ERR_UNSUPPORTED_SHAPE;
  AVR_TRY(check_nvfp4(w_fwd, n, m));
  AVR_TRY(check_nvfp4(w_dgrad, m, n));
  if (!aligned16(W)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, m, n, 0, &w));
  AVR_TRY(device_ok());
  // amax of W, then W_bar_dgrad = Q_4(W) along n and W_bar_fwd = Q_4(W^T) along m
  AVR_TRY(split_chain(W, wt, m, n, 0, AVR_RNE, 0, 0, 6u, 0u, nullptr, nullptr, w_dgrad, nullptr,
                      nullptr, nullptr, w, stream));
  QuantTransposedArgs t;
  t.W = W;
  t.wt = wt;
  t.m = m;
  t.n = n;
  t.n_tiles = n_tiles(n);
  t.slot_amax = w.slot_xr();
  t.codes = w_fwd->codes;
  t.scales = w_fwd->scales;
  t.g_dec = w_fwd->g_dec;
  return cuda_status(launch_quant_transposed(t, stream));
}

avr_status averis_bias_row(const avr_nvfp4* mu_q, const avr_nvfp4* w_q, float* bias, void* ws,
                           size_t ws_bytes, avr_stream stream) {
  if (!mu_q || !w_q || !bias) return AVR_ERR_INVALID_ARG;
  if (!k_ok(mu_q->K) || !n_ok(w_q->rows)) return AVR_ERR_UNSUPPORTED_SHAPE;
  AVR_TRY(check_nvfp4(mu_q, 1, mu_q->K));
  AVR_TRY(check_nvfp4(w_q, w_q->rows, mu_q->K));
  if (!aligned16(bias)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, 0, mu_q->K, 0, &w));
  AVR_TRY(device_ok());
  BiasArgs b;
  b.mu_codes = mu_q->codes;
  b.mu_scales = mu_q->scales;
  b.mu_gdec = mu_q->g_dec;
  b.w_codes = w_q->codes;
  b.w_scales = w_q->scales;
  b.w_gdec = w_q->g_dec;
  b.K = mu_q->K;
  b.n_out = w_q->rows;
  b.bias = bias;
  return cuda_status(launch_bias(b, stream));
}

avr_status nvfp4_gemm(const avr_nvfp4* a, const avr_nvfp4* b, const float* bias, void* Y,
                      avr_dtype yt, void* ws, size_t ws_bytes, avr_stream stream) {
  if (!a || !b || !dtype_ok(yt)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(a->K) || !l_ok(a->rows) || !n_ok(b->rows)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (a->rows == 0) return AVR_OK;
  if (!Y) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(a, a->rows, a->K));
  AVR_TRY(check_nvfp4(b, b->rows, a->K));
  if (!aligned16(Y) || !aligned16(bias)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, 0, a->K, 0, &w));
  AVR_TRY(device_ok());
  return gemm(a, b, bias, Y, yt, w.status(), stream);
}

static avr_status linear(const void* X, avr_dtype xt, int64_t l, int64_t K, int64_t N,
                         const avr_nvfp4* wq, int split, avr_round rm, uint64_t seed,
                         uint64_t offset, uint32_t tag, uint32_t tag_mu, void* Y, avr_dtype yt,
                         const avr_nvfp4* save_xr, const avr_nvfp4* save_mu, void* ws,
                         size_t ws_bytes, avr_stream stream) {
  if (!dtype_ok(xt) || !dtype_ok(yt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(K) || !n_ok(N) || !l_ok(l)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (l == 0) return AVR_OK;
  if (!X || !Y) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(wq, N, K));
  if (save_xr) AVR_TRY(check_nvfp4(save_xr, l, K));
  if (save_mu) AVR_TRY(check_nvfp4(save_mu, 1, K));
  if (!aligned16(X) || !aligned16(Y)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, l, K, N, &w));
  AVR_TRY(device_ok());
  avr_nvfp4 xr_ws = {w.at<uint8_t>(w.lay.xr_codes), w.at<uint8_t>(w.lay.xr_scales),
                     w.at<float>(w.lay.xr_gdec), l, K};
  avr_nvfp4 mu_ws = {w.at<uint8_t>(w.lay.mu_codes), w.at<uint8_t>(w.lay.mu_scales),
                     w.at<float>(w.lay.mu_gdec), 1, K};
  const avr_nvfp4* xr = save_xr ? save_xr : &xr_ws;
  const avr_nvfp4* muq = save_mu ? save_mu : &mu_ws;
  float* bias = split ? w.at<float>(w.lay.bias) : nullptr;
  AVR_TRY(split_chain(X, xt, l, K, split, rm, seed, offset, tag, tag_mu, w.at<float>(w.lay.mu),
                      split ? muq : nullptr, xr, nullptr, split ? wq : nullptr, bias, w, stream));
  return gemm(xr, wq, bias, Y, yt, w.status(), stream);
}

avr_status averis_linear_fwd(const void* X, avr_dtype xt, int64_t l, int64_t m, int64_t n,
                             const avr_nvfp4* w_fwd, avr_round rm, uint64_t seed, uint64_t offset,
                             void* Y, avr_dtype yt, const avr_nvfp4* save_xr,
                             const avr_nvfp4* save_mu, void* ws, size_t ws_bytes,
                             avr_stream stream) {
  return linear(X, xt, l, m, n, w_fwd, 1, rm, seed, offset, 1u, 2u, Y, yt, save_xr, save_mu, ws,
                ws_bytes, stream);
}

avr_status averis_linear_dgrad(const void* D, avr_dtype dt, int64_t l, int64_t m, int64_t n,
                               const avr_nvfp4* w_dgrad, avr_round rm, uint64_t seed,
                               uint64_t offset, void* dX, avr_dtype xt, void* ws, size_t ws_bytes,
                               avr_stream stream) {
  return linear(D, dt, l, n, m, w_dgrad, 1, rm, seed, offset, 3u, 4u, dX, xt, nullptr, nullptr, ws,
                ws_bytes, stream);
}

avr_status nvfp4_linear_fwd(const void* X, avr_dtype xt, int64_t l, int64_t m, int64_t n,
                            const avr_nvfp4* w_fwd, avr_round rm, uint64_t seed, uint64_t offset,
                            void* Y, avr_dtype yt, void* ws, size_t ws_bytes, avr_stream stream) {
  return linear(X, xt, l, m, n, w_fwd, 0, rm, seed, offset, 7u, 0u, Y, yt, nullptr, nullptr, ws,
                ws_bytes, stream);
}

avr_status nvfp4_linear_dgrad(const void* D, avr_dtype dt, int64_t l, int64_t m, int64_t n,
                              const avr_nvfp4* w_dgrad, avr_round rm, uint64_t seed,
                              uint64_t offset, void* dX, avr_dtype xt, void* ws, size_t ws_bytes,
                              avr_stream stream) {
  return linear(D, dt, l, n, m, w_dgrad, 0, rm, seed, offset, 8u, 0u, dX, xt, nullptr, nullptr, ws,
                ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// weight gradient
// ---------------------------------------------------------------------------
static avr_status quant_tokens_entry(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                                     uint64_t seed, uint64_t offset, int split, uint32_t tag,
                                     uint32_t tag_mu, float* mu, const avr_nvfp4* mu_q,
                                     const avr_nvfp4* xt_q, void* ws, size_t ws_bytes, avr_stream stream) {
  if (!dtype_ok(xt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(K) || !l_ok(l)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (l == 0) return AVR_OK;   // no tokens: nothing is read or written
  if (!X) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(xt_q, K, padded_tokens(l)));
  if (mu_q) AVR_TRY(check_nvfp4(mu_q, 1, K));
  if (!aligned16(X) || !aligned16(mu)) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, l, K, 0, &w));
  AVR_TRY(device_ok());
  float* mu_buf = mu ? mu : w.at<float>(w.lay.mu);
  return split_chain_tokens(X, xt, l, K, split, rm, seed, offset, tag, tag_mu, mu_buf, mu_q, xt_q, w, stream);
}

avr_status averis_split_quant_t(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                                uint64_t seed, uint64_t offset, int grad, float* mu,
                                const avr_nvfp4* mu_q, const avr_nvfp4* xrt_q, void* ws,
                                size_t ws_bytes, avr_stream stream) {
  return quant_tokens_entry(X, xt, l, K, rm, seed, offset, 1, grad ? 10u : 9u, grad ? 4u : 2u, mu, mu_q,
                            xrt_q, ws, ws_bytes, stream);
}

avr_status nvfp4_quant_t(const void* X, avr_dtype xt, int64_t l, int64_t K, avr_round rm,
                         uint64_t seed, uint64_t offset, int grad, const avr_nvfp4* out, void* ws,
                         size_t ws_bytes, avr_stream stream) {
  return quant_tokens_entry(X, xt, l, K, rm, seed, offset, 0, grad ? 12u : 11u, 0u, nullptr, nullptr, out,
                            ws, ws_bytes, stream);
}

size_t averis_wgrad_workspace_size(int64_t l, int64_t m, int64_t n) {
  if (l < 0 || m <= 0 || n <= 0) return 0;
  return wgrad_layout(l, m, n).total;
}

static avr_status make_wg(void* ws, size_t ws_bytes, int64_t l, int64_t m, int64_t n, WgLayout* lay, Ws* w) {
  if (!ws) return AVR_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return AVR_ERR_MISALIGNED;
  *lay = wgrad_layout(l, m, n);
  if (ws_bytes < lay->total) return AVR_ERR_WORKSPACE_TOO_SMALL;
  w->base = static_cast<char*>(ws);
  w->lay = lay->base;
  return AVR_OK;
}

// dW = alpha acc (+ u v^T) once the four operands are in place
static avr_status wgrad_product(const avr_nvfp4* xt_q, const avr_nvfp4* dt_q, const avr_nvfp4* mu_x_q,
                                const avr_nvfp4* mu_d_q, int64_t l, void* dW, avr_dtype wt, const Ws& w,
                                const WgLayout& lay, cudaStream_t s) {
  if (!mu_x_q) return gemm(xt_q, dt_q, nullptr, dW, wt, w.status(), s);
  float* u = w.at<float>(lay.u);
  float* v = w.at<float>(lay.v);
  AVR_TRY(cuda_status(launch_mean_dequant(mu_x_q->codes, mu_x_q->scales, mu_x_q->g_dec, xt_q->rows, mu_d_q->codes,
                                          mu_d_q->scales, mu_d_q->g_dec, dt_q->rows, l, u, v, s, true)));
  return gemm(xt_q, dt_q, v, dW, wt, w.status(), s, u);
}

avr_status averis_wgrad_gemm(const avr_nvfp4* xrt_q, const avr_nvfp4* drt_q, const avr_nvfp4* mu_x_q,
                             const avr_nvfp4* mu_d_q, int64_t l, void* dW, avr_dtype wt, void* ws,
                             size_t ws_bytes, avr_stream stream) {
  if (!xrt_q || !drt_q || !dtype_ok(wt)) return AVR_ERR_INVALID_ARG;
  if ((mu_x_q == nullptr) != (mu_d_q == nullptr)) return AVR_ERR_INVALID_ARG;
  const int64_t m = xrt_q->rows, n = drt_q->rows, L = xrt_q->K;
  if (!k_ok(m) || !n_ok(n) || !k_ok(L) || l < 1 || padded_tokens(l) != L) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (!dW) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(xrt_q, m, L));
  AVR_TRY(check_nvfp4(drt_q, n, L));
  if (mu_x_q) {
    AVR_TRY(check_nvfp4(mu_x_q, 1, m));
    AVR_TRY(check_nvfp4(mu_d_q, 1, n));
  }
  if (!aligned16(dW)) return AVR_ERR_MISALIGNED;
  WgLayout lay;
  Ws w;
  AVR_TRY(make_wg(ws, ws_bytes, l, m, n, &lay, &w));
  AVR_TRY(device_ok());
  return wgrad_product(xrt_q, drt_q, mu_x_q, mu_d_q, l, dW, wt, w, lay, stream);
}

static avr_status linear_wgrad(const void* X, avr_dtype xt, const void* D, avr_dtype dt, int64_t l,
                               int64_t m, int64_t n, int split, avr_round rm, uint64_t seed,
                               uint64_t offset, void* dW, avr_dtype wt, void* ws, size_t ws_bytes,
                               avr_stream stream) {
  if (!dtype_ok(xt) || !dtype_ok(dt) || !dtype_ok(wt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(m) || !n_ok(n) || !l_ok(l)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (!dW) return AVR_ERR_INVALID_ARG;
  if (!aligned16(dW)) return AVR_ERR_MISALIGNED;
  if (l == 0) {   // an empty sum over tokens
    AVR_TRY(device_ok());
    const size_t bytes = static_cast<size_t>(m) * static_cast<size_t>(n) * (wt == AVR_BF16 ? 2 : 4);
    return cuda_status(cudaMemsetAsync(dW, 0, bytes, stream));
  }
  if (!X || !D) return AVR_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(D)) return AVR_ERR_MISALIGNED;
  WgLayout lay;
  Ws w;
  AVR_TRY(make_wg(ws, ws_bytes, l, m, n, &lay, &w));
  AVR_TRY(device_ok());
  const int64_t L = padded_tokens(l);
  float* g = w.at<float>(lay.gdec);
  avr_nvfp4 xq = {w.at<uint8_t>(lay.xt_codes), w.at<uint8_t>(lay.xt_scales), g, m, L};
  avr_nvfp4 dq = {w.at<uint8_t>(lay.dt_codes), w.at<uint8_t>(lay.dt_scales), g + 1, n, L};
  avr_nvfp4 mxq = {w.at<uint8_t>(lay.mux_codes), w.at<uint8_t>(lay.mux_scales), g + 2, 1, m};
  avr_nvfp4 mdq = {w.at<uint8_t>(lay.mud_codes), w.at<uint8_t>(lay.mud_scales), g + 3, 1, n};
  float* mu_buf = w.at<float>(w.lay.mu);
  AVR_TRY(split_chain_tokens(X, xt, l, m, split, rm, seed, offset, split ? 9u : 11u, 2u, mu_buf,
                             split ? &mxq : nullptr, &xq, w, stream));
  AVR_TRY(split_chain_tokens(D, dt, l, n, split, rm, seed, offset, split ? 10u : 12u, 4u, mu_buf,
                             split ? &mdq : nullptr, &dq, w, stream));
  return wgrad_product(&xq, &dq, split ? &mxq : nullptr, split ? &mdq : nullptr, l, dW, wt, w, lay, stream);
}

avr_status averis_linear_wgrad(const void* X, avr_dtype xt, const void* D, avr_dtype dt, int64_t l,
                               int64_t m, int64_t n, avr_round rm, uint64_t seed, uint64_t offset,
                               void* dW, avr_dtype wt, void* ws, size_t ws_bytes, avr_stream stream) {
  return linear_wgrad(X, xt, D, dt, l, m, n, 1, rm, seed, offset, dW, wt, ws, ws_bytes, stream);
}

avr_status nvfp4_linear_wgrad(const void* X, avr_dtype xt, const void* D, avr_dtype dt, int64_t l,
                              int64_t m, int64_t n, avr_round rm, uint64_t seed, uint64_t offset,
                              void* dW, avr_dtype wt, void* ws, size_t ws_bytes, avr_stream stream) {
  return linear_wgrad(X, xt, D, dt, l, m, n, 0, rm, seed, offset, dW, wt, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// mixture of experts
// ---------------------------------------------------------------------------
static int moe_c_max(int64_t l_cap, int E) {
  return static_cast<int>((l_cap + kChunkRows - 1) / kChunkRows) + E;
}

// status, tickets and slots at the fixed offsets of WsLayout, then the
// grouped reduce's partials, the segment table, the per-expert means, their
// NVFP4 form, the rank-one rows and the split residual
struct MoeLayout {
  WsLayout base;              // status, tickets, slots, partials [3][c_max][K]
  size_t seg = 0, totals = 0, chunk_expert = 0, block_expert = 0;
  size_t mu = 0, mu_codes = 0, mu_scales = 0, mu_gdec = 0, xr_gdec = 0, bias = 0;
  size_t xr_codes = 0, xr_scales = 0;
  size_t total = 0;
};

static MoeLayout moe_layout(int64_t l_cap, int64_t K, int64_t N, int E) {
  MoeLayout w;
  const size_t C = static_cast<size_t>(moe_c_max(l_cap, E));
  const size_t Ks = static_cast<size_t>(K), Ns = static_cast<size_t>(N), Es = static_cast<size_t>(E);
  size_t off = round_up(w.base.slots + 2 * sizeof(float) * kMaxColTiles, 256);
  w.base.partials = off; off = round_up(off + 3 * C * Ks * sizeof(float), 256);
  w.seg = off;           off = round_up(off + Es * sizeof(MoeSeg), 256);
  w.totals = off;        off += 256;
  w.chunk_expert = off;  off = round_up(off + C * sizeof(int32_t), 256);
  w.block_expert = off;  off = round_up(off + static_cast<size_t>(l_cap / 128) * sizeof(int32_t), 256);
  w.mu = off;            off = round_up(off + Es * Ks * sizeof(float), 256);
  w.mu_codes = off;      off = round_up(off + Es * Ks / 2, 256);
  w.mu_scales = off;     off = round_up(off + scales_bytes(E, K), 256);
  w.mu_gdec = off;       off = round_up(off + Es * sizeof(float), 256);
  w.xr_gdec = off;       off = round_up(off + Es * sizeof(float), 256);
  w.bias = off;          off = round_up(off + Es * Ns * sizeof(float), 256);
  w.xr_codes = off;      off = round_up(off + static_cast<size_t>(l_cap) * Ks / 2, 256);
  w.xr_scales = off;     off = round_up(off + scales_bytes(l_cap, K), 256);
  w.total = off;
  return w;
}

static bool moe_shape_ok(int64_t l_cap, int E, int64_t K) {
  return l_cap >= 0 && l_cap % 128 == 0 && l_cap <= kMaxDim && E >= 1 && E <= 1024 && k_ok(K) &&
         static_cast<int64_t>(E) * ((K + kColTile - 1) / kColTile) <= kMaxColTiles;
}

static avr_status make_moe_ws(void* ws, size_t ws_bytes, int64_t l_cap, int64_t K, int64_t N, int E,
                              MoeLayout* lay, Ws* w) {
  if (!ws) return AVR_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return AVR_ERR_MISALIGNED;
  *lay = moe_layout(l_cap, K, N, E);
  if (ws_bytes < lay->total) return AVR_ERR_WORKSPACE_TOO_SMALL;
  w->base = static_cast<char*>(ws);
  w->lay = lay->base;
  return AVR_OK;
}

// segment table, grouped reduce and grouped quantizer (the per-expert split)
static avr_status moe_split_chain(const void* X, avr_dtype xt, int64_t l_cap, const int32_t* counts, int E,
                                  int64_t K, avr_round rm, uint64_t seed, uint64_t offset, uint32_t tag,
                                  uint32_t tag_mu, float* mu, const avr_nvfp4* mu_q, const avr_nvfp4* xr_q,
                                  const Ws& w, const MoeLayout& lay, cudaStream_t s) {
  const int c_max = moe_c_max(l_cap, E);
  MoeSeg* seg = w.at<MoeSeg>(lay.seg);
  int32_t* totals = w.at<int32_t>(lay.totals);
  int32_t* chunk_expert = w.at<int32_t>(lay.chunk_expert);
  int32_t* block_expert = w.at<int32_t>(lay.block_expert);
  AVR_TRY(cuda_status(launch_moe_table(counts, E, l_cap, c_max, seg, chunk_expert, block_expert, totals,
                                       w.status(), s, true)));
  ColReduceArgs ca;
  ca.X = X;
  ca.xt = xt;
  ca.l = l_cap;
  ca.K = K;
  ca.split = 1;
  ca.mu_out = mu;
  ca.energy = 0;
  ca.ws = w.base;
  ca.lay = &w.lay;
  ca.seg = seg;
  ca.chunk_expert = chunk_expert;
  ca.totals = totals;
  ca.c_max = c_max;
  AVR_TRY(cuda_status(launch_colreduce(ca, s, true)));
  MoeQuantArgs qa = {};
  qa.X = X;
  qa.xt = xt;
  qa.l_cap = l_cap;
  qa.K = K;
  qa.E = E;
  qa.seg = seg;
  qa.block_expert = block_expert;
  qa.totals = totals;
  qa.mu = mu;
  qa.slot_xr = w.slot_xr();
  qa.slot_mu = w.slot_mu();
  qa.codes = xr_q->codes;
  qa.scales = xr_q->scales;
  qa.g_dec = xr_q->g_dec;
  if (mu_q) {
    qa.mu_codes = mu_q->codes;
    qa.mu_scales = mu_q->scales;
    qa.mu_gdec = mu_q->g_dec;
  }
  qa.seed = seed;
  qa.offset = offset;
  qa.tag = tag;
  qa.tag_mu = tag_mu;
  qa.sr = rm == AVR_SR;
  qa.status = w.status();
  return cuda_status(launch_moe_quant(qa, s, true));
}

size_t averis_moe_workspace_size(int64_t l_cap, int64_t K, int64_t N, int E) {
  if (!moe_shape_ok(l_cap, E, K) || N < 0) return 0;
  return moe_layout(l_cap, K, N, E).total;
}

avr_status averis_moe_split_quant(const void* X, avr_dtype xt, int64_t l_cap, const int32_t* counts, int E,
                                  int64_t K, avr_round rm, uint64_t seed, uint64_t offset, int grad, float* mu,
                                  const avr_nvfp4* mu_q, const avr_nvfp4* xr_q, void* ws, size_t ws_bytes,
                                  avr_stream stream) {
  if (!dtype_ok(xt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!moe_shape_ok(l_cap, E, K)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (!X || !counts || !xr_q || !xr_q->g_dec) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(xr_q, l_cap, K));
  if (mu_q) AVR_TRY(check_nvfp4(mu_q, E, K));
  if (!aligned16(X) || !aligned16(mu) || (reinterpret_cast<uintptr_t>(counts) & 3u)) return AVR_ERR_MISALIGNED;
  MoeLayout lay;
  Ws w;
  AVR_TRY(make_moe_ws(ws, ws_bytes, l_cap, K, 0, E, &lay, &w));
  AVR_TRY(device_ok());
  if (l_cap == 0) return AVR_OK;
  return moe_split_chain(X, xt, l_cap, counts, E, K, rm, seed, offset, grad ? 3u : 1u, grad ? 4u : 2u,
                         mu ? mu : w.at<float>(lay.mu), mu_q, xr_q, w, lay, stream);
}

avr_status averis_moe_quant_weights(const void* W, avr_dtype wt, int E, int64_t m, int64_t n,
                                    const avr_nvfp4* w_fwd, const avr_nvfp4* w_dgrad, void* ws, size_t ws_bytes,
                                    avr_stream stream) {
  if (!W || !dtype_ok(wt) || E < 1 || E > 1024) return AVR_ERR_INVALID_ARG;
  if (!k_ok(m) || !k_ok(n) || m % 128 || n % 128) return AVR_ERR_UNSUPPORTED_SHAPE;
  AVR_TRY(check_nvfp4(w_fwd, static_cast<int64_t>(E) * n, m));
  AVR_TRY(check_nvfp4(w_dgrad, static_cast<int64_t>(E) * m, n));
  const size_t elem = wt == AVR_BF16 ? 2 : 4;
  for (int e = 0; e < E; ++e) {
    // expert e's slices: its W [m, n], rows e n .. of W_bar_fwd, e m .. of W_bar_dgrad
    const avr_nvfp4 f = {w_fwd->codes + static_cast<size_t>(e) * n * (m / 2),
                         w_fwd->scales + static_cast<size_t>(e) * scales_bytes(n, m), w_fwd->g_dec + e, n, m};
    const avr_nvfp4 d = {w_dgrad->codes + static_cast<size_t>(e) * m * (n / 2),
                         w_dgrad->scales + static_cast<size_t>(e) * scales_bytes(m, n), w_dgrad->g_dec + e, m, n};
    AVR_TRY(averis_quant_weight(static_cast<const char*>(W) + static_cast<size_t>(e) * m * n * elem, wt, m, n, &f,
                                &d, ws, ws_bytes, stream));
  }
  return AVR_OK;
}

static avr_status moe_linear(const void* X, avr_dtype xt, int64_t l_cap, const int32_t* counts, int E, int64_t K,
                             int64_t N, const avr_nvfp4* wq, avr_round rm, uint64_t seed, uint64_t offset,
                             uint32_t tag, uint32_t tag_mu, void* Y, avr_dtype yt, void* ws, size_t ws_bytes,
                             avr_stream stream) {
  if (!dtype_ok(xt) || !dtype_ok(yt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!moe_shape_ok(l_cap, E, K) || !n_ok(N) || N % 128) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (!X || !Y || !counts) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(wq, static_cast<int64_t>(E) * N, K));
  if (!aligned16(X) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(counts) & 3u)) return AVR_ERR_MISALIGNED;
  MoeLayout lay;
  Ws w;
  AVR_TRY(make_moe_ws(ws, ws_bytes, l_cap, K, N, E, &lay, &w));
  AVR_TRY(device_ok());
  if (l_cap == 0) return AVR_OK;
  const avr_nvfp4 xr = {w.at<uint8_t>(lay.xr_codes), w.at<uint8_t>(lay.xr_scales), w.at<float>(lay.xr_gdec),
                        l_cap, K};
  const avr_nvfp4 muq = {w.at<uint8_t>(lay.mu_codes), w.at<uint8_t>(lay.mu_scales), w.at<float>(lay.mu_gdec),
                         E, K};
  AVR_TRY(moe_split_chain(X, xt, l_cap, counts, E, K, rm, seed, offset, tag, tag_mu, w.at<float>(lay.mu), &muq,
                          &xr, w, lay, stream));
  MoeBiasArgs ba;
  ba.seg = w.at<MoeSeg>(lay.seg);
  ba.totals = w.at<int32_t>(lay.totals);
  ba.E = E;
  ba.K = K;
  ba.N = N;
  ba.mu_codes = muq.codes;
  ba.mu_scales = muq.scales;
  ba.mu_gdec = muq.g_dec;
  ba.w_codes = wq->codes;
  ba.w_scales = wq->scales;
  ba.w_gdec = wq->g_dec;
  ba.bias = w.at<float>(lay.bias);
  AVR_TRY(cuda_status(launch_moe_bias(ba, stream, true)));
  GemmArgs g;
  g.a_codes = xr.codes;
  g.a_scales = xr.scales;
  g.a_gdec = xr.g_dec;
  g.b_codes = wq->codes;
  g.b_scales = wq->scales;
  g.b_gdec = wq->g_dec;
  g.M = l_cap;
  g.N = N;
  g.K = K;
  g.bias = ba.bias;
  g.Y = Y;
  g.yt = yt;
  g.status = w.status();
  g.groups = E;
  g.block_expert = w.at<int32_t>(lay.block_expert);
  g.totals = ba.totals;
  return cuda_status(launch_gemm(g, stream, true));
}

avr_status averis_moe_linear_fwd(const void* X, avr_dtype xt, int64_t l_cap, const int32_t* counts, int E,
                                 int64_t m, int64_t n, const avr_nvfp4* w_fwd, avr_round rm, uint64_t seed,
                                 uint64_t offset, void* Y, avr_dtype yt, void* ws, size_t ws_bytes,
                                 avr_stream stream) {
  return moe_linear(X, xt, l_cap, counts, E, m, n, w_fwd, rm, seed, offset, 1u, 2u, Y, yt, ws, ws_bytes, stream);
}

avr_status averis_moe_linear_dgrad(const void* D, avr_dtype dt, int64_t l_cap, const int32_t* counts, int E,
                                   int64_t m, int64_t n, const avr_nvfp4* w_dgrad, avr_round rm, uint64_t seed,
                                   uint64_t offset, void* dX, avr_dtype xt, void* ws, size_t ws_bytes,
                                   avr_stream stream) {
  return moe_linear(D, dt, l_cap, counts, E, n, m, w_dgrad, rm, seed, offset, 3u, 4u, dX, xt, ws, ws_bytes, stream);
}

avr_status averis_probe_convert(const float* in, uint8_t* e4m3, uint8_t* e2m1, int64_t n,
                                avr_stream stream) {
  if (!in || n < 0) return AVR_ERR_INVALID_ARG;
  if (n == 0) return AVR_OK;
  AVR_TRY(device_ok());
  return cuda_status(launch_probe_convert(in, e4m3, e2m1, n, stream));
}

avr_status averis_probe_convert_sr(const float* in, const uint32_t* rbits, uint16_t* out, int64_t n,
                                   avr_stream stream) {
  if (!in || !rbits || !out || n < 0) return AVR_ERR_INVALID_ARG;
  if (!aligned16(in) || (reinterpret_cast<uintptr_t>(rbits) & 3u) || (reinterpret_cast<uintptr_t>(out) & 1u))
    return AVR_ERR_MISALIGNED;
  if (n == 0) return AVR_OK;
  AVR_TRY(device_ok());
  return cuda_status(launch_probe_convert_sr(in, rbits, out, n, stream));
}

avr_status averis_probe_mma_rate(int iters, int grid, uint64_t* ns, void* ws, size_t ws_bytes, avr_stream stream) {
  if (iters < 1 || grid < 1 || !ns) return AVR_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ns) & 7u) return AVR_ERR_MISALIGNED;
  Ws w;
  AVR_TRY(make_ws(ws, ws_bytes, 0, 64, 0, &w));
  AVR_TRY(device_ok());
  return cuda_status(launch_mma_rate(iters, grid, ns, w.status(), stream));
}

avr_status averis_probe_philox(uint64_t seed, uint64_t offset, uint32_t tag, int64_t n,
                               uint32_t* out, avr_stream stream) {
  if (!out || n < 0) return AVR_ERR_INVALID_ARG;
  if (!aligned16(out)) return AVR_ERR_MISALIGNED;
  if (n == 0) return AVR_OK;
  AVR_TRY(device_ok());
  return cuda_status(launch_probe_philox(seed, offset, tag, n, out, stream));
}

}  // extern "C"
