// averis_split_quant_noalloc: the split quantizer for callers that cannot
// hand the library a workspace.
//
// Some callers have no way to allocate device memory at the point where
// they quantize: a plugin that receives only its input and output pointers
// from a host framework that owns every allocation, or latency-critical code
// that must not call cudaMalloc/cudaFree, which synchronize the device and
// can stall every stream.  This entry point keeps the column reduce's scratch
// (status word, tickets, amax slots, chunk partials, the mean) in a
// fixed-size array that lives in the library's own module, so the caller
// passes only inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it (kNoAllocScratchBytes) until the process exits, and every
// call shares it, so two calls that overlap on the GPU (for example on two
// streams) race and must not be issued.  Host code cannot use the array's
// name as a device address; the first call on each device looks the address
// up with cudaGetSymbolAddress (with that device current) and reuses it.
#include <mutex>

#include "internal.h"

namespace avr {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static avr_status noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* ptr[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AVR_ERR_NO_DEVICE;
  if (dev < 0 || dev >= 256) return AVR_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> g(mu);
  if (ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return AVR_ERR_CUDA;
    ptr[dev] = p;
  }
  *out = ptr[dev];
  return AVR_OK;
}

// Forward the first error latched in the scratch status word to the caller's.
__global__ void forward_status(const uint32_t* scratch_status, uint32_t* caller_status) {
  const uint32_t s = *scratch_status;
  if (s != 0u) atomicCAS(caller_status, 0u, s);
}

}  // namespace avr

using namespace avr;

extern "C" avr_status averis_split_quant_noalloc(const void* X, avr_dtype xt, int64_t l, int64_t K,
                                                 avr_round rm, uint64_t seed, uint64_t offset,
                                                 int grad, float* mu, const avr_nvfp4* mu_q,
                                                 const avr_nvfp4* xr_q, float* xr_debug,
                                                 uint32_t* device_status, avr_stream stream) {
  if (!(xt == AVR_F32 || xt == AVR_BF16) || !(rm == AVR_RNE || rm == AVR_SR)) return AVR_ERR_INVALID_ARG;
  if (K <= 0 || K % 64 != 0 || K > int64_t{kColTile} * kMaxColTiles || l < 0 || l > INT32_MAX)
    return AVR_ERR_UNSUPPORTED_SHAPE;
  if (l == 0) return AVR_OK;
  if (!X || !xr_q || !xr_q->codes || !xr_q->scales || !xr_q->g_dec) return AVR_ERR_INVALID_ARG;
  if (xr_q->rows != l || xr_q->K != K) return AVR_ERR_INVALID_ARG;
  if (mu_q && (!mu_q->codes || !mu_q->scales || !mu_q->g_dec || mu_q->rows != 1 || mu_q->K != K))
    return AVR_ERR_INVALID_ARG;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(X) || !a16(mu) || !a16(xr_debug) || !a16(xr_q->codes) || !a16(xr_q->scales) ||
      (mu_q && (!a16(mu_q->codes) || !a16(mu_q->scales))) ||
      (reinterpret_cast<uintptr_t>(device_status) & 3u))
    return AVR_ERR_MISALIGNED;

  // The reduce needs the status word, tickets, amax slots, chunk partials and
  // the mean: everything in the workspace layout before the mean's codes.
  const WsLayout lay = ws_layout(l, K, 0);
  if (lay.mu_codes > kNoAllocScratchBytes) return AVR_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  avr_status st = noalloc_scratch(&scratch);
  if (st != AVR_OK) return st;
  char* base = static_cast<char*>(scratch);
  cudaStream_t s = stream;

  // The array keeps the previous call's contents: the status word and the
  // tickets must start at zero (slots, partials and mean are written before
  // they are read).
  if (cudaMemsetAsync(base, 0, lay.slots, s) != cudaSuccess) return AVR_ERR_CUDA;

  float* mu_buf = mu ? mu : reinterpret_cast<float*>(base + lay.mu);
  ColReduceArgs ca;
  ca.X = X;
  ca.xt = xt;
  ca.l = l;
  ca.K = K;
  ca.split = 1;
  ca.mu_out = mu_buf;
  ca.energy = 0;
  ca.ws = base;
  ca.lay = &lay;
  if (launch_colreduce(ca, s, false) != cudaSuccess) return AVR_ERR_CUDA;

  QuantArgs qa = {};
  qa.X = X;
  qa.xt = xt;
  qa.rows = l;
  qa.K = K;
  qa.mu = mu_buf;
  qa.n_tiles = static_cast<int>((K + kColTile - 1) / kColTile);
  qa.slot_xr = reinterpret_cast<float*>(base + lay.slots);
  qa.codes = xr_q->codes;
  qa.scales = xr_q->scales;
  qa.g_dec = xr_q->g_dec;
  qa.xr_debug = xr_debug;
  qa.seed = seed;
  qa.offset = offset;
  qa.tag = grad ? 3u : 1u;
  qa.sr = rm == AVR_SR;
  qa.status = reinterpret_cast<uint32_t*>(base + lay.status);
  qa.slot_mu = qa.slot_xr + kMaxColTiles;
  qa.tag_mu = grad ? 4u : 2u;
  if (mu_q) {
    qa.mu_codes = mu_q->codes;
    qa.mu_scales = mu_q->scales;
    qa.mu_gdec = mu_q->g_dec;
  }
  if (launch_quant(qa, s, false) != cudaSuccess) return AVR_ERR_CUDA;
  if (device_status) {
    forward_status<<<1, 1, 0, s>>>(reinterpret_cast<const uint32_t*>(base + lay.status), device_status);
    if (cudaGetLastError() != cudaSuccess) return AVR_ERR_CUDA;
  }
  return AVR_OK;
}
