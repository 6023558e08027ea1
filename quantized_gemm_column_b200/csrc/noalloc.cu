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
// name as a device address; the address is looked up with
// cudaGetSymbolAddress (with the device current) on the first call in each
// device context and reused while that context lives.  A cudaDeviceReset
// ends the context and its module, so the next call looks the address up
// again instead of writing through a stale one.
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace avr {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The unique ID of the calling thread's current context (false if none is
// current yet, or the driver lacks the call).
static bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

static avr_status noalloc_scratch(void** out) {
  struct Entry {
    unsigned long long ctx;
    void* ptr;
  };
  static std::mutex mu;
  static Entry cache[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AVR_ERR_NO_DEVICE;
  if (dev < 0 || dev >= 256) return AVR_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> g(mu);
  unsigned long long ctx = 0;
  if (cache[dev].ptr == nullptr || !current_context_id(&ctx) || ctx != cache[dev].ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return AVR_ERR_CUDA;
    // the lookup made the device's context current, so its ID exists now
    if (!current_context_id(&ctx)) return AVR_ERR_CUDA;
    cache[dev].ctx = ctx;
    cache[dev].ptr = p;
  }
  *out = cache[dev].ptr;
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
  // the same checks, in the same order, as averis_split_quant
  if (!dtype_ok(xt) || !round_ok(rm)) return AVR_ERR_INVALID_ARG;
  if (!k_ok(K) || !l_ok(l)) return AVR_ERR_UNSUPPORTED_SHAPE;
  if (l == 0) return AVR_OK;   // no tokens: nothing is read or written
  if (!X) return AVR_ERR_INVALID_ARG;
  AVR_TRY(check_nvfp4(xr_q, l, K));
  if (mu_q) AVR_TRY(check_nvfp4(mu_q, 1, K));
  if (!aligned16(X) || !aligned16(mu) || !aligned16(xr_debug) ||
      (reinterpret_cast<uintptr_t>(device_status) & 3u))
    return AVR_ERR_MISALIGNED;

  // The reduce needs the status word, tickets, amax slots, chunk partials and
  // the mean: everything in the workspace layout before the mean's codes.
  Ws w;
  w.lay = ws_layout(l, K, 0);
  if (w.lay.mu_codes > kNoAllocScratchBytes) return AVR_ERR_WORKSPACE_TOO_SMALL;
  AVR_TRY(device_ok());
  void* scratch = nullptr;
  AVR_TRY(noalloc_scratch(&scratch));
  w.base = static_cast<char*>(scratch);
  cudaStream_t s = stream;

  // The array keeps the previous call's contents: the status word and the
  // tickets must start at zero (slots, partials and mean are written before
  // they are read).
  if (cudaMemsetAsync(w.base, 0, w.lay.slots, s) != cudaSuccess) return AVR_ERR_CUDA;
  float* mu_buf = mu ? mu : w.at<float>(w.lay.mu);
  AVR_TRY(split_chain(X, xt, l, K, 1, rm, seed, offset, grad ? 3u : 1u, grad ? 4u : 2u, mu_buf, mu_q, xr_q,
                      xr_debug, nullptr, nullptr, w, s, false, false));
  if (device_status) {
    forward_status<<<1, 1, 0, s>>>(w.status(), device_status);
    if (cudaGetLastError() != cudaSuccess) return AVR_ERR_CUDA;
  }
  return AVR_OK;
}
