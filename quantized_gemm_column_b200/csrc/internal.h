// Host-side interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/averis.h"

namespace avr {

constexpr int kChunkRows = 256;      // rows per partial of the fixed-order mean
constexpr int kColTile = 128;        // columns per column-reduce CTA
constexpr int kMaxColTiles = 4096;   // K <= 524288
constexpr int kStripCols = 512;      // columns per warp in the quantizer (16 per lane)

// Workspace layout (byte offsets, 256-aligned).  The status word and the
// per-column-tile tickets sit at fixed offsets whatever the sizes, so a
// workspace can be reused across shapes; everything after them is scratch
// that each call writes before it reads.
// The first 256 bytes of a workspace are its status block: the status word
// at 0, the one-kernel split's barrier counter and generation at 64 and 128,
// and at kWaitLimitOffset the bound (uint64 ns, 0 = the default 2 s) of the
// waits on other CTAs.
constexpr size_t kWaitLimitOffset = 192;

struct WsLayout {
  size_t status = 0;
  size_t tickets = 256;
  size_t slots = 256 + 4 * kMaxColTiles;           // float[2][kMaxColTiles]
  size_t partials = 0;                              // float[3][C][K]
  size_t mu = 0;                                    // float[K]
  size_t mu_codes = 0, mu_scales = 0, mu_gdec = 0;  // Q_4(mu), 1 x K
  size_t xr_gdec = 0;
  size_t bias = 0;                                  // float[N]
  size_t xr_codes = 0, xr_scales = 0;               // Q_4(X_R), l x K
  size_t energy_partials = 0, energy = 0;           // float[C][K], float[K]: the R monitor's sums of squares
  size_t total = 0;
};
WsLayout ws_layout(int64_t l, int64_t K, int64_t N);

// Weight-gradient workspace: the split's regions for K = max(m, n), then the
// four token-axis operands (L = l rounded up to 64), their decode scales and
// the rank-one factors u [m], v [n].
int64_t padded_tokens(int64_t l);
struct WgLayout {
  WsLayout base;
  size_t xt_codes = 0, xt_scales = 0, dt_codes = 0, dt_scales = 0;
  size_t mux_codes = 0, mux_scales = 0, mud_codes = 0, mud_scales = 0;
  size_t gdec = 0;        // float[4]: X_R^T, D_R^T, mu_bar_X, mu_bar_D
  size_t u = 0, v = 0;
  size_t total = 0;
};
WgLayout wgrad_layout(int64_t l, int64_t m, int64_t n);

size_t scales_bytes(int64_t rows, int64_t K);

// ---------------- K1: fixed-order column reduce ----------------
// One expert's segment of a token buffer permuted by expert (MoE): rows
// [row0, row0 + rows) of the buffer, its chunks of 256 rows numbered
// chunk0 .. chunk0 + chunks - 1 among all experts' chunks.
struct MoeSeg {
  int32_t row0, rows, chunk0, chunks;
};

struct ColReduceArgs {
  const void* X;
  avr_dtype xt;
  int64_t l, K;
  int split;              // 1: mean + residual amax; 0: amax of X only (vanilla)
  float* mu_out;          // [K] ([E][K] grouped), written when split (nullable otherwise)
  int energy;             // 1: also the column sums of squares (the R monitor)
  char* ws;               // workspace base
  const WsLayout* lay;
  // grouped (MoE) mode, null for a dense matrix: per-expert segments, the
  // expert of every chunk, the number of chunks in use; c_max chunks launched
  const MoeSeg* seg = nullptr;
  const int32_t* chunk_expert = nullptr;
  const int32_t* totals = nullptr;
  int c_max = 0;
};
cudaError_t launch_colreduce(const ColReduceArgs& a, cudaStream_t s, bool pdl);

// R = ||mu|| / sqrt(E||x||^2 / m) from mu [K] and the column sums of squares [K]
cudaError_t launch_energy_ratio(const float* mu, const float* energy, int64_t K, int64_t l, float* R,
                                uint32_t* status, cudaStream_t s, bool pdl);

// ---------------- K2: split quantizer (+ mean quantizer, rank-one row) ----------------
struct QuantArgs {
  const void* X;
  avr_dtype xt;
  int64_t rows, K;
  const float* mu;          // [K] subtracted from every row; NULL = vanilla
  int n_tiles;              // column tiles whose amax slots hold max |X_R|
  const float* slot_xr;     // [n_tiles]
  uint8_t* codes;
  uint8_t* scales;
  float* g_dec;
  float* xr_debug;          // nullable
  uint64_t seed, offset;
  uint32_t tag;
  int sr;
  uint32_t* status;
  // mean quantization and rank-one row (run by extra CTAs when mu != NULL)
  const float* slot_mu;     // [n_tiles] max |mu| per tile
  uint32_t tag_mu;
  uint8_t* mu_codes;        // nullable: where Q_4(mu) is stored
  uint8_t* mu_scales;
  float* mu_gdec;
  const uint8_t* w_codes;   // nullable: no rank-one row
  const uint8_t* w_scales;
  const float* w_gdec;
  int64_t n_out;            // rows of w = entries of bias
  float* bias;
};
cudaError_t launch_quant(const QuantArgs& a, cudaStream_t s, bool pdl);

// zero the scale bytes of the padding rows [rows, next multiple of 128) (no-op when rows % 128 == 0)
cudaError_t launch_zero_scale_padding(uint8_t* scales, int64_t rows, int64_t K, cudaStream_t s);

// K1 + K2 as one persistent kernel (one CTA per SM, grid-wide barriers): the
// same outputs as launch_colreduce followed by launch_quant, without the
// X_R debug output or the monitor's sums of squares.
cudaError_t launch_split_fused(const ColReduceArgs& ca, const QuantArgs& qa, cudaStream_t s, bool pdl);

// The same split quantized along the tokens (a.rows = l tokens, a.K
// features): codes [K][L/2] and scales of a K x L tensor, L = l rounded up to
// 64, zero padding.  xr_debug and the rank-one row (w_*) are not used.
cudaError_t launch_quant_tokens(const QuantArgs& a, cudaStream_t s, bool pdl);

// ---------------- mixture of experts (moe.cu) ----------------
// segment table from the per-expert token counts (device), see moe.cu
cudaError_t launch_moe_table(const int32_t* counts, int E, int64_t l_cap, int c_max, MoeSeg* seg,
                             int32_t* chunk_expert, int32_t* block_expert, int32_t* totals, uint32_t* status,
                             cudaStream_t s, bool pdl);

struct MoeQuantArgs {
  const void* X;
  avr_dtype xt;
  int64_t l_cap, K;
  int E;
  const MoeSeg* seg;
  const int32_t* block_expert;
  const int32_t* totals;
  const float* mu;              // [E][K] (null: vanilla)
  const float* slot_xr;         // [E][T] (T = K / 128 rounded up)
  const float* slot_mu;
  uint8_t* codes;               // [l_cap][K/2]
  uint8_t* scales;
  float* g_dec;                 // [E]
  uint8_t* mu_codes;            // [E][K/2] (null: no mean quantization)
  uint8_t* mu_scales;
  float* mu_gdec;               // [E]
  uint64_t seed, offset;
  uint32_t tag, tag_mu;
  int sr;
  uint32_t* status;
};
cudaError_t launch_moe_quant(const MoeQuantArgs& a, cudaStream_t s, bool pdl);

struct MoeBiasArgs {
  const MoeSeg* seg;
  const int32_t* totals;
  int E;
  int64_t K, N;                 // mean length; output features per expert
  const uint8_t* mu_codes;      // [E][K/2] with scales and mu_gdec [E]
  const uint8_t* mu_scales;
  const float* mu_gdec;
  const uint8_t* w_codes;       // [E * N][K/2], experts stacked
  const uint8_t* w_scales;
  const float* w_gdec;          // [E]
  float* bias;                  // [E][N]
};
cudaError_t launch_moe_bias(const MoeBiasArgs& a, cudaStream_t s, bool pdl);

// u = l * deq(mu_bar_X) [m], v = deq(mu_bar_D) [n]
cudaError_t launch_mean_dequant(const uint8_t* codes_x, const uint8_t* scales_x, const float* gdec_x, int64_t m,
                                const uint8_t* codes_d, const uint8_t* scales_d, const float* gdec_d, int64_t n,
                                int64_t l, float* u, float* v, cudaStream_t s, bool pdl);

// Q_4 of T = W^T for W [m, n] (T [n, m], blocks along m), round to nearest even.
struct QuantTransposedArgs {
  const void* W;
  avr_dtype wt;
  int64_t m, n;
  int n_tiles;
  const float* slot_amax;
  uint8_t* codes;
  uint8_t* scales;
  float* g_dec;
};
cudaError_t launch_quant_transposed(const QuantTransposedArgs& a, cudaStream_t s);

// rank-one row only
struct BiasArgs {
  const uint8_t* mu_codes;
  const uint8_t* mu_scales;
  const float* mu_gdec;
  const uint8_t* w_codes;
  const uint8_t* w_scales;
  const float* w_gdec;
  int64_t K, n_out;
  float* bias;
};
cudaError_t launch_bias(const BiasArgs& a, cudaStream_t s);

// ---------------- K3: tcgen05 block-scaled FP4 GEMM ----------------
struct GemmArgs {
  const uint8_t* a_codes;
  const uint8_t* a_scales;
  const float* a_gdec;
  const uint8_t* b_codes;
  const uint8_t* b_scales;
  const float* b_gdec;
  int64_t M, N, K;
  const float* bias;   // nullable
  const float* row_scale = nullptr;   // nullable: Y = alpha acc + row_scale[i] * bias[j] (rank-one term)
  // grouped (MoE): B holds `groups` experts' [N, K] matrices stacked; a_gdec,
  // b_gdec and bias are per expert; A's 128-row blocks map to experts through
  // block_expert, and totals[1] rows are in use (null: one GEMM)
  int64_t groups = 1;
  const int32_t* block_expert = nullptr;
  const int32_t* totals = nullptr;
  void* Y;
  avr_dtype yt;
  uint32_t* status;
};
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, bool pdl);
// the 2-CTA kernel (gemm2.cu): dense bf16 outputs, 256 x 256 tiles on CTA pairs
bool gemm_pair_applies(const GemmArgs& a);
cudaError_t launch_gemm_pair(const GemmArgs& a, cudaStream_t s, bool pdl);
// the short-contraction pair kernel (K <= 1024; B's column block resident)
bool gemm_pair_short_applies(const GemmArgs& a);
cudaError_t launch_gemm_pair_short(const GemmArgs& a, cudaStream_t s, bool pdl);
// tensor maps of the pair kernels: codes as (128 bytes, rows, K/256 chunks),
// scale atoms as (256 x 8 bytes, K/256 chunks, row groups of 128)
bool pair_codes_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K, uint32_t box_rows, uint32_t box_chunks);
bool pair_scales_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K, uint32_t box_chunks,
                     uint32_t box_groups);

// ---------------- host-side validation and the split chain (api.cu) ----------------
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool dtype_ok(avr_dtype t) { return t == AVR_F32 || t == AVR_BF16; }
inline bool round_ok(avr_round r) { return r == AVR_RNE || r == AVR_SR; }
constexpr int64_t kMaxDim = (int64_t{1} << 31) - 1;
inline bool k_ok(int64_t K) { return K > 0 && K % 64 == 0 && K <= int64_t{kColTile} * kMaxColTiles; }
inline bool l_ok(int64_t l) { return l >= 0 && l <= kMaxDim; }
inline bool n_ok(int64_t N) { return N > 0 && N % 64 == 0 && N <= kMaxDim; }
inline avr_status cuda_status(cudaError_t e) { return e == cudaSuccess ? AVR_OK : AVR_ERR_CUDA; }

#define AVR_TRY(expr)                  \
  do {                                 \
    avr_status st_ = (expr);           \
    if (st_ != AVR_OK) return st_;     \
  } while (0)

// AVR_OK when the current device is an sm_100 part, else AVR_ERR_NO_DEVICE
avr_status device_ok();
// an NVFP4 descriptor of `rows` x K: non-null parts, matching shape, codes and
// scales 16-byte aligned, g_dec 4-byte aligned
avr_status check_nvfp4(const avr_nvfp4* t, int64_t rows, int64_t K);

// a workspace (or any scratch laid out like one) and its regions
struct Ws {
  char* base;
  WsLayout lay;
  uint32_t* status() const { return reinterpret_cast<uint32_t*>(base + lay.status); }
  float* slot_xr() const { return reinterpret_cast<float*>(base + lay.slots); }
  float* slot_mu() const { return slot_xr() + kMaxColTiles; }
  template <typename T>
  T* at(size_t off) const { return reinterpret_cast<T*>(base + off); }
};

// K1 + K2 on `ws` (+ mean quantizer and rank-one row when mu_q / w are
// given); fused: the one-kernel split; pdl: chain the launches with
// programmatic dependent launch
avr_status split_chain(const void* X, avr_dtype xt, int64_t l, int64_t K, int split, avr_round rm,
                       uint64_t seed, uint64_t offset, uint32_t tag, uint32_t tag_mu, float* mu_buf,
                       const avr_nvfp4* mu_q, const avr_nvfp4* xr_q, float* xr_debug, const avr_nvfp4* w,
                       float* bias, const Ws& ws, cudaStream_t s, bool fused = false, bool pdl = true);

// ---------------- diagnostics ----------------
cudaError_t launch_probe_convert(const float* in, uint8_t* e4m3, uint8_t* e2m1, int64_t n,
                                 cudaStream_t s);
cudaError_t launch_probe_convert_sr(const float* in, const uint32_t* rbits, uint16_t* out, int64_t n,
                                    cudaStream_t s);
cudaError_t launch_mma_rate(int iters, int grid, uint64_t* ns, uint32_t* status, cudaStream_t s);
cudaError_t launch_probe_philox(uint64_t seed, uint64_t offset, uint32_t tag, int64_t n,
                                uint32_t* out, cudaStream_t s);

// ---------------- tensor maps ----------------
// 2-D row-major tensor [rows, cols] of elem_bytes-sized elements.
bool make_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                        int elem_bytes, uint64_t rows, uint64_t cols, uint32_t box_rows,
                        uint32_t box_cols, CUtensorMapSwizzle swizzle);

// 3-D tensor of elem-sized elements: dims[0] contiguous, byte strides of
// dims 1 and 2.
bool make_tensor_map_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, const uint64_t dims[3],
                        const uint64_t strides[2], const uint32_t box[3],
                        CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE);

// cudaFuncAttributeMaxDynamicSharedMemorySize for the current device (set
// once per device and function).
cudaError_t set_max_dynamic_smem(const void* func, size_t bytes);

// Resident CTAs per SM of `func` with this block size and dynamic shared
// memory on the current device (cached).
int blocks_per_sm(const void* func, int threads, size_t smem);

// Streaming multiprocessors of the current device.
int sm_count();

// launch with the programmatic-stream-serialization attribute when pdl
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t s, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace avr
