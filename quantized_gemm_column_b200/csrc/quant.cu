// K2: the split quantizer -- the "subtract" and Q_4 of the Averis split.
//
// X_bar_R = Q_4(X - 1 mu_X) and mu_bar_X = Q_4(mu_X) (Lighthouse review of
// "The Curse and Blessing of Mean Bias in FP4-Quantized LLM Training",
// section 二 "Averis 方法"), with Q_4 the E2M1 NVFP4 quantizer, stochastic
// rounding by default (section 三 3.1).  Per 16-element block along K:
//   x_R = fl(x - mu_j); a = max |x_R|; S = E4M3(fl(fl(a / 6) * g_enc));
//   r = g_enc / value(S) (0 if S = 0); y = fl(x_R * r); code = E2M1(y)
// with g_enc = 2688 / amax(X_R) from the column reduce.  The codes are
// packed two per byte and the scales written straight into the tcgen05
// 128x4 scale-atom layout, so the GEMM consumes them without any reshuffle.
//
// Work split: a warp owns a 256-column strip and walks rows; lane i holds 8
// consecutive columns (one 16-byte bf16 load), so a lane pair is one block
// (amax by one shuffle), eight lanes are one 4-scale atom word, and one
// Philox4x32-10 call gives the 8 x 16 random bits of the lane's elements.
// Extra CTAs at the end of the grid quantize mu and form the rank-one row
// mu_bar W_bar that the GEMM adds as a bias.
#include "device.cuh"
#include "internal.h"

namespace avr {

constexpr int kQuantThreads = 256;
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kRowsPerCta = 32;            // rows per CTA (4 per warp)
constexpr int kBiasRowsPerCta = 64;        // rank-one-row outputs per extra CTA

struct QuantParams {
  const void* X;
  int64_t rows, K;
  const float* mu;
  int n_tiles;
  const float* slot_xr;
  uint8_t* codes;
  uint8_t* scales;
  float* g_dec;
  float* xr_debug;
  uint64_t seed, offset;
  uint32_t tag;
  uint32_t* status;
  int n_strips;
  int n_quant_ctas;
  // extra CTAs
  const float* slot_mu;
  uint32_t tag_mu;
  uint8_t* mu_codes;
  uint8_t* mu_scales;
  float* mu_gdec;
  const uint8_t* w_codes;
  const uint8_t* w_scales;
  const float* w_gdec;
  int64_t n_out;
  float* bias;
};

__device__ __forceinline__ float max_of_slots(const float* slots, int n) {
  float a = 0.0f;
  for (int i = threadIdx.x & 31; i < n; i += 32) a = fmaxf(a, __ldcg(slots + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  return a;
}

// Load 8 consecutive elements as fp32.
template <bool kBf16>
__device__ __forceinline__ void load8(const void* base, int64_t idx, bool active, float (&x)[8]) {
  if (kBf16) {
    uint4 w = make_uint4(0, 0, 0, 0);
    if (active) w = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + idx));
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
    x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
    x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
  } else {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (active) {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
      a = __ldcs(p);
      b = __ldcs(p + 1);
    }
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

// Quantize the 8 values of this lane (its lane pair forms one 16-block).
// Returns the packed codes (8 nibbles) and the block's scale code in *S.
template <bool kSR>
__device__ __forceinline__ uint32_t quant8(const float (&xr)[8], float g_enc, uint64_t seed,
                                           uint64_t offset, uint32_t tag, uint64_t elem0,
                                           uint32_t* S_out, float* rscale_out) {
  float am = 0.0f;
#pragma unroll
  for (int t = 0; t < 8; ++t) am = fmaxf(am, fabsf(xr[t]));
  am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
  const uint32_t S = e4m3_rn_satfinite(__fmul_rn(__fdiv_rn(am, 6.0f), g_enc));
  const float r = S == 0u ? 0.0f : __fdiv_rn(g_enc, e4m3_value(S));
  float y[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) y[t] = __fmul_rn(xr[t], r);
  uint32_t packed = 0;
  if (kSR) {
    const uint4 rnd = philox_block(seed, offset, tag, elem0 >> 3);
    const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint32_t r16 = (w[t >> 1] >> ((t & 1) * 16)) & 0xFFFFu;
      packed |= e2m1_sr(y[t], r16) << (4 * t);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) packed |= e2m1x2_rn(y[2 * k], y[2 * k + 1]) << (8 * k);
  }
  *S_out = S;
  if (rscale_out) *rscale_out = e4m3_value(S);
  return packed;
}

// Lane 8q gathers the scale codes of lanes 8q, 8q+2, 8q+4, 8q+6 (four
// consecutive blocks) into one little-endian word.
__device__ __forceinline__ uint32_t gather_scale_word(uint32_t S) {
  const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, S, 2);
  const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, S, 4);
  const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, S, 6);
  return S | (s1 << 8) | (s2 << 16) | (s3 << 24);
}

// sum_k mu_val[k] * value(w)[j, k] for the rows j of this warp; mu_val holds
// e2m1 * e4m3 of mu (tensor scale applied by the caller).
__device__ void bias_rows(const float* s_mu, int64_t K, const uint8_t* w_codes,
                          const uint8_t* w_scales, float g_dec_prod, int64_t j_begin,
                          int64_t j_end, float* bias) {
  const int lane = threadIdx.x & 31;
  const uint32_t n_kb64 = static_cast<uint32_t>(K / 64);
  for (int64_t j = j_begin; j < j_end; ++j) {
    float acc = 0.0f;
    for (int64_t k0 = static_cast<int64_t>(lane) * 32; k0 < K; k0 += 32 * 32) {
      const uint4 cw = __ldg(reinterpret_cast<const uint4*>(w_codes + j * (K / 2) + k0 / 2));
      const uint32_t c16 = static_cast<uint32_t>(k0 / 16);
      const float s0 = e4m3_value(__ldg(w_scales + scale_offset(j, c16, n_kb64)));
      const float s1 = e4m3_value(__ldg(w_scales + scale_offset(j, c16 + 1, n_kb64)));
      const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float sc = q < 2 ? s0 : s1;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float wv = e2m1_value((words[q] >> (4 * t)) & 0xFu) * sc;
          acc = fmaf(wv, s_mu[k0 + q * 8 + t], acc);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) bias[j] = acc * g_dec_prod;
  }
}

template <bool kSR>
__device__ void mean_and_bias_block(const QuantParams& p, int e, float* s_mu) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TensorScale ts = tensor_scale(max_of_slots(p.slot_mu, p.n_tiles));
  const uint32_t n_kb64 = static_cast<uint32_t>(p.K / 64);
  const bool writer = (e == 0) && p.mu_codes != nullptr;
  if (writer) {
    if (threadIdx.x == 0) *p.mu_gdec = ts.g_dec;
    // zero the padding rows 1..127 of every scale atom (row 0 is written below)
    uint32_t* w = reinterpret_cast<uint32_t*>(p.mu_scales);
    const int64_t n_words = static_cast<int64_t>(n_kb64) * 128;
    for (int64_t i = threadIdx.x; i < n_words; i += kQuantThreads)
      if ((i & 127) != 0) w[i] = 0u;
  }
  for (int strip = warp; strip < p.n_strips; strip += kQuantWarps) {
    const int64_t col0 = static_cast<int64_t>(strip) * kStripCols + lane * 8;
    const bool active = col0 < p.K;
    float x[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) x[t] = active ? __ldcg(p.mu + col0 + t) : 0.0f;
    uint32_t S;
    float sv;
    const uint32_t packed = quant8<kSR>(x, ts.g_enc, p.seed, p.offset, p.tag_mu,
                                        static_cast<uint64_t>(col0), &S, &sv);
    const uint32_t sw = gather_scale_word(S);
    if (active) {
      if (writer) {
        *reinterpret_cast<uint32_t*>(p.mu_codes + col0 / 2) = packed;
        if ((lane & 7) == 0)
          *reinterpret_cast<uint32_t*>(p.mu_scales + scale_offset(0, static_cast<uint32_t>(col0 / 16), n_kb64)) = sw;
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) s_mu[col0 + t] = e2m1_value((packed >> (4 * t)) & 0xFu) * sv;
    }
  }
  __syncthreads();
  if (p.w_codes == nullptr) return;
  const float gprod = ts.g_dec * __ldg(p.w_gdec);
  const int64_t j0 = static_cast<int64_t>(e) * kBiasRowsPerCta;
  const int64_t per_warp = kBiasRowsPerCta / kQuantWarps;
  const int64_t jb = j0 + warp * per_warp;
  const int64_t je = min64(jb + per_warp, p.n_out);
  if (jb < je) bias_rows(s_mu, p.K, p.w_codes, p.w_scales, gprod, jb, je, p.bias);
}

template <bool kBf16, bool kSR>
__global__ void __launch_bounds__(kQuantThreads) quant_kernel(const QuantParams p) {
  extern __shared__ float s_mu[];   // extra CTAs only: dequantized mu (K floats)
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  if (static_cast<int>(blockIdx.x) >= p.n_quant_ctas) {
    mean_and_bias_block<kSR>(p, blockIdx.x - p.n_quant_ctas, s_mu);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TensorScale ts = tensor_scale(max_of_slots(p.slot_xr, p.n_tiles));
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.g_dec = ts.g_dec;

  const int strip = blockIdx.x % p.n_strips;
  const int64_t row_base = static_cast<int64_t>(blockIdx.x / p.n_strips) * kRowsPerCta;
  const int64_t col0 = static_cast<int64_t>(strip) * kStripCols + lane * 8;
  const bool active = col0 < p.K;
  const uint32_t n_kb64 = static_cast<uint32_t>(p.K / 64);

  float mu[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) mu[t] = (p.mu != nullptr && active) ? __ldcg(p.mu + col0 + t) : 0.0f;

  constexpr int kRowsPerWarp = kRowsPerCta / kQuantWarps;
  float x[kRowsPerWarp][8];
  bool rv[kRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int64_t r = row_base + warp + i * kQuantWarps;
    rv[i] = r < p.rows;
    load8<kBf16>(p.X, r * p.K + col0, active && rv[i], x[i]);
  }
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int64_t r = row_base + warp + i * kQuantWarps;
    float xr[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) xr[t] = __fsub_rn(x[i][t], mu[t]);
    uint32_t S;
    const uint32_t packed = quant8<kSR>(xr, ts.g_enc, p.seed, p.offset, p.tag,
                                        static_cast<uint64_t>(r * p.K + col0), &S, nullptr);
    const uint32_t sw = gather_scale_word(S);
    if (active && rv[i]) {
      *reinterpret_cast<uint32_t*>(p.codes + r * (p.K / 2) + col0 / 2) = packed;
      if ((lane & 7) == 0)
        *reinterpret_cast<uint32_t*>(p.scales + scale_offset(static_cast<uint64_t>(r),
                                                             static_cast<uint32_t>(col0 / 16), n_kb64)) = sw;
      if (p.xr_debug) {
        float4* d = reinterpret_cast<float4*>(p.xr_debug + r * p.K + col0);
        d[0] = make_float4(xr[0], xr[1], xr[2], xr[3]);
        d[1] = make_float4(xr[4], xr[5], xr[6], xr[7]);
      }
    }
  }
}

// Zero the scale bytes of the padding rows [rows, next multiple of 128).
__global__ void zero_scale_padding(uint8_t* scales, int64_t rows, int64_t K) {
  const int64_t pad0 = rows, pad1 = (rows + 127) / 128 * 128;
  const int64_t ncols = K / 16;
  const int64_t total = (pad1 - pad0) * ncols;
  const uint32_t n_kb64 = static_cast<uint32_t>(K / 64);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = pad0 + i / ncols;
    const uint32_t c = static_cast<uint32_t>(i % ncols);
    scales[scale_offset(static_cast<uint64_t>(r), c, n_kb64)] = 0;
  }
}

template <bool kBf16, bool kSR>
static cudaError_t launch_quant_t(const QuantParams& p, int n_extra, size_t smem, cudaStream_t s,
                                  bool pdl) {
  if (smem > 48 * 1024) {
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(quant_kernel<kBf16, kSR>), smem);
    if (e != cudaSuccess) return e;
  }
  return launch_ex(quant_kernel<kBf16, kSR>, dim3(p.n_quant_ctas + n_extra), dim3(kQuantThreads),
                   smem, s, pdl, p);
}

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t s, bool pdl) {
  QuantParams p = {};
  p.X = a.X;
  p.rows = a.rows;
  p.K = a.K;
  p.mu = a.mu;
  p.n_tiles = a.n_tiles;
  p.slot_xr = a.slot_xr;
  p.codes = a.codes;
  p.scales = a.scales;
  p.g_dec = a.g_dec;
  p.xr_debug = a.xr_debug;
  p.seed = a.seed;
  p.offset = a.offset;
  p.tag = a.tag;
  p.status = a.status;
  p.n_strips = static_cast<int>((a.K + kStripCols - 1) / kStripCols);
  p.n_quant_ctas = static_cast<int>((a.rows + kRowsPerCta - 1) / kRowsPerCta) * p.n_strips;
  p.slot_mu = a.slot_mu;
  p.tag_mu = a.tag_mu;
  p.mu_codes = a.mu_codes;
  p.mu_scales = a.mu_scales;
  p.mu_gdec = a.mu_gdec;
  p.w_codes = a.w_codes;
  p.w_scales = a.w_scales;
  p.w_gdec = a.w_gdec;
  p.n_out = a.n_out;
  p.bias = a.bias;
  int n_extra = 0;
  size_t smem = 0;
  if (a.mu != nullptr && (a.mu_codes != nullptr || a.w_codes != nullptr)) {
    n_extra = a.w_codes ? static_cast<int>((a.n_out + kBiasRowsPerCta - 1) / kBiasRowsPerCta) : 1;
    if (n_extra < 1) n_extra = 1;
    smem = static_cast<size_t>(p.n_strips) * kStripCols * sizeof(float);
  }
  // Padding rows of the scale atoms are written here so every output byte is
  // defined; the quantizer itself touches rows < a.rows only.
  if (a.rows % 128 != 0) {
    zero_scale_padding<<<32, 256, 0, s>>>(a.scales, a.rows, a.K);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    pdl = false;
  }
  if (a.xt == AVR_BF16)
    return a.sr ? launch_quant_t<true, true>(p, n_extra, smem, s, pdl)
                : launch_quant_t<true, false>(p, n_extra, smem, s, pdl);
  return a.sr ? launch_quant_t<false, true>(p, n_extra, smem, s, pdl)
              : launch_quant_t<false, false>(p, n_extra, smem, s, pdl);
}

// ---------------------------------------------------------------------------
// Q_4 of W^T for a weight W [m, n]: T[r][k] = W[k][r], blocks along k (= m).
// A lane owns one row r of T (a column of W) and 64 consecutive k, so the 32
// lanes of a warp read 32 adjacent columns of W row by row (coalesced).
// ---------------------------------------------------------------------------
struct QuantTParams {
  const void* W;
  int64_t m, n;
  int n_tiles;
  const float* slot_amax;
  uint8_t* codes;
  uint8_t* scales;
  float* g_dec;
};

template <bool kBf16>
__global__ void __launch_bounds__(256) quant_transposed_kernel(const QuantTParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TensorScale ts = tensor_scale(max_of_slots(p.slot_amax, p.n_tiles));
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.g_dec = ts.g_dec;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 32 + lane;      // row of T = column of W
  const int64_t k0 = (static_cast<int64_t>(blockIdx.y) * 8 + warp) * 64; // 64 elements along m
  if (r >= p.n || k0 >= p.m) return;
  const uint32_t n_kb64 = static_cast<uint32_t>(p.m / 64);
  uint32_t sw = 0;
  uint32_t packed[8];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    float v[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const int64_t idx = (k0 + b * 16 + t) * p.n + r;
      v[t] = kBf16 ? __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(p.W)[idx]) << 16)
                   : static_cast<const float*>(p.W)[idx];
    }
    float am = 0.0f;
#pragma unroll
    for (int t = 0; t < 16; ++t) am = fmaxf(am, fabsf(v[t]));
    const uint32_t S = e4m3_rn_satfinite(__fmul_rn(__fdiv_rn(am, 6.0f), ts.g_enc));
    const float rs = S == 0u ? 0.0f : __fdiv_rn(ts.g_enc, e4m3_value(S));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t w = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        w |= e2m1x2_rn(__fmul_rn(v[h * 8 + 2 * k], rs), __fmul_rn(v[h * 8 + 2 * k + 1], rs)) << (8 * k);
      packed[b * 2 + h] = w;
    }
    sw |= S << (8 * b);
  }
  uint4* dst = reinterpret_cast<uint4*>(p.codes + r * (p.m / 2) + k0 / 2);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  *reinterpret_cast<uint32_t*>(p.scales + scale_offset(static_cast<uint64_t>(r), static_cast<uint32_t>(k0 / 16), n_kb64)) = sw;
}

cudaError_t launch_quant_transposed(const QuantTransposedArgs& a, cudaStream_t s) {
  QuantTParams p;
  p.W = a.W;
  p.m = a.m;
  p.n = a.n;
  p.n_tiles = a.n_tiles;
  p.slot_amax = a.slot_amax;
  p.codes = a.codes;
  p.scales = a.scales;
  p.g_dec = a.g_dec;
  if (a.n % 128 != 0) {
    zero_scale_padding<<<32, 256, 0, s>>>(a.scales, a.n, a.m);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  dim3 grid(static_cast<unsigned>((a.n + 31) / 32), static_cast<unsigned>((a.m / 64 + 7) / 8));
  if (a.wt == AVR_BF16)
    quant_transposed_kernel<true><<<grid, 256, 0, s>>>(p);
  else
    quant_transposed_kernel<false><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// rank-one row alone, from an already quantized mu
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQuantThreads) bias_kernel(const BiasArgs a) {
  extern __shared__ float s_mu[];
  const int warp = threadIdx.x >> 5;
  const uint32_t n_kb64 = static_cast<uint32_t>(a.K / 64);
  for (int64_t k = threadIdx.x; k < a.K; k += kQuantThreads) {
    const uint32_t byte = a.mu_codes[k / 2];
    const uint32_t code = (k & 1) ? (byte >> 4) : (byte & 0xFu);
    s_mu[k] = e2m1_value(code) * e4m3_value(a.mu_scales[scale_offset(0, static_cast<uint32_t>(k / 16), n_kb64)]);
  }
  __syncthreads();
  const float gprod = __ldg(a.mu_gdec) * __ldg(a.w_gdec);
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kBiasRowsPerCta;
  const int64_t per_warp = kBiasRowsPerCta / kQuantWarps;
  const int64_t jb = j0 + warp * per_warp;
  const int64_t je = min64(jb + per_warp, a.n_out);
  if (jb < je) bias_rows(s_mu, a.K, a.w_codes, a.w_scales, gprod, jb, je, a.bias);
}

cudaError_t launch_bias(const BiasArgs& a, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(a.K) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(bias_kernel), smem);
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = static_cast<unsigned>((a.n_out + kBiasRowsPerCta - 1) / kBiasRowsPerCta);
  bias_kernel<<<grid, kQuantThreads, smem, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// diagnostics
// ---------------------------------------------------------------------------
__global__ void probe_convert_kernel(const float* in, uint8_t* e4m3, uint8_t* e2m1, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = in[i];
    if (e4m3) e4m3[i] = static_cast<uint8_t>(e4m3_rn_satfinite(fabsf(v)));
    if (e2m1) e2m1[i] = static_cast<uint8_t>(e2m1x2_rn(v, 0.0f) & 0xFu);
  }
}

__global__ void probe_philox_kernel(uint64_t seed, uint64_t offset, uint32_t tag, int64_t n,
                                    uint32_t* out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 r = philox_block(seed, offset, tag, static_cast<uint64_t>(i));
    reinterpret_cast<uint4*>(out)[i] = r;
  }
}

cudaError_t launch_probe_convert(const float* in, uint8_t* e4m3, uint8_t* e2m1, int64_t n,
                                 cudaStream_t s) {
  const int64_t blocks = min64((n + 255) / 256, 148 * 16);
  probe_convert_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(in, e4m3, e2m1, n);
  return cudaGetLastError();
}

cudaError_t launch_probe_philox(uint64_t seed, uint64_t offset, uint32_t tag, int64_t n,
                                uint32_t* out, cudaStream_t s) {
  const int64_t blocks = min64((n + 255) / 256, 148 * 16);
  probe_philox_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(seed, offset, tag, n, out);
  return cudaGetLastError();
}

}  // namespace avr
