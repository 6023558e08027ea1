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
// Work split: a warp owns a 512-column strip and walks rows; lane i holds one
// 16-element block (two 16-byte bf16 loads), so the block amax needs no
// shuffle, four lanes make one 4-scale atom word, one Philox4x32-10 call
// gives the block's four 32-bit random words, and stochastic rounding is the
// hardware convert cvt.rs.satfinite.e2m1x4 (four elements per instruction).
// A few leading "aux" CTAs quantize mu and form the rank-one row
// mu_bar W_bar that the GEMM adds as a bias, beside the quantizing CTAs.
#include "quant_common.cuh"

namespace avr {

template <bool kBf16, bool kSR>
__global__ void __launch_bounds__(kQuantThreads) quant_kernel(const QuantParams p) {
  extern __shared__ uint16_t s_mu16[];   // aux CTAs: a window of mu_bar values (f16)
  __shared__ float r_tab[128];
  __shared__ float s_genc, s_gdec;
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  if (static_cast<int>(blockIdx.x) < p.n_aux) {
    __shared__ float s_part[kQuantWarps * kRowGroup];
    aux_cta<kSR>(p, s_mu16, s_part, r_tab);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bid = static_cast<int>(blockIdx.x) - p.n_aux;
  const int n_ctas = static_cast<int>(gridDim.x) - p.n_aux;
  const int gw = bid * kQuantWarps + warp;

  // this warp's strip and first rows do not depend on the tensor scale:
  // start their loads before it is known
  const int warps_per_strip = (n_ctas * kQuantWarps) / p.n_strips;
  const bool has_work = gw < warps_per_strip * p.n_strips;
  const int strip = gw % p.n_strips;
  const int64_t row_step = static_cast<int64_t>(warps_per_strip) * kRowsPerIter;
  const int64_t col0 = static_cast<int64_t>(strip) * kStripCols + lane * 16;
  const bool active = has_work && col0 < p.K;
  int64_t r0 = static_cast<int64_t>(gw / p.n_strips) * kRowsPerIter;

  Raw16<kBf16> cur[kRowsPerIter];
#pragma unroll
  for (int i = 0; i < kRowsPerIter; ++i) load16<kBf16>(p.X, (r0 + i) * p.K + col0, active && r0 + i < p.rows, cur[i]);
  float mu[16];
  if (p.mu != nullptr && active) {
    load_f32x16(p.mu + col0, mu);
  } else {
#pragma unroll
    for (int t = 0; t < 16; ++t) mu[t] = 0.0f;
  }

  if (warp == 0) {
    const TensorScale ts = tensor_scale(max_of_slots(p.slot_xr, p.n_tiles));
    if (lane == 0) {
      s_genc = ts.g_enc;
      s_gdec = ts.g_dec;
    }
  }
  __syncthreads();
  const float g_enc = s_genc;
  fill_rscale_table(r_tab, g_enc);
  __syncthreads();
  if (bid == 0 && threadIdx.x == 0) *p.g_dec = s_gdec;
  if (!has_work) return;
  const uint32_t n_kb64 = static_cast<uint32_t>(p.K / 64);

  // Rows r0 and r0 + 1 of each iteration; the next iteration's rows are loaded
  // into the other buffer while these are quantized (two buffers, unrolled
  // by two, so no register copies).  Pointers and the Philox counter advance
  // by constant strides.
  const int elem = kBf16 ? 2 : 4;
  const uint8_t* xp = static_cast<const uint8_t*>(p.X) + (r0 * p.K + col0) * elem;
  const int64_t x_row = p.K * elem, x_step = row_step * p.K * elem;
  uint8_t* cp = p.codes + r0 * (p.K / 2) + col0 / 2;
  const int64_t c_row = p.K / 2, c_step = row_step * (p.K / 2);
  uint64_t g = p.offset + static_cast<uint64_t>((r0 * p.K + col0) / 16);
  const uint64_t g_row = static_cast<uint64_t>(p.K / 16), g_step = static_cast<uint64_t>(row_step * (p.K / 16));
  const uint32_t c16 = static_cast<uint32_t>(col0 / 16);
  PhiloxKeys keys;
  if (kSR) keys = philox_keys(p.seed);

  auto do_rows = [&](const Raw16<kBf16> (&buf)[kRowsPerIter]) {
#pragma unroll
    for (int i = 0; i < kRowsPerIter; ++i) {
      const int64_t r = r0 + i;
      float xr[16];
      sub_mu16<kBf16>(buf[i], mu, xr);
      const uint4 rw = kSR ? philox_keyed(g + i * g_row, p.tag, keys) : make_uint4(0u, 0u, 0u, 0u);
      uint32_t S;
      const uint2 packed = quant16<kSR>(xr, g_enc, r_tab, rw, &S);
      const uint32_t sw = gather_scale_word(S);
      if (active && r < p.rows) {
        *reinterpret_cast<uint2*>(cp + i * c_row) = packed;
        if ((lane & 3) == 0)
          *reinterpret_cast<uint32_t*>(p.scales + scale_offset(static_cast<uint64_t>(r), c16, n_kb64)) = sw;
        if (p.xr_debug) {
          float4* d = reinterpret_cast<float4*>(p.xr_debug + r * p.K + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) d[q] = make_float4(xr[4 * q], xr[4 * q + 1], xr[4 * q + 2], xr[4 * q + 3]);
        }
      }
    }
    r0 += row_step;
    xp += x_step;
    cp += c_step;
    g += g_step;
  };
  auto load_rows = [&](Raw16<kBf16> (&buf)[kRowsPerIter]) {   // the rows after the current ones
#pragma unroll
    for (int i = 0; i < kRowsPerIter; ++i)
      load16_ptr<kBf16>(xp + x_step + i * x_row, active && r0 + row_step + i < p.rows, buf[i]);
  };
  Raw16<kBf16> nxt[kRowsPerIter];
  while (r0 < p.rows) {
    load_rows(nxt);
    do_rows(cur);
    if (r0 >= p.rows) break;
    load_rows(cur);
    do_rows(nxt);
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

cudaError_t launch_zero_scale_padding(uint8_t* scales, int64_t rows, int64_t K, cudaStream_t s) {
  if (rows % 128 == 0) return cudaSuccess;
  zero_scale_padding<<<32, 256, 0, s>>>(scales, rows, K);
  return cudaGetLastError();
}

template <bool kBf16, bool kSR>
static cudaError_t launch_quant_t(const QuantParams& p, int64_t tasks, size_t smem, cudaStream_t s,
                                  bool pdl) {
  const void* fn = reinterpret_cast<const void*>(quant_kernel<kBf16, kSR>);
  cudaError_t e = set_max_dynamic_smem(fn, smem);
  if (e != cudaSuccess) return e;
  // one warp per task if they all fit at once, else one full wave of
  // resident CTAs (less the aux CTAs), each warp walking rows of its strip
  int64_t n = (tasks + kQuantWarps - 1) / kQuantWarps;
  int64_t cap = static_cast<int64_t>(sm_count()) * blocks_per_sm(fn, kQuantThreads, smem) - p.n_aux;
  if (n > cap) n = cap;
  const int64_t min_ctas = (p.n_strips + kQuantWarps - 1) / kQuantWarps;
  if (n < min_ctas) n = min_ctas;
  return launch_ex(quant_kernel<kBf16, kSR>, dim3(static_cast<unsigned>(n + p.n_aux)), dim3(kQuantThreads),
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
  size_t smem = 0;
  if (a.mu != nullptr && (a.mu_codes != nullptr || a.w_codes != nullptr)) {
    int64_t n_aux = 1;
    if (a.w_codes != nullptr) {
      // one aux CTA per 32 output rows, at most one per two SMs: the GEMM
      // waits for the rank-one row, so the aux CTAs must not finish later
      // than the quantizing ones (measured on the QKV shapes: X's 4096 rows
      // want about a quarter of the CTAs, dY's 1024 rows an eighth)
      n_aux = (a.n_out + kRowGroup - 1) / kRowGroup;
      const int64_t max_aux = sm_count() / 2 > 1 ? sm_count() / 2 : 1;
      n_aux = n_aux > max_aux ? max_aux : n_aux;
    }
    p.n_aux = static_cast<int>(n_aux);
    smem = static_cast<size_t>(min64(a.K, kBiasWindow)) * sizeof(uint16_t);
  }
  const int64_t tasks = ((a.rows + kRowsPerIter - 1) / kRowsPerIter) * p.n_strips;
  // Padding rows of the scale atoms are written here so every output byte is
  // defined; the quantizer itself touches rows < a.rows only.
  if (a.rows % 128 != 0) {
    zero_scale_padding<<<32, 256, 0, s>>>(a.scales, a.rows, a.K);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    pdl = false;
  }
  if (a.xt == AVR_BF16)
    return a.sr ? launch_quant_t<true, true>(p, tasks, smem, s, pdl) : launch_quant_t<true, false>(p, tasks, smem, s, pdl);
  return a.sr ? launch_quant_t<false, true>(p, tasks, smem, s, pdl) : launch_quant_t<false, false>(p, tasks, smem, s, pdl);
}

// ---------------------------------------------------------------------------
// The split quantized along the tokens, for the weight gradient:
// T = (X - 1 mu)^T [K, L] with L = l rounded up to 64 and T[j][i] = 0 for
// i >= l, quantized along its rows (16-token blocks), so that dW = X^T D
// splits into X_bar_R^T D_bar_R on the tensor cores plus a rank-one term.
// The tensor scale is the row-wise residual's (same amax, from the column
// reduce); the random stream of element (j, i) of T counts from
// offset + (j L + i) / 16.
//
// A CTA takes 128 tokens x 128 features: one TMA box into shared memory
// (tokens beyond l read as zero and are replaced by exact zeros), then
// thread t owns feature 128 c0 + t % 128 and 64 consecutive tokens: four
// blocks, 32 bytes of codes (one full sector) and one 4-scale atom word.
// With mean quantization asked for, CTA 0 is an aux CTA that quantizes mu
// exactly as the row-wise quantizer does (same function, same tag).
// ---------------------------------------------------------------------------
constexpr int kTokTile = 128;     // tokens per CTA
constexpr int kFeatTile = 128;    // features per CTA

template <bool kBf16, bool kSR>
__global__ void __launch_bounds__(kQuantThreads) quant_tokens_kernel(const __grid_constant__ CUtensorMap map,
                                                                     const QuantParams p) {
  extern __shared__ __align__(1024) uint8_t smem_tile[];   // the X tile, or (aux CTA) mu_bar in f16
  __shared__ float r_tab[128];
  __shared__ uint64_t bar;
  __shared__ float s_genc, s_gdec;
  __shared__ uint32_t s_ok;
  constexpr uint32_t kElem = kBf16 ? 2u : 4u;
  constexpr uint32_t kTileBytes = kTokTile * kFeatTile * kElem;
  if (static_cast<int>(blockIdx.x) < p.n_aux) {
    __shared__ float s_part[kQuantWarps * kRowGroup];
    pdl_wait_prior_grid();
    pdl_allow_next_grid();
    aux_cta<kSR>(p, reinterpret_cast<uint16_t*>(smem_tile), s_part, r_tab);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bid = static_cast<int>(blockIdx.x) - p.n_aux;
  const int tiles_k = static_cast<int>((p.K + kFeatTile - 1) / kFeatTile);
  const int64_t f0 = static_cast<int64_t>(bid % tiles_k) * kFeatTile;   // first feature
  const int64_t t0 = static_cast<int64_t>(bid / tiles_k) * kTokTile;    // first token
  if (tid == 0) {
    prefetch_tensormap(&map);
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar, kTileBytes);
    tma_load_2d(smem_tile, &map, &bar, static_cast<int32_t>(f0), static_cast<int32_t>(t0));
  }
  const int c = tid % kFeatTile, grp = tid / kFeatTile;
  const int64_t j = f0 + c;                                  // feature = row of T
  const int64_t i0 = t0 + 64 * grp;                          // first token of this thread
  const float mu = (p.mu != nullptr && j < p.K) ? __ldg(p.mu + j) : 0.0f;
  if (warp == 0) {
    const TensorScale ts = tensor_scale(max_of_slots(p.slot_xr, p.n_tiles));
    if (lane == 0) {
      s_genc = ts.g_enc;
      s_gdec = ts.g_dec;
    }
  }
  __syncthreads();
  fill_rscale_table(r_tab, s_genc);
  if (tid == 0) {
    s_ok = mbar_wait(&bar, 0, p.status) ? 1u : 0u;
    if (!s_ok) mbar_wait(&bar, 0, nullptr);   // a second bounded wait for the copy in flight
  }
  __syncthreads();
  if (bid == 0 && tid == 0) *p.g_dec = s_gdec;
  if (!s_ok || j >= p.K || i0 >= p.lp) return;

  const float g_enc = s_genc;
  PhiloxKeys keys;
  if (kSR) keys = philox_keys(p.seed);
  const uint64_t g = p.offset + static_cast<uint64_t>((j * p.lp + i0) / 16);
  uint32_t packed[8], sw = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    float xr[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const int rr = 64 * grp + 16 * b + t;                 // token within the tile
      const uint32_t idx = static_cast<uint32_t>(rr * kFeatTile + c);
      const float x = kBf16 ? __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(smem_tile)[idx]) << 16)
                            : reinterpret_cast<const float*>(smem_tile)[idx];
      xr[t] = (t0 + rr < p.rows) ? __fsub_rn(x, mu) : 0.0f;
    }
    const uint4 rw = kSR ? philox_keyed(g + b, p.tag, keys) : make_uint4(0u, 0u, 0u, 0u);
    uint32_t S;
    const uint2 pk = quant16<kSR>(xr, g_enc, r_tab, rw, &S);
    packed[2 * b] = pk.x;
    packed[2 * b + 1] = pk.y;
    sw |= S << (8 * b);
  }
  uint4* dst = reinterpret_cast<uint4*>(p.codes + j * (p.lp / 2) + i0 / 2);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  *reinterpret_cast<uint32_t*>(p.scales + scale_offset(static_cast<uint64_t>(j), static_cast<uint32_t>(i0 / 16),
                                                       static_cast<uint32_t>(p.lp / 64))) = sw;
}

template <bool kBf16, bool kSR>
static cudaError_t launch_quant_tokens_t(const CUtensorMap& map, const QuantParams& p, int64_t ctas, size_t smem,
                                         cudaStream_t s, bool pdl) {
  const void* fn = reinterpret_cast<const void*>(quant_tokens_kernel<kBf16, kSR>);
  cudaError_t e = set_max_dynamic_smem(fn, smem);
  if (e != cudaSuccess) return e;
  return launch_ex(quant_tokens_kernel<kBf16, kSR>, dim3(static_cast<unsigned>(ctas)), dim3(kQuantThreads), smem, s,
                   pdl, map, p);
}

cudaError_t launch_quant_tokens(const QuantArgs& a, cudaStream_t s, bool pdl) {
  const bool bf16 = a.xt == AVR_BF16;
  const int elem = bf16 ? 2 : 4;
  CUtensorMap map;
  if (!make_tensor_map_2d(&map, a.X, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                          elem, static_cast<uint64_t>(a.rows), static_cast<uint64_t>(a.K), kTokTile, kFeatTile,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  QuantParams p = {};
  p.rows = a.rows;
  p.K = a.K;
  p.lp = (a.rows + 63) / 64 * 64;
  p.mu = a.mu;
  p.n_tiles = a.n_tiles;
  p.slot_xr = a.slot_xr;
  p.codes = a.codes;
  p.scales = a.scales;
  p.g_dec = a.g_dec;
  p.seed = a.seed;
  p.offset = a.offset;
  p.tag = a.tag;
  p.status = a.status;
  p.slot_mu = a.slot_mu;
  p.tag_mu = a.tag_mu;
  p.mu_codes = a.mu_codes;
  p.mu_scales = a.mu_scales;
  p.mu_gdec = a.mu_gdec;
  size_t smem = static_cast<size_t>(kTokTile) * kFeatTile * elem;
  if (a.mu != nullptr && a.mu_codes != nullptr) {
    p.n_aux = 1;
    const size_t aux = static_cast<size_t>(min64(a.K, kBiasWindow)) * sizeof(uint16_t);
    if (aux > smem) smem = aux;
  }
  // scale rows K .. next multiple of 128 (features past K) are zero
  if (a.K % 128 != 0) {
    zero_scale_padding<<<32, 256, 0, s>>>(a.scales, a.K, p.lp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    pdl = false;
  }
  const int64_t ctas = p.n_aux + ((a.K + kFeatTile - 1) / kFeatTile) * ((p.lp + kTokTile - 1) / kTokTile);
  if (bf16)
    return a.sr ? launch_quant_tokens_t<true, true>(map, p, ctas, smem, s, pdl)
                : launch_quant_tokens_t<true, false>(map, p, ctas, smem, s, pdl);
  return a.sr ? launch_quant_tokens_t<false, true>(map, p, ctas, smem, s, pdl)
              : launch_quant_tokens_t<false, false>(map, p, ctas, smem, s, pdl);
}

// ---------------------------------------------------------------------------
// dequantized means for the weight gradient's rank-one term:
// u[i] = l * deq(mu_bar_X)[i], v[j] = deq(mu_bar_D)[j], deq = e2m1 * e4m3 * g_dec
// ---------------------------------------------------------------------------
__global__ void mean_dequant_kernel(const uint8_t* codes_x, const uint8_t* scales_x, const float* gdec_x, int64_t m,
                                    const uint8_t* codes_d, const uint8_t* scales_d, const float* gdec_d, int64_t n,
                                    float l, float* u, float* v) {
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const float gx = __ldg(gdec_x), gd = __ldg(gdec_d);
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < m + n;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool is_x = k < m;
    const int64_t e = is_x ? k : k - m;
    const int64_t K = is_x ? m : n;
    const uint8_t* codes = is_x ? codes_x : codes_d;
    const uint8_t* scales = is_x ? scales_x : scales_d;
    const uint32_t byte = codes[e / 2];
    const uint32_t code = (e & 1) ? (byte >> 4) : (byte & 0xFu);
    const float sv = e4m3_value(scales[scale_offset(0, static_cast<uint32_t>(e / 16), static_cast<uint32_t>(K / 64))]);
    const float val = __fmul_rn(__fmul_rn(e2m1_value(code), sv), is_x ? gx : gd);
    if (is_x)
      u[e] = __fmul_rn(l, val);
    else
      v[e] = val;
  }
}

cudaError_t launch_mean_dequant(const uint8_t* codes_x, const uint8_t* scales_x, const float* gdec_x, int64_t m,
                                const uint8_t* codes_d, const uint8_t* scales_d, const float* gdec_d, int64_t n,
                                int64_t l, float* u, float* v, cudaStream_t s, bool pdl) {
  const int64_t blocks = min64((m + n + 255) / 256, 148);
  return launch_ex(mean_dequant_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, pdl, codes_x, scales_x,
                   gdec_x, m, codes_d, scales_d, gdec_d, n, static_cast<float>(l), u, v);
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
  extern __shared__ uint16_t s_mu16[];
  __shared__ float s_part[kQuantWarps * kRowGroup];
  const uint32_t n_kb64 = static_cast<uint32_t>(a.K / 64);
  const float gprod = __ldg(a.mu_gdec) * __ldg(a.w_gdec);
  for (int64_t k_lo = 0; k_lo < a.K; k_lo += kBiasWindow) {
    const int64_t k_hi = min64(a.K, k_lo + kBiasWindow);
    for (int64_t k = k_lo + threadIdx.x; k < k_hi; k += kQuantThreads) {
      const uint32_t byte = a.mu_codes[k / 2];
      const uint32_t code = (k & 1) ? (byte >> 4) : (byte & 0xFu);
      const float v = e2m1_value(code) * e4m3_value(a.mu_scales[scale_offset(0, static_cast<uint32_t>(k / 16), n_kb64)]);
      s_mu16[k - k_lo] = __half_as_ushort(__float2half_rn(v));
    }
    __syncthreads();
    bias_window(s_mu16, s_part, k_lo, k_hi, a.K, a.w_codes, a.w_scales, gprod, a.n_out,
                static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x), a.bias);
    __syncthreads();
  }
}

cudaError_t launch_bias(const BiasArgs& a, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(min64(a.K, kBiasWindow)) * sizeof(uint16_t);
  const unsigned grid = static_cast<unsigned>((a.n_out + kRowGroup - 1) / kRowGroup);
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

__global__ void probe_convert_sr_kernel(const float4* in, const uint32_t* rbits, uint16_t* out, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = in[i];
    out[i] = static_cast<uint16_t>(e2m1x4_sr(v.x, v.y, v.z, v.w, rbits[i]));
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

cudaError_t launch_probe_convert_sr(const float* in, const uint32_t* rbits, uint16_t* out, int64_t n,
                                    cudaStream_t s) {
  const int64_t blocks = min64((n + 255) / 256, 148 * 16);
  probe_convert_sr_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(reinterpret_cast<const float4*>(in), rbits,
                                                                         out, n);
  return cudaGetLastError();
}

cudaError_t launch_probe_philox(uint64_t seed, uint64_t offset, uint32_t tag, int64_t n,
                                uint32_t* out, cudaStream_t s) {
  const int64_t blocks = min64((n + 255) / 256, 148 * 16);
  probe_philox_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(seed, offset, tag, n, out);
  return cudaGetLastError();
}

}  // namespace avr
