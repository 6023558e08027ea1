// Device code shared by the split quantizers (quant.cu, split_fused.cu):
// the per-block NVFP4 quantizer, the scale-word gather, the E4M3 reciprocal
// table, and the aux work (Q_4(mu) and the rank-one row mu_bar W_bar) that
// runs beside the quantizing CTAs.
#pragma once

#include "device.cuh"
#include "internal.h"

namespace avr {

constexpr int kQuantThreads = 256;
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kRowsPerIter = 2;            // rows a warp computes per iteration (the next ones are in flight)
constexpr int kBiasWindow = 8192;          // mu_bar values staged in shared memory at a time

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
  int n_aux;              // leading CTAs that quantize mu and form the rank-one row
  // mean quantization and rank-one row
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
  int64_t lp;             // token-axis quantizer: tokens rounded up to a multiple of 64
};

__device__ __forceinline__ float max_of_slots(const float* slots, int n) {
  float a = 0.0f;
  for (int i = threadIdx.x & 31; i < n; i += 32) a = fmaxf(a, __ldcg(slots + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  return a;
}

// 16 consecutive input elements of one lane, kept as loaded (bf16: two
// 16-byte words; fp32: four).
template <bool kBf16>
struct Raw16 {
  uint4 w[kBf16 ? 2 : 4];
};

template <bool kBf16>
__device__ __forceinline__ void load16_ptr(const uint8_t* ptr, bool active, Raw16<kBf16>& r) {
#pragma unroll
  for (int i = 0; i < (kBf16 ? 2 : 4); ++i) r.w[i] = make_uint4(0, 0, 0, 0);
  if (!active) return;
  const uint4* q = reinterpret_cast<const uint4*>(ptr);
#pragma unroll
  for (int i = 0; i < (kBf16 ? 2 : 4); ++i) r.w[i] = __ldcs(q + i);
}

template <bool kBf16>
__device__ __forceinline__ void load16(const void* base, int64_t idx, bool active, Raw16<kBf16>& r) {
#pragma unroll
  for (int i = 0; i < (kBf16 ? 2 : 4); ++i) r.w[i] = make_uint4(0, 0, 0, 0);
  if (!active) return;
  const uint4* p = kBf16 ? reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + idx)
                         : reinterpret_cast<const uint4*>(static_cast<const float*>(base) + idx);
#pragma unroll
  for (int i = 0; i < (kBf16 ? 2 : 4); ++i) r.w[i] = __ldcs(p + i);
}

// xr = fl(x - mu) for the 16 loaded elements of a lane
template <bool kBf16>
__device__ __forceinline__ void sub_mu16(const Raw16<kBf16>& r, const float (&mu)[16], float (&xr)[16]) {
  if (kBf16) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t u[4] = {r.w[i].x, r.w[i].y, r.w[i].z, r.w[i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        sub_bf16x2_f32(u[k], mu[8 * i + 2 * k], mu[8 * i + 2 * k + 1], xr[8 * i + 2 * k], xr[8 * i + 2 * k + 1]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xr[4 * i] = __fsub_rn(__uint_as_float(r.w[i].x), mu[4 * i]);
      xr[4 * i + 1] = __fsub_rn(__uint_as_float(r.w[i].y), mu[4 * i + 1]);
      xr[4 * i + 2] = __fsub_rn(__uint_as_float(r.w[i].z), mu[4 * i + 2]);
      xr[4 * i + 3] = __fsub_rn(__uint_as_float(r.w[i].w), mu[4 * i + 3]);
    }
  }
}

// r_tab[S] = fl(g_enc / value(S)) for every E4M3 code S (0 for S = 0), one
// IEEE division per code instead of one per block.
__device__ __forceinline__ void fill_rscale_table(float* r_tab, float g_enc) {
  for (int c = threadIdx.x; c < 128; c += blockDim.x)
    r_tab[c] = (c == 0 || c == 0x7F) ? 0.0f : __fdiv_rn(g_enc, e4m3_value(static_cast<uint32_t>(c)));
}

// Quantize one 16-element block: returns the 16 packed codes (element 2k in
// the low nibble of byte k) and the block's E4M3 scale code in *S.
// `blk` = element index of the block's first element / 16 (its Philox counter).
// `rw` holds the block's four random words (stochastic rounding only).
template <bool kSR>
__device__ __forceinline__ uint2 quant16(const float (&xr)[16], float g_enc, const float* r_tab, uint4 rw,
                                         uint32_t* S_out) {
  float am = fmax3(fabsf(xr[0]), fabsf(xr[1]), fabsf(xr[2]));
#pragma unroll
  for (int t = 3; t < 15; t += 2) am = fmax3(am, fabsf(xr[t]), fabsf(xr[t + 1]));
  am = fmaxf(am, fabsf(xr[15]));
  const uint32_t S = e4m3_rn_satfinite(__fmul_rn(__fdiv_rn(am, 6.0f), g_enc));
  const float r = r_tab[S];
  float y[16];
#pragma unroll
  for (int t = 0; t < 16; t += 2) fmul2(xr[t], xr[t + 1], r, y[t], y[t + 1]);
  uint2 packed;
  if (kSR) {
    const uint4 w = rw;
    packed.x = e2m1x4_sr(y[0], y[1], y[2], y[3], w.x) | (e2m1x4_sr(y[4], y[5], y[6], y[7], w.y) << 16);
    packed.y = e2m1x4_sr(y[8], y[9], y[10], y[11], w.z) | (e2m1x4_sr(y[12], y[13], y[14], y[15], w.w) << 16);
  } else {
    uint32_t b[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) b[k] = e2m1x2_rn(y[2 * k], y[2 * k + 1]);
    packed.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    packed.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
  }
  *S_out = S;
  return packed;
}

// Lane 4q gathers the scale codes of lanes 4q .. 4q+3 (four consecutive
// blocks) into one little-endian word.
__device__ __forceinline__ uint32_t gather_scale_word(uint32_t S) {
  const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, S, 1);
  const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, S, 2);
  const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, S, 3);
  return S | (s1 << 8) | (s2 << 16) | (s3 << 24);
}

// ---------------------------------------------------------------------------
// Rank-one row mu_bar W_bar: bias[j] = g_dec(mu) g_dec(w) sum_k mu_val[k] value(w)[j, k],
// mu_val = e2m1 * e4m3 of mu_bar.  Every mu_val is exact in f16 (an E2M1
// magnitude has 2 significant bits and an E4M3 one 4, and the product lies
// in [2^-10, 2688]), and so is every E2M1 value, so the per-element product
// is taken exactly with the mixed f16 x f16 + f32 FMA and summed in fp32.
// ---------------------------------------------------------------------------
constexpr int kRowGroup = 32;   // output rows per aux CTA when the aux CTAs are counted

// two packed E2M1 codes (one byte, element 2i in the low nibble) -> f16x2
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t h;
  asm("{ .reg .b8 b; cvt.u8.u32 b, %1; cvt.rn.f16x2.e2m1x2 %0, b; }" : "=r"(h) : "r"(byte));
  return h;
}

// c + lo(a) lo(b) + hi(a) hi(b) with f16x2 a, b and an fp32 accumulator
__device__ __forceinline__ float fma2_f16_f32(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{ .reg .f16 al, ah, bl, bh; .reg .f32 t;\n\t"
      "mov.b32 {al, ah}, %1; mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 t, al, bl, %3; fma.rn.f32.f16 %0, ah, bh, t; }"
      : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}

// The rows of w over the window [k_lo, k_hi) of the f16 values
// s_mu16[k - k_lo]: warp w of CTA `cta` takes the rows cta * 8 + w + t R,
// R = 8 n_ctas, four at a time.  Lane l takes the 16-element blocks l,
// l + 32, ... of the window (8 bytes of codes each: a warp reads 256
// contiguous bytes of a row per block step); the loads of four rows x two
// block steps are issued before any is used, and each mu_bar block read from
// shared memory serves the four rows.  The block's E4M3 scale is applied to
// its 16-element partial, and the lanes' sums are added by a fixed
// butterfly.  The first window stores into out[j], later windows add to it,
// and the last one scales by g_dec_prod.  (s_part is not used.)
static __device__ void bias_window(const uint16_t* s_mu16, float* s_part, int64_t k_lo, int64_t k_hi, int64_t K,
                                   const uint8_t* w_codes, const uint8_t* w_scales, float g_dec_prod,
                                   int64_t n_out, int cta, int n_ctas, float* out) {
  (void)s_part;
  constexpr int kRows = 4, kSteps = 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t n_kb64 = static_cast<uint32_t>(K / 64);
  const int64_t row_step = static_cast<int64_t>(n_ctas) * kQuantWarps;
  for (int64_t j0 = static_cast<int64_t>(cta) * kQuantWarps + warp; j0 < n_out; j0 += kRows * row_step) {
    float acc[kRows];
#pragma unroll
    for (int t = 0; t < kRows; ++t) acc[t] = 0.0f;
    for (int64_t kb = k_lo + 16 * lane; kb < k_hi; kb += 16 * 32 * kSteps) {
      uint2 c[kSteps][kRows];
      uint32_t sb[kSteps][kRows];
#pragma unroll
      for (int u = 0; u < kSteps; ++u) {
        const int64_t k = kb + 16 * 32 * u;
#pragma unroll
        for (int t = 0; t < kRows; ++t) {
          const int64_t j = j0 + t * row_step;
          if (k < k_hi && j < n_out) {
            c[u][t] = __ldg(reinterpret_cast<const uint2*>(w_codes + j * (K / 2) + k / 2));
            sb[u][t] = __ldg(w_scales + scale_offset(static_cast<uint64_t>(j), static_cast<uint32_t>(k / 16), n_kb64));
          } else {
            c[u][t] = make_uint2(0u, 0u);
            sb[u][t] = 0u;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kSteps; ++u) {
        const int64_t k = kb + 16 * 32 * u;
        if (k >= k_hi) break;
        const uint4* m = reinterpret_cast<const uint4*>(s_mu16 + (k - k_lo));   // 16 f16 = 2 x 16 B
        const uint4 m0 = m[0], m1 = m[1];
        const uint32_t mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
        for (int t = 0; t < kRows; ++t) {
          float part = 0.0f;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t byte = ((q < 4 ? c[u][t].x : c[u][t].y) >> (8 * (q % 4))) & 0xFFu;
            part = fma2_f16_f32(e2m1x2_to_f16x2(byte), mv[q], part);
          }
          acc[t] = fmaf(part, e4m3_value(sb[u][t]), acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kRows; ++t) {
      float v = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
      const int64_t j = j0 + t * row_step;
      if (lane == 0 && j < n_out) {
        if (k_lo != 0) v += out[j];
        out[j] = k_hi == K ? v * g_dec_prod : v;
      }
    }
  }
}

// 16 fp32 values of a 64-byte aligned row; kL2: through L2 only, for data
// other CTAs of the same grid wrote (L1 does not see their stores).  The
// plain form lets the warps of an SM that read the same mean share L1 lines.
template <bool kL2 = false>
__device__ __forceinline__ void load_f32x16(const float* p, float (&v)[16]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 t = kL2 ? __ldcg(q + i) : q[i];
    v[4 * i] = t.x;
    v[4 * i + 1] = t.y;
    v[4 * i + 2] = t.z;
    v[4 * i + 3] = t.w;
  }
}

// Q_4(mu) for the window [k_lo, k_hi) by all warps of the CTA:
// s_mu16[k - k_lo] = e2m1 * e4m3 of mu_bar in f16 (exact; the tensor scale
// left out); with `writer` set the codes and scale words are also stored to
// mu_bar.
template <bool kSR, bool kL2>
__device__ void quantize_mean_window(const QuantParams& p, float g_enc, const float* r_tab, int64_t k_lo,
                                     int64_t k_hi, bool writer, uint16_t* s_mu16) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t n_kb64 = static_cast<uint32_t>(p.K / 64);
  for (int64_t s0 = k_lo + static_cast<int64_t>(warp) * kStripCols; s0 < k_hi; s0 += kQuantWarps * kStripCols) {
    const int64_t col0 = s0 + lane * 16;
    const bool active = col0 < k_hi;
    float x[16];
    if (active) {
      load_f32x16<kL2>(p.mu + col0, x);
    } else {
#pragma unroll
      for (int t = 0; t < 16; ++t) x[t] = 0.0f;
    }
    uint32_t S;
    const uint4 rw = kSR ? philox_block(p.seed, p.offset, p.tag_mu, static_cast<uint64_t>(col0 / 16))
                         : make_uint4(0u, 0u, 0u, 0u);
    const uint2 packed = quant16<kSR>(x, g_enc, r_tab, rw, &S);
    const uint32_t sw = gather_scale_word(S);
    if (active) {
      if (writer) {
        *reinterpret_cast<uint2*>(p.mu_codes + col0 / 2) = packed;
        if ((lane & 3) == 0)
          *reinterpret_cast<uint32_t*>(p.mu_scales + scale_offset(0, static_cast<uint32_t>(col0 / 16), n_kb64)) = sw;
      }
      const float sv = e4m3_value(S);
      uint16_t* d = s_mu16 + (col0 - k_lo);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        d[t] = __half_as_ushort(__float2half_rn(e2m1_value((packed.x >> (4 * t)) & 0xFu) * sv));
        d[8 + t] = __half_as_ushort(__float2half_rn(e2m1_value((packed.y >> (4 * t)) & 0xFu) * sv));
      }
    }
  }
}

// The aux CTAs of the split quantizer: Q_4(mu) (CTA 0 stores mu_bar when
// asked) and the rank-one row mu_bar W_bar, whose rows are shared out over
// the warps of all aux CTAs.  They run beside the quantizing CTAs.
template <bool kSR, bool kL2 = false>
__device__ void aux_cta(const QuantParams& p, uint16_t* s_mu16, float* s_part, float* r_tab) {
  const TensorScale ts = tensor_scale(max_of_slots(p.slot_mu, p.n_tiles));
  const bool writer = blockIdx.x == 0 && p.mu_codes != nullptr;
  fill_rscale_table(r_tab, ts.g_enc);
  if (writer) {
    if (threadIdx.x == 0) *p.mu_gdec = ts.g_dec;
    // zero the padding rows 1..127 of every scale atom (row 0 is written below)
    uint32_t* w = reinterpret_cast<uint32_t*>(p.mu_scales);
    const int64_t n_words = (p.K / 64) * 128;
    for (int64_t i = threadIdx.x; i < n_words; i += kQuantThreads)
      if ((i & 127) != 0) w[i] = 0u;
  }
  const bool bias = p.w_codes != nullptr;
  if (!bias && !writer) return;
  const float gprod = bias ? ts.g_dec * __ldg(p.w_gdec) : 0.0f;
  __syncthreads();
  for (int64_t k_lo = 0; k_lo < p.K; k_lo += kBiasWindow) {
    const int64_t k_hi = min64(p.K, k_lo + kBiasWindow);
    quantize_mean_window<kSR, kL2>(p, ts.g_enc, r_tab, k_lo, k_hi, writer, s_mu16);
    __syncthreads();
    if (bias)
      bias_window(s_mu16, s_part, k_lo, k_hi, p.K, p.w_codes, p.w_scales, gprod, p.n_out,
                  static_cast<int>(blockIdx.x), p.n_aux, p.bias);
    __syncthreads();
  }
}

}  // namespace avr
