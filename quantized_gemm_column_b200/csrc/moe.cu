// The Averis split for a mixture-of-experts layer: one split per expert over
// a token buffer permuted by expert (the method is applied to the Qwen3
// 7B-A1.5B MoE model in "The Curse and Blessing of Mean Bias in FP4-Quantized
// LLM Training", arXiv abstract page; every expert is its own linear layer).
//
// Layout: expert e owns rows [o_e, o_e + n_e) of the buffer, o_0 = 0 and
// o_{e+1} = o_e + n_e rounded up to 128, so every 128-row block belongs to one
// expert and the NVFP4 scale atoms of a block are that expert's.  The counts
// n_e live on the device (a router writes them); a one-CTA kernel turns them
// into the segment table the other kernels read:
//   seg[e]          = {o_e, n_e, first chunk, chunks}  (256-row chunks from o_e)
//   chunk_expert[c] = the expert of global chunk c
//   block_expert[b] = the expert of 128-row block b, or -1 past the last segment
//   totals          = {chunks in use, rows in use (o_E), 1 if they fit}
// The grouped column reduce (colreduce.cu) then gives mu_e and the per-expert
// amax slots; this file's quantizer quantizes each row with its expert's mean
// and tensor scale, and its rank-one kernel forms b_e = mu_bar_e W_bar_e for
// the grouped GEMM's epilogue.
#include "quant_common.cuh"

namespace avr {

// ---------------------------------------------------------------------------
// segment table
// ---------------------------------------------------------------------------
constexpr int kMoeTableThreads = 1024;

__global__ void __launch_bounds__(kMoeTableThreads) moe_table_kernel(const int32_t* counts, int E, int64_t l_cap,
                                                                     int c_max, MoeSeg* seg, int32_t* chunk_expert,
                                                                     int32_t* block_expert, int32_t* totals,
                                                                     uint32_t* status) {
  __shared__ int64_t s_rows[kMoeTableThreads], s_chunks[kMoeTableThreads];
  __shared__ int32_t s_bad;
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const int e = threadIdx.x;
  int32_t n = 0;
  if (e < E) n = __ldg(counts + e);
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  if (n < 0 || n > l_cap) atomicOr(&s_bad, 1);
  const int32_t n_ok = (n < 0 || n > l_cap) ? 0 : n;
  const int64_t padded = (static_cast<int64_t>(n_ok) + 127) / 128 * 128;
  const int64_t chunks = (static_cast<int64_t>(n_ok) + kChunkRows - 1) / kChunkRows;
  // inclusive prefix sums (Hillis-Steele over the block)
  s_rows[e] = padded;
  s_chunks[e] = chunks;
  __syncthreads();
  for (int d = 1; d < kMoeTableThreads; d <<= 1) {
    const int64_t r = e >= d ? s_rows[e - d] : 0, c = e >= d ? s_chunks[e - d] : 0;
    __syncthreads();
    s_rows[e] += r;
    s_chunks[e] += c;
    __syncthreads();
  }
  const int64_t row0 = s_rows[e] - padded, chunk0 = s_chunks[e] - chunks;
  const int64_t rows_used = E > 0 ? s_rows[E - 1] : 0;
  const int64_t chunks_used = E > 0 ? s_chunks[E - 1] : 0;
  const bool fits = s_bad == 0 && rows_used <= l_cap && chunks_used <= c_max;
  if (e < E && fits) {
    seg[e] = MoeSeg{static_cast<int32_t>(row0), n_ok, static_cast<int32_t>(chunk0), static_cast<int32_t>(chunks)};
    for (int64_t c = 0; c < chunks; ++c) chunk_expert[chunk0 + c] = e;
    for (int64_t b = 0; b < padded / 128; ++b) block_expert[row0 / 128 + b] = e;
  }
  const int64_t n_blocks = l_cap / 128;
  for (int64_t b = (fits ? rows_used / 128 : 0) + threadIdx.x; b < n_blocks; b += kMoeTableThreads)
    block_expert[b] = -1;
  if (threadIdx.x == 0) {
    totals[0] = fits ? static_cast<int32_t>(chunks_used) : 0;
    totals[1] = fits ? static_cast<int32_t>(rows_used) : 0;
    totals[2] = fits ? 1 : 0;
    if (!fits) raise_status(status, AVR_ERR_INVALID_ARG);
  }
}

cudaError_t launch_moe_table(const int32_t* counts, int E, int64_t l_cap, int c_max, MoeSeg* seg,
                             int32_t* chunk_expert, int32_t* block_expert, int32_t* totals, uint32_t* status,
                             cudaStream_t s, bool pdl) {
  if (E < 1 || E > kMoeTableThreads) return cudaErrorInvalidValue;
  return launch_ex(moe_table_kernel, dim3(1), dim3(kMoeTableThreads), 0, s, pdl, counts, E, l_cap, c_max, seg,
                   chunk_expert, block_expert, totals, status);
}

// ---------------------------------------------------------------------------
// grouped split quantizer
// ---------------------------------------------------------------------------
constexpr int kGroupRows = 32;   // rows of one task (a task lies in one 128-row block)

struct MoeQuantParams {
  const void* X;
  int64_t l_cap, K;
  int E, T;                     // experts; amax slots per expert (128-column tiles)
  const MoeSeg* seg;
  const int32_t* block_expert;
  const int32_t* totals;        // [2] = 1 when the segments fit the buffer
  const float* mu;              // [E][K] (null: vanilla)
  const float* slot_xr;         // [E][T]
  const float* slot_mu;         // [E][T]
  uint8_t* codes;
  uint8_t* scales;
  float* g_dec;                 // [E]
  uint8_t* mu_codes;            // [E][K/2] (null: no mean quantization)
  uint8_t* mu_scales;
  float* mu_gdec;               // [E]
  uint64_t seed, offset;
  uint32_t tag, tag_mu;
  uint32_t* status;
  int n_strips, n_aux;
};

// max over this expert's T amax slots, by one warp
__device__ __forceinline__ float expert_amax(const float* slots, int e, int T) {
  float a = 0.0f;
  for (int i = threadIdx.x & 31; i < T; i += 32) a = fmaxf(a, __ldcg(slots + static_cast<int64_t>(e) * T + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  return a;
}

// r_tab[S] = fl(g_enc / value(S)) filled by one warp
__device__ __forceinline__ void fill_rscale_table_warp(float* r_tab, float g_enc) {
  for (int c = threadIdx.x & 31; c < 128; c += 32)
    r_tab[c] = (c == 0 || c == 0x7F) ? 0.0f : __fdiv_rn(g_enc, e4m3_value(static_cast<uint32_t>(c)));
  __syncwarp();
}

template <bool kBf16, bool kSR>
__global__ void __launch_bounds__(kQuantThreads) moe_quant_kernel(const MoeQuantParams p) {
  __shared__ float s_rtab[kQuantWarps][128];
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* r_tab = s_rtab[warp];
  const uint32_t n_kb64 = static_cast<uint32_t>(p.K / 64);
  PhiloxKeys keys;
  if (kSR) keys = philox_keys(p.seed);

  if (__ldcg(p.totals + 2) == 0) return;     // the segments did not fit: nothing to quantize
  if (static_cast<int>(blockIdx.x) < p.n_aux) {
    // Q_4(mu_e) as row e of an [E, K] tensor, its own tensor scale; warp w of
    // aux CTA a takes experts a * 8 + w, + 8 n_aux, ...
    for (int e = static_cast<int>(blockIdx.x) * kQuantWarps + warp; e < p.E; e += p.n_aux * kQuantWarps) {
      if (p.seg[e].rows == 0) continue;
      const TensorScale ts = tensor_scale(expert_amax(p.slot_mu, e, p.T));
      fill_rscale_table_warp(r_tab, ts.g_enc);
      if (lane == 0) p.mu_gdec[e] = ts.g_dec;
      for (int64_t s0 = 0; s0 < p.K; s0 += kStripCols) {   // every lane takes every step
        const int64_t col0 = s0 + lane * 16;
        const bool act = col0 < p.K;
        float x[16];
        if (act) {
          load_f32x16(p.mu + static_cast<int64_t>(e) * p.K + col0, x);
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) x[q] = 0.0f;
        }
        const uint4 rw = kSR ? philox_keyed(p.offset + static_cast<uint64_t>((static_cast<int64_t>(e) * p.K + col0) / 16),
                                            p.tag_mu, keys)
                             : make_uint4(0u, 0u, 0u, 0u);
        uint32_t S;
        const uint2 packed = quant16<kSR>(x, ts.g_enc, r_tab, rw, &S);
        const uint32_t sw = gather_scale_word(S);
        if (act) {
          *reinterpret_cast<uint2*>(p.mu_codes + static_cast<int64_t>(e) * (p.K / 2) + col0 / 2) = packed;
          if ((lane & 3) == 0)
            *reinterpret_cast<uint32_t*>(p.mu_scales + scale_offset(static_cast<uint64_t>(e),
                                                                    static_cast<uint32_t>(col0 / 16), n_kb64)) = sw;
        }
      }
      __syncwarp();
    }
    return;
  }

  // tasks: (512-column strip, 32-row group) with every row of the group in
  // one expert's segment (or past all of them)
  // each warp takes a contiguous range of tasks, so that consecutive tasks
  // mostly share the expert (and its tensor scale and reciprocal table)
  const int n_ctas = static_cast<int>(gridDim.x) - p.n_aux;
  const int64_t n_groups = p.l_cap / kGroupRows;
  const int64_t n_tasks = n_groups * p.n_strips;
  const int64_t n_warps = static_cast<int64_t>(n_ctas) * kQuantWarps;
  const int64_t gw0 = static_cast<int64_t>(static_cast<int>(blockIdx.x) - p.n_aux) * kQuantWarps + warp;
  const int64_t t_per = (n_tasks + n_warps - 1) / n_warps;
  const int64_t t_end = min64(n_tasks, (gw0 + 1) * t_per);
  int cached_e = -1;
  TensorScale ts = {1.0f, 1.0f};
  for (int64_t task = gw0 * t_per; task < t_end; ++task) {
    const int strip = static_cast<int>(task % p.n_strips);
    const int64_t r_first = (task / p.n_strips) * kGroupRows;
    const int e = __ldg(p.block_expert + r_first / 128);
    if (e < 0) continue;
    const MoeSeg sg = p.seg[e];
    if (e != cached_e) {
      ts = tensor_scale(expert_amax(p.slot_xr, e, p.T));
      fill_rscale_table_warp(r_tab, ts.g_enc);
      cached_e = e;
    }
    const int64_t col0 = static_cast<int64_t>(strip) * kStripCols + lane * 16;
    const bool active = col0 < p.K;
    float mu[16];
    if (p.mu != nullptr && active) {
      load_f32x16(p.mu + static_cast<int64_t>(e) * p.K + col0, mu);
    } else {
#pragma unroll
      for (int q = 0; q < 16; ++q) mu[q] = 0.0f;
    }
    if (strip == 0 && r_first == sg.row0 && lane == 0) p.g_dec[e] = ts.g_dec;
    const int64_t r_end = static_cast<int64_t>(sg.row0) + sg.rows;   // rows past it are padding
    const uint32_t c16 = static_cast<uint32_t>(col0 / 16);
    // rows kRowsInFlight at a time, the next ones loading meanwhile (the
    // buffer is usually read from HBM: it does not fit in L2 with the reduce's pass)
    constexpr int kRowsInFlight = 2;
    Raw16<kBf16> cur[kRowsInFlight], nxt[kRowsInFlight];
#pragma unroll
    for (int q = 0; q < kRowsInFlight; ++q)
      load16<kBf16>(p.X, (r_first + q) * p.K + col0, active && r_first + q < r_end, cur[q]);
#pragma unroll 1
    for (int i = 0; i < kGroupRows; i += kRowsInFlight) {
      if (i + kRowsInFlight < kGroupRows) {
#pragma unroll
        for (int q = 0; q < kRowsInFlight; ++q) {
          const int64_t rn = r_first + i + kRowsInFlight + q;
          load16<kBf16>(p.X, rn * p.K + col0, active && rn < r_end, nxt[q]);
        }
      }
#pragma unroll
      for (int q = 0; q < kRowsInFlight; ++q) {
        const int64_t r = r_first + i + q;
        float xr[16];
        sub_mu16<kBf16>(cur[q], mu, xr);
        if (r >= r_end) {
#pragma unroll
          for (int t = 0; t < 16; ++t) xr[t] = 0.0f;   // padding rows: zero codes and scales
        }
        const uint4 rw = kSR ? philox_keyed(p.offset + static_cast<uint64_t>((r * p.K + col0) / 16), p.tag, keys)
                             : make_uint4(0u, 0u, 0u, 0u);
        uint32_t S;
        const uint2 packed = quant16<kSR>(xr, ts.g_enc, r_tab, rw, &S);
        const uint32_t sw = gather_scale_word(S);
        if (active) {
          *reinterpret_cast<uint2*>(p.codes + r * (p.K / 2) + col0 / 2) = packed;
          if ((lane & 3) == 0)
            *reinterpret_cast<uint32_t*>(p.scales + scale_offset(static_cast<uint64_t>(r), c16, n_kb64)) = sw;
        }
      }
#pragma unroll
      for (int q = 0; q < kRowsInFlight; ++q) cur[q] = nxt[q];
    }
  }
}

template <bool kBf16, bool kSR>
static cudaError_t launch_moe_quant_t(const MoeQuantParams& p, cudaStream_t s, bool pdl) {
  const void* fn = reinterpret_cast<const void*>(moe_quant_kernel<kBf16, kSR>);
  const int64_t tasks = (p.l_cap / kGroupRows) * p.n_strips;
  int64_t n = (tasks + kQuantWarps - 1) / kQuantWarps;
  const int64_t cap = static_cast<int64_t>(sm_count()) * blocks_per_sm(fn, kQuantThreads, 0) - p.n_aux;
  if (n > cap) n = cap;
  if (n < 1) n = 1;
  return launch_ex(moe_quant_kernel<kBf16, kSR>, dim3(static_cast<unsigned>(n + p.n_aux)), dim3(kQuantThreads), 0, s,
                   pdl, p);
}

cudaError_t launch_moe_quant(const MoeQuantArgs& a, cudaStream_t s, bool pdl) {
  MoeQuantParams p = {};
  p.X = a.X;
  p.l_cap = a.l_cap;
  p.K = a.K;
  p.E = a.E;
  p.T = static_cast<int>((a.K + kColTile - 1) / kColTile);
  p.seg = a.seg;
  p.block_expert = a.block_expert;
  p.totals = a.totals;
  p.mu = a.mu;
  p.slot_xr = a.slot_xr;
  p.slot_mu = a.slot_mu;
  p.codes = a.codes;
  p.scales = a.scales;
  p.g_dec = a.g_dec;
  p.mu_codes = a.mu_codes;
  p.mu_scales = a.mu_scales;
  p.mu_gdec = a.mu_gdec;
  p.seed = a.seed;
  p.offset = a.offset;
  p.tag = a.tag;
  p.tag_mu = a.tag_mu;
  p.status = a.status;
  p.n_strips = static_cast<int>((a.K + kStripCols - 1) / kStripCols);
  p.n_aux = (a.mu != nullptr && a.mu_codes != nullptr) ? (a.E + kQuantWarps - 1) / kQuantWarps : 0;
  if (a.mu_codes != nullptr) {   // scale rows E .. next multiple of 128 of the [E, K] mean tensor
    cudaError_t e = launch_zero_scale_padding(a.mu_scales, a.E, a.K, s);
    if (e != cudaSuccess) return e;
    if (a.E % 128 != 0) pdl = false;
  }
  if (a.xt == AVR_BF16)
    return a.sr ? launch_moe_quant_t<true, true>(p, s, pdl) : launch_moe_quant_t<true, false>(p, s, pdl);
  return a.sr ? launch_moe_quant_t<false, true>(p, s, pdl) : launch_moe_quant_t<false, false>(p, s, pdl);
}

// ---------------------------------------------------------------------------
// rank-one rows b_e = mu_bar_e W_bar_e: a warp per output row, so the 32 lanes
// read the row's codes with coalesced 16-byte loads (32 elements per lane per
// step); products of E2M1 x (E2M1 x E4M3) values are exact in f16 and summed
// in fp32 per 16-element block, scaled by the block's E4M3 scale, then the
// lanes' partial sums are added by a shuffle tree.  CTA (x, e) takes rows
// 64 x .. 64 x + 63 of expert e.
// ---------------------------------------------------------------------------
constexpr int kBiasRowsPerCta = 64;

__global__ void __launch_bounds__(kQuantThreads) moe_bias_kernel(const MoeBiasArgs a) {
  extern __shared__ uint16_t s_mu16[];         // mu_bar_e as f16, one window of K
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const int e = static_cast<int>(blockIdx.y);
  if (__ldcg(a.totals + 2) == 0) return;       // the segments did not fit
  if (a.seg[e].rows == 0) return;             // no tokens: the GEMM has no tile of this expert
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t n_kb64 = static_cast<uint32_t>(a.K / 64);
  const float gprod = __ldcg(a.mu_gdec + e) * __ldg(a.w_gdec + e);
  const uint8_t* w_codes = a.w_codes + static_cast<int64_t>(e) * a.N * (a.K / 2);
  const uint8_t* w_scales = a.w_scales + static_cast<int64_t>(e) * a.N * (a.K / 16);
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kBiasRowsPerCta;
  float acc[kBiasRowsPerCta / kQuantWarps];
#pragma unroll
  for (int r = 0; r < kBiasRowsPerCta / kQuantWarps; ++r) acc[r] = 0.0f;
  for (int64_t k_lo = 0; k_lo < a.K; k_lo += kBiasWindow) {
    const int64_t k_hi = min64(a.K, k_lo + kBiasWindow);
    __syncthreads();                            // the previous window is no longer read
    for (int64_t k = k_lo + threadIdx.x; k < k_hi; k += kQuantThreads) {
      const uint32_t byte = a.mu_codes[static_cast<int64_t>(e) * (a.K / 2) + k / 2];
      const uint32_t code = (k & 1) ? (byte >> 4) : (byte & 0xFu);
      const float v = e2m1_value(code) *
                      e4m3_value(a.mu_scales[scale_offset(static_cast<uint64_t>(e), static_cast<uint32_t>(k / 16), n_kb64)]);
      s_mu16[k - k_lo] = __half_as_ushort(__float2half_rn(v));
    }
    __syncthreads();
    // per 1024-column step: the codes and scales of all this warp's rows are
    // requested before any product, so a warp keeps 8 row loads in flight
    for (int64_t ks = k_lo; ks < k_hi; ks += 32 * 32) {
      const int64_t k = ks + lane * 32;
      const bool kv = k < k_hi;
      uint4 c[kBiasRowsPerCta / kQuantWarps];
      uint32_t sc[kBiasRowsPerCta / kQuantWarps];
#pragma unroll
      for (int r = 0; r < kBiasRowsPerCta / kQuantWarps; ++r) {
        const int64_t j = j0 + r * kQuantWarps + warp;
        c[r] = make_uint4(0u, 0u, 0u, 0u);
        sc[r] = 0u;
        if (kv && j < a.N) {
          c[r] = __ldg(reinterpret_cast<const uint4*>(w_codes + j * (a.K / 2) + k / 2));   // 32 codes
          sc[r] = __ldg(reinterpret_cast<const uint16_t*>(
              w_scales + scale_offset(static_cast<uint64_t>(j), static_cast<uint32_t>(k / 16), n_kb64)));
        }
      }
      if (!kv) continue;
      uint32_t mv[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 m = *reinterpret_cast<const uint4*>(s_mu16 + (k - k_lo) + 8 * q);
        mv[4 * q] = m.x;
        mv[4 * q + 1] = m.y;
        mv[4 * q + 2] = m.z;
        mv[4 * q + 3] = m.w;
      }
#pragma unroll
      for (int r = 0; r < kBiasRowsPerCta / kQuantWarps; ++r) {
        const uint32_t words[4] = {c[r].x, c[r].y, c[r].z, c[r].w};
#pragma unroll
        for (int b = 0; b < 2; ++b) {           // two 16-element blocks
          float part = 0.0f;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t byte = (words[2 * b + q / 4] >> (8 * (q % 4))) & 0xFFu;
            part = fma2_f16_f32(e2m1x2_to_f16x2(byte), mv[8 * b + q], part);
          }
          acc[r] = fmaf(part, e4m3_value((sc[r] >> (8 * b)) & 0xFFu), acc[r]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kBiasRowsPerCta / kQuantWarps; ++r) {
    float v = acc[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const int64_t j = j0 + r * kQuantWarps + warp;
    if (lane == 0 && j < a.N) a.bias[static_cast<int64_t>(e) * a.N + j] = v * gprod;
  }
}

cudaError_t launch_moe_bias(const MoeBiasArgs& a, cudaStream_t s, bool pdl) {
  const size_t smem = static_cast<size_t>(min64(a.K, kBiasWindow)) * sizeof(uint16_t);
  const dim3 grid(static_cast<unsigned>((a.N + kBiasRowsPerCta - 1) / kBiasRowsPerCta), static_cast<unsigned>(a.E));
  return launch_ex(moe_bias_kernel, grid, dim3(kQuantThreads), smem, s, pdl, a);
}

}  // namespace avr
