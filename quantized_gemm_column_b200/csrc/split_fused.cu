// K1 + K2 in one persistent kernel: the Averis split with a single pass over
// its input (mu_X = (1/l) 1^T X, X_bar_R = Q_4(X - 1 mu_X), mu_bar_X = Q_4(mu_X)
// and the rank-one row mu_bar W_bar; Lighthouse review of "The Curse and
// Blessing of Mean Bias in FP4-Quantized LLM Training", section 二 "Averis
// 方法": a reduce and a subtract before FP4 quantization).
//
// Two CTAs per SM (one for fp32 input), all resident, three phases separated
// by grid-wide barriers:
//  1. reduce: X [l, K] is cut into units of one 256-row chunk x 128 columns;
//     CTA b takes units b, b + G, b + 2G, ... (tiles fastest, so the CTAs
//     running together read whole rows), each by one TMA copy into its unit
//     buffer, and threads 0..127 form the unit's column partials (sum, max,
//     min) in the fixed order of the column reduce.  The CTA's last unit
//     stays in shared memory.
//  2. fold: CTA b folds a contiguous range of columns, one warp per column:
//     lane c loads chunk c's partials (32 chunks per round trip) and every
//     lane adds them up in chunk order from broadcast shuffles, giving mu_j
//     and max(fl(colmax - mu), fl(mu - colmin)), the residual's amax over its
//     columns, into slot b.
//  3. quantize: the tensor scale is the maximum of the G slots; the leading
//     aux CTAs first quantize mu and form the rank-one row; every CTA then
//     quantizes its units, the resident ones straight from shared memory and
//     the others copied in again (from L2, where phase 1 left them).
// The results are bit for bit those of the two-kernel split (same order of
// every sum, same quantizer, same random stream).
#include "quant_common.cuh"

namespace avr {

constexpr int kFuCols = 128;             // columns per unit (one thread each in the reduce)
constexpr int kFuThreads = 256;

struct FusedParams {
  int64_t l, K;
  int C, T, n_units;        // chunks, column tiles, units = C * T
  int split;                // 1: Averis (mu subtracted); 0: vanilla (amax of X only)
  float* part;              // [3][C][K] chunk partials: sum, max, min
  float* mu_out;            // [K]
  float* slot_xr;           // [G] per-CTA max |X_R| (or max |X|)
  float* slot_mu;           // [G] per-CTA max |mu|
  uint32_t* bar_count;
  uint32_t* bar_gen;
  const uint64_t* wait_limit;   // ns for the grid barriers' waits (0: the default bound)
  uint8_t* codes;
  uint8_t* scales;
  float* g_dec;
  uint64_t seed, offset;
  uint32_t tag;
  uint32_t* status;
  QuantParams aux;          // mean quantization and rank-one row (n_aux leading CTAs)
};

template <bool kBf16, bool kSR>
struct FuCfg {
  static constexpr int kElem = kBf16 ? 2 : 4;
  static constexpr uint32_t kUnitBytes = kChunkRows * kFuCols * kElem;
  static constexpr int kRing = 1;
  static constexpr size_t kAuxOffset = static_cast<size_t>(kRing) * kUnitBytes;
  static constexpr size_t kSmemBytes = kAuxOffset + static_cast<size_t>(kBiasWindow) * sizeof(uint16_t);
};

template <bool kBf16, bool kSR>
__global__ void __launch_bounds__(kFuThreads, kBf16 ? 2 : 1) split_fused_kernel(const __grid_constant__ CUtensorMap map,
                                                                    const FusedParams p) {
  using Cfg = FuCfg<kBf16, kSR>;
  constexpr int kRing = Cfg::kRing;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint16_t* s_mu16 = reinterpret_cast<uint16_t*>(smem + Cfg::kAuxOffset);
  __shared__ uint64_t full[kRing];
  __shared__ float r_tab[128], r_tab_mu[128];
  __shared__ float s_part[kQuantWarps * kRowGroup];
  __shared__ float s_red[2][kFuThreads / 32];
  __shared__ float s_genc, s_gdec;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = static_cast<int>(blockIdx.x), G = static_cast<int>(gridDim.x);
  const int n_mine = b < p.n_units ? (p.n_units - b + G - 1) / G : 0;
  uint32_t phase_bits = 0;   // bit s: parity of the next completion of ring slot s
  uint32_t inflight = 0;     // bit s: a copy into slot s has been issued and not yet waited for

  auto issue = [&](int i, int slot) {   // my unit i into ring slot `slot` (thread 0)
    const int u = b + i * G;
    const int c = u / p.T, t = u - (u / p.T) * p.T;
    mbar_arrive_expect_tx(&full[slot], Cfg::kUnitBytes);
    tma_load_2d(ring + static_cast<size_t>(slot) * Cfg::kUnitBytes, &map, &full[slot], t * kFuCols,
                c * kChunkRows);
    inflight |= 1u << slot;
  };
  auto wait_slot = [&](int slot) {       // every thread; true if the copy landed in time
    const bool ok = mbar_wait(&full[slot], (phase_bits >> slot) & 1u, p.status);
    if (ok) {
      phase_bits ^= 1u << slot;
      inflight &= ~(1u << slot);
    }
    return __syncthreads_and(ok) != 0;
  };
  auto drain = [&]() {                   // bounded waits for copies still in flight, then leave
    if (tid == 0)
      for (int s = 0; s < kRing; ++s)
        if ((inflight >> s) & 1u) mbar_wait(&full[s], (phase_bits >> s) & 1u, nullptr);
    __syncthreads();
  };

  if (smem_u32(smem) & 127u) {                // TMA destinations need 128-byte alignment
    if (tid == 0) raise_status(p.status, AVR_ERR_MISALIGNED);
    return;
  }
  if (tid == 0) {
    prefetch_tensormap(&map);
#pragma unroll
    for (int s = 0; s < kRing; ++s) mbar_init(&full[s], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const uint64_t wait_limit = __ldcg(p.wait_limit);

  // ---------------- phase 1: chunk partials, units kept resident ----------------
  const int n_res = min(kRing, n_mine);        // units that stay in shared memory
  const int first_res = n_mine - n_res;
  if (tid == 0)
    for (int i = 0; i < n_res; ++i) issue(i, i);
  for (int i = 0; i < n_mine; ++i) {
    const int slot = i % kRing;
    if (!wait_slot(slot)) {
      drain();
      return;
    }
    const int u = b + i * G;
    const int c = u / p.T, t = u - c * p.T;
    const int64_t col = static_cast<int64_t>(t) * kFuCols + tid;
    if (tid < kFuCols && col < p.K) {
      const int64_t row0 = static_cast<int64_t>(c) * kChunkRows;
      const int rows = static_cast<int>(min64(kChunkRows, p.l - row0));
      float s = 0.0f, mx = -INFINITY, mn = INFINITY;
      const uint8_t* tile = ring + static_cast<size_t>(slot) * Cfg::kUnitBytes;
      if (kBf16) {
        const uint16_t* v = reinterpret_cast<const uint16_t*>(tile) + tid;
#pragma unroll 8
        for (int r = 0; r < rows; ++r) {
          const float x = __uint_as_float(static_cast<uint32_t>(v[r * kFuCols]) << 16);
          s = __fadd_rn(s, x);
          mx = fmaxf(mx, x);
          mn = fminf(mn, x);
        }
      } else {
        const float* v = reinterpret_cast<const float*>(tile) + tid;
#pragma unroll 8
        for (int r = 0; r < rows; ++r) {
          const float x = v[r * kFuCols];
          s = __fadd_rn(s, x);
          mx = fmaxf(mx, x);
          mn = fminf(mn, x);
        }
      }
      const int64_t o = static_cast<int64_t>(c) * p.K + col;
      const int64_t plane = static_cast<int64_t>(p.C) * p.K;
      p.part[o] = s;
      p.part[plane + o] = mx;
      p.part[2 * plane + o] = mn;
    }
    if (i + kRing < n_mine) {                  // this unit is not resident: reuse its slot
      __syncthreads();
      if (tid == 0) issue(i + kRing, slot);
    }
  }

  if (!grid_barrier(p.bar_count, p.bar_gen, static_cast<uint32_t>(G), p.status, wait_limit)) {
    drain();
    return;
  }

  // ---------------- phase 2: fold a column range, chunks in order ----------------
  {
    const int64_t per = (p.K + G - 1) / G;
    const int64_t j0 = static_cast<int64_t>(b) * per, j1 = min64(p.K, j0 + per);
    const int64_t plane = static_cast<int64_t>(p.C) * p.K;
    float a_xr = 0.0f, a_mu = 0.0f;
    for (int64_t jb = j0; jb < j1; jb += kFuThreads / 32) {
      const int64_t j = jb + warp;                     // this warp's column
      const bool jv = j < j1;
      float S = 0.0f, cmax = -INFINITY, cmin = INFINITY;
      for (int c0 = 0; c0 < p.C; c0 += 32) {
        const int c = c0 + lane;
        float ps = 0.0f, px = -INFINITY, pn = INFINITY;
        if (jv && c < p.C) {
          const int64_t o = static_cast<int64_t>(c) * p.K + j;
          ps = __ldcg(&p.part[o]);
          px = __ldcg(&p.part[plane + o]);
          pn = __ldcg(&p.part[2 * plane + o]);
        }
        const int n = min(32, p.C - c0);
        for (int q = 0; q < n; ++q) {                  // chunk order, the same in every lane
          S = __fadd_rn(S, __shfl_sync(0xFFFFFFFFu, ps, q));
          cmax = fmaxf(cmax, __shfl_sync(0xFFFFFFFFu, px, q));
          cmin = fminf(cmin, __shfl_sync(0xFFFFFFFFu, pn, q));
        }
      }
      if (jv) {
        if (!isfinite(S)) raise_status(p.status, AVR_ERR_NONFINITE);
        if (p.split) {
          const float mu = __fdiv_rn(S, static_cast<float>(p.l));
          if (!isfinite(mu)) raise_status(p.status, AVR_ERR_NONFINITE);
          a_xr = fmaxf(a_xr, fmaxf(__fsub_rn(cmax, mu), __fsub_rn(mu, cmin)));
          a_mu = fmaxf(a_mu, fabsf(mu));
          if (lane == 0) p.mu_out[j] = mu;
        } else {
          a_xr = fmaxf(a_xr, fmaxf(cmax, -cmin));
        }
      }
    }
    if (lane == 0) {
      s_red[0][warp] = a_xr;
      s_red[1][warp] = a_mu;
    }
    __syncthreads();
    if (tid == 0) {
      float x = s_red[0][0], m = s_red[1][0];
#pragma unroll
      for (int w = 1; w < kFuThreads / 32; ++w) {
        x = fmaxf(x, s_red[0][w]);
        m = fmaxf(m, s_red[1][w]);
      }
      p.slot_xr[b] = x;
      p.slot_mu[b] = m;
    }
  }

  if (!grid_barrier(p.bar_count, p.bar_gen, static_cast<uint32_t>(G), p.status, wait_limit)) {
    drain();
    return;
  }

  // ---------------- phase 3: quantize ----------------
  if (warp == 0) {
    const TensorScale ts = tensor_scale(max_of_slots(p.slot_xr, G));
    if (lane == 0) {
      s_genc = ts.g_enc;
      s_gdec = ts.g_dec;
    }
  }
  __syncthreads();
  const float g_enc = s_genc;
  fill_rscale_table(r_tab, g_enc);
  __syncthreads();
  if (b == 0 && tid == 0) *p.g_dec = s_gdec;
  if (b < p.aux.n_aux) aux_cta<kSR, true>(p.aux, s_mu16, s_part, r_tab_mu);

  PhiloxKeys keys;
  if (kSR) keys = philox_keys(p.seed);
  const uint32_t n_kb64 = static_cast<uint32_t>(p.K / 64);
  const int blk = lane & 7, sub = lane >> 3;   // lane: 16-column block, row within a group of 4

  // one unit from ring slot `slot`: 256 rows, a warp does 4 rows x 128 columns per step
  auto quant_unit = [&](int i, int slot) {
    const int u = b + i * G;
    const int c = u / p.T, t = u - c * p.T;
    const int64_t col0 = static_cast<int64_t>(t) * kFuCols + 16 * blk;
    const bool col_ok = col0 < p.K;
    float mu[16];
    if (p.split && col_ok) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(p.mu_out + col0) + q);
        mu[4 * q] = v.x;
        mu[4 * q + 1] = v.y;
        mu[4 * q + 2] = v.z;
        mu[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 16; ++q) mu[q] = 0.0f;
    }
    const uint8_t* tile = ring + static_cast<size_t>(slot) * Cfg::kUnitBytes;
    const int64_t row0 = static_cast<int64_t>(c) * kChunkRows;
    const uint64_t g0 = p.offset + static_cast<uint64_t>((row0 * p.K + col0) / 16);
    const uint64_t g_row = static_cast<uint64_t>(p.K / 16);
    const uint32_t c16 = static_cast<uint32_t>(col0 / 16);
#pragma unroll 2
    for (int st = 0; st < kChunkRows / (kQuantWarps * 4); ++st) {
      const int rr = (st * kQuantWarps + warp) * 4 + sub;        // row within the unit
      const int64_t row = row0 + rr;
      Raw16<kBf16> raw;
      const uint4* src = reinterpret_cast<const uint4*>(tile + (static_cast<size_t>(rr) * kFuCols + 16 * blk) * Cfg::kElem);
#pragma unroll
      for (int q = 0; q < (kBf16 ? 2 : 4); ++q) raw.w[q] = src[q];
      float xr[16];
      sub_mu16<kBf16>(raw, mu, xr);
      const uint4 rw = kSR ? philox_keyed(g0 + static_cast<uint64_t>(rr) * g_row, p.tag, keys)
                           : make_uint4(0u, 0u, 0u, 0u);
      uint32_t S;
      const uint2 packed = quant16<kSR>(xr, g_enc, r_tab, rw, &S);
      const uint32_t sw = gather_scale_word(S);
      if (col_ok && row < p.l) {
        *reinterpret_cast<uint2*>(p.codes + row * (p.K / 2) + col0 / 2) = packed;
        if ((lane & 3) == 0)
          *reinterpret_cast<uint32_t*>(p.scales + scale_offset(static_cast<uint64_t>(row), c16, n_kb64)) = sw;
      }
    }
  };

  // the resident units first; each freed slot takes one of the other units,
  // copied in again, in order (unit k goes to slot (first_res + k) % kRing)
  for (int i = first_res; i < n_mine; ++i) {
    quant_unit(i, i % kRing);
    const int k = i - first_res;
    if (k < first_res) {
      __syncthreads();
      if (tid == 0) issue(k, i % kRing);
    }
  }
  for (int k = 0; k < first_res; ++k) {
    const int slot = (first_res + k) % kRing;
    if (!wait_slot(slot)) {
      drain();
      return;
    }
    quant_unit(k, slot);
    if (k + n_res < first_res) {
      __syncthreads();
      if (tid == 0) issue(k + n_res, slot);
    }
  }
}

template <bool kBf16, bool kSR>
static cudaError_t launch_split_fused_t(const CUtensorMap& map, const FusedParams& p, int grid, cudaStream_t s,
                                        bool pdl) {
  using Cfg = FuCfg<kBf16, kSR>;
  const void* fn = reinterpret_cast<const void*>(split_fused_kernel<kBf16, kSR>);
  cudaError_t e = set_max_dynamic_smem(fn, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (blocks_per_sm(fn, kFuThreads, Cfg::kSmemBytes) < 1) return cudaErrorInvalidConfiguration;
  // A cooperative launch: the runtime refuses a grid whose CTAs cannot all be
  // resident at once, instead of leaving the grid barriers to time out.  It
  // is not combined with programmatic dependent launch.
  (void)pdl;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kFuThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, split_fused_kernel<kBf16, kSR>, map, p);
}

cudaError_t launch_split_fused(const ColReduceArgs& ca, const QuantArgs& qa, cudaStream_t s, bool pdl) {
  const bool bf16 = ca.xt == AVR_BF16;
  CUtensorMap map;
  if (!make_tensor_map_2d(&map, ca.X, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                          bf16 ? 2 : 4, static_cast<uint64_t>(ca.l), static_cast<uint64_t>(ca.K), kChunkRows,
                          kFuCols, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  FusedParams p = {};
  p.l = ca.l;
  p.K = ca.K;
  p.C = static_cast<int>((ca.l + kChunkRows - 1) / kChunkRows);
  p.T = static_cast<int>((ca.K + kFuCols - 1) / kFuCols);
  if (static_cast<int64_t>(p.C) * p.T > int64_t{0x7FFFFFFF}) return cudaErrorInvalidValue;
  p.n_units = p.C * p.T;
  p.split = ca.split;
  p.part = reinterpret_cast<float*>(ca.ws + ca.lay->partials);
  p.mu_out = ca.mu_out;
  p.slot_xr = reinterpret_cast<float*>(ca.ws + ca.lay->slots);
  p.slot_mu = p.slot_xr + kMaxColTiles;
  p.status = reinterpret_cast<uint32_t*>(ca.ws + ca.lay->status);
  p.bar_count = p.status + 16;      // 64 and 128 bytes into the status block
  p.bar_gen = p.status + 32;
  p.wait_limit = reinterpret_cast<const uint64_t*>(ca.ws + ca.lay->status + kWaitLimitOffset);
  p.codes = qa.codes;
  p.scales = qa.scales;
  p.g_dec = qa.g_dec;
  p.seed = qa.seed;
  p.offset = qa.offset;
  p.tag = qa.tag;
  // every CTA of the grid must be resident at once (grid-wide barriers)
  const void* fn = bf16 ? (qa.sr ? reinterpret_cast<const void*>(split_fused_kernel<true, true>)
                                 : reinterpret_cast<const void*>(split_fused_kernel<true, false>))
                        : (qa.sr ? reinterpret_cast<const void*>(split_fused_kernel<false, true>)
                                 : reinterpret_cast<const void*>(split_fused_kernel<false, false>));
  const size_t smem = bf16 ? FuCfg<true, true>::kSmemBytes : FuCfg<false, true>::kSmemBytes;
  {
    cudaError_t e = set_max_dynamic_smem(fn, smem);
    if (e != cudaSuccess) return e;
  }
  const int per_sm = blocks_per_sm(fn, kFuThreads, smem);
  const int resident = sm_count() * (per_sm < 1 ? 1 : per_sm);
  const int grid = p.n_units < resident ? p.n_units : resident;
  // mean quantization and rank-one row, as the split quantizer's aux CTAs do them
  QuantParams& a = p.aux;
  a.K = ca.K;
  a.mu = ca.split ? ca.mu_out : nullptr;
  a.seed = qa.seed;
  a.offset = qa.offset;
  a.status = p.status;
  a.slot_mu = p.slot_mu;
  a.n_tiles = grid;
  a.tag_mu = qa.tag_mu;
  a.mu_codes = qa.mu_codes;
  a.mu_scales = qa.mu_scales;
  a.mu_gdec = qa.mu_gdec;
  a.w_codes = qa.w_codes;
  a.w_scales = qa.w_scales;
  a.w_gdec = qa.w_gdec;
  a.n_out = qa.n_out;
  a.bias = qa.bias;
  a.n_aux = 0;
  if (ca.split && (qa.mu_codes != nullptr || qa.w_codes != nullptr)) {
    int n_aux = 1;
    if (qa.w_codes != nullptr) {
      const int64_t want = (qa.n_out + kRowGroup - 1) / kRowGroup;
      const int cap = grid / 8 > 1 ? grid / 8 : 1;
      n_aux = static_cast<int>(want < cap ? want : cap);
    }
    a.n_aux = n_aux < grid ? n_aux : grid;
  }
  if (ca.l % 128 != 0) {
    cudaError_t e = launch_zero_scale_padding(qa.scales, ca.l, ca.K, s);
    if (e != cudaSuccess) return e;
    pdl = false;
  }
  if (bf16)
    return qa.sr ? launch_split_fused_t<true, true>(map, p, grid, s, pdl)
                 : launch_split_fused_t<true, false>(map, p, grid, s, pdl);
  return qa.sr ? launch_split_fused_t<false, true>(map, p, grid, s, pdl)
               : launch_split_fused_t<false, false>(map, p, grid, s, pdl);
}

}  // namespace avr
