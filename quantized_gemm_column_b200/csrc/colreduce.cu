// K1: deterministic column reduce -- the "reduce" of the Averis split.
//
// mu_X = (1/l) 1^T X (Lighthouse review of "The Curse and Blessing of Mean
// Bias in FP4-Quantized LLM Training", section 二 2.1), computed in a fixed
// fp32 order so that every run and the CPU oracle give the same bits:
//   p[c][j] = (((+0 + x[256c][j]) + x[256c+1][j]) + ...)    rows of chunk c in order
//   S[j]    = (((+0 + p[0][j]) + p[1][j]) + ...)              chunks in order
//   mu[j]   = S[j] / l                                        IEEE division
// The same pass keeps the column max and min, so the fold of a column tile
// can also give max_i |fl(x_ij - mu_j)| = max(fl(colmax - mu), fl(mu - colmin))
// (rounded subtraction is monotone), the amax the residual's tensor scale
// needs, without a third pass over X.
//
// colreduce_kernel: grid (column tiles of 128, chunks of 256 rows).  One TMA
// copy brings the 256 x 128 tile into shared memory; thread j then runs the
// sequential sum of column j over the chunk, and the partials go to the
// workspace.  The tile's fold (the partials summed in chunk order, mu and the
// tile's amax slots) is then either a separate fold_kernel launch (the dense
// split and vanilla amax: the reduce takes no tickets), or run by the CTA
// that takes the tile's last ticket (the R monitor's and the MoE layer's
// reduces; atomicInc wraps the ticket back to 0).
#include "device.cuh"
#include "internal.h"

namespace avr {

struct ColReduceParams {
  int64_t l, K;
  int C;                  // chunks
  int split;
  float* part;            // [3][C][K]: sum, max, min
  uint32_t* tickets;      // [T]
  float* slot_xr;         // [T] max |X_R| (split) or max |X| (vanilla)
  float* slot_mu;         // [T] max |mu|
  float* mu_out;          // [K]
  float* part_e;          // [C][K]: sum of squares (energy pass only)
  float* energy;          // [K] column sums of squares, chunks in order (energy pass only)
  uint32_t* status;
  // grouped (MoE) mode: blockIdx.y is a global chunk index; chunk_expert maps it
  // to its expert, whose segment, chunk range, mean and slots it uses (null: dense)
  const MoeSeg* seg;
  const int32_t* chunk_expert;
  const int32_t* totals;  // [1]: chunks in use
  int T;                  // column tiles (slot and ticket stride per expert)
};

// Sequential fp32 sum, max and min (and sum of squares) of column `tid` of a
// 256 x 128 chunk in shared memory, rows in order.  The shared-memory loads
// of kRowBatch rows are issued before the first add of the batch, so the
// thread waits for one load latency per batch, not per row.
constexpr int kRowBatch = 16;

__device__ __forceinline__ void stats_step(float x, float& s, float& mx, float& mn) {
  s = __fadd_rn(s, x);
  mx = fmaxf(mx, x);
  mn = fminf(mn, x);
}

template <bool kBf16, bool kEnergy>
__device__ __forceinline__ void chunk_column_stats(const uint8_t* tile, int tid, int rows, float& s, float& mx,
                                                   float& mn, float& e) {
  s = 0.0f;
  mx = -INFINITY;
  mn = INFINITY;
  e = 0.0f;
  int i = 0;
  if (kBf16) {
    const uint16_t* v = reinterpret_cast<const uint16_t*>(tile) + tid;
    for (; i + kRowBatch <= rows; i += kRowBatch) {
      uint32_t w[kRowBatch];
#pragma unroll
      for (int k = 0; k < kRowBatch; ++k) w[k] = v[(i + k) * kColTile];
#pragma unroll
      for (int k = 0; k < kRowBatch; ++k) {
        const float x = __uint_as_float(w[k] << 16);
        stats_step(x, s, mx, mn);
        if (kEnergy) e = __fmaf_rn(x, x, e);
      }
    }
    for (; i < rows; ++i) {
      const float x = __uint_as_float(static_cast<uint32_t>(v[i * kColTile]) << 16);
      stats_step(x, s, mx, mn);
      if (kEnergy) e = __fmaf_rn(x, x, e);
    }
  } else {
    const float* v = reinterpret_cast<const float*>(tile) + tid;
    for (; i + kRowBatch <= rows; i += kRowBatch) {
      float w[kRowBatch];
#pragma unroll
      for (int k = 0; k < kRowBatch; ++k) w[k] = v[(i + k) * kColTile];
#pragma unroll
      for (int k = 0; k < kRowBatch; ++k) {
        stats_step(w[k], s, mx, mn);
        if (kEnergy) e = __fmaf_rn(w[k], w[k], e);
      }
    }
    for (; i < rows; ++i) {
      const float x = v[i * kColTile];
      stats_step(x, s, mx, mn);
      if (kEnergy) e = __fmaf_rn(x, x, e);
    }
  }
}

template <bool kEnergy>
__device__ __forceinline__ void store_partials(const ColReduceParams& p, int c, int64_t col, float s, float mx,
                                               float mn, float e) {
  if (kEnergy) p.part_e[static_cast<int64_t>(c) * p.K + col] = e;
  const int64_t o = static_cast<int64_t>(c) * p.K + col;
  const int64_t plane = static_cast<int64_t>(p.C) * p.K;
  p.part[o] = s;
  p.part[plane + o] = mx;
  p.part[2 * plane + o] = mn;
}

// The fold of one column tile, run by every thread of a fold_kernel CTA or of
// the CTA that took the tile's last ticket.  The tile's chunk partials (three
// planes) come into the CTA's shared buffer by TMA, kFoldRows chunks of each plane per round,
// one round trip per round; each thread then sums its column's partials in
// chunk order from shared memory, writes mu and, through a CTA max, the
// tile's two amax slots.  `phase` is the parity of the tile barrier's next
// phase.  Returns false if a copy never landed (status set).
constexpr int kFoldRows = 40;                      // 3 planes x 40 x 128 fp32 = 60 KB of the tile buffer
constexpr uint32_t kFoldPlaneBytes = kFoldRows * kColTile * 4;

template <bool kEnergy>
__device__ __forceinline__ bool fold_tile(const ColReduceParams& p, int tid, int64_t col, int t, int c_first,
                                          int c_count, int64_t n_rows, float* mu_out, int slot,
                                          float (*s_red)[kColTile / 32], uint8_t* tile, uint64_t* bar,
                                          const CUtensorMap* pmap, uint32_t phase, uint32_t* s_ok) {
  float a_xr = 0.0f, a_mu = 0.0f;
  float S = 0.0f, cmax = -INFINITY, cmin = INFINITY;
  const float* sp = reinterpret_cast<const float*>(tile);
  for (int c0 = 0; c0 < c_count; c0 += kFoldRows) {
    const int n = c_count - c0 < kFoldRows ? c_count - c0 : kFoldRows;
    __syncthreads();                                // the buffer's previous contents are no longer read
    if (tid == 0) {
      fence_proxy_async_smem();                     // ... before the copies overwrite it
      fence_proxy_async_global();                   // the acquired partials, for the copy engine
      mbar_arrive_expect_tx(bar, 3 * kFoldPlaneBytes);
#pragma unroll
      for (int pl = 0; pl < 3; ++pl)
        tma_load_2d(tile + pl * kFoldPlaneBytes, pmap, bar, t * kColTile, pl * p.C + c_first + c0);
      *s_ok = mbar_wait(bar, phase, p.status) ? 1u : 0u;
      if (!*s_ok) mbar_wait(bar, phase, nullptr);   // a second bounded wait for the copies in flight
    }
    __syncthreads();
    if (!*s_ok) return false;
    phase ^= 1u;
    if (col < p.K) {
#pragma unroll 8
      for (int u = 0; u < n; ++u) {
        S = __fadd_rn(S, sp[u * kColTile + tid]);
        cmax = fmaxf(cmax, sp[(kFoldRows + u) * kColTile + tid]);
        cmin = fminf(cmin, sp[(2 * kFoldRows + u) * kColTile + tid]);
      }
    }
  }
  if (col < p.K && kEnergy) {
    // the column's sum of squares, chunks in order
    constexpr int kBatch = 16;
    float E = 0.0f;
    for (int c0 = 0; c0 < p.C; c0 += kBatch) {
      float pe[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (c0 + u < p.C) pe[u] = __ldcg(&p.part_e[static_cast<int64_t>(c0 + u) * p.K + col]);
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (c0 + u < p.C) E = __fadd_rn(E, pe[u]);
    }
    p.energy[col] = E;
  }
  if (col < p.K) {
    if (!isfinite(S)) raise_status(p.status, AVR_ERR_NONFINITE);
    if (p.split) {
      const float mu = __fdiv_rn(S, static_cast<float>(n_rows));
      if (!isfinite(mu)) raise_status(p.status, AVR_ERR_NONFINITE);
      a_xr = fmaxf(__fsub_rn(cmax, mu), __fsub_rn(mu, cmin));
      a_mu = fabsf(mu);
      mu_out[col] = mu;
    } else {
      a_xr = fmaxf(cmax, -cmin);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a_xr = fmaxf(a_xr, __shfl_xor_sync(0xFFFFFFFFu, a_xr, o));
    a_mu = fmaxf(a_mu, __shfl_xor_sync(0xFFFFFFFFu, a_mu, o));
  }
  if ((tid & 31) == 0) {
    s_red[0][tid >> 5] = a_xr;
    s_red[1][tid >> 5] = a_mu;
  }
  __syncthreads();
  if (tid == 0) {
    float x = s_red[0][0], m = s_red[1][0];
#pragma unroll
    for (int w = 1; w < kColTile / 32; ++w) {
      x = fmaxf(x, s_red[0][w]);
      m = fmaxf(m, s_red[1][w]);
    }
    p.slot_xr[slot] = x;
    p.slot_mu[slot] = m;
  }
  return true;
}

template <bool kBf16, bool kEnergy, bool kGrouped, bool kDeferFold>
__global__ void __launch_bounds__(kColTile) colreduce_kernel(const __grid_constant__ CUtensorMap map,
                                                             const __grid_constant__ CUtensorMap pmap,
                                                             const ColReduceParams p) {
  extern __shared__ __align__(1024) uint8_t tile[];
  __shared__ uint64_t bar;
  __shared__ uint32_t s_last, s_ok;
  __shared__ float s_red[2][kColTile / 32];

  const int tid = threadIdx.x;
  const int t = blockIdx.x;
  const int c = blockIdx.y;                    // chunk index into the partials
  const int64_t col = static_cast<int64_t>(t) * kColTile + tid;
  // this chunk's rows, the chunks folded with it, the slot and mean it feeds
  int64_t row0 = static_cast<int64_t>(c) * kChunkRows;
  int64_t n_rows = p.l;                        // rows of the (expert's) matrix
  int c_first = 0, c_count = p.C, slot = t;
  float* mu_out = p.mu_out;
  if (kGrouped) {
    pdl_wait_prior_grid();                     // the segment table comes from the previous launch
    if (c >= __ldcg(p.totals)) return;         // a chunk past the last expert's
    const int e = __ldcg(p.chunk_expert + c);
    const MoeSeg sg = p.seg[e];
    c_first = sg.chunk0;
    c_count = sg.chunks;
    row0 = sg.row0 + static_cast<int64_t>(c - sg.chunk0) * kChunkRows;
    n_rows = sg.rows;
    slot = e * p.T + t;
    mu_out = p.mu_out + static_cast<int64_t>(e) * p.K;
  }
  const int rows = static_cast<int>(min64(kChunkRows, n_rows - static_cast<int64_t>(c - c_first) * kChunkRows));
  constexpr uint32_t kElem = kBf16 ? 2u : 4u;
  constexpr uint32_t kTileBytes = kChunkRows * kColTile * kElem;

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
    tma_load_2d(tile, &map, &bar, t * kColTile, static_cast<int32_t>(row0));
    s_ok = mbar_wait(&bar, 0, p.status) ? 1u : 0u;
    if (!s_ok) mbar_wait(&bar, 0, nullptr);   // a second bounded wait for the copy in flight
  }
  __syncthreads();
  if (!s_ok) return;

  // Sequential fp32 sum of this column over the chunk, plus max and min.
  if (col < p.K) {
    float sum, mx, mn, e;
    chunk_column_stats<kBf16, kEnergy>(tile, tid, rows, sum, mx, mn, e);
    store_partials<kEnergy>(p, c, col, sum, mx, mn, e);
  }

  if (kDeferFold) return;   // fold_kernel, the next launch, folds every tile

  // Last CTA of this column tile finalizes it.  The CTA barrier orders every
  // thread's partial stores before thread 0's ticket, an acquire-release
  // increment at GPU scope: it publishes them (release, cumulative over the
  // barrier) and, for the last CTA, makes every other CTA's partials visible
  // to the fold below (acquire, passed on by the second barrier).
  __syncthreads();
  if (tid == 0) s_last = ticket_inc_acq_rel(&p.tickets[slot], static_cast<uint32_t>(c_count - 1)) ==
                         static_cast<uint32_t>(c_count - 1);
  __syncthreads();
  if (!s_last) return;

  if (tid == 0) prefetch_tensormap(&pmap);
  fold_tile<kEnergy>(p, tid, col, t, c_first, c_count, n_rows, mu_out, slot, s_red, tile, &bar, &pmap, 1u, &s_ok);
}

// The fold as its own launch, one CTA per column tile, after a reduce that
// took no tickets (the dense split and vanilla amax): the partials are
// complete once the reduce grid is, so its CTAs hold their SM slots only for
// the copy and the sum.
__global__ void __launch_bounds__(kColTile) fold_kernel(const __grid_constant__ CUtensorMap pmap,
                                                        const ColReduceParams p) {
  extern __shared__ __align__(1024) uint8_t buf[];
  __shared__ uint64_t bar;
  __shared__ uint32_t s_ok;
  __shared__ float s_red[2][kColTile / 32];
  const int tid = threadIdx.x, t = blockIdx.x;
  if (tid == 0) {
    prefetch_tensormap(&pmap);
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  fold_tile<false>(p, tid, static_cast<int64_t>(t) * kColTile + tid, t, 0, p.C, p.l, p.mu_out, t, s_red, buf, &bar,
                   &pmap, 0u, &s_ok);
}

template <bool kBf16, bool kEnergy, bool kGrouped, bool kDeferFold = false>
static cudaError_t launch_colreduce_t(const CUtensorMap& map, const CUtensorMap& pmap, const ColReduceParams& p,
                                      dim3 grid, size_t smem, cudaStream_t s, bool pdl) {
  const void* fn = reinterpret_cast<const void*>(colreduce_kernel<kBf16, kEnergy, kGrouped, kDeferFold>);
  cudaError_t e = set_max_dynamic_smem(fn, smem);
  if (e != cudaSuccess) return e;
  e = launch_ex(colreduce_kernel<kBf16, kEnergy, kGrouped, kDeferFold>, grid, dim3(kColTile), smem, s, pdl, map,
                pmap, p);
  if (e != cudaSuccess || !kDeferFold) return e;
  const size_t fold_smem = 3 * static_cast<size_t>(kFoldPlaneBytes);
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(fold_kernel), fold_smem);
  if (e != cudaSuccess) return e;
  return launch_ex(fold_kernel, dim3(grid.x), dim3(kColTile), fold_smem, s, true, pmap, p);
}

cudaError_t launch_colreduce(const ColReduceArgs& a, cudaStream_t s, bool pdl) {
  const bool bf16 = a.xt == AVR_BF16;
  const int elem = bf16 ? 2 : 4;
  CUtensorMap map;
  if (!make_tensor_map_2d(&map, a.X, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                          elem, static_cast<uint64_t>(a.l), static_cast<uint64_t>(a.K), kChunkRows,
                          kColTile, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  ColReduceParams p;
  p.l = a.l;
  p.K = a.K;
  p.C = a.seg ? a.c_max : static_cast<int>((a.l + kChunkRows - 1) / kChunkRows);
  p.split = a.split;
  p.part = reinterpret_cast<float*>(a.ws + a.lay->partials);
  p.tickets = reinterpret_cast<uint32_t*>(a.ws + a.lay->tickets);
  p.slot_xr = reinterpret_cast<float*>(a.ws + a.lay->slots);
  p.slot_mu = p.slot_xr + kMaxColTiles;
  p.mu_out = a.mu_out;
  p.part_e = reinterpret_cast<float*>(a.ws + a.lay->energy_partials);
  p.energy = reinterpret_cast<float*>(a.ws + a.lay->energy);
  p.status = reinterpret_cast<uint32_t*>(a.ws + a.lay->status);
  p.seg = a.seg;
  p.chunk_expert = a.chunk_expert;
  p.totals = a.totals;
  const int T = static_cast<int>((a.K + kColTile - 1) / kColTile);
  p.T = T;
  if (p.C < 1) return cudaSuccess;
  // the partials as a [3 C, K] fp32 array, for the fold's copies
  CUtensorMap pmap;
  if (!make_tensor_map_2d(&pmap, p.part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 3 * static_cast<uint64_t>(p.C),
                          static_cast<uint64_t>(a.K), kFoldRows, kColTile, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(kChunkRows) * kColTile * elem;
  static_assert(3 * kFoldPlaneBytes <= kChunkRows * kColTile * 2, "fold rounds fit the bf16 tile buffer");
  const dim3 grid(T, p.C);
  if (a.seg != nullptr)   // grouped (MoE): no energy pass
    return bf16 ? launch_colreduce_t<true, false, true>(map, pmap, p, grid, smem, s, pdl)
                : launch_colreduce_t<false, false, true>(map, pmap, p, grid, smem, s, pdl);
  if (a.energy) {
    return bf16 ? launch_colreduce_t<true, true, false>(map, pmap, p, grid, smem, s, pdl)
                : launch_colreduce_t<false, true, false>(map, pmap, p, grid, smem, s, pdl);
  }
  return bf16 ? launch_colreduce_t<true, false, false, true>(map, pmap, p, grid, smem, s, pdl)
              : launch_colreduce_t<false, false, false, true>(map, pmap, p, grid, smem, s, pdl);
}

// ---------------------------------------------------------------------------
// Mean-energy ratio R = ||mu||_2 / sqrt(E||x||^2 / m) (Lighthouse review,
// 实践建议 item 2, with N read as the feature count m), from the reduce's mu
// and column sums of squares: E||x||^2 = (1/l) sum_j energy_j.  One CTA; the
// two sums run in fp64 in a fixed order (thread t over columns t, t + 256,
// ..., then a fixed tree).
// ---------------------------------------------------------------------------
constexpr int kRatioThreads = 256;

__global__ void __launch_bounds__(kRatioThreads) energy_ratio_kernel(const float* mu, const float* energy, int64_t K,
                                                                     int64_t l, float* R, uint32_t* status) {
  __shared__ double s_m[kRatioThreads], s_e[kRatioThreads];
  pdl_wait_prior_grid();
  double sm = 0.0, se = 0.0;
  for (int64_t j = threadIdx.x; j < K; j += kRatioThreads) {
    const double u = static_cast<double>(__ldcg(mu + j));
    sm = fma(u, u, sm);
    se += static_cast<double>(__ldcg(energy + j));
  }
  s_m[threadIdx.x] = sm;
  s_e[threadIdx.x] = se;
  __syncthreads();
  for (int w = kRatioThreads / 2; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) {
      s_m[threadIdx.x] += s_m[threadIdx.x + w];
      s_e[threadIdx.x] += s_e[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double mean_sq = s_e[0] / static_cast<double>(l) / static_cast<double>(K);   // E||x||^2 / m
    const double r = mean_sq > 0.0 ? sqrt(s_m[0]) / sqrt(mean_sq) : 0.0;
    if (!isfinite(r)) raise_status(status, AVR_ERR_NONFINITE);
    *R = static_cast<float>(r);
  }
}

cudaError_t launch_energy_ratio(const float* mu, const float* energy, int64_t K, int64_t l, float* R,
                                uint32_t* status, cudaStream_t s, bool pdl) {
  return launch_ex(energy_ratio_kernel, dim3(1), dim3(kRatioThreads), 0, s, pdl, mu, energy, K, l, R, status);
}

}  // namespace avr
