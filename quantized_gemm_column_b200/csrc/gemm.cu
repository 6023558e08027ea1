// K3: block-scaled FP4 GEMM on the 5th-generation tensor cores (tcgen05),
// with the Averis rank-one row as a broadcast bias in the epilogue.
//
// Y = 1 (mu_bar W_bar) + X_bar_R W_bar (Lighthouse review of "The Curse and
// Blessing of Mean Bias in FP4-Quantized LLM Training", section 二 "Averis
// 方法"): the product X_bar_R W_bar runs here on E2M1 operands with E4M3
// per-16 scales, and the row mu_bar W_bar (one value per output column) is
// added to every output row:
//   Y[i, j] = g_dec(A) g_dec(B) * acc[i, j] + bias[j].
// The weight gradient's rank-one term l mu_bar_X^T mu_bar_D uses the same
// epilogue with a row factor: Y[i, j] = alpha acc[i, j] + u[i] v[j].
//
// Persistent kernel, one CTA per SM; each CTA takes a contiguous run of
// output tiles, M fastest, so consecutive tiles share their B (weight)
// columns.  K is staged 256 elements (128 bytes per row, 128-byte swizzle) at
// a time.
//   warp 0     : allocates tensor memory; one thread copies the scale atoms
//                shared -> tensor memory (tcgen05.cp 32x128b, replicated into
//                the four lane quarters) and issues
//                tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M 128, K 64);
//   warps 1..4 : producers, one TMA operation each per stage -- the A code
//                tile, the B code tile, and A's and B's 512-byte scale atoms
//                (2-D copies over the atom array, out-of-range atoms read as
//                zero).  A thread issues one bulk copy at a time, so the
//                copies of a stage go out from separate warps;
//   warps 5..  : epilogue -- the tile's bias row is fetched into registers
//                while the mainloop runs; tcgen05.ld of the accumulator (each
//                warp one 32-lane quarter and a run of columns), alpha * acc +
//                bias, convert, a 128-byte-swizzled staging tile, TMA store.
//
// Resident weight scales (bf16 output, K <= 1792): the scale copies cost as
// much tensor-pipe time as the MMAs they feed, and B's scales repeat for
// every tile of a column block.  So when all of K's B scales fit in tensor
// memory beside the accumulator, warp 4 loads them once per column block into
// a shared buffer, the MMA thread copies them into tensor memory once, and a
// stage then needs only A's four scale copies.
#include "device.cuh"
#include "internal.h"

namespace avr {

// Two tile shapes:
//  BN = 256 (bf16 output): MMAs of M 128 x N 256, the shape that reaches the
//    tensor cores' rate; 3 stages; one accumulator of 256 columns, released to
//    the MMA thread as soon as its last tcgen05.ld lands; the 64 KB output
//    tile leaves through a 32 KB staging buffer in two rounds.
//  BN = 128 (fp32 output): 4 stages; two accumulators, so the epilogue
//    overlaps the next tile's mainloop; a 64 KB staging tile.
template <int BN, bool kBf16Out>
struct GemmCfg {
  static constexpr int kBM = 128, kBN = BN;
  static constexpr int kStageK = 256;                      // fp4 elements per stage
  static constexpr int kRowBytes = kStageK / 2;            // 128 bytes per row
  static constexpr int kStages = BN == 256 ? 3 : 4;
  static constexpr int kKbPerStage = kStageK / 64;         // MMAs per stage
  static constexpr int kAccBufs = BN == 256 ? 1 : 2;
  static constexpr int kEpiWarps = BN / 32;                // 8 or 4
  static constexpr int kFirstEpiWarp = 5;
  static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
  static constexpr uint32_t kSwizzle = kLayoutSwizzle128B;
  static constexpr uint32_t kSbo = 8 * kRowBytes;          // 8-row swizzle atom
  static constexpr int kABytes = kBM * kRowBytes;
  static constexpr int kBBytes = kBN * kRowBytes;
  static constexpr int kSfaBytes = kKbPerStage * 512;      // one 128-row group
  static constexpr int kSfbBytes = (kBN / 128) * kKbPerStage * 512;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kOutElem = kBf16Out ? 2 : 4;
  static constexpr int kBoxCols = 128 / kOutElem;          // columns per 128-byte swizzled store box
  static constexpr int kOutRounds = kBf16Out ? 2 : 1;      // staging rounds per tile
  static constexpr int kStageOutBytes = kBM * kBN * kOutElem / kOutRounds;
  static constexpr int kBoxesPerRound = kBN / kBoxCols / kOutRounds;
  // resident B scales (bf16 output only): up to kResMaxKb k-blocks
  static constexpr int kAccCols = kBN;
  static constexpr int kSfaCols = kKbPerStage * 4;
  static constexpr int kSfbCols = kKbPerStage * (kBN / 32);
  static constexpr int kSfCol = kAccBufs * kAccCols;       // scale buffers after the accumulators
  static constexpr int kTmemCols = 512;
  static constexpr int kResSfbCol = kSfCol + 2 * kSfaCols;  // resident mode: SFA x2, then all of SFB
  static constexpr int kResMaxKb = kBf16Out ? (kTmemCols - kResSfbCol) / (kBN / 32) : 0;
  static constexpr int kResMaxStages = kResMaxKb / kKbPerStage;
  static constexpr int kResBytes = kResMaxStages * kSfbBytes;
  static constexpr int kOutOffset = kStages * kStageBytes;
  static constexpr int kResOffset = kOutOffset + kStageOutBytes;
  static constexpr int kBarOffset = kResOffset + kResBytes;
  // dynamic shared memory starts 1024-aligned when a kernel has no static
  // shared memory; the kernel checks it and refuses to run otherwise
  static constexpr int kSmemBytes = kBarOffset + 128;
  static_assert(kSfCol + 2 * (kSfaCols + kSfbCols) <= kTmemCols, "tensor memory budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  // instruction descriptor: E2M1 A and B (format 1), UE4M3 scales, K-major
  // operands, N >> 3 at bit 17, M >> 4 at bit 24
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                                     (static_cast<uint32_t>(kBM >> 4) << 24);
};

struct GemmParams {
  int64_t M, N, K;
  int tiles_m, num_tiles;
  int sfb_resident;       // 1: B's scales for all of K live in tensor memory
  const float* gdec_a;
  const float* gdec_b;
  const float* bias;
  const float* row_scale;   // rank-one epilogue only: Y = alpha acc + row_scale[i] bias[j]
  uint32_t* status;
  // grouped (MoE) mode, null for one GEMM: A's 128-row block b belongs to
  // expert block_expert[b], whose B rows start at e * N (experts stacked), and
  // whose decode scales and bias row are gdec_a[e], gdec_b[e], bias + e * N;
  // totals[1] = the rows in use (a multiple of 128)
  const int32_t* block_expert;
  const int32_t* totals;
};

// The contiguous run of tiles [first, first + count) of this CTA; tile t is
// (m block t mod tiles_m, n block t / tiles_m).
struct TileRun {
  int first, count;
  __device__ __forceinline__ TileRun(int num_tiles) {
    const int q = num_tiles / static_cast<int>(gridDim.x), r = num_tiles % static_cast<int>(gridDim.x);
    const int b = static_cast<int>(blockIdx.x);
    first = b * q + (b < r ? b : r);
    count = q + (b < r ? 1 : 0);
  }
};

template <int BN, bool kBf16Out, bool kRank1, bool kGrouped>
__global__ void __launch_bounds__(GemmCfg<BN, kBf16Out>::kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                      const __grid_constant__ CUtensorMap map_y, const GemmParams p) {
  using Cfg = GemmCfg<BN, kBf16Out>;
  constexpr int kEpiThreads = 32 * Cfg::kEpiWarps;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {            // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) raise_status(p.status, AVR_ERR_MISALIGNED);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sA = smem;
  uint8_t* sB = sA + Cfg::kStages * Cfg::kABytes;
  uint8_t* sSfa = sB + Cfg::kStages * Cfg::kBBytes;
  uint8_t* sSfb = sSfa + Cfg::kStages * Cfg::kSfaBytes;
  uint8_t* sOut = smem + Cfg::kOutOffset;
  uint8_t* sRes = smem + Cfg::kResOffset;      // resident B scales, one kSfbBytes slab per stage of K
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);
  uint64_t* empty = full + Cfg::kStages;
  uint64_t* acc_full = empty + Cfg::kStages;   // [kAccBufs]
  uint64_t* acc_empty = acc_full + 2;          // [kAccBufs]
  uint64_t* res_full = acc_empty + 2;          // resident B scales loaded
  uint64_t* res_empty = res_full + 1;          // resident B scales copied to tensor memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_empty + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_kst = static_cast<int>((p.K + Cfg::kStageK - 1) / Cfg::kStageK);
  const bool res = p.sfb_resident != 0;
  constexpr bool grouped = kGrouped;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
    prefetch_tensormap(&map_sfa);
    prefetch_tensormap(&map_sfb);
    prefetch_tensormap(&map_y);
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], res ? 3 : 4);        // one arrival per per-stage producer warp
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < Cfg::kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], Cfg::kEpiWarps);   // one arrival per epilogue warp
    }
    mbar_init(res_full, 1);
    mbar_init(res_empty, 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  // grouped: only the blocks of the experts' segments are tiles (a device count)
  int tiles_m = p.tiles_m, num_tiles = p.num_tiles;
  if (grouped) {
    tiles_m = __ldcg(p.totals + 1) / Cfg::kBM;
    num_tiles = tiles_m * (p.num_tiles / p.tiles_m);
  }
  const TileRun run(num_tiles);
  auto expert_of = [&](int32_t m0) { return grouped ? __ldg(p.block_expert + m0 / Cfg::kBM) : 0; };

  if (warp >= 1 && warp <= 4) {
    if (lane == 0) {
      // ---------------- producers: warp 1 A, 2 B, 3 A's scales, 4 B's scales ----------------
      const int role = warp - 1;
      if (role == 3 && res) {
        // B's scales for all of K, once per column block
        int n_prev = -1, uses = 0;
        for (int i = 0; i < run.count; ++i) {
          const int n_blk = (run.first + i) / tiles_m;
          if (n_blk == n_prev) continue;
          n_prev = n_blk;
          if (uses >= 1 && !mbar_wait(res_empty, static_cast<uint32_t>(uses - 1) & 1u, p.status)) break;
          ++uses;
          mbar_arrive_expect_tx(res_full, static_cast<uint32_t>(n_kst * Cfg::kSfbBytes));
          for (int ks = 0; ks < n_kst; ++ks)
            tma_load_2d(sRes + ks * Cfg::kSfbBytes, &map_sfb, res_full, ks * 256, n_blk * (Cfg::kBN / 128));
        }
      } else {
        uint32_t st = 0, ph = 0;
        int it = 0;
        bool ok = true;
        for (int i = 0; i < run.count && ok; ++i) {
          const int tile = run.first + i;
          const int32_t m0 = (tile % tiles_m) * Cfg::kBM;
          const int32_t n0 = (tile / tiles_m) * Cfg::kBN;
          const int32_t nb0 = n0 + (grouped ? expert_of(m0) * static_cast<int32_t>(p.N) : 0);   // B's first row
          for (int ks = 0; ks < n_kst; ++ks, ++it) {
            if (it >= Cfg::kStages && !mbar_wait(&empty[st], ph ^ 1u, p.status)) {
              ok = false;
              break;
            }
            if (role == 0) {
              mbar_arrive_expect_tx(&full[st], Cfg::kABytes);
              tma_load_2d(sA + st * Cfg::kABytes, &map_a, &full[st], ks * Cfg::kRowBytes, m0);
            } else if (role == 1) {
              mbar_arrive_expect_tx(&full[st], Cfg::kBBytes);
              tma_load_2d(sB + st * Cfg::kBBytes, &map_b, &full[st], ks * Cfg::kRowBytes, nb0);
            } else if (role == 2) {
              // 4 atoms (2 KB) of the tile's 128-row group, as 256 eight-byte elements
              mbar_arrive_expect_tx(&full[st], Cfg::kSfaBytes);
              tma_load_2d(sSfa + st * Cfg::kSfaBytes, &map_sfa, &full[st], ks * 256, m0 / 128);
            } else {
              mbar_arrive_expect_tx(&full[st], Cfg::kSfbBytes);
              tma_load_2d(sSfb + st * Cfg::kSfbBytes, &map_sfb, &full[st], ks * 256, nb0 / 128);
            }
            if (++st == Cfg::kStages) {
              st = 0;
              ph ^= 1u;
            }
          }
        }
      }
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      // The issuing thread is on the critical path: every tcgen05 instruction
      // it is late with idles the tensor pipe, so the loop keeps its
      // bookkeeping to increments (stage, phase and scale-buffer counters)
      // and issues a full stage's copies and MMAs unrolled, with descriptors
      // advanced by constants (16-byte units: +32 per 512-byte scale atom, +2
      // per 32-byte k-block step).  A tile's first copies go out before the
      // wait for its accumulator: they write the scale area, not the
      // accumulator, and so overlap the previous tile's epilogue.
      uint32_t st = 0, ph = 0, sf_buf = 0;
      const int n_full = static_cast<int>(p.K / Cfg::kStageK);               // stages of kKbPerStage k-blocks
      const int tail_kb = static_cast<int>((p.K % Cfg::kStageK) / 64);       // k-blocks of a last, partial stage
      const uint32_t sfa_stride = res ? Cfg::kSfaCols : Cfg::kSfaCols + Cfg::kSfbCols;
      auto wait_acc_empty = [&](int ab, int use) {
        if (!mbar_wait_poll(&acc_empty[ab], static_cast<uint32_t>(use - 1) & 1u, p.status)) return false;
        tc_fence_after();
        return true;
      };
      int n_prev = -1, res_uses = 0;
      bool ok = true;
      for (int i = 0; i < run.count && ok; ++i) {
        const int tile = run.first + i;
        const int ab = i % Cfg::kAccBufs;
        const int use = i / Cfg::kAccBufs;
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(ab * Cfg::kAccCols);
        if (res && tile / tiles_m != n_prev) {
          // a new column block: its B scales, all of K, into tensor memory
          n_prev = tile / tiles_m;
          if (!mbar_wait(res_full, static_cast<uint32_t>(res_uses) & 1u, p.status)) break;
          tc_fence_after();
          const uint64_t r_d = smem_desc(smem_u32(sRes), 0, 128, kLayoutSwizzleNone);
          for (int ks = 0; ks < n_kst; ++ks)
#pragma unroll
            for (int kb = 0; kb < Cfg::kKbPerStage; ++kb)
#pragma unroll
              for (int g = 0; g < Cfg::kBN / 128; ++g)
                tc_cp_32x128b_warpx4(tmem + Cfg::kResSfbCol + (Cfg::kBN / 32) * (ks * Cfg::kKbPerStage + kb) + 4 * g,
                                     r_d + static_cast<uint64_t>(32 * ((ks * (Cfg::kBN / 128) + g) * Cfg::kKbPerStage + kb)));
          tc_commit(res_empty);
          ++res_uses;
        }
        for (int ks = 0; ks < n_kst; ++ks) {
          if (!mbar_wait(&full[st], ph, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + Cfg::kSfCol + sf_buf * sfa_stride;
          const uint32_t sfb_t = res ? tmem + Cfg::kResSfbCol + (Cfg::kBN / 32) * (ks * Cfg::kKbPerStage)
                                     : sfa_t + Cfg::kSfaCols;
          const uint64_t sfa_d = smem_desc(smem_u32(sSfa + st * Cfg::kSfaBytes), 0, 128, kLayoutSwizzleNone);
          const uint64_t sfb_d = smem_desc(smem_u32(sSfb + st * Cfg::kSfbBytes), 0, 128, kLayoutSwizzleNone);
          const uint64_t a0 = smem_desc(smem_u32(sA + st * Cfg::kABytes), 16, Cfg::kSbo, Cfg::kSwizzle);
          const uint64_t b0 = smem_desc(smem_u32(sB + st * Cfg::kBBytes), 16, Cfg::kSbo, Cfg::kSwizzle);
          if (ks < n_full) {
#pragma unroll
            for (int kb = 0; kb < Cfg::kKbPerStage; ++kb) {
              tc_cp_32x128b_warpx4(sfa_t + 4 * kb, sfa_d + static_cast<uint64_t>(32 * kb));
              if (!res) {
#pragma unroll
                for (int g = 0; g < Cfg::kBN / 128; ++g)
                  tc_cp_32x128b_warpx4(sfb_t + (Cfg::kBN / 32) * kb + 4 * g,
                                       sfb_d + static_cast<uint64_t>(32 * (g * Cfg::kKbPerStage + kb)));
              }
            }
            if (ks == 0 && use >= 1 && !wait_acc_empty(ab, use)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int kb = 0; kb < Cfg::kKbPerStage; ++kb)
              mma_nvf4(d_tmem, a0 + static_cast<uint64_t>(2 * kb), b0 + static_cast<uint64_t>(2 * kb), Cfg::kIdesc,
                       sfa_t + 4 * kb, sfb_t + (Cfg::kBN / 32) * kb, (ks > 0 || kb > 0) ? 1u : 0u);
          } else {
            for (int kb = 0; kb < tail_kb; ++kb) {
              tc_cp_32x128b_warpx4(sfa_t + 4 * kb, sfa_d + static_cast<uint64_t>(32 * kb));
              if (!res)
                for (int g = 0; g < Cfg::kBN / 128; ++g)
                  tc_cp_32x128b_warpx4(sfb_t + (Cfg::kBN / 32) * kb + 4 * g,
                                       sfb_d + static_cast<uint64_t>(32 * (g * Cfg::kKbPerStage + kb)));
            }
            if (ks == 0 && use >= 1 && !wait_acc_empty(ab, use)) {
              ok = false;
              break;
            }
            for (int kb = 0; kb < tail_kb; ++kb)
              mma_nvf4(d_tmem, a0 + static_cast<uint64_t>(2 * kb), b0 + static_cast<uint64_t>(2 * kb), Cfg::kIdesc,
                       sfa_t + 4 * kb, sfb_t + (Cfg::kBN / 32) * kb, (ks > 0 || kb > 0) ? 1u : 0u);
          }
          tc_commit(&empty[st]);
          sf_buf ^= 1u;
          if (++st == Cfg::kStages) {
            st = 0;
            ph ^= 1u;
          }
        }
        tc_commit(&acc_full[ab]);
      }
    }
  } else {
    // ---------------- epilogue ----------------
    const int ew = warp - Cfg::kFirstEpiWarp;  // epilogue warp index
    const int q = warp & 3;                    // lane quarter of tensor memory this warp may read
    const int h = ew / 4;                      // which 128-column half (BN = 256)
    const int r = 32 * q + lane;               // row of the tile
    const bool leader = (ew == 0 && lane == 0);
    float alpha = __ldg(p.gdec_a) * __ldg(p.gdec_b);
    for (int i = 0; i < run.count; ++i) {
      const int tile = run.first + i;
      const int ab = i % Cfg::kAccBufs;
      const int64_t m0 = static_cast<int64_t>(tile % tiles_m) * Cfg::kBM;
      const int64_t n0 = static_cast<int64_t>(tile / tiles_m) * Cfg::kBN;
      const float* bias = p.bias;
      if (grouped) {
        const int e = expert_of(static_cast<int32_t>(m0));
        alpha = __ldg(p.gdec_a + e) * __ldg(p.gdec_b + e);
        if (bias != nullptr) bias += static_cast<int64_t>(e) * p.N;
      }
      // lane l holds the bias of column 32 cc + l of each of its chunks, fetched
      // before the accumulator is ready so the load hides behind the mainloop
      float bias_l[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int64_t col = n0 + 32 * (4 * h + c) + lane;
        bias_l[c] = (bias != nullptr && col < p.N) ? __ldg(bias + col) : 0.0f;
      }
      // rank-one epilogue: this thread's row factor (the bias row becomes the column factor)
      float u_r = 1.0f;
      if (kRank1) u_r = (m0 + r < p.M) ? __ldg(p.row_scale + m0 + r) : 0.0f;
      uint32_t okw = 0;
      if (lane == 0) okw = mbar_wait_poll(&acc_full[ab], static_cast<uint32_t>(i / Cfg::kAccBufs) & 1u, p.status) ? 1u : 0u;
      const bool ok = __shfl_sync(0xFFFFFFFFu, okw, 0) != 0;
      // all epilogue threads agree, so the .sync.aligned loads below run in
      // every lane of every warp or in none
      if (named_barrier_or(1, kEpiThreads, !ok)) break;
      tc_fence_after();
      const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(ab * Cfg::kAccCols);
      // chunk c (of this warp's four) = alpha * acc + bias, converted, into the staging buffer
      auto emit = [&](int c, const uint32_t (&v)[32]) {
        const int cc = 4 * h + c;              // 32-column chunk of the tile
        if (kBf16Out) {
          // 32 bf16 = 64 bytes = four 16-byte pieces of row r in box h of this round
          uint8_t* box = sOut + h * (Cfg::kBM * 128);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int j = 8 * u + 2 * k;
              float b0 = __shfl_sync(0xFFFFFFFFu, bias_l[c], j);
              float b1 = __shfl_sync(0xFFFFFFFFu, bias_l[c], j + 1);
              if (kRank1) {
                b0 = __fmul_rn(u_r, b0);
                b1 = __fmul_rn(u_r, b1);
              }
              const __nv_bfloat162 pr = __floats2bfloat162_rn(fmaf(alpha, __uint_as_float(v[j]), b0),
                                                              fmaf(alpha, __uint_as_float(v[j + 1]), b1));
              w[k] = *reinterpret_cast<const uint32_t*>(&pr);
            }
            const int piece = ((cc & 1) * 4 + u) ^ (r & 7);
            *reinterpret_cast<uint4*>(box + r * 128 + piece * 16) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          // 32 fp32 = 128 bytes = one full row of box cc
          uint8_t* box = sOut + cc * (Cfg::kBM * 128);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float f[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              float b = __shfl_sync(0xFFFFFFFFu, bias_l[c], 4 * u + k);
              if (kRank1) b = __fmul_rn(u_r, b);
              f[k] = fmaf(alpha, __uint_as_float(v[4 * u + k]), b);
            }
            *reinterpret_cast<float4*>(box + r * 128 + ((u ^ (r & 7)) * 16)) = make_float4(f[0], f[1], f[2], f[3]);
          }
        }
      };
      // the staging buffer is free once the previous store has read it
      auto staging_free = [&]() {
        if (leader) bulk_wait_group_read<0>();
        named_barrier(1, kEpiThreads);
      };
      auto store_round = [&](int first_box_col) {   // make the round visible to the TMA engine, store it
        fence_proxy_async_smem();
        named_barrier(1, kEpiThreads);
        if (leader) {
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxesPerRound; ++bx) {
            const int64_t col = n0 + first_box_col + bx * (kBf16Out ? 128 : Cfg::kBoxCols);
            if (col < p.N)
              tma_store_2d(&map_y, sOut + bx * (Cfg::kBM * 128), static_cast<int32_t>(col), static_cast<int32_t>(m0));
          }
          bulk_commit_group();
        }
      };
      // two chunks per tensor-memory round trip; the accumulator goes back to
      // the MMA thread as soon as the last two are in registers
#pragma unroll
      for (int c2 = 0; c2 < 4; c2 += 2) {
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(32 * (4 * h + c2)), v0);
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(32 * (4 * h + c2 + 1)), v1);
        tmem_ld_wait();
        if (c2 == 2) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
        if (kBf16Out || c2 == 0) staging_free();
        emit(c2, v0);
        emit(c2 + 1, v1);
        // bf16: one round per chunk pair (box h holds columns 128 h + 64 (c2/2) .. +63)
        if (kBf16Out) store_round(64 * (c2 / 2));
      }
      if (!kBf16Out) store_round(0);
    }
    if (leader) bulk_wait_group_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

template <int BN, bool kBf16Out, bool kRank1, bool kGrouped>
static cudaError_t launch_gemm_t(const GemmArgs& a, cudaStream_t s, bool pdl) {
  using Cfg = GemmCfg<BN, kBf16Out>;
  constexpr CUtensorMapSwizzle kOpSwizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap ma, mb, msa, msb, my;
  if (!make_tensor_map_2d(&ma, a.a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(a.M),
                          static_cast<uint64_t>(a.K / 2), Cfg::kBM, Cfg::kRowBytes, kOpSwizzle))
    return cudaErrorInvalidValue;
  const uint64_t b_rows = static_cast<uint64_t>(a.N) * static_cast<uint64_t>(a.groups);   // experts stacked
  if (!make_tensor_map_2d(&mb, a.b_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, b_rows,
                          static_cast<uint64_t>(a.K / 2), Cfg::kBN, Cfg::kRowBytes, kOpSwizzle))
    return cudaErrorInvalidValue;
  // scale atoms as a [row groups, K/64 * 64] array of 8-byte elements; a box of
  // 256 elements is the 4 atoms (2 KB) of one stage of one 128-row group
  const uint64_t sf_cols = static_cast<uint64_t>(a.K / 64) * 64;
  if (!make_tensor_map_2d(&msa, a.a_scales, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, static_cast<uint64_t>((a.M + 127) / 128),
                          sf_cols, 1, 256, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (!make_tensor_map_2d(&msb, a.b_scales, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, (b_rows + 127) / 128,
                          sf_cols, Cfg::kBN / 128, 256, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (!make_tensor_map_2d(&my, a.Y, kBf16Out ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                          Cfg::kOutElem, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.N), Cfg::kBM,
                          Cfg::kBoxCols, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  GemmParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.block_expert = a.block_expert;
  p.totals = a.totals;
  p.tiles_m = static_cast<int>((a.M + Cfg::kBM - 1) / Cfg::kBM);
  p.num_tiles = p.tiles_m * static_cast<int>((a.N + Cfg::kBN - 1) / Cfg::kBN);
  const int64_t n_kst = (a.K + Cfg::kStageK - 1) / Cfg::kStageK;
  p.sfb_resident = (Cfg::kResMaxStages > 0 && n_kst <= Cfg::kResMaxStages && a.block_expert == nullptr) ? 1 : 0;
  p.gdec_a = a.a_gdec;
  p.gdec_b = a.b_gdec;
  p.bias = a.bias;
  p.row_scale = a.row_scale;
  p.status = a.status;
  auto kern = gemm_nvfp4_kernel<BN, kBf16Out, kRank1, kGrouped>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < sm_count() ? p.num_tiles : sm_count();
  return launch_ex(kern, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmemBytes, s, pdl, ma, mb, msa, msb, my, p);
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, bool pdl) {
  if (a.row_scale != nullptr) {
    if (a.bias == nullptr || a.block_expert != nullptr) return cudaErrorInvalidValue;
    return a.yt == AVR_BF16 ? launch_gemm_t<256, true, true, false>(a, s, pdl)
                            : launch_gemm_t<128, false, true, false>(a, s, pdl);
  }
  if (a.block_expert != nullptr)
    return a.yt == AVR_BF16 ? launch_gemm_t<256, true, false, true>(a, s, pdl)
                            : launch_gemm_t<128, false, false, true>(a, s, pdl);
  return a.yt == AVR_BF16 ? launch_gemm_t<256, true, false, false>(a, s, pdl)
                          : launch_gemm_t<128, false, false, false>(a, s, pdl);
}

}  // namespace avr
