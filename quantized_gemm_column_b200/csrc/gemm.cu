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
//   warp 0     : allocates tensor memory; one thread issues
//                tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M 128, K 64)
//                from the staged operands and the scale slots;
//   warps 1..4 : TMA producers, one operand each: the A code tile, the B code
//                tile, A's and B's 512-byte scale atoms (2-D copies over the
//                atom array, out-of-range atoms read as zero), and warp 4
//                also the resident B scales (below).  A thread's bulk copies
//                complete one after another, about one per 350 ns whatever
//                their size, so every operand of a stage has a thread of its
//                own;
//   warp 5     : scale copier: one thread moves each stage's scale atoms from
//                shared into tensor memory (tcgen05.cp 32x128b, replicated
//                into the four lane quarters) into one of two scale slots.
//                Copies issued by a thread of their own run beside the MMAs
//                instead of between them;
//   warps 6..  : epilogue -- the tile's bias row staged in shared memory,
//                tcgen05.ld of the accumulator (each warp one 32-lane quarter
//                and a run of columns), alpha * acc + bias, convert, a
//                128-byte-swizzled staging tile, TMA store.
//
// The scale copies are what limits a block-scaled FP4 GEMM with 128 x 256
// tiles on this part: one 64-deep k-block needs A's atom (2 KB of tensor
// memory after replication) and two of B's (4 KB), and the copies move about
// 55 bytes per ns, longer than the 73 ns MMA they feed.  So the first stages
// of B's scales (up to kResMaxStages of them) stay resident in tensor memory
// for as long as a CTA works on one column block: warp 4 loads them into a
// shared buffer (one 3-D copy) when the column block changes, warp 5 copies
// them once, and those stages then need only A's copies.  With K <= 1280
// (bf16 output) every stage is resident.
//
// bf16 output: one 256-column accumulator; the epilogue takes it out of
// tensor memory in two rounds of 64 columns per warp and hands it back to the
// MMA thread before the second round goes to the staging buffer.
// fp32 output: 128-column tiles, two accumulators, so the epilogue overlaps
// the next tile's mainloop.
#include "device.cuh"
#include "internal.h"

namespace avr {

template <int BN, bool kBf16Out>
struct GemmCfg {
  static constexpr int kBM = 128, kBN = BN;
  static constexpr int kStageK = 256;                      // fp4 elements per stage
  static constexpr int kRowBytes = kStageK / 2;            // 128 bytes per row
  static constexpr int kStages = 3;
  static constexpr int kKbPerStage = kStageK / 64;         // MMAs per stage
  static constexpr int kAccBufs = BN == 256 ? 1 : 2;
  static constexpr int kEpiWarps = BN / 32;                // 8 or 4
  static constexpr int kFirstEpiWarp = 6;
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
  // tensor memory: accumulators, two scale slots (A's and B's atoms of one
  // stage), then the resident B scales
  static constexpr int kAccCols = kBN;
  static constexpr int kSfaCols = kKbPerStage * 4;         // 4 columns per replicated atom
  static constexpr int kSfbKbCols = kBN / 32;              // B's atoms of one k-block
  static constexpr int kSfbCols = kKbPerStage * kSfbKbCols;
  static constexpr int kSlots = 2;
  static constexpr int kSlotCols = kSfaCols + kSfbCols;
  static constexpr int kSlotCol = kAccBufs * kAccCols;
  static constexpr int kResCol = kSlotCol + kSlots * kSlotCols;
  static constexpr int kTmemCols = 512;
  static constexpr int kResMaxStages = (kTmemCols - kResCol) / kSfbCols;
  static constexpr int kResBytes = kResMaxStages * kSfbBytes;
  // shared memory
  static constexpr int kOutOffset = kStages * kStageBytes;
  static constexpr int kResOffset = kOutOffset + kStageOutBytes;
  static constexpr int kBiasOffset = kResOffset + kResBytes;
  static constexpr int kBarOffset = kBiasOffset + kAccBufs * kBN * 4;
  // dynamic shared memory starts 1024-aligned when a kernel has no static
  // shared memory; the kernel checks it and refuses to run otherwise
  static constexpr int kSmemBytes = kBarOffset + 256;
  static_assert(kResMaxStages >= 1 && kResCol + kResMaxStages * kSfbCols <= kTmemCols, "tensor memory budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  // instruction descriptor: E2M1 A and B (format 1), UE4M3 scales, K-major
  // operands, N >> 3 at bit 17, M >> 4 at bit 24
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                                     (static_cast<uint32_t>(kBM >> 4) << 24);
};

struct GemmParams {
  int64_t M, N, K;
  int tiles_m, num_tiles;
  int res_stages;         // full stages of K whose B scales stay resident per column block (0: none)
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
                      const __grid_constant__ CUtensorMap map_sfb_res, const __grid_constant__ CUtensorMap map_y,
                      const GemmParams p) {
  using Cfg = GemmCfg<BN, kBf16Out>;
  constexpr int kEpiThreads = 32 * Cfg::kEpiWarps;
  constexpr int kNbGroups = Cfg::kBN / 128;    // 128-row atom groups of a B tile
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
  uint8_t* sRes = smem + Cfg::kResOffset;      // resident B scales: [row group][stage][4 atoms]
  float* sBias = reinterpret_cast<float*>(smem + Cfg::kBiasOffset);   // [kAccBufs][kBN]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);   // [kStages] operands landed
  uint64_t* empty = full + Cfg::kStages;        // [kStages] operands consumed by the MMAs
  uint64_t* sf_full = empty + Cfg::kStages;     // [kSlots] scale slot copied
  uint64_t* sf_empty = sf_full + Cfg::kSlots;   // [kSlots] scale slot read by the MMAs
  uint64_t* acc_full = sf_empty + Cfg::kSlots;  // [kAccBufs]
  uint64_t* acc_empty = acc_full + 2;           // [kAccBufs]
  uint64_t* res_load = acc_empty + 2;           // resident B scales in shared memory
  uint64_t* res_cp = res_load + 1;              // resident B scales copied to tensor memory
  uint64_t* res_free = res_cp + 1;              // the MMAs of a column block are done with them
  uint64_t* drained = res_free + 1;             // [2] the MMA and copy threads' last operations completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_kst = static_cast<int>((p.K + Cfg::kStageK - 1) / Cfg::kStageK);
  const int n_full = static_cast<int>(p.K / Cfg::kStageK);                // stages of kKbPerStage k-blocks
  const int tail_kb = static_cast<int>((p.K % Cfg::kStageK) / 64);        // k-blocks of a last, partial stage
  const int res_st = p.res_stages;
  constexpr bool grouped = kGrouped;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
    prefetch_tensormap(&map_sfa);
    prefetch_tensormap(&map_sfb);
    prefetch_tensormap(&map_sfb_res);
    prefetch_tensormap(&map_y);
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 4);                   // one arrival per producer warp
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < Cfg::kSlots; ++s) {
      mbar_init(&sf_full[s], 1);
      mbar_init(&sf_empty[s], 1);
    }
    for (int b = 0; b < Cfg::kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], Cfg::kEpiWarps);   // one arrival per epilogue warp
    }
    mbar_init(res_load, 1);
    mbar_init(res_cp, 1);
    mbar_init(res_free, 1);
    mbar_init(&drained[0], 1);
    mbar_init(&drained[1], 1);
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
  // does tile i of the run start a new column block (its resident B scales must be loaded)?
  auto new_block = [&](int i) { return i == 0 || (run.first + i) / tiles_m != (run.first + i - 1) / tiles_m; };
  auto last_of_block = [&](int i) { return i + 1 == run.count || (run.first + i + 1) / tiles_m != (run.first + i) / tiles_m; };

  if (warp >= 1 && warp <= 4) {
    if (lane == 0) {
      // ---------------- producers: warp 1 A, 2 B, 3 A's scales, 4 B's scales (+ resident) ----------------
      const int role = warp - 1;
      uint32_t st = 0, ph = 0;
      int it = 0, res_uses = 0;
      bool ok = true;
      for (int i = 0; i < run.count && ok; ++i) {
        const int tile = run.first + i;
        const int32_t m0 = (tile % tiles_m) * Cfg::kBM;
        const int32_t n0 = (tile / tiles_m) * Cfg::kBN;
        const int32_t nb0 = n0 + (grouped ? expert_of(m0) * static_cast<int32_t>(p.N) : 0);   // B's first row
        if (role == 3 && res_st > 0 && new_block(i)) {
          // the resident buffer is free once the previous column block's copies have run
          if (res_uses >= 1 && !mbar_wait(res_cp, static_cast<uint32_t>(res_uses - 1) & 1u, p.status)) break;
          ++res_uses;
          mbar_arrive_expect_tx(res_load, static_cast<uint32_t>(res_st * Cfg::kSfbBytes));
          tma_load_3d(sRes, &map_sfb_res, res_load, 0, 0, nb0 / 128);
        }
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
          } else if (ks >= res_st) {
            mbar_arrive_expect_tx(&full[st], Cfg::kSfbBytes);
            tma_load_2d(sSfb + st * Cfg::kSfbBytes, &map_sfb, &full[st], ks * 256, nb0 / 128);
          } else {
            mbar_arrive(&full[st]);               // this stage's B scales are resident
          }
          if (++st == Cfg::kStages) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ---------------- scale copier ----------------
      uint32_t st = 0, ph = 0, sl = 0, sph = 0;
      int it = 0, res_uses = 0;
      bool ok = true;
      const uint64_t res_d = smem_desc(smem_u32(sRes), 0, 128, kLayoutSwizzleNone);
      for (int i = 0; i < run.count && ok; ++i) {
        if (res_st > 0 && new_block(i)) {
          // the previous column block's MMAs must be done with the resident columns
          if (res_uses >= 1 && !mbar_wait_poll(res_free, static_cast<uint32_t>(res_uses - 1) & 1u, p.status)) break;
          if (!mbar_wait_poll(res_load, static_cast<uint32_t>(res_uses) & 1u, p.status)) break;
          ++res_uses;
          tc_fence_after();
          for (int ks = 0; ks < res_st; ++ks)
#pragma unroll
            for (int kb = 0; kb < Cfg::kKbPerStage; ++kb)
#pragma unroll
              for (int g = 0; g < kNbGroups; ++g)
                tc_cp_32x128b_warpx4(tmem + Cfg::kResCol + Cfg::kSfbKbCols * (ks * Cfg::kKbPerStage + kb) + 4 * g,
                                     res_d + static_cast<uint64_t>(32 * ((g * res_st + ks) * Cfg::kKbPerStage + kb)));
          tc_commit(res_cp);
        }
        for (int ks = 0; ks < n_kst; ++ks, ++it) {
          if (!mbar_wait_poll(&full[st], ph, p.status)) {
            ok = false;
            break;
          }
          if (it >= Cfg::kSlots && !mbar_wait_poll(&sf_empty[sl], sph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + Cfg::kSlotCol + sl * Cfg::kSlotCols;
          const uint32_t sfb_t = sfa_t + Cfg::kSfaCols;
          const uint64_t sfa_d = smem_desc(smem_u32(sSfa + st * Cfg::kSfaBytes), 0, 128, kLayoutSwizzleNone);
          const uint64_t sfb_d = smem_desc(smem_u32(sSfb + st * Cfg::kSfbBytes), 0, 128, kLayoutSwizzleNone);
          const bool sfb = ks >= res_st;
          if (ks < n_full) {
#pragma unroll
            for (int kb = 0; kb < Cfg::kKbPerStage; ++kb) tc_cp_32x128b_warpx4(sfa_t + 4 * kb, sfa_d + static_cast<uint64_t>(32 * kb));
            if (sfb) {
#pragma unroll
              for (int kb = 0; kb < Cfg::kKbPerStage; ++kb)
#pragma unroll
                for (int g = 0; g < kNbGroups; ++g)
                  tc_cp_32x128b_warpx4(sfb_t + Cfg::kSfbKbCols * kb + 4 * g,
                                       sfb_d + static_cast<uint64_t>(32 * (g * Cfg::kKbPerStage + kb)));
            }
          } else {
            for (int kb = 0; kb < tail_kb; ++kb) {
              tc_cp_32x128b_warpx4(sfa_t + 4 * kb, sfa_d + static_cast<uint64_t>(32 * kb));
              if (sfb)
                for (int g = 0; g < kNbGroups; ++g)
                  tc_cp_32x128b_warpx4(sfb_t + Cfg::kSfbKbCols * kb + 4 * g,
                                       sfb_d + static_cast<uint64_t>(32 * (g * Cfg::kKbPerStage + kb)));
            }
          }
          tc_commit(&sf_full[sl]);
          if (++st == Cfg::kStages) {
            st = 0;
            ph ^= 1u;
          }
          if (++sl == Cfg::kSlots) {
            sl = 0;
            sph ^= 1u;
          }
        }
      }
      // every copy this thread issued has completed before the CTA tears down
      tc_commit(&drained[1]);
      mbar_wait(&drained[1], 0, p.status);
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      // The issuing thread is on the critical path: the loop keeps its
      // bookkeeping to increments and issues a full stage's MMAs unrolled,
      // with descriptors advanced by constants (16-byte units: +2 per 32-byte
      // k-block step).
      uint32_t st = 0, ph = 0, sl = 0, sph = 0;
      int res_uses = 0;
      bool ok = true;
      for (int i = 0; i < run.count && ok; ++i) {
        const int ab = i % Cfg::kAccBufs;
        const int use = i / Cfg::kAccBufs;
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(ab * Cfg::kAccCols);
        if (res_st > 0 && new_block(i)) {
          if (!mbar_wait_poll(res_cp, static_cast<uint32_t>(res_uses) & 1u, p.status)) break;
          ++res_uses;
        }
        for (int ks = 0; ks < n_kst; ++ks) {
          if (!mbar_wait_poll(&sf_full[sl], sph, p.status) || !mbar_wait_poll(&full[st], ph, p.status)) {
            ok = false;
            break;
          }
          if (ks == 0 && use >= 1 && !mbar_wait_poll(&acc_empty[ab], static_cast<uint32_t>(use - 1) & 1u, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + Cfg::kSlotCol + sl * Cfg::kSlotCols;
          const uint32_t sfb_t = ks < res_st ? tmem + Cfg::kResCol + Cfg::kSfbKbCols * (ks * Cfg::kKbPerStage)
                                             : sfa_t + Cfg::kSfaCols;
          const uint64_t a0 = smem_desc(smem_u32(sA + st * Cfg::kABytes), 16, Cfg::kSbo, Cfg::kSwizzle);
          const uint64_t b0 = smem_desc(smem_u32(sB + st * Cfg::kBBytes), 16, Cfg::kSbo, Cfg::kSwizzle);
          if (ks < n_full) {
#pragma unroll
            for (int kb = 0; kb < Cfg::kKbPerStage; ++kb)
              mma_nvf4(d_tmem, a0 + static_cast<uint64_t>(2 * kb), b0 + static_cast<uint64_t>(2 * kb), Cfg::kIdesc,
                       sfa_t + 4 * kb, sfb_t + Cfg::kSfbKbCols * kb, (ks > 0 || kb > 0) ? 1u : 0u);
          } else {
            for (int kb = 0; kb < tail_kb; ++kb)
              mma_nvf4(d_tmem, a0 + static_cast<uint64_t>(2 * kb), b0 + static_cast<uint64_t>(2 * kb), Cfg::kIdesc,
                       sfa_t + 4 * kb, sfb_t + Cfg::kSfbKbCols * kb, (ks > 0 || kb > 0) ? 1u : 0u);
          }
          tc_commit(&empty[st]);
          tc_commit(&sf_empty[sl]);
          if (++st == Cfg::kStages) {
            st = 0;
            ph ^= 1u;
          }
          if (++sl == Cfg::kSlots) {
            sl = 0;
            sph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[ab]);
        if (res_st > 0 && last_of_block(i)) tc_commit(res_free);
      }
      tc_commit(&drained[0]);
      mbar_wait(&drained[0], 0, p.status);
    }
  } else {
    // ---------------- epilogue ----------------
    const int ew = warp - Cfg::kFirstEpiWarp;  // epilogue warp index
    const int q = warp & 3;                    // lane quarter of tensor memory this warp may read
    const int h = ew / 4;                      // which 128-column half (BN = 256)
    const int r = 32 * q + lane;               // row of the tile
    const int et = ew * 32 + lane;             // epilogue thread index = the bias column it stages
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
      // The staging buffer is free once the previous tile's last store has
      // read it, and the bias buffer once every thread is past the previous
      // tile; then this tile's bias row goes into shared memory.
      if (leader) bulk_wait_group_read<0>();
      named_barrier(1, kEpiThreads);
      float* bias_s = sBias + ab * Cfg::kBN;
      {
        const int64_t col = n0 + et;
        bias_s[et] = (bias != nullptr && col < p.N) ? __ldg(bias + col) : 0.0f;
      }
      // rank-one epilogue: this thread's row factor (the bias row becomes the column factor)
      float u_r = 1.0f;
      if (kRank1) u_r = (m0 + r < p.M) ? __ldg(p.row_scale + m0 + r) : 0.0f;
      uint32_t okw = 0;
      if (lane == 0) okw = mbar_wait_poll(&acc_full[ab], static_cast<uint32_t>(i / Cfg::kAccBufs) & 1u, p.status) ? 1u : 0u;
      const bool ok = __shfl_sync(0xFFFFFFFFu, okw, 0) != 0;
      // all epilogue threads agree, so the .sync.aligned loads below run in
      // every lane of every warp or in none; the barrier also publishes the
      // bias row
      if (named_barrier_or(1, kEpiThreads, !ok)) break;
      tc_fence_after();
      const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(ab * Cfg::kAccCols);
      // alpha * acc + bias of chunk c (of this warp's four), 32 columns of row r
      auto value = [&](const float* b, int j, uint32_t v) {
        float bj = b[j];
        if (kRank1) bj = __fmul_rn(u_r, bj);
        return fmaf(alpha, __uint_as_float(v), bj);
      };
      // chunk c as 16 bf16 pairs
      auto pack_bf16 = [&](int c, const uint32_t (&v)[32], uint32_t (&w)[16]) {
        const float* b = bias_s + 32 * (4 * h + c);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const __nv_bfloat162 pr = __floats2bfloat162_rn(value(b, 2 * k, v[2 * k]), value(b, 2 * k + 1, v[2 * k + 1]));
          w[k] = *reinterpret_cast<const uint32_t*>(&pr);
        }
      };
      // 16 bf16 pairs of chunk c = 64 bytes = four 16-byte pieces of row r in
      // box h of the staging buffer (a box is 128 rows x 64 columns)
      auto stage_bf16 = [&](int c, const uint32_t (&w)[16]) {
        uint8_t* box = sOut + h * (Cfg::kBM * 128);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int piece = ((c & 1) * 4 + u) ^ (r & 7);
          *reinterpret_cast<uint4*>(box + r * 128 + piece * 16) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      };
      // fp32: chunk c = 128 bytes = one full row of box c
      auto stage_f32 = [&](int c, const uint32_t (&v)[32]) {
        const float* b = bias_s + 32 * c;
        uint8_t* box = sOut + c * (Cfg::kBM * 128);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float f[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) f[k] = value(b, 4 * u + k, v[4 * u + k]);
          *reinterpret_cast<float4*>(box + r * 128 + ((u ^ (r & 7)) * 16)) = make_float4(f[0], f[1], f[2], f[3]);
        }
      };
      auto store_round = [&](int first_col) {   // make the round visible to the TMA engine, store it
        fence_proxy_async_smem();
        named_barrier(1, kEpiThreads);
        if (leader) {
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxesPerRound; ++bx) {
            // bf16: box bx is the 64 columns of half bx starting at first_col; fp32: box bx = columns 32 bx
            const int64_t col = n0 + first_col + bx * (kBf16Out ? 128 : Cfg::kBoxCols);
            if (col < p.N)
              tma_store_2d(&map_y, sOut + bx * (Cfg::kBM * 128), static_cast<int32_t>(col), static_cast<int32_t>(m0));
          }
          bulk_commit_group();
        }
      };
      auto release_acc = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
      };
      uint32_t v0[32], v1[32];
      tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(32 * (4 * h + 0)), v0);
      tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(32 * (4 * h + 1)), v1);
      tmem_ld_wait();
      if (kBf16Out) {
        // round 0: columns 128 h + 0..63
        {
          uint32_t w[16];
          pack_bf16(0, v0, w);
          stage_bf16(0, w);
          pack_bf16(1, v1, w);
          stage_bf16(1, w);
        }
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(32 * (4 * h + 2)), v0);
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(32 * (4 * h + 3)), v1);
        tmem_ld_wait();
        release_acc();
        uint32_t w2[16], w3[16];
        pack_bf16(2, v0, w2);
        pack_bf16(3, v1, w3);
        store_round(0);
        // round 1 (columns 128 h + 64..127) reuses the staging buffer once
        // the TMA engine has read round 0
        if (leader) bulk_wait_group_read<0>();
        named_barrier(1, kEpiThreads);
        stage_bf16(2, w2);
        stage_bf16(3, w3);
        store_round(64);
      } else {
        stage_f32(0, v0);
        stage_f32(1, v1);
        tmem_ld_32x32b_x32(t_row + 64, v0);
        tmem_ld_32x32b_x32(t_row + 96, v1);
        tmem_ld_wait();
        release_acc();
        stage_f32(2, v0);
        stage_f32(3, v1);
        store_round(0);
      }
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
  // B's scales of the first full stages stay resident per column block (not
  // in grouped mode, where consecutive tiles may belong to different experts):
  // one 3-D copy of [row groups][stages][4 atoms] brings them in
  const int64_t n_full = a.K / Cfg::kStageK;
  const int res_stages = a.block_expert == nullptr ? static_cast<int>(min64(n_full, Cfg::kResMaxStages)) : 0;
  CUtensorMap msr = msb;
  if (res_stages > 0) {
    const uint64_t dims[3] = {256, static_cast<uint64_t>(n_full), (b_rows + 127) / 128};
    const uint64_t strides[2] = {2048, sf_cols * 8};
    const uint32_t box[3] = {256, static_cast<uint32_t>(res_stages), Cfg::kBN / 128};
    if (!make_tensor_map_3d(&msr, a.b_scales, CU_TENSOR_MAP_DATA_TYPE_UINT64, dims, strides, box))
      return cudaErrorInvalidValue;
  }
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
  p.res_stages = res_stages;
  p.gdec_a = a.a_gdec;
  p.gdec_b = a.b_gdec;
  p.bias = a.bias;
  p.row_scale = a.row_scale;
  p.status = a.status;
  auto kern = gemm_nvfp4_kernel<BN, kBf16Out, kRank1, kGrouped>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < sm_count() ? p.num_tiles : sm_count();
  return launch_ex(kern, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmemBytes, s, pdl, ma, mb, msa, msb, msr, my, p);
}

// MMA-only loop: the tensor pipe's block-scaled FP4 rate on this device.
// Each CTA (one per SM) fills shared memory with constant E2M1 codes and
// E4M3 scales, copies the scales into tensor memory once, then issues `iters`
// stages of four M 128 x N 256 x K 64 MMAs into one accumulator, waiting on
// a commit every 16 stages; ns[b] = the CTA's elapsed time.  A measurement
// aid for the roofline, not part of the method.
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int iters, uint64_t* ns, uint32_t* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) raise_status(status, AVR_ERR_MISALIGNED);
    return;
  }
  uint8_t* sA = smem_raw;                 // 128 rows x 128 B
  uint8_t* sB = sA + 16384;               // 256 rows x 128 B
  uint8_t* sSF = sB + 32768;              // SFA 4 atoms, SFB 8 atoms
  uint64_t* bar = reinterpret_cast<uint64_t*>(sSF + 6144);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  for (int i = threadIdx.x; i < (16384 + 32768) / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sA)[i] = 0x22222222u;
  for (int i = threadIdx.x; i < 6144 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sSF)[i] = 0x38383838u;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbarrier_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = GemmCfg<256, true>::kIdesc;
    const uint32_t sfa = tmem + 256, sfb = tmem + 272;
    for (int kb = 0; kb < 4; ++kb) {
      tc_cp_32x128b_warpx4(sfa + 4 * kb, smem_desc(smem_u32(sSF + kb * 512), 0, 128, kLayoutSwizzleNone));
      for (int g = 0; g < 2; ++g)
        tc_cp_32x128b_warpx4(sfb + 8 * kb + 4 * g,
                             smem_desc(smem_u32(sSF + 2048 + (g * 4 + kb) * 512), 0, 128, kLayoutSwizzleNone));
    }
    tc_commit(bar);
    uint32_t phase = 0;
    bool ok = mbar_wait(bar, phase, status);
    phase ^= 1u;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t a0 = smem_desc(smem_u32(sA), 16, 1024, kLayoutSwizzle128B);
    const uint64_t b0 = smem_desc(smem_u32(sB), 16, 1024, kLayoutSwizzle128B);
    for (int it = 0; it < iters && ok; ++it) {
#pragma unroll
      for (int kb = 0; kb < 4; ++kb)
        mma_nvf4(tmem, a0 + static_cast<uint64_t>(2 * kb), b0 + static_cast<uint64_t>(2 * kb), idesc, sfa + 4 * kb,
                 sfb + 8 * kb, (it | kb) ? 1u : 0u);
      if ((it & 15) == 15) {
        tc_commit(bar);
        ok = mbar_wait(bar, phase, status);
        phase ^= 1u;
      }
    }
    tc_commit(bar);
    if (ok) mbar_wait(bar, phase, status);
    ns[blockIdx.x] = globaltimer_ns() - t0;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_mma_rate(int iters, int grid, uint64_t* ns, uint32_t* status, cudaStream_t s) {
  // more than half of the SM's shared memory, so one CTA per SM
  constexpr int kSmem = 16384 + 32768 + 6144 + 64 + 64 * 1024;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(mma_rate_kernel), kSmem);
  if (e != cudaSuccess) return e;
  mma_rate_kernel<<<grid, 128, kSmem, s>>>(iters, ns, status);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, bool pdl) {
  if (gemm_pair_short_applies(a)) return launch_gemm_pair_short(a, s, pdl);
  if (gemm_pair_applies(a)) return launch_gemm_pair(a, s, pdl);
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
