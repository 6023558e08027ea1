// K3 on CTA pairs: the block-scaled FP4 GEMM with 2-CTA tcgen05 MMAs, for
// bf16 output.
//
// Y = 1 (mu_bar W_bar) + X_bar_R W_bar (Lighthouse review of "The Curse and
// Blessing of Mean Bias in FP4-Quantized LLM Training", section 二 "Averis
// 方法"): the product X_bar_R W_bar on E2M1 operands with E4M3 per-16 scales,
// the row mu_bar W_bar added to every output row as a bias:
//   Y[i, j] = g_dec(A) g_dec(B) * acc[i, j] + bias[j].
//
// Why pairs.  A 128 x 256 tile of one CTA needs 12 KB of operands (A 4 KB,
// B 8 KB) per 64-deep k-block, 48 KB per 256-deep stage plus scales, and one
// SM brings in about 70 bytes per clock from L2: longer than the 73 ns the
// k-block's MMA takes, and with three stages in shared memory the load
// latency (about 0.8 us per stage) is not covered either.  Two CTAs on two
// SMs of a cluster share one 256 x 256 tile: each holds its 128 rows of A
// and half (128 rows) of B, and the MMA issued by the first CTA
// (tcgen05.mma.cta_group::2, M 256, N 256, K 64) reads A from each CTA's own
// shared memory and B from both.  Each SM then loads 8 KB per k-block, a
// stage is 38 KB with scales, and four stages fit.
//
// Roles (both CTAs have the same warps; CTA rank 0 of the pair leads):
//   warp 0     : tensor-memory allocation (cta_group::2, in both CTAs); in
//                the leading CTA one thread issues the pair's MMAs;
//   warps 1..8 : TMA producers in both CTAs, two per operand taking
//                alternate stages (A rows, B rows, A's scale atoms, B's
//                scale atoms for all 256 columns plus the resident ones).
//                The copies of A, B and B's scales complete on the leading
//                CTA's barrier, whose producers expect the bytes of both
//                CTAs; A's scale atoms are each CTA's own and complete on
//                its own barrier;
//   warps 9, 10: in the leading CTA, B's scale copiers, alternate stages
//                (tcgen05.cp cta_group::2: each CTA's atoms into its own
//                tensor memory);
//   warps 11..14: A's scales into tensor memory, one warp per lane quarter
//                in each CTA, by tcgen05.st from registers (the image a
//                32x128b.warpx4 copy makes).  Tensor memory takes writes at
//                a limited rate while the MMAs run: splitting them between
//                the copy engine (B) and the stores (A) spreads the load;
//   warps 15..22: epilogue in both CTAs, each over its own 128 x 256
//                accumulator: the bias row staged in shared memory,
//                tcgen05.ld, alpha * acc + bias, bf16, TMA store.
// The leading CTA's MMA commits signal both CTAs' barriers (multicast
// commit); the second CTA's epilogue hands the accumulator back through a
// remote arrive on the leading CTA's barrier.  No TMA load is multicast.
//
// B's scales of the first full stages (up to kResMaxStages) stay resident in
// tensor memory while a pair works on one column block, as in the one-CTA
// kernel.
#include <map>
#include <mutex>

#include "device.cuh"
#include "internal.h"
#include "pair.cuh"

namespace avr {

using namespace pair;

struct Gemm2Cfg {
  static constexpr int kBM = 128;                          // rows per CTA (256 per pair)
  static constexpr int kBN = 256;                          // columns per tile
  static constexpr int kBNHalf = kBN / 2;                  // B rows per CTA
  static constexpr int kChunkK = 256;                      // K per 128-byte swizzled row chunk
  static constexpr int kChunks = 1;                        // chunks per stage
  static constexpr int kStageK = kChunkK * kChunks;        // 256
  static constexpr int kStages = 5;
  static constexpr int kKbPerStage = kStageK / 64;         // 4 MMAs per stage
  static constexpr int kEpiWarps = 8;
  static constexpr int kProducers = 8;                     // two per operand, alternate stages
  static constexpr int kSfWarps = 4;                       // one per lane quarter
  static constexpr int kCopyWarp = 1 + kProducers;
  static constexpr int kCopyWarps = 2;                     // B's scale copies, alternate stages
  static constexpr int kFirstSfWarp = kCopyWarp + kCopyWarps;
  static constexpr int kFirstEpiWarp = kFirstSfWarp + kSfWarps;
  static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
  static constexpr uint32_t kSbo = 8 * 128;                // 8-row swizzle atom of 128-byte rows
  static constexpr int kAChunkBytes = kBM * 128;           // 16 KB
  static constexpr int kABytes = kChunks * kAChunkBytes;   // 16 KB
  static constexpr int kBChunkBytes = kBNHalf * 128;       // 16 KB
  static constexpr int kBBytes = kChunks * kBChunkBytes;   // 16 KB
  static constexpr int kSfaBytes = kKbPerStage * 512;      // 2 KB: 4 atoms
  static constexpr int kSfbBytes = 2 * kKbPerStage * 512;  // 4 KB: [row group][4 atoms]
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kStageOutBytes = kBM * kBN * 2 / 2; // 32 KB: half the bf16 tile per round
  // tensor memory (the same columns in both CTAs): accumulator, A's scale
  // slots (one per stage), then B's scales: all of K resident (K <= 1280,
  // as many k-blocks as the streamed slots hold) or one slot per stage
  static constexpr int kAccCols = kBN;
  static constexpr int kSfaSlotCols = kKbPerStage * 4;     // 16
  static constexpr int kSfaCol = kAccCols;
  static constexpr int kSfbKbCols = kBN / 32;              // 8
  static constexpr int kSfbStageCols = kKbPerStage * kSfbKbCols;   // 32
  static constexpr int kSfbCol = kSfaCol + kStages * kSfaSlotCols; // 336
  static constexpr int kTmemCols = 512;
  static constexpr int kResAllStages = kStages;                    // resident: the slots' columns, K <= 1280
  static constexpr int kStreamSlotCol = kSfbCol;
  static_assert(kSfbCol + kStages * kSfbStageCols <= kTmemCols, "tensor memory budget");
  // shared memory; the resident B scales reuse the per-stage B-scale buffers
  // (contiguous, kStages * kSfbBytes), which resident mode does not stream into
  static constexpr int kOutOffset = kStages * kStageBytes;
  static constexpr int kResOffset = kOutOffset + kStageOutBytes;
  static constexpr int kBiasOffset = kResOffset;
  static constexpr int kBarOffset = kBiasOffset + kBN * 4;
  static constexpr int kSmemBytes = kBarOffset + 512;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  // instruction descriptor: E2M1 A and B, UE4M3 scales, K-major, N >> 3 at
  // bit 17, M >> 4 at bit 24 (M = 256 for the pair)
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                                     (static_cast<uint32_t>((2 * kBM) >> 4) << 24);
};

struct Gemm2Params {
  int64_t M, N, K;
  int tiles_m, num_tiles;   // pair tiles of 256 x 256, M fastest
  int res_stages;           // stages whose B scales stay resident per column block (all of K, or 1)
  const float* gdec_a;
  const float* gdec_b;
  const float* bias;
  uint32_t* status;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Gemm2Cfg::kThreads, 1)
    gemm2_nvfp4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                       const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                       const __grid_constant__ CUtensorMap map_y, const Gemm2Params p) {
  using Cfg = Gemm2Cfg;
  constexpr int kEpiThreads = 32 * Cfg::kEpiWarps;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled tiles need 1024-byte alignment; a CTA without it still takes
  // part in the pair's cluster barriers and allocation, but does no work
  const bool aligned = (smem_u32(smem_raw) & 1023u) == 0;
  uint8_t* smem = smem_raw;
  uint8_t* sA = smem;
  uint8_t* sB = sA + Cfg::kStages * Cfg::kABytes;
  uint8_t* sSfa = sB + Cfg::kStages * Cfg::kBBytes;
  uint8_t* sSfb = sSfa + Cfg::kStages * Cfg::kSfaBytes;
  uint8_t* sOut = smem + Cfg::kOutOffset;
  uint8_t* sRes = sSfb;                        // resident mode: [2 row groups][chunk][4 atoms]
  float* bias_s = reinterpret_cast<float*>(smem + Cfg::kBiasOffset);
  uint64_t* full_ab = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);  // [kStages] leading CTA: A, B landed
  uint64_t* full_sfb = full_ab + Cfg::kStages;  // [kStages] leading CTA: B's scale atoms landed in both CTAs
  uint64_t* full_sfa = full_sfb + Cfg::kStages; // [kStages] both CTAs: this CTA's A scale atoms landed
  uint64_t* empty = full_sfa + Cfg::kStages;    // [kStages] both CTAs
  uint64_t* sf_full = empty + Cfg::kStages;     // [kStages] leading CTA: the stage's scales are in tensor memory
  uint64_t* acc_full = sf_full + Cfg::kStages;  // both CTAs
  uint64_t* acc_empty = acc_full + 1;           // leading CTA: both epilogues arrive
  uint64_t* res_load = acc_empty + 1;           // leading CTA: resident scales landed in both CTAs
  uint64_t* res_cp = res_load + 1;              // both CTAs: resident scales copied
  uint64_t* res_free = res_cp + 1;              // leading CTA: the MMAs of a column block are done
  uint64_t* drained = res_free + 1;             // [1 + kCopyWarps] leading CTA: MMA and copy threads drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1 + Cfg::kCopyWarps);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;
  const int n_kst = static_cast<int>((p.K + Cfg::kStageK - 1) / Cfg::kStageK);
  const int n_kb = static_cast<int>(p.K / 64);
  const int res_st = p.res_stages;
  // B's scales of stage ks in tensor memory: resident, or a streamed slot
  auto sfb_tmem_of = [&](uint32_t tmem, int ks, int st) -> uint32_t {
    return ks < res_st ? tmem + Cfg::kSfbCol + Cfg::kSfbStageCols * ks
                       : tmem + Cfg::kStreamSlotCol + Cfg::kSfbStageCols * st;
  };

  if (threadIdx.x == 0) {
    if (!aligned) raise_status(p.status, AVR_ERR_MISALIGNED);
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
    prefetch_tensormap(&map_sfa);
    prefetch_tensormap(&map_sfb);
    prefetch_tensormap(&map_y);
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full_ab[s], 2);                // the leading CTA's A and B producers
      mbar_init(&full_sfb[s], 1);               // ... and its B-scale producer
      mbar_init(&full_sfa[s], 1);               // this CTA's A-scale producer
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 2 * Cfg::kSfWarps + 1);   // the A-scale warps of both CTAs, the B-scale copies
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * Cfg::kEpiWarps);   // every epilogue warp of both CTAs
    mbar_init(res_load, 1);
    mbar_init(res_cp, 1);
    mbar_init(res_free, 1);
    for (int d = 0; d <= Cfg::kCopyWarps; ++d) mbar_init(&drained[d], 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();          // barriers initialised and tensor memory allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_prior_grid();
  pdl_allow_next_grid();

  // the pair's run of tiles: pair q of G / 2 takes tiles [first, first + count)
  const int pairs = static_cast<int>(gridDim.x) / 2, pair = static_cast<int>(blockIdx.x) / 2;
  int first = 0, count = 0;
  {
    const int q = p.num_tiles / pairs, r = p.num_tiles % pairs;
    first = pair * q + (pair < r ? pair : r);
    count = aligned ? q + (pair < r ? 1 : 0) : 0;
  }
  auto new_block = [&](int i) { return i == 0 || (first + i) / p.tiles_m != (first + i - 1) / p.tiles_m; };
  auto last_of_block = [&](int i) { return i + 1 == count || (first + i + 1) / p.tiles_m != (first + i) / p.tiles_m; };
  // barriers of the leading CTA, as shared::cluster addresses
  const uint32_t full_ab_lead = mapa_shared(smem_u32(full_ab), 0);
  const uint32_t full_sfb_lead = mapa_shared(smem_u32(full_sfb), 0);
  const uint32_t sf_full_lead = mapa_shared(smem_u32(sf_full), 0);
  const uint32_t res_load_lead = mapa_shared(smem_u32(res_load), 0);
  const uint32_t acc_empty_lead = mapa_shared(smem_u32(acc_empty), 0);

  if (warp >= 1 && warp <= Cfg::kProducers) {
    if (lane == 0) {
      // ---------------- producers: A, B, A's scales, B's scales (+ resident) ----------------
      // One copy per operand and stage.  A thread's copies complete one after
      // another, so each operand has two threads, taking the even and the odd
      // stages of the sequence.
      const int role = (warp - 1) >> 1, parity = (warp - 1) & 1;
      int it = 0, res_uses = 0;
      bool ok = true;
      for (int i = 0; i < count && ok; ++i) {
        const int tile = first + i;
        const int32_t m0 = (tile % p.tiles_m) * (2 * Cfg::kBM) + static_cast<int32_t>(rank) * Cfg::kBM;
        const int32_t n0 = (tile / p.tiles_m) * Cfg::kBN;
        if (role == 3 && parity == 0 && res_st > 0 && new_block(i)) {
          // both CTAs' resident buffers are free once the previous block's copies ran
          if (res_uses >= 1 && !mbar_wait_backoff(res_cp, static_cast<uint32_t>(res_uses - 1) & 1u, p.status)) break;
          ++res_uses;
          if (lead) mbar_arrive_expect_tx(res_load, static_cast<uint32_t>(2 * res_st * Cfg::kSfbBytes));
          // box of res_st * 2 chunks: this launch's B-scale map is sized for it (see the launch)
          tma_load_3d_pair(sRes, &map_sfb, res_load_lead, 0, 0, n0 / 128);
        }
        for (int ks = 0; ks < n_kst; ++ks, ++it) {
          if ((it & 1) != parity) continue;
          const uint32_t st = static_cast<uint32_t>(it % Cfg::kStages);
          const uint32_t ph = static_cast<uint32_t>(it / Cfg::kStages) & 1u;
          if (it >= Cfg::kStages && !mbar_wait_backoff(&empty[st], ph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          const uint32_t bar_ab = full_ab_lead + static_cast<uint32_t>(st * 8);
          const uint32_t bar_sfb = full_sfb_lead + static_cast<uint32_t>(st * 8);
          if (role == 0) {
            if (lead) mbar_arrive_expect_tx(&full_ab[st], 2 * Cfg::kABytes);
            tma_load_3d_pair(sA + st * Cfg::kABytes, &map_a, bar_ab, 0, m0, Cfg::kChunks * ks);
          } else if (role == 1) {
            if (lead) mbar_arrive_expect_tx(&full_ab[st], 2 * Cfg::kBBytes);
            tma_load_3d_pair(sB + st * Cfg::kBBytes, &map_b, bar_ab, 0, n0 + static_cast<int32_t>(rank) * Cfg::kBNHalf,
                             Cfg::kChunks * ks);
          } else if (role == 2) {
            mbar_arrive_expect_tx(&full_sfa[st], Cfg::kSfaBytes);
            tma_load_3d(sSfa + st * Cfg::kSfaBytes, &map_sfa, &full_sfa[st], 0, Cfg::kChunks * ks, m0 / 128);
          } else if (ks >= res_st) {
            if (lead) mbar_arrive_expect_tx(&full_sfb[st], 2 * Cfg::kSfbBytes);
            tma_load_3d_pair(sSfb + st * Cfg::kSfbBytes, &map_sfb, bar_sfb, 0, Cfg::kChunks * ks, n0 / 128);
          } else if (lead) {
            mbar_arrive(&full_sfb[st]);           // this stage's B scales are resident
          }
        }
      }
    }
  } else if (warp >= Cfg::kCopyWarp && warp < Cfg::kCopyWarp + Cfg::kCopyWarps) {
    if (lead && lane == 0) {
      // ---------------- B's scale copiers (leading CTA; each copy fills both CTAs) ----------------
      // Copier cw takes the stages it with it % kCopyWarps == cw, so one
      // thread's waits and commits run beside the other's copies.  Stage
      // ks's copies go to the slots of its stage buffer st: the slot's
      // previous MMAs completed before the stage was refilled.  Copier 0
      // also copies the resident scales of a new column block.
      const int cw = warp - Cfg::kCopyWarp;
      int it = 0, res_uses = 0;
      bool ok = true;
      const uint64_t res_d = smem_desc(smem_u32(sRes), 0, 128, kLayoutSwizzleNone);
      for (int i = 0; i < count && ok; ++i) {
        if (cw == 0 && res_st > 0 && new_block(i)) {
          if (res_uses >= 1 && !mbar_wait_poll(res_free, static_cast<uint32_t>(res_uses - 1) & 1u, p.status)) break;
          if (!mbar_wait_poll(res_load, static_cast<uint32_t>(res_uses) & 1u, p.status)) break;
          ++res_uses;
          tc_fence_after();
          // sRes: [group g][k-block kb of the resident stages], 512 bytes each
          const int res_kb = min(res_st * Cfg::kKbPerStage, n_kb);
          for (int kb = 0; kb < res_kb; ++kb)
#pragma unroll
            for (int g = 0; g < 2; ++g)
              tc_cp_32x128b_warpx4_pair(tmem + Cfg::kSfbCol + Cfg::kSfbKbCols * kb + 4 * g,
                                        res_d + static_cast<uint64_t>(32 * (g * res_st * Cfg::kKbPerStage + kb)));
          tc_commit_pair_both(res_cp);
        }
        for (int ks = 0; ks < n_kst; ++ks, ++it) {
          if (it % Cfg::kCopyWarps != cw) continue;
          const uint32_t st = static_cast<uint32_t>(it % Cfg::kStages);
          const uint32_t ph = static_cast<uint32_t>(it / Cfg::kStages) & 1u;
          if (!mbar_wait_poll(&full_sfb[st], ph, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (ks >= res_st) {
            const uint32_t sfb_t = sfb_tmem_of(tmem, ks, static_cast<int>(st));
            const uint64_t sfb_d = smem_desc(smem_u32(sSfb + st * Cfg::kSfbBytes), 0, 128, kLayoutSwizzleNone);
            const int nkb = min(Cfg::kKbPerStage, n_kb - ks * Cfg::kKbPerStage);
            for (int kb = 0; kb < nkb; ++kb)
#pragma unroll
              for (int g = 0; g < 2; ++g)
                tc_cp_32x128b_warpx4_pair(sfb_t + Cfg::kSfbKbCols * kb + 4 * g,
                                          sfb_d + static_cast<uint64_t>(32 * (g * Cfg::kKbPerStage + kb)));
          }
          tc_commit_pair(&sf_full[st]);
        }
      }
      tc_commit_pair(&drained[1 + cw]);
      mbar_wait(&drained[1 + cw], 0, p.status);
    }
  } else if (warp >= Cfg::kFirstSfWarp && warp < Cfg::kFirstEpiWarp) {
    // ---------------- A's scales into tensor memory (both CTAs) ----------------
    // Each warp stores A's atoms of every stage (its CTA's rows) into the
    // stage's slot in its own lane quarter.  A slot's previous MMAs completed
    // before its stage was refilled, so the slot is free once the stage's
    // atoms have landed.
    const uint32_t t_quarter = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    uint32_t st = 0, ph = 0;
    for (int it = 0; it < count * n_kst; ++it) {
      uint32_t okw = 1u;
      if (lane == 0) okw = mbar_wait_backoff(&full_sfa[st], ph, p.status) ? 1u : 0u;
      if (__shfl_sync(0xFFFFFFFFu, okw, 0) == 0u) break;
      tc_fence_after();
      // lane l's 16 bytes of atom kb are columns 4 kb .. 4 kb + 3 of its lane
      const uint8_t* src = sSfa + st * Cfg::kSfaBytes + 16 * lane;
      uint32_t w[16];
#pragma unroll
      for (int kb = 0; kb < Cfg::kKbPerStage; ++kb) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + kb * 512);
        w[4 * kb] = v.x;
        w[4 * kb + 1] = v.y;
        w[4 * kb + 2] = v.z;
        w[4 * kb + 3] = v.w;
      }
      tmem_st_32x32b_x16(t_quarter + Cfg::kSfaCol + Cfg::kSfaSlotCols * st, w);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(sf_full_lead + static_cast<uint32_t>(st * 8));
      if (++st == Cfg::kStages) {
        st = 0;
        ph ^= 1u;
      }
    }
  } else if (warp == 0) {
    if (lead && lane == 0) {
      // ---------------- MMA issuer (leading CTA) ----------------
      uint32_t st = 0, ph = 0;
      int res_uses = 0;
      bool ok = true;
      for (int i = 0; i < count && ok; ++i) {
        if (res_st > 0 && new_block(i)) {
          if (!mbar_wait_poll(res_cp, static_cast<uint32_t>(res_uses) & 1u, p.status)) break;
          ++res_uses;
        }
        for (int ks = 0; ks < n_kst; ++ks) {
          if (!mbar_wait_poll(&sf_full[st], ph, p.status) || !mbar_wait_poll(&full_ab[st], ph, p.status)) {
            ok = false;
            break;
          }
          if (ks == 0 && i >= 1 && !mbar_wait_poll(acc_empty, static_cast<uint32_t>(i - 1) & 1u, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + Cfg::kSfaCol + Cfg::kSfaSlotCols * st;
          const uint32_t sfb_t = sfb_tmem_of(tmem, ks, static_cast<int>(st));
          // k-block kb: chunk kb / 4 (16 KB tiles), 32-byte step kb % 4 inside it
          const uint64_t a0 = smem_desc(smem_u32(sA + st * Cfg::kABytes), 16, Cfg::kSbo, kLayoutSwizzle128B);
          const uint64_t b0 = smem_desc(smem_u32(sB + st * Cfg::kBBytes), 16, Cfg::kSbo, kLayoutSwizzle128B);
          const int nkb = min(Cfg::kKbPerStage, n_kb - ks * Cfg::kKbPerStage);
          if (nkb == Cfg::kKbPerStage) {
#pragma unroll
            for (int kb = 0; kb < Cfg::kKbPerStage; ++kb) {
              const uint64_t step = static_cast<uint64_t>((kb >> 2) * (Cfg::kAChunkBytes >> 4) + 2 * (kb & 3));
              const uint64_t stepb = static_cast<uint64_t>((kb >> 2) * (Cfg::kBChunkBytes >> 4) + 2 * (kb & 3));
              mma_nvf4_pair(tmem, a0 + step, b0 + stepb, Cfg::kIdesc, sfa_t + 4 * kb, sfb_t + Cfg::kSfbKbCols * kb,
                            (ks > 0 || kb > 0) ? 1u : 0u);
            }
          } else {
            for (int kb = 0; kb < nkb; ++kb) {
              const uint64_t step = static_cast<uint64_t>((kb >> 2) * (Cfg::kAChunkBytes >> 4) + 2 * (kb & 3));
              const uint64_t stepb = static_cast<uint64_t>((kb >> 2) * (Cfg::kBChunkBytes >> 4) + 2 * (kb & 3));
              mma_nvf4_pair(tmem, a0 + step, b0 + stepb, Cfg::kIdesc, sfa_t + 4 * kb, sfb_t + Cfg::kSfbKbCols * kb,
                            (ks > 0 || kb > 0) ? 1u : 0u);
            }
          }
          tc_commit_pair_both(&empty[st]);        // both CTAs' producers may refill the stage
          if (++st == Cfg::kStages) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_both(acc_full);
        if (res_st > 0 && last_of_block(i)) tc_commit_pair(res_free);
      }
      tc_commit_pair(&drained[0]);
      mbar_wait(&drained[0], 0, p.status);
    }
  } else {
    // ---------------- epilogue (both CTAs, own rows) ----------------
    // The whole 128-column slice of a warp is taken out of tensor memory and
    // packed to bf16 in registers, chunk by chunk, before the accumulator is
    // handed back; only then is it staged and stored.
    const int ew = warp - Cfg::kFirstEpiWarp;
    const int q = warp & 3;                    // lane quarter of tensor memory this warp may read
    const int h = ew / 4;                      // which 128-column half
    const int r = 32 * q + lane;               // row of this CTA's 128
    const bool store_thr = (ew == 0 && lane == 0);
    const float alpha = __ldg(p.gdec_a) * __ldg(p.gdec_b);
    for (int i = 0; i < count; ++i) {
      const int tile = first + i;
      const int64_t m0 = static_cast<int64_t>(tile % p.tiles_m) * (2 * Cfg::kBM) + static_cast<int64_t>(rank) * Cfg::kBM;
      const int64_t n0 = static_cast<int64_t>(tile / p.tiles_m) * Cfg::kBN;
      if (store_thr) bulk_wait_group_read<0>();
      named_barrier(1, kEpiThreads);
      {
        const int64_t col = n0 + ew * 32 + lane;
        bias_s[ew * 32 + lane] = (p.bias != nullptr && col < p.N) ? __ldg(p.bias + col) : 0.0f;
      }
      uint32_t okw = 0;
      if (lane == 0) okw = mbar_wait_backoff(acc_full, static_cast<uint32_t>(i) & 1u, p.status) ? 1u : 0u;
      const bool ok = __shfl_sync(0xFFFFFFFFu, okw, 0) != 0;
      if (named_barrier_or(1, kEpiThreads, !ok)) break;
      tc_fence_after();
      const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * q) << 16);
      // chunk c of this warp's four: alpha * acc + bias as 16 bf16 pairs
      auto load_pack = [&](int c, uint32_t (&w)[16]) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(32 * (4 * h + c)), v);
        tmem_ld_wait();
        const float* b = bias_s + 32 * (4 * h + c);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 bb = *reinterpret_cast<const float2*>(b + 2 * k);
          const __nv_bfloat162 pr = __floats2bfloat162_rn(fmaf(alpha, __uint_as_float(v[2 * k]), bb.x),
                                                          fmaf(alpha, __uint_as_float(v[2 * k + 1]), bb.y));
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
      auto store_round = [&](int first_col) {
        fence_proxy_async_smem();
        named_barrier(1, kEpiThreads);
        if (store_thr) {
          if (m0 < p.M) {
#pragma unroll
            for (int bx = 0; bx < 2; ++bx) {
              const int64_t col = n0 + first_col + bx * 128;
              if (col < p.N)
                tma_store_2d(&map_y, sOut + bx * (Cfg::kBM * 128), static_cast<int32_t>(col), static_cast<int32_t>(m0));
            }
          }
          bulk_commit_group();
        }
      };
      // round 0's chunks go straight to the (free) staging buffer; round 1's
      // stay in registers; the accumulator goes back to the leading CTA's MMA
      // thread as soon as the last chunk is out of tensor memory
      {
        uint32_t w[16];
        load_pack(0, w);
        stage_bf16(0, w);
        load_pack(1, w);
        stage_bf16(1, w);
      }
      uint32_t w2[16], w3[16];
      load_pack(2, w2);
      load_pack(3, w3);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_lead);
      store_round(0);
      if (store_thr) bulk_wait_group_read<0>();
      named_barrier(1, kEpiThreads);
      stage_bf16(2, w2);
      stage_bf16(3, w3);
      store_round(64);
    }
    if (store_thr) bulk_wait_group_all();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();          // no CTA leaves while its pair may still signal its barriers
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::kTmemCols);
  }
}

// Clusters of two CTAs of gemm2_nvfp4_kernel that can be resident at once on
// the current device (cached per device).
static int resident_pairs() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> g(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * (sm_count() / 2)));
  cfg.blockDim = dim3(Gemm2Cfg::kThreads);
  cfg.dynamicSmemBytes = Gemm2Cfg::kSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(gemm2_nvfp4_kernel), &cfg) != cudaSuccess || n < 1)
    n = sm_count() / 2;
  cache[dev] = n;
  return n;
}

// The pair kernel serves dense bf16 outputs with K a multiple of 256 (its
// operand copies take whole 256-deep chunks); its tiles are 256 x 256.
bool gemm_pair_applies(const GemmArgs& a) {
  return a.yt == AVR_BF16 && a.block_expert == nullptr && a.row_scale == nullptr && a.groups == 1 && a.K % 256 == 0;
}

// [rows, K/2 bytes] codes as a 3-D tensor (128 bytes, rows, K/256 chunks):
// a box of (128, box_rows, box_chunks) brings box_chunks 128-byte-swizzled
// chunk tiles of box_rows rows, one after the other
bool pair_codes_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K, uint32_t box_rows, uint32_t box_chunks) {
  const uint64_t dims[3] = {128, static_cast<uint64_t>(rows), static_cast<uint64_t>(K / 256)};
  const uint64_t strides[2] = {static_cast<uint64_t>(K / 2), 128};
  const uint32_t box[3] = {128, box_rows, box_chunks};
  return make_tensor_map_3d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// scale atoms as a 3-D tensor of 8-byte elements (256 = one chunk's 4
// atoms, K/256 chunks, row groups of 128)
bool pair_scales_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K, uint32_t box_chunks,
                     uint32_t box_groups) {
  const uint64_t dims[3] = {256, static_cast<uint64_t>(K / 256), static_cast<uint64_t>((rows + 127) / 128)};
  const uint64_t strides[2] = {2048, static_cast<uint64_t>(K / 64) * 512};
  const uint32_t box[3] = {256, box_chunks, box_groups};
  return make_tensor_map_3d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT64, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

cudaError_t launch_gemm_pair(const GemmArgs& a, cudaStream_t s, bool pdl) {
  using Cfg = Gemm2Cfg;
  if (!gemm_pair_applies(a)) return cudaErrorInvalidValue;
  const int n_kst = static_cast<int>((a.K + Cfg::kStageK - 1) / Cfg::kStageK);
  // B's scales: all of K resident when they fit, else streamed per stage
  const int res_stages = n_kst <= Cfg::kResAllStages ? n_kst : 0;
  CUtensorMap ma, mb, msa, msb, my;
  if (!pair_codes_map(&ma, a.a_codes, a.M, a.K, Cfg::kBM, Cfg::kChunks) ||
      !pair_codes_map(&mb, a.b_codes, a.N, a.K, Cfg::kBNHalf, Cfg::kChunks) ||
      !pair_scales_map(&msa, a.a_scales, a.M, a.K, Cfg::kChunks, 1))
    return cudaErrorInvalidValue;
  // one map for B's scales: its box is the resident block (res_stages stages
  // of both row groups) when every stage is resident, else one stage
  if (!pair_scales_map(&msb, a.b_scales, a.N, a.K, static_cast<uint32_t>(Cfg::kChunks * (res_stages > 0 ? res_stages : 1)), 2))
    return cudaErrorInvalidValue;
  if (!make_tensor_map_2d(&my, a.Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, static_cast<uint64_t>(a.M),
                          static_cast<uint64_t>(a.N), Cfg::kBM, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  Gemm2Params p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.tiles_m = static_cast<int>((a.M + 2 * Cfg::kBM - 1) / (2 * Cfg::kBM));
  p.num_tiles = p.tiles_m * static_cast<int>((a.N + Cfg::kBN - 1) / Cfg::kBN);
  p.res_stages = res_stages;
  p.gdec_a = a.a_gdec;
  p.gdec_b = a.b_gdec;
  p.bias = a.bias;
  p.status = a.status;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(gemm2_nvfp4_kernel), Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  // one pair per two SMs that can hold pairs at once: the run of tiles is
  // split statically, so a pair that had to wait for another would double the time
  const int max_pairs = resident_pairs();
  const int pairs = p.num_tiles < max_pairs ? p.num_tiles : max_pairs;
  return launch_ex(gemm2_nvfp4_kernel, dim3(2 * pairs), dim3(Cfg::kThreads), Cfg::kSmemBytes, s, pdl, ma, mb, msa,
                   msb, my, p);
}

}  // namespace avr
