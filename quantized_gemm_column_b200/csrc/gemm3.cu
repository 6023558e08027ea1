// K3 on CTA pairs for short contractions (K <= 1024, a multiple of 256):
// the block-scaled FP4 GEMM with bf16 output.
//
// Y = 1 (mu_bar W_bar) + X_bar_R W_bar (Lighthouse review of "The Curse and
// Blessing of Mean Bias in FP4-Quantized LLM Training", section 二 "Averis
// 方法"): the product X_bar_R W_bar on E2M1 operands with E4M3 per-16 scales,
// the row mu_bar W_bar added to every output row as a bias:
//   Y[i, j] = g_dec(A) g_dec(B) * acc[i, j] + bias[j].
//
// Why a second pair kernel.  At K <= 1024 a 256 x 256 tile is at most four
// 256-deep stages of MMAs (about 1.2 us).  The long-contraction kernel
// streams A and B for every stage, and at this depth the operand copies, not
// the MMAs, set the pace (without any epilogue it still runs at about 40% of
// the MMA rate): B is fetched again for every tile although it did not
// change.  Here B's codes (shared memory) and scales (tensor memory) for the
// pair's column block stay resident while the pair's run of tiles stays in
// that block (tiles go M fastest); only A and its scales stream, through a
// ring of six 256-deep stages (one and a half tiles).
//
// Roles (both CTAs have the same warps; CTA rank 0 of the pair leads):
//   warp 0     : tensor-memory allocation (cta_group::2, in both CTAs); in
//                the leading CTA one thread issues the pair's MMAs;
//   warps 1..4 : A's rows, stage it from warp 1 + it % 4; the copies
//                complete on the leading CTA's barrier, which expects both
//                CTAs' bytes;
//   warp 5     : A's scale atoms of this CTA, on its own barrier;
//   warp 6     : per column block, B's rows (the 128 this CTA holds) and
//                B's scale atoms for all 256 columns, on the leading CTA's
//                barrier;
//   warp 7     : in the leading CTA, B's scale atoms into tensor memory
//                (tcgen05.cp cta_group::2) per column block;
//   warps 8..11: A's scales into tensor memory, one warp per lane quarter,
//                by tcgen05.st from registers;
//   warps 12..19: epilogue, each warp 32 rows x 128 columns: tcgen05.ld,
//                alpha * acc + bias, bf16, staged in the warp's own 4 KB in
//                two rounds of 64 columns and stored by its own TMA copies.
// No TMA load is multicast.
#include <map>
#include <mutex>
#include <utility>

#include "device.cuh"
#include "internal.h"
#include "pair.cuh"

namespace avr {

using namespace pair;

struct Gemm3Cfg {
  static constexpr int kBM = 128;                          // rows per CTA (256 per pair)
  static constexpr int kBN = 256;                          // columns per tile
  static constexpr int kMaxChunks = 4;                     // K <= 1024: 256-deep chunks
  static constexpr int kAStages = 6;
  static constexpr int kKbPerStage = 4;                    // 64-deep MMAs per chunk
  static constexpr int kEpiWarps = 8;
  static constexpr int kSfWarps = 4;
  static constexpr int kAWarp0 = 1;
  static constexpr int kAWarps = 4;                        // one TMA thread's copies complete one after another
  static constexpr int kSfaWarp = kAWarp0 + kAWarps;
  static constexpr int kResWarp = kSfaWarp + 1;
  static constexpr int kCopyWarp = kResWarp + 1;
  static constexpr int kFirstSfWarp = kCopyWarp + 1;
  static constexpr int kFirstEpiWarp = kFirstSfWarp + kSfWarps;
  static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
  static constexpr uint32_t kSbo = 8 * 128;                // 8-row swizzle atom of 128-byte rows
  static constexpr int kABytes = kBM * 128;                // 16 KB: 128 rows x 256 K
  static constexpr int kSfaBytes = kKbPerStage * 512;      // 2 KB: 4 atoms
  static constexpr int kBChunkBytes = 128 * 128;           // 16 KB: this CTA's 128 rows x 256 K
  static constexpr int kSfbResBytes = 2 * kMaxChunks * kKbPerStage * 512;   // 16 KB: [group][k-block] atoms
  static constexpr int kOutBytes = kEpiWarps * 32 * 128;   // 32 KB: per epilogue warp, 32 rows x 64 columns
  static constexpr int kSfaOffset = kAStages * kABytes;
  static constexpr int kBOffset = kSfaOffset + kAStages * kSfaBytes;
  static constexpr int kSfbResOffset = kBOffset + kMaxChunks * kBChunkBytes;
  static constexpr int kOutOffset = kSfbResOffset + kSfbResBytes;
  static constexpr int kBiasOffset = kOutOffset + kOutBytes;
  static constexpr int kBarOffset = kBiasOffset + 2 * kBN * 4;   // the bias row, double-buffered by tile
  static constexpr int kSmemBytes = kBarOffset + 512;
  static_assert(kBOffset % 1024 == 0 && kOutOffset % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  // tensor memory (the same columns in both CTAs): the 256-column
  // accumulator, A's scale slots (one per stage), B's resident scales
  static constexpr int kSfaCol = kBN;
  static constexpr int kSfaSlotCols = kKbPerStage * 4;     // 16
  static constexpr int kSfbCol = kSfaCol + kAStages * kSfaSlotCols;   // 352
  static constexpr int kSfbKbCols = 8;                     // two groups of 128 columns, 4 columns each
  static constexpr int kTmemCols = 512;
  static_assert(kSfbCol + kMaxChunks * kKbPerStage * kSfbKbCols <= kTmemCols, "tensor memory budget");
  // instruction descriptor: E2M1 A and B, UE4M3 scales, K-major, N = 256
  // (N >> 3 at bit 17), M = 256 for the pair (M >> 4 at bit 24)
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                                     (static_cast<uint32_t>((2 * kBM) >> 4) << 24);
};

struct Gemm3Params {
  int64_t M, N, K;
  int tiles_m, num_tiles;   // pair tiles of 256 x 256, M fastest
  const float* gdec_a;
  const float* gdec_b;
  const float* bias;
  uint32_t* status;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Gemm3Cfg::kThreads, 1)
    gemm3_nvfp4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                       const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                       const __grid_constant__ CUtensorMap map_y, const Gemm3Params p) {
  using Cfg = Gemm3Cfg;
  constexpr int kEpiThreads = 32 * Cfg::kEpiWarps;
  extern __shared__ __align__(1024) uint8_t smem[];
  // the swizzled tiles need 1024-byte alignment; a CTA without it still takes
  // part in the pair's cluster barriers and allocation, but does no work
  const bool aligned = (smem_u32(smem) & 1023u) == 0;
  uint8_t* sA = smem;
  uint8_t* sSfa = smem + Cfg::kSfaOffset;
  uint8_t* sB = smem + Cfg::kBOffset;                  // [chunk][128 rows x 128 B]
  uint8_t* sSfbRes = smem + Cfg::kSfbResOffset;        // [group][k-block] atoms of 512 B
  uint8_t* sOut = smem + Cfg::kOutOffset;
  float* bias_s = reinterpret_cast<float*>(smem + Cfg::kBiasOffset);   // [2][256]
  uint64_t* full_a = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);  // [kAStages] leading CTA: A of both CTAs
  uint64_t* full_sfa = full_a + Cfg::kAStages;    // [kAStages] both CTAs: this CTA's A scale atoms
  uint64_t* empty = full_sfa + Cfg::kAStages;     // [kAStages] both CTAs: the stage's MMAs completed
  uint64_t* sf_full = empty + Cfg::kAStages;      // [kAStages] leading CTA: A's scales of both CTAs stored
  uint64_t* acc_full = sf_full + Cfg::kAStages;   // both CTAs: a tile's MMAs completed
  uint64_t* acc_empty = acc_full + 1;             // leading CTA: both epilogues took the accumulator
  uint64_t* res_load = acc_empty + 1;             // leading CTA: the block's B rows and atoms landed in both CTAs
  uint64_t* res_cp = res_load + 1;                // both CTAs: the block's B scales are in tensor memory
  uint64_t* res_free = res_cp + 1;                // both CTAs: the MMAs of the block's last tile completed
  uint64_t* drained = res_free + 1;               // [2] leading CTA: MMA and copy threads drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;
  const int n_kst = static_cast<int>(p.K / 256);
  const int n_kb = static_cast<int>(p.K / 64);

  if (threadIdx.x == 0) {
    if (!aligned) raise_status(p.status, AVR_ERR_MISALIGNED);
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
    prefetch_tensormap(&map_sfa);
    prefetch_tensormap(&map_sfb);
    prefetch_tensormap(&map_y);
    for (int s = 0; s < Cfg::kAStages; ++s) {
      mbar_init(&full_a[s], 1);                 // the leading CTA's A producer
      mbar_init(&full_sfa[s], 1);               // this CTA's A-scale producer
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 2 * Cfg::kSfWarps);   // the A-scale warps of both CTAs
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * Cfg::kEpiWarps);   // every epilogue warp of both CTAs
    mbar_init(res_load, 1);
    mbar_init(res_cp, 1);
    mbar_init(res_free, 1);
    mbar_init(&drained[0], 1);
    mbar_init(&drained[1], 1);
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
  const int pairs = static_cast<int>(gridDim.x) / 2, pair_id = static_cast<int>(blockIdx.x) / 2;
  int first = 0, count = 0;
  {
    const int q = p.num_tiles / pairs, r = p.num_tiles % pairs;
    first = pair_id * q + (pair_id < r ? pair_id : r);
    count = aligned ? q + (pair_id < r ? 1 : 0) : 0;
  }
  auto new_block = [&](int i) { return i == 0 || (first + i) / p.tiles_m != (first + i - 1) / p.tiles_m; };
  auto last_of_block = [&](int i) { return i + 1 == count || (first + i + 1) / p.tiles_m != (first + i) / p.tiles_m; };
  auto row0 = [&](int i) {   // this CTA's first row of tile first + i
    return static_cast<int32_t>(((first + i) % p.tiles_m) * (2 * Cfg::kBM) + static_cast<int>(rank) * Cfg::kBM);
  };
  auto col0 = [&](int i) { return static_cast<int32_t>(((first + i) / p.tiles_m) * Cfg::kBN); };
  // barriers of the leading CTA, as shared::cluster addresses
  const uint32_t full_a_lead = mapa_shared(smem_u32(full_a), 0);
  const uint32_t sf_full_lead = mapa_shared(smem_u32(sf_full), 0);
  const uint32_t res_load_lead = mapa_shared(smem_u32(res_load), 0);
  const uint32_t acc_empty_lead = mapa_shared(smem_u32(acc_empty), 0);

  if (warp >= Cfg::kAWarp0 && warp < Cfg::kAWarp0 + Cfg::kAWarps) {
    if (lane == 0) {
      // ---------------- A's rows (both CTAs; stage it from thread it % kAWarps) ----------------
      // A thread's copies complete one after another (about 16 KB per
      // 265 ns), so the stages are spread over several threads.
      const int parity = warp - Cfg::kAWarp0;
      int it = 0;
      for (int i = 0; i < count; ++i) {
        const int32_t m0 = row0(i);
        bool ok = true;
        for (int ks = 0; ks < n_kst; ++ks, ++it) {
          if (it % Cfg::kAWarps != parity) continue;
          const uint32_t st = static_cast<uint32_t>(it % Cfg::kAStages);
          const uint32_t ph = static_cast<uint32_t>(it / Cfg::kAStages) & 1u;
          if (it >= Cfg::kAStages && !mbar_wait_backoff(&empty[st], ph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          if (lead) mbar_arrive_expect_tx(&full_a[st], 2 * Cfg::kABytes);
          tma_load_3d_pair(sA + st * Cfg::kABytes, &map_a, full_a_lead + static_cast<uint32_t>(st * 8), 0, m0, ks);
        }
        if (!ok) break;
      }
    }
  } else if (warp == Cfg::kSfaWarp) {
    if (lane == 0) {
      // ---------------- A's scale atoms (both CTAs, each its own rows) ----------------
      int it = 0;
      for (int i = 0; i < count; ++i) {
        const int32_t g0 = row0(i) / 128;
        bool ok = true;
        for (int ks = 0; ks < n_kst; ++ks, ++it) {
          const uint32_t st = static_cast<uint32_t>(it % Cfg::kAStages);
          const uint32_t ph = static_cast<uint32_t>(it / Cfg::kAStages) & 1u;
          if (it >= Cfg::kAStages && !mbar_wait_backoff(&empty[st], ph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_sfa[st], Cfg::kSfaBytes);
          tma_load_3d(sSfa + st * Cfg::kSfaBytes, &map_sfa, &full_sfa[st], 0, ks, g0);
        }
        if (!ok) break;
      }
    }
  } else if (warp == Cfg::kResWarp) {
    if (lane == 0) {
      // ---------------- B's rows and scale atoms per column block (both CTAs) ----------------
      // The previous block's MMAs must have completed before its rows are
      // overwritten (its atoms were copied out before those MMAs ran).
      int res_uses = 0;
      for (int i = 0; i < count; ++i) {
        if (!new_block(i)) continue;
        if (res_uses >= 1 && !mbar_wait_backoff(res_free, static_cast<uint32_t>(res_uses - 1) & 1u, p.status)) break;
        ++res_uses;
        const int32_t n0 = col0(i);
        if (lead)
          mbar_arrive_expect_tx(res_load,
                                static_cast<uint32_t>(2 * n_kst * (Cfg::kBChunkBytes + 2 * Cfg::kKbPerStage * 512)));
        // rows n0 + 128 rank .. + 128, all chunks (a box of n_kst chunks)
        tma_load_3d_pair(sB, &map_b, res_load_lead, 0, n0 + 128 * static_cast<int32_t>(rank), 0);
        tma_load_3d_pair(sSfbRes, &map_sfb, res_load_lead, 0, 0, n0 / 128);
      }
    }
  } else if (warp == Cfg::kCopyWarp) {
    if (lead && lane == 0) {
      // ---------------- B's scales into tensor memory per column block (leading CTA) ----------------
      int res_uses = 0;
      const uint64_t res_d = smem_desc(smem_u32(sSfbRes), 0, 128, kLayoutSwizzleNone);
      for (int i = 0; i < count; ++i) {
        if (!new_block(i)) continue;
        if (res_uses >= 1 && !mbar_wait_backoff(res_free, static_cast<uint32_t>(res_uses - 1) & 1u, p.status)) break;
        if (!mbar_wait_backoff(res_load, static_cast<uint32_t>(res_uses) & 1u, p.status)) break;
        ++res_uses;
        tc_fence_after();
        for (int kb = 0; kb < n_kb; ++kb)
#pragma unroll
          for (int g = 0; g < 2; ++g)
            tc_cp_32x128b_warpx4_pair(tmem + Cfg::kSfbCol + Cfg::kSfbKbCols * kb + 4 * g,
                                      res_d + static_cast<uint64_t>(32 * (g * n_kb + kb)));
        tc_commit_pair_both(res_cp);
      }
      tc_commit_pair(&drained[1]);
      mbar_wait(&drained[1], 0, p.status);
    }
  } else if (warp >= Cfg::kFirstSfWarp && warp < Cfg::kFirstEpiWarp) {
    // ---------------- A's scales into tensor memory (both CTAs) ----------------
    // Each warp stores A's atoms of every stage (its CTA's rows) into the
    // stage's slot in its own lane quarter: the image a 32x128b.warpx4 copy
    // makes.  A slot's previous MMAs completed before its stage was
    // refilled, so the slot is free once the stage's atoms have landed.
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
      if (++st == Cfg::kAStages) {
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
        if (new_block(i)) {
          if (!mbar_wait_poll(res_cp, static_cast<uint32_t>(res_uses) & 1u, p.status)) break;
          ++res_uses;
        }
        for (int ks = 0; ks < n_kst; ++ks) {
          if (!mbar_wait_poll(&sf_full[st], ph, p.status) || !mbar_wait_poll(&full_a[st], ph, p.status)) {
            ok = false;
            break;
          }
          if (ks == 0 && i >= 1 && !mbar_wait_poll(acc_empty, static_cast<uint32_t>(i - 1) & 1u, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + Cfg::kSfaCol + Cfg::kSfaSlotCols * st;
          const uint32_t sfb_t = tmem + Cfg::kSfbCol + Cfg::kSfbKbCols * (Cfg::kKbPerStage * ks);
          // k-block kb: a 32-byte step inside the 128-byte swizzled rows
          const uint64_t a0 = smem_desc(smem_u32(sA + st * Cfg::kABytes), 16, Cfg::kSbo, kLayoutSwizzle128B);
          const uint64_t b0 = smem_desc(smem_u32(sB + ks * Cfg::kBChunkBytes), 16, Cfg::kSbo, kLayoutSwizzle128B);
#pragma unroll
          for (int kb = 0; kb < Cfg::kKbPerStage; ++kb)
            mma_nvf4_pair(tmem, a0 + 2 * kb, b0 + 2 * kb, Cfg::kIdesc, sfa_t + 4 * kb, sfb_t + Cfg::kSfbKbCols * kb,
                          (ks > 0 || kb > 0) ? 1u : 0u);
          tc_commit_pair_both(&empty[st]);        // both CTAs' producers may refill the stage
          if (++st == Cfg::kAStages) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_both(acc_full);
        if (last_of_block(i)) tc_commit_pair_both(res_free);
      }
      tc_commit_pair(&drained[0]);
      mbar_wait(&drained[0], 0, p.status);
    }
  } else {
    // ---------------- epilogue (both CTAs, own rows) ----------------
    // Warp (q, h) owns rows 32 q .. 32 q + 31 of this CTA and columns
    // 128 h .. 128 h + 127 of the tile.  Chunks 0 and 1 (columns + 0 .. 63)
    // go to the warp's own 4 KB staging block as they come out of tensor
    // memory, chunks 2 and 3 stay in registers; the accumulator is handed
    // back, then the two 32 x 64 blocks are stored by the warp's own TMA
    // copies.  The warps meet once per tile (the bias row; a failed wait
    // ends every warp's loop there).
    const int ew = warp - Cfg::kFirstEpiWarp;
    const int q = warp & 3;                    // lane quarter of tensor memory this warp may read
    const int h = ew / 4;                      // which 128 columns
    const float alpha = __ldg(p.gdec_a) * __ldg(p.gdec_b);
    const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * q) << 16);
    uint8_t* stg = sOut + ew * 4096;           // 32 rows x 128 bytes, 128-byte swizzle
    bool ok = true;
    for (int i = 0; i < count; ++i) {
      const int32_t m0 = row0(i) + 32 * q;
      const int32_t n0 = col0(i);
      // the bias row of this tile, in the buffer of its parity: every warp has
      // finished tile i - 2 (it passed the barrier below at tile i - 1)
      float* bias_t = bias_s + (i & 1) * Cfg::kBN;
      {
        const int64_t col = static_cast<int64_t>(n0) + ew * 32 + lane;
        bias_t[ew * 32 + lane] = (p.bias != nullptr && col < p.N) ? __ldg(p.bias + col) : 0.0f;
      }
      if (named_barrier_or(1, kEpiThreads, !ok)) break;
      uint32_t okw = 1u;
      if (lane == 0) {
        bulk_wait_group_read<0>();             // this warp's last store has read its staging block
        okw = mbar_wait_poll(acc_full, static_cast<uint32_t>(i) & 1u, p.status) ? 1u : 0u;
      }
      ok = __shfl_sync(0xFFFFFFFFu, okw, 0) != 0;
      if (!ok) continue;
      tc_fence_after();
      // chunk c of the warp's four: alpha * acc + bias as 16 bf16 pairs
      auto load_pack = [&](int c, uint32_t (&w)[16]) {
        const int col = 128 * h + 32 * c;
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(col), v);
        tmem_ld_wait();
        const float* bsrc = bias_t + col;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 bb = *reinterpret_cast<const float2*>(bsrc + 2 * k);
          const __nv_bfloat162 pr = __floats2bfloat162_rn(fmaf(alpha, __uint_as_float(v[2 * k]), bb.x),
                                                          fmaf(alpha, __uint_as_float(v[2 * k + 1]), bb.y));
          w[k] = *reinterpret_cast<const uint32_t*>(&pr);
        }
      };
      // chunk c's 64 bytes of row `lane` in the staging block (64 columns)
      auto stage = [&](int c, const uint32_t (&w)[16]) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int piece = ((c & 1) * 4 + u) ^ (lane & 7);
          *reinterpret_cast<uint4*>(stg + lane * 128 + piece * 16) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      };
      auto store = [&](int first_col) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int64_t col = static_cast<int64_t>(n0) + 128 * h + first_col;
          if (m0 < p.M && col < p.N) tma_store_2d(&map_y, stg, static_cast<int32_t>(col), m0);
          bulk_commit_group();
        }
      };
      {
        uint32_t w[16];
        load_pack(0, w);
        stage(0, w);
        load_pack(1, w);
        stage(1, w);
      }
      uint32_t w2[16], w3[16];
      load_pack(2, w2);
      load_pack(3, w3);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_lead);
      store(0);
      if (lane == 0) bulk_wait_group_read<0>();
      __syncwarp();
      stage(2, w2);
      stage(3, w3);
      store(64);
    }
    if (lane == 0) bulk_wait_group_all();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();          // no CTA leaves while its pair may still signal its barriers
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::kTmemCols);
  }
}

// Clusters of two CTAs of gemm3_nvfp4_kernel that can be resident at once on
// the current device (cached per device).
static int resident_pairs_short() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> g(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * (sm_count() / 2)));
  cfg.blockDim = dim3(Gemm3Cfg::kThreads);
  cfg.dynamicSmemBytes = Gemm3Cfg::kSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(gemm3_nvfp4_kernel), &cfg) != cudaSuccess || n < 1)
    n = sm_count() / 2;
  cache[dev] = n;
  return n;
}

// Dense bf16 outputs with K a multiple of 256 up to 1024.
bool gemm_pair_short_applies(const GemmArgs& a) {
  return gemm_pair_applies(a) && a.K <= 256 * Gemm3Cfg::kMaxChunks;
}

cudaError_t launch_gemm_pair_short(const GemmArgs& a, cudaStream_t s, bool pdl) {
  using Cfg = Gemm3Cfg;
  if (!gemm_pair_short_applies(a)) return cudaErrorInvalidValue;
  const uint32_t n_kst = static_cast<uint32_t>(a.K / 256);
  CUtensorMap ma, mb, msa, msb, my;
  if (!pair_codes_map(&ma, a.a_codes, a.M, a.K, Cfg::kBM, 1) || !pair_codes_map(&mb, a.b_codes, a.N, a.K, Cfg::kBM, n_kst) ||
      !pair_scales_map(&msa, a.a_scales, a.M, a.K, 1, 1) || !pair_scales_map(&msb, a.b_scales, a.N, a.K, n_kst, 2))
    return cudaErrorInvalidValue;
  if (!make_tensor_map_2d(&my, a.Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, static_cast<uint64_t>(a.M),
                          static_cast<uint64_t>(a.N), 32, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  Gemm3Params p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.tiles_m = static_cast<int>((a.M + 2 * Cfg::kBM - 1) / (2 * Cfg::kBM));
  p.num_tiles = p.tiles_m * static_cast<int>((a.N + Cfg::kBN - 1) / Cfg::kBN);
  p.gdec_a = a.a_gdec;
  p.gdec_b = a.b_gdec;
  p.bias = a.bias;
  p.status = a.status;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(gemm3_nvfp4_kernel), Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  // one pair per two SMs that can hold pairs at once: the run of tiles is
  // split statically, so a pair that had to wait for another would double the time
  const int max_pairs = resident_pairs_short();
  const int pairs = p.num_tiles < max_pairs ? p.num_tiles : max_pairs;
  return launch_ex(gemm3_nvfp4_kernel, dim3(2 * pairs), dim3(Cfg::kThreads), Cfg::kSmemBytes, s, pdl, ma, mb, msa,
                   msb, my, p);
}

}  // namespace avr
