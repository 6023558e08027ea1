// K3: block-scaled FP4 GEMM on the 5th-generation tensor cores (tcgen05),
// with the Averis rank-one row as a broadcast bias in the epilogue.
//
// Y = 1 (mu_bar W_bar) + X_bar_R W_bar (Lighthouse review of "The Curse and
// Blessing of Mean Bias in FP4-Quantized LLM Training", section 二 "Averis
// 方法"): the product X_bar_R W_bar runs here on E2M1 operands with E4M3
// per-16 scales, and the row mu_bar W_bar (one value per output column) is
// added to every output row:
//   Y[i, j] = g_dec(A) g_dec(B) * acc[i, j] + bias[j].
//
// CTA tile 128 x BN, K staged 256 elements (128 bytes per row) at a time.
//   warp 0     : TMA producer -- 2-D tensor copies of the A and B code tiles
//                (128-byte swizzle) and 1-D bulk copies of the matching
//                512-byte scale atoms, all completing on the stage's mbarrier;
//   warp 1     : allocates tensor memory; one thread copies the scale atoms
//                shared -> tensor memory (tcgen05.cp 32x128b, replicated to the
//                four lane quarters) and issues the
//                tcgen05.mma.kind::mxf4nvf4.block_scale.block16 instructions
//                (M 128, N BN, K 64 each), then commits to free the stage;
//   warps 2..5 : epilogue -- tcgen05.ld of the fp32 accumulator (each warp its
//                32-lane quarter), scale, add the bias, convert, store.
// Two CTAs share an SM, so one CTA's epilogue overlaps the other's mainloop.
#include "device.cuh"
#include "internal.h"

namespace avr {

template <int BN>
struct GemmCfg {
  static constexpr int kBM = 128;
  static constexpr int kStages = 3;
  static constexpr int kStageK = 256;                      // fp4 elements per stage
  static constexpr int kKbPerStage = kStageK / 64;         // MMAs per stage
  static constexpr int kABytes = kBM * 128;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kSfaBytes = kKbPerStage * 512;
  static constexpr int kSfbBytes = (BN / 128) * kKbPerStage * 512;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;   // + barriers + alignment slack
  static constexpr int kTmemCols = BN <= 128 ? 256 : 512;
  static constexpr int kSfaCol = BN;                           // 2 buffers x 16 columns
  static constexpr int kSfbCol = BN + 2 * kKbPerStage * 4;     // 2 buffers x 4 k-blocks x BN/32
  static constexpr int kSfbColsPerKb = BN / 32;
  static_assert(kSfbCol + 2 * kKbPerStage * kSfbColsPerKb <= kTmemCols, "tensor memory budget");
  // instruction descriptor: E2M1 A and B (format 1), UE4M3 scales, K-major
  // operands, N >> 3 at bit 17, M >> 4 at bit 24
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                     (static_cast<uint32_t>(kBM >> 4) << 24);
};

struct GemmParams {
  int64_t M, N, K;
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* gdec_a;
  const float* gdec_b;
  const float* bias;
  void* Y;
  uint32_t* status;
};

template <int BN, bool kBf16Out>
__global__ void __launch_bounds__(192, 1) gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap map_a,
                                                            const __grid_constant__ CUtensorMap map_b,
                                                            const GemmParams p) {
  using Cfg = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + Cfg::kStages * Cfg::kABytes;
  uint8_t* sSfa = sB + Cfg::kStages * Cfg::kBBytes;
  uint8_t* sSfb = sSfa + Cfg::kStages * Cfg::kSfaBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);
  uint64_t* empty = full + Cfg::kStages;
  uint64_t* acc_bar = empty + Cfg::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * Cfg::kBM;
  const int n_stages = static_cast<int>((p.K + Cfg::kStageK - 1) / Cfg::kStageK);
  const uint32_t kb64 = static_cast<uint32_t>(p.K / 64);

  if (threadIdx.x == 0) {
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_bar, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_prior_grid();
  pdl_allow_next_grid();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer ----------------
      for (int ks = 0; ks < n_stages; ++ks) {
        const int st = ks % Cfg::kStages;
        if (ks >= Cfg::kStages &&
            !mbar_wait(&empty[st], static_cast<uint32_t>((ks / Cfg::kStages) - 1) & 1u, p.status))
          break;
        const int nkb = static_cast<int>(min64(Cfg::kKbPerStage, (p.K - static_cast<int64_t>(ks) * Cfg::kStageK) / 64));
        const uint32_t sf_bytes = static_cast<uint32_t>(nkb) * 512u;
        mbar_arrive_expect_tx(&full[st], Cfg::kABytes + Cfg::kBBytes + sf_bytes * (1 + BN / 128));
        tma_load_2d(sA + st * Cfg::kABytes, &map_a, &full[st], ks * 128, static_cast<int32_t>(m0));
        tma_load_2d(sB + st * Cfg::kBBytes, &map_b, &full[st], ks * 128, static_cast<int32_t>(n0));
        const uint64_t a_atom = (static_cast<uint64_t>(m0 / 128) * kb64 + static_cast<uint64_t>(ks) * Cfg::kKbPerStage) * 512u;
        bulk_load(sSfa + st * Cfg::kSfaBytes, p.sfa + a_atom, sf_bytes, &full[st]);
#pragma unroll
        for (int g = 0; g < BN / 128; ++g) {
          const uint64_t b_atom = (static_cast<uint64_t>(n0 / 128 + g) * kb64 + static_cast<uint64_t>(ks) * Cfg::kKbPerStage) * 512u;
          bulk_load(sSfb + st * Cfg::kSfbBytes + g * Cfg::kKbPerStage * 512, p.sfb + b_atom, sf_bytes, &full[st]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      for (int ks = 0; ks < n_stages; ++ks) {
        const int st = ks % Cfg::kStages;
        if (!mbar_wait(&full[st], static_cast<uint32_t>(ks / Cfg::kStages) & 1u, p.status)) break;
        tc_fence_after();
        const int nkb = static_cast<int>(min64(Cfg::kKbPerStage, (p.K - static_cast<int64_t>(ks) * Cfg::kStageK) / 64));
        const uint32_t buf = static_cast<uint32_t>(ks & 1);
        const uint32_t sfa_t = tmem + Cfg::kSfaCol + buf * (Cfg::kKbPerStage * 4);
        const uint32_t sfb_t = tmem + Cfg::kSfbCol + buf * (Cfg::kKbPerStage * Cfg::kSfbColsPerKb);
        for (int kb = 0; kb < nkb; ++kb) {
          tc_cp_32x128b_warpx4(sfa_t + 4 * kb,
                               smem_desc(smem_u32(sSfa + st * Cfg::kSfaBytes + kb * 512), 0, 128, kLayoutSwizzleNone));
#pragma unroll
          for (int g = 0; g < BN / 128; ++g)
            tc_cp_32x128b_warpx4(sfb_t + Cfg::kSfbColsPerKb * kb + 4 * g,
                                 smem_desc(smem_u32(sSfb + st * Cfg::kSfbBytes + g * Cfg::kKbPerStage * 512 + kb * 512),
                                           0, 128, kLayoutSwizzleNone));
        }
        const uint32_t a_base = smem_u32(sA + st * Cfg::kABytes);
        const uint32_t b_base = smem_u32(sB + st * Cfg::kBBytes);
        for (int kb = 0; kb < nkb; ++kb) {
          const uint64_t adesc = smem_desc(a_base + kb * 32, 16, 1024, kLayoutSwizzle128B);
          const uint64_t bdesc = smem_desc(b_base + kb * 32, 16, 1024, kLayoutSwizzle128B);
          mma_nvf4(tmem, adesc, bdesc, Cfg::kIdesc, sfa_t + 4 * kb, sfb_t + Cfg::kSfbColsPerKb * kb,
                   (ks > 0 || kb > 0) ? 1u : 0u);
        }
        tc_commit(&empty[st]);
      }
      tc_commit(acc_bar);
    }
  } else {
    // ---------------- epilogue ----------------
    const int q = warp & 3;
    const int64_t row = m0 + 32 * q + lane;
    // warp-uniform, so that the .sync.aligned tensor-memory loads below are
    // executed by all 32 lanes or by none
    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_bar, 0u, p.status) ? 1 : 0) != 0;
    tc_fence_after();
    if (ok) {
      const float alpha = __ldg(p.gdec_a) * __ldg(p.gdec_b);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int64_t col = n0 + 32 * c;
        if (col >= p.N) break;
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(32 * c), r);
        tmem_ld_wait();
        float b[32];
        if (p.bias) {
          const float4* bp = reinterpret_cast<const float4*>(p.bias + col);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 t = __ldg(bp + v);
            b[4 * v] = t.x; b[4 * v + 1] = t.y; b[4 * v + 2] = t.z; b[4 * v + 3] = t.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) b[j] = 0.0f;
        }
        if (row < p.M) {
          if (kBf16Out) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float y0 = fmaf(alpha, __uint_as_float(r[2 * j]), b[2 * j]);
              const float y1 = fmaf(alpha, __uint_as_float(r[2 * j + 1]), b[2 * j + 1]);
              const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
              w[j] = *reinterpret_cast<const uint32_t*>(&h);
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.Y) + row * p.N + col);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.Y) + row * p.N + col);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(fmaf(alpha, __uint_as_float(r[4 * v]), b[4 * v]),
                                   fmaf(alpha, __uint_as_float(r[4 * v + 1]), b[4 * v + 1]),
                                   fmaf(alpha, __uint_as_float(r[4 * v + 2]), b[4 * v + 2]),
                                   fmaf(alpha, __uint_as_float(r[4 * v + 3]), b[4 * v + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

template <int BN, bool kBf16Out>
static cudaError_t launch_gemm_t(const CUtensorMap& ma, const CUtensorMap& mb, const GemmParams& p,
                                 cudaStream_t s, bool pdl) {
  using Cfg = GemmCfg<BN>;
  auto kern = gemm_nvfp4_kernel<BN, kBf16Out>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((p.N + BN - 1) / BN), static_cast<unsigned>((p.M + Cfg::kBM - 1) / Cfg::kBM));
  return launch_ex(kern, grid, dim3(192), Cfg::kSmemBytes, s, pdl, ma, mb, p);
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, bool pdl) {
  constexpr int BN = 128;
  CUtensorMap ma, mb;
  if (!make_tensor_map_2d(&ma, a.a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(a.M),
                          static_cast<uint64_t>(a.K / 2), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_tensor_map_2d(&mb, a.b_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(a.N),
                          static_cast<uint64_t>(a.K / 2), BN, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  GemmParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.sfa = a.a_scales;
  p.sfb = a.b_scales;
  p.gdec_a = a.a_gdec;
  p.gdec_b = a.b_gdec;
  p.bias = a.bias;
  p.Y = a.Y;
  p.status = a.status;
  return a.yt == AVR_BF16 ? launch_gemm_t<BN, true>(ma, mb, p, s, pdl)
                          : launch_gemm_t<BN, false>(ma, mb, p, s, pdl);
}

}  // namespace avr
