// Device-side building blocks shared by the kernels of libaveris: status
// reporting, bounded mbarrier waits, TMA and bulk copies, tcgen05 (TMEM,
// block-scaled MMA, scale-factor copies), Philox4x32-10 and the NVFP4
// conversions.  sm_100a only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/averis.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libaveris is built for sm_100a only"
#endif

namespace avr {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// ---------------------------------------------------------------------------
// status word (first 4 bytes of every workspace): first error wins
// ---------------------------------------------------------------------------
__device__ __forceinline__ void raise_status(uint32_t* status, uint32_t code) {
  if (status) atomicCAS(status, 0u, code);
}

// atomicInc (wrapping to 0 after `limit`) with acquire-release semantics at GPU
// scope; returns the old value.
__device__ __forceinline__ uint32_t ticket_inc_acq_rel(uint32_t* addr, uint32_t limit) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(limit) : "memory");
  return old;
}

// Wall-clock bound for every spin-wait: after this many nanoseconds of
// waiting the kernel records AVR_ERR_DEVICE_TIMEOUT and gives up.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Grid-wide barrier for a grid whose CTAs are all resident at once.  Thread 0
// of each CTA arrives on *count (acquire-release at GPU scope, after a CTA
// barrier, so it publishes every thread's prior writes); the last of n
// arrivals resets *count and advances *gen, which the others poll, reading
// the clock after every poll, for at most limit_ns (0: kWaitLimitNs).  *count
// is back at 0 after every completed barrier.  Returns false (and records
// AVR_ERR_DEVICE_TIMEOUT) if the other CTAs did not come in time; *count is
// then left part-way and the caller's status block must be cleared before
// the next barrier.
__device__ __forceinline__ bool grid_barrier(uint32_t* count, uint32_t* gen, uint32_t n, uint32_t* status,
                                             uint64_t limit_ns) {
  const uint64_t limit = limit_ns != 0 ? limit_ns : kWaitLimitNs;
  __shared__ uint32_t s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t ok = 1u, g0, old;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g0) : "l"(gen) : "memory");
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(count) : "memory");
    if (old == n - 1u) {
      asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(count) : "memory");
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(gen) : "memory");
    } else {
      const uint64_t t0 = globaltimer_ns();
      uint32_t g;
      for (;;) {
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g) : "l"(gen) : "memory");
        if (g != g0) break;
        if (globaltimer_ns() - t0 > limit) {   // one clock read per poll: a poll is an L2 round trip
          raise_status(status, AVR_ERR_DEVICE_TIMEOUT);
          ok = 0u;
          break;
        }
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0u;
}

// Wait for the phase with the given parity to complete.  Returns false (and
// records a timeout in *status) if it has not completed within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (((++spins) & 255u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) {
      raise_status(status, AVR_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Like mbar_wait, but polling with test_wait, which never suspends the
// thread: for hand-offs on the critical path, where waking from a suspended
// try_wait costs a few hundred nanoseconds.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_poll(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (!mbar_test(bar, parity)) {
    if (((++spins) & 1023u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) {
      raise_status(status, AVR_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Polling with a short sleep between polls, for waiters off the critical
// path: a warp spinning on test_wait keeps the shared-memory pipe busy, and
// the MMA issuer's own barrier and tcgen05 operations queue behind it.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity)) {
    __nanosleep(64);
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      raise_status(status, AVR_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// TMA (tensor) loads and bulk copies, global -> shared, completing on an
// mbarrier.  No cluster multicast anywhere in this library.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// TMA tensor store shared -> global (bulk-group completion) and its waits.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_group_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Named barrier over `count` threads; returns the OR of `pred` over them.
__device__ __forceinline__ bool named_barrier_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r) : "r"(pred ? 1u : 0u), "r"(id), "r"(count) : "memory");
  return r != 0;
}
__device__ __forceinline__ void named_barrier(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------
// programmatic dependent launch
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_allow_next_grid() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, block-scaled MMA, scale copies, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on *bar when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with per-16-element E4M3 scales of A and B
// taken from tensor memory; E2M1 operands, fp32 accumulator.
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
      "}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem)
      : "memory");
}

// Copy a 32-row x 16-byte block from shared memory into tensor memory,
// replicated into all four 32-lane sub-partitions (4 columns of 32 bits).
__device__ __forceinline__ void tc_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane
// (32 * (warp % 4) + t) of the addressed columns.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start address, leading
// and stride byte offsets (16-byte units), descriptor version 1, layout type.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}
constexpr uint32_t kLayoutSwizzleNone = 0;
constexpr uint32_t kLayoutSwizzle128B = 2;
constexpr uint32_t kLayoutSwizzle64B = 4;

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    // one 32 x 32 -> 64-bit multiply gives both halves of each product
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
    const uint32_t lo0 = static_cast<uint32_t>(p0), hi0 = static_cast<uint32_t>(p0 >> 32);
    const uint32_t lo1 = static_cast<uint32_t>(p1), hi1 = static_cast<uint32_t>(p1 >> 32);
    c = make_uint4(hi1 ^ c.y ^ (k0 + static_cast<uint32_t>(r) * 0x9E3779B9u), lo1,
                   hi0 ^ c.w ^ (k1 + static_cast<uint32_t>(r) * 0xBB67AE85u), lo0);
  }
  return c;
}

// Philox4x32-10 with its round keys computed once: a thread that draws many
// blocks under one (seed, tag) keeps k0 + r W0 and k1 + r W1 in registers.
struct PhiloxKeys {
  uint32_t k0[10], k1[10];
};
__device__ __forceinline__ PhiloxKeys philox_keys(uint64_t seed) {
  PhiloxKeys k;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    k.k0[r] = static_cast<uint32_t>(seed) + static_cast<uint32_t>(r) * 0x9E3779B9u;
    k.k1[r] = static_cast<uint32_t>(seed >> 32) + static_cast<uint32_t>(r) * 0xBB67AE85u;
  }
  return k;
}
// counter (lo32 g, hi32 g, tag, 0)
__device__ __forceinline__ uint4 philox_keyed(uint64_t g, uint32_t tag, const PhiloxKeys& k) {
  uint4 c = make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), tag, 0u);
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k.k0[r], static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k.k1[r], static_cast<uint32_t>(p0));
  }
  return c;
}

// The 128 random bits of the 16 elements e with floor(e/16) = blk (word k
// for elements 16 blk + 4k .. 16 blk + 4k + 3): counter (lo32(offset+blk),
// hi32(offset+blk), tag, 0), key (lo32(seed), hi32(seed)).
__device__ __forceinline__ uint4 philox_block(uint64_t seed, uint64_t offset, uint32_t tag,
                                              uint64_t blk) {
  const uint64_t g = offset + blk;
  return philox4x32_10(make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), tag, 0u),
                       static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
}

// ---------------------------------------------------------------------------
// NVFP4 arithmetic
// ---------------------------------------------------------------------------
constexpr float kFp4Fp8Product = 2688.0f;   // 6 (E2M1 max) * 448 (E4M3 max)

struct TensorScale {
  float g_enc, g_dec;
};
__device__ __forceinline__ TensorScale tensor_scale(float amax) {
  TensorScale t;
  if (amax == 0.0f) {
    t.g_enc = 1.0f;
    t.g_dec = 1.0f;
  } else {
    t.g_enc = fminf(__fdiv_rn(kFp4Fp8Product, amax), 3.402823466e38f);
    t.g_dec = __fdiv_rn(amax, kFp4Fp8Product);
  }
  return t;
}

// fp32 -> unsigned E4M3 code, round to nearest even, saturating to 448.
__device__ __forceinline__ uint32_t e4m3_rn_satfinite(float s) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(0.0f), "f"(s));
  return static_cast<uint32_t>(d & 0xFFu);
}

// E4M3 code (0..0x7E) -> its exact fp32 value.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
  return e == 0u ? static_cast<float>(m) * 0.001953125f
                 : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Two fp32 -> one byte of two E2M1 codes (lo in bits 0..3), nearest even,
// saturating; the hardware keeps the sign of values that round to zero.
__device__ __forceinline__ uint32_t e2m1x2_rn(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Stochastic rounding of four fp32 values to E2M1 codes (element 0 in bits
// 0..3 of the result) with one 32-bit random word, by the hardware convert.
// For each element the fraction of |y| inside its E2M1 interval, truncated to
// 16 bits, is added to a 16-bit random value and a carry rounds up (|y| > 6
// saturates to 6; the sign is kept).  The random values the instruction takes
// from the word (bytes b0..b3): W = b2:b0 for element 0, bitrev16(W) for
// element 1, V = b3:b1 for element 2 and bitrev16(V) for element 3.  The
// instruction puts its first operand in the top nibble, so the elements are
// passed in reverse order.
__device__ __forceinline__ uint32_t e2m1x4_sr(float e0, float e1, float e2, float e3, uint32_t rbits) {
  uint16_t r;
  asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %3, %4}, %5;"
      : "=h"(r) : "f"(e3), "f"(e2), "f"(e1), "f"(e0), "r"(rbits));
  return static_cast<uint32_t>(r);
}

// E2M1 code -> value.  Codes 2..7 are normal: 2^((c>>1) - 1) * (1 + (c&1)/2).
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t m = c & 7u;
  const float v = m >= 2u ? __uint_as_float(((126u + (m >> 1)) << 23) | ((m & 1u) << 22))
                          : (m == 1u ? 0.5f : 0.0f);
  return (c & 8u) ? -v : v;
}

// Byte offset of the scale of (row r, 16-element block column c) in the
// tcgen05 128x4 atom layout (512-byte atoms, row-group major).
__device__ __forceinline__ uint64_t scale_offset(uint64_t r, uint32_t c, uint32_t n_kb64) {
  return ((r >> 7) * n_kb64 + (c >> 2)) * 512ull + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (c & 3u);
}

// fl(a - c) for the two bf16 halves of w (element 2i in the low half) and
// fp32 c: the mixed-precision subtract widens the bf16 exactly, then rounds
// once, i.e. the same bits as __fsub_rn(float(a), c).
__device__ __forceinline__ void sub_bf16x2_f32(uint32_t w, float c_lo, float c_hi, float& d_lo, float& d_hi) {
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "sub.rn.f32.bf16 %0, l, %3;\n\t"
      "sub.rn.f32.bf16 %1, h, %4;\n\t}"
      : "=f"(d_lo), "=f"(d_hi) : "r"(w), "f"(c_lo), "f"(c_hi));
}

// max(a, b, c) in one three-input instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (a0 * b, a1 * b) rounded to nearest, as one packed f32x2 multiply
__device__ __forceinline__ void fmul2(float a0, float a1, float b, float& d0, float& d1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %4};\n\t"
      "mul.rn.f32x2 d, a, b;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b));
}


}  // namespace avr
