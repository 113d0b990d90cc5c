// dsa_common.cuh — device helpers shared by the indexer kernels (sm_100a).
//
// PTX wrappers for mbarriers, TMA tile loads and tcgen05 (TMEM allocation,
// MMA issue, commit, TMEM loads), order-preserving float keys, and the
// bounded-wait error protocol: a wait on an mbarrier sleeps in the hardware
// until the phase completes and gives up after a time budget, records
// DSA_ERR_TIMEOUT in the workspace status word and raises a per-CTA abort
// flag so that all roles leave their loops.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "dsa_index.h"

namespace dsa {

// ----------------------------------------------------------------------------
// workspace header: status word + scratch counters (first 256 bytes)
// ----------------------------------------------------------------------------
struct WsHeader {
  int status;      // first device-side error (0 = none)
  int info;        // where it happened
  int offsets_ok;  // decode groups: 1 when the call's offsets passed their device check
  int pad[61];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

__device__ __forceinline__ void report_error(int* status, int code, int info) {
  if (atomicCAS(status, 0, code) == 0) status[1] = info;
}

// Debug bounds checks, compiled in by -DDSA_DEBUG_BOUNDS=1 (the library's
// debug build, libdsa_index_debug.so): an index a kernel is about to use is
// checked against the extent of its buffer; a failing check records
// DSA_ERR_INTERNAL with info 100 + site in the status word and the access is
// skipped.  In the normal build in_bounds is constant true and costs nothing.
#ifndef DSA_DEBUG_BOUNDS
#define DSA_DEBUG_BOUNDS 0
#endif
__device__ __forceinline__ bool in_bounds(bool ok, int* status, int site) {
  if constexpr (DSA_DEBUG_BOUNDS != 0) {
    if (!ok) report_error(status, DSA_ERR_INTERNAL, 100 + site);
    return ok;
  } else {
    (void)status;
    (void)site;
    return true;
  }
}

// A call whose device offsets failed their check (offsets_ok == 0) runs none
// of its later kernels' work; null means the kernel checks its own.
__device__ __forceinline__ bool offsets_bad(const int* ok) {
  return ok != nullptr && *(volatile const int*)ok == 0;
}

// ----------------------------------------------------------------------------
// order-preserving float <-> uint32 and the coarse score bins
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t f2o(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 1024 bins of 1/16 binade over positive scores in [2^-40, 2^24); everything
// <= 2^-40 (zero and negatives included) is bin 0, everything >= 2^24 is
// bin 1023.  Monotone non-decreasing in the score.
constexpr int kBins = 1024;
constexpr int kBinExpLo = 127 - 40;
__device__ __forceinline__ int score_bin(float f) {
  int b = (int)__float_as_uint(f);
  if (b <= 0) return 0;                      // +0 and every negative value
  int key = (b >> 19) - kBinExpLo * 16;      // exponent(8) | top 4 mantissa bits
  return key < 0 ? 0 : (key > kBins - 1 ? kBins - 1 : key);
}

// The smallest score whose bin is b: for every finite score f,
// score_bin(f) >= b  <=>  f >= bin_floor(b).  (Bin 0 holds every score up to
// 2^-40, negatives included, so its floor is -inf; inside bins 1..1023 the
// bin is the score's top 13 bits offset by the exponent floor, and positive
// floats order like their bits.)
__device__ __forceinline__ float bin_floor(int b) {
  return b <= 0 ? __int_as_float(0xff800000) : __uint_as_float((uint32_t)(b + kBinExpLo * 16) << 19);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// 64-bit selection key: larger = better (higher score, then lower index).
__device__ __forceinline__ uint64_t sel_key(uint2 e) {
  return ((uint64_t)f2o(__uint_as_float(e.x)) << 32) | (uint64_t)(~e.y);
}

// ----------------------------------------------------------------------------
// shared-memory addressing, barriers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Longest single suspension of a waiting thread when the wait is far off the
// critical path (the TMA producer, drains): try_wait sleeps until the phase
// completes or this many nanoseconds pass, so the warp takes no issue slots
// meanwhile.  Waits on the critical path use the plain form, whose short
// hardware suspension wakes sooner.
constexpr uint32_t kSuspendNs = 20000;

template <bool kLongSleep>
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  if constexpr (kLongSleep) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendNs)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
  }
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Time budget of one bounded wait: far beyond any legitimate wait of these
// kernels (microseconds), short enough that a failure returns promptly.
constexpr uint64_t kWaitNs = 2000000000ull;

// Returns false when the wait gave up (abort raised elsewhere, or the
// `budget_ns` ran out — then the status word and the abort flag are set).
template <bool kLongSleep = false>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, int where, uint64_t budget_ns = kWaitNs) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait<kLongSleep>(a, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (*abort_flag) return false;
    if (mbar_try_wait<kLongSleep>(a, parity)) return true;
    if (global_ns() - t0 > budget_ns) {
      report_error(status, DSA_ERR_TIMEOUT, where);
      *abort_flag = 1;
      return false;
    }
  }
}

// The wait for work this CTA has already issued (a TMA copy, an MMA) before
// it leaves: it ignores the abort flag, since a copy in flight must land
// before the CTA's shared memory is released, and keeps the full budget.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, int* status, int where) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait<true>(a, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait<true>(a, parity)) return true;
    if (global_ns() - t0 > kWaitNs) {
      report_error(status, DSA_ERR_TIMEOUT, where);
      return false;
    }
  }
}

// ----------------------------------------------------------------------------
// TMA (tiled, no multicast)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// L2 eviction policies (cache hints for loads and stores): data read once
// (queries, outputs, streamed decode keys) goes first, data read again (the
// prefill keys, the candidate lists until the final select) stays.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// A 2-D TMA tile load with an L2 eviction policy.
__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void st_global_hint(uint2* p, uint2 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v2.u32 [%0], {%1, %2}, %3;" ::"l"(p), "r"(v.x), "r"(v.y), "l"(pol)
               : "memory");
}

__device__ __forceinline__ uint2 ld_global_hint(const uint2* p, uint64_t pol) {
  uint2 v;
  asm volatile("ld.global.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;" : "=r"(v.x), "=r"(v.y) : "l"(p), "l"(pol));
  return v;
}

// Brings a tile into L2 ahead of its load (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05
// ----------------------------------------------------------------------------
// Shared-memory matrix descriptor, K-major operand in the 128-byte swizzled
// layout that a TMA box of 64 bf16 x R rows with SWIZZLE_128B produces:
// rows of 128 B, 8-row groups 1024 B apart (stride byte offset), version 1,
// layout type 2 = SWIZZLE_128B.  The leading byte offset is unused for this
// layout (set to 1).  Tiles start 1024-byte aligned (base offset 0); moving
// along K inside the 128-byte row is a plain start-address advance.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B, fp32 accumulate,
// both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive fp32 columns per warp; thread i gets lane
// (taddr.lane + i), registers r[j] = column (taddr.col + j).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// The same for 16 consecutive columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ----------------------------------------------------------------------------
// input element loads (exact conversion to fp32)
// ----------------------------------------------------------------------------
__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
  return __half2float(*reinterpret_cast<__half*>(&h));
}

}  // namespace dsa
