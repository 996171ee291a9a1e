// Device-side helpers shared by the quantize and decode kernels (sm_100a only).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kivi.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace kivi {

constexpr int kHeadDim = 128;

// ---- fp16 <-> fp32 / fp64 -------------------------------------------------------------------
__device__ __forceinline__ float h2f(uint16_t bits) { return __half2float(__ushort_as_half(bits)); }

// binary16 of a double, round to nearest even, one rounding (PTX cvt.rn.f16.f64).
__device__ __forceinline__ uint16_t f64_to_h_rn(double x) {
  uint16_t r;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(r) : "d"(x));
  return r;
}

// ---- integer dot products on bytes ----------------------------------------------------------
// d = sum_i a.byte[i] * b.byte[i] + c with a unsigned and b unsigned / signed bytes.
__device__ __forceinline__ int dp4a_uu(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ---- shared-memory addresses, mbarriers and 1-D bulk copies ----------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// try_wait that may suspend the thread for up to `hint_ns` while the phase is incomplete (the
// thread resumes as soon as it completes), so a waiting warp does not spin through issue slots.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

#ifndef KIVI_WAIT_HINT_NS
#define KIVI_WAIT_HINT_NS 20000u  // longest suspension of one try of a bounded wait
#endif

// Bounded wait on an mbarrier phase: gives up after `limit_ns` of wall time (checked every 16
// tries, each suspending for at most KIVI_WAIT_HINT_NS) and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 0;; ++spin) {
    if (mbar_try_wait_hint(bar, parity, KIVI_WAIT_HINT_NS)) return true;
    if ((spin & 15u) == 15u && global_timer_ns() - t0 > limit_ns) return false;
  }
}

// Global -> shared bulk copy (TMA, no tensor map, no multicast), completion counted in bytes on
// `bar`.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before later async-proxy
// (bulk copy) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void report_status(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// ---- debug build (nvcc -DKIVI_DEBUG): device-side bounds checks ------------------------------
// dbg_check(cond, status) is true in a release build (the condition is not evaluated at run time).
// In a debug build a false condition records KIVI_ERR_INTERNAL in `status` (if given) and in the
// translation unit's own debug word (read and cleared by kivi_debug_status), without a trap; the
// caller then skips the access it guards.
#ifdef KIVI_DEBUG
constexpr bool kDebugBuild = true;
static __device__ int32_t g_debug_status = 0;  // one per translation unit
#else
constexpr bool kDebugBuild = false;
#endif

__device__ __forceinline__ bool dbg_check(bool cond, int32_t* status = nullptr) {
#ifdef KIVI_DEBUG
  if (!cond) {
    report_status(status, KIVI_ERR_INTERNAL);
    atomicCAS(&g_debug_status, 0, KIVI_ERR_INTERNAL);
    return false;
  }
#endif
  (void)cond;
  (void)status;
  return true;
}

// Host side: reads and clears this translation unit's debug word (0 in a release build).
static inline cudaError_t take_debug_status_tu(int32_t* out) {
#ifdef KIVI_DEBUG
  cudaError_t e = cudaMemcpyFromSymbol(out, g_debug_status, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  const int32_t zero = 0;
  return cudaMemcpyToSymbol(g_debug_status, &zero, sizeof(int32_t));
#else
  *out = 0;
  return cudaSuccess;
#endif
}

}  // namespace kivi
