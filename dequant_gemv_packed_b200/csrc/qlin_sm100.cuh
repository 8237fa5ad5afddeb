// Thin wrappers over the sm_100a PTX used by the qlin kernels: mbarriers,
// bulk asynchronous copies (global -> shared), named barriers, grid-dependency
// control, and the mixed-precision fp16 x fp16 + fp32 fused multiply-add.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace qlin {

// Iteration bound of every spin on an mbarrier (try_wait itself suspends for a
// while per iteration); on expiry the waiter records an error and goes on.
constexpr uint32_t kSpinLimit = 1u << 22;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Makes mbarrier initialisation visible to the async proxy and other threads.
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Sleep bound of one try_wait: the waiting warp is suspended (issues nothing)
// until the phase completes or this many nanoseconds pass.
constexpr uint32_t kSuspendHintNs = 200000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Longest wait for one barrier phase before the waiter gives up.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Bounded wait for the phase with the given parity; false if it did not come
// within kWaitLimitNs, or as soon as `abort_word` (a sticky device error word)
// is nonzero, so that one failed wait ends every other wait quickly.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const volatile unsigned* abort_word) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 0; n < kSpinLimit; ++n) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_word) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return false;
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_wait for a phase that has usually completed already: a few cheap
// non-blocking tests first (no suspension when the data is there), then the
// bounded blocking wait.
__device__ __forceinline__ bool mbar_wait_poll(uint64_t* bar, uint32_t parity, const volatile unsigned* abort_word) {
#pragma unroll 1
  for (int i = 0; i < 4; ++i)
    if (mbar_test_wait(bar, parity)) return true;
  return mbar_wait(bar, parity, abort_word);
}

// Bulk copy of `bytes` (multiple of 16; both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing on `bar` (tx bytes).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Barrier among the first `threads` threads of the CTA (id 1..15).
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's memory, and
// allow the next grid to start launching.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint16_t lo16(uint32_t v) {
  uint16_t lo;
  asm("{\n\t.reg .b16 t;\n\tmov.b32 {%0, t}, %1;\n\t}" : "=h"(lo) : "r"(v));
  return lo;
}

__device__ __forceinline__ uint16_t hi16(uint32_t v) {
  uint16_t hi;
  asm("{\n\t.reg .b16 t;\n\tmov.b32 {t, %0}, %1;\n\t}" : "=h"(hi) : "r"(v));
  return hi;
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_addr(p)));
  return v;
}

}  // namespace qlin
