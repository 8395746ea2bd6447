// mbar.cuh -- shared-memory mbarriers with bounded waits, for the kernels
// whose roles hand work to one another inside a CTA.
//
// Every wait is bounded (about 2 s of %globaltimer by default); a wait that
// runs out records a code in the device error word and raises a CTA-wide abort
// flag, so a fault in a pipeline can never hang the GPU.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace b200conv {
namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: true when the phase completed; false after limit_ns of
// %globaltimer or when another role raised the abort flag.  The inlined form
// is for kernels that repartition registers between roles (setmaxnreg), which
// cannot call out of line.
__device__ __forceinline__ bool mbar_wait_inl(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err,
                                              int code, unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = gtimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*abort_flag) return false;
      if (gtimer() - t0 > limit_ns) {
        *abort_flag = 1;
        if (code) atomicCAS(err, 0, code);
        return false;
      }
    }
  }
}
// Bounded wait that sleeps between polls (32 ns doubling to 2 us), for roles
// that may wait a long time beside warps that need the issue slots.
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err,
                                                int code, unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = gtimer();
  unsigned ns = 32;
  for (;;) {
    __nanosleep(ns);
    if (mbar_try(bar, parity)) return true;
    if (ns < 2048) ns *= 2;
    if (*abort_flag) return false;
    if (gtimer() - t0 > limit_ns) {
      *abort_flag = 1;
      if (code) atomicCAS(err, 0, code);
      return false;
    }
  }
}
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err, int code,
                                       unsigned long long limit_ns = kWaitLimitNs) {
  return mbar_wait_inl(bar, parity, abort_flag, err, code, limit_ns);
}

}  // namespace
}  // namespace b200conv
