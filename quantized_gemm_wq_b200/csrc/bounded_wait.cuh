// bounded_wait.cuh -- the library's one definition of a bounded mbarrier wait.
//
// Every pipeline wait of every kernel is bounded in time, so a pipeline that
// never completes (a copy that never lands, a lost arrival) cannot hold the
// GPU: the wait gives up after kPipeWaitNs, raises the kernel's device flag
// (read and cleared by wq_last_device_error) and the kernel drains the copies
// it has in flight and returns.  Exit-path drains use their own limit,
// kDrainNs, which is never shortened: every issued copy must land before its
// CTA exits.  WQ_PIPE_WAIT_NS may be defined at build time (a test build uses
// 0 so that every wait that is not already complete expires).
#pragma once
#include <cstdint>

#ifndef WQ_PIPE_WAIT_NS
#define WQ_PIPE_WAIT_NS 1000000000ull   // 1 s: far beyond any healthy wait
#endif

namespace wq {
namespace bw {

constexpr uint64_t kPipeWaitNs = WQ_PIPE_WAIT_NS;
constexpr uint64_t kDrainNs = 200000000ull;        // 0.2 s per in-flight stage on exit paths

static __device__ __forceinline__ bool try_parity(uint32_t bar, uint32_t parity) {
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

static __device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of the mbarrier at shared address `bar`.  Returns
// true once it completed; false when the CTA's abort word (optional) was set
// by another wait, or when kPipeWaitNs passed: then the abort word and the
// kernel's device flag are raised.
static __device__ __noinline__ bool pipe_wait(uint32_t bar, uint32_t parity, unsigned int* flag,
                                              volatile uint32_t* abort) {
  if (try_parity(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (uint32_t i = 1;; ++i) {
    if (try_parity(bar, parity)) return true;
    if ((i & 15u) == 0) {
      if (abort && *abort) return false;
      if (now_ns() - t0 > kPipeWaitNs) {
        if (abort) *abort = 1u;
        atomicExch(flag, 1u);
        return false;
      }
    }
  }
}

// Exit-path wait for copies or MMAs still in flight: ignores the abort word;
// gives up (raising the flag) only after kDrainNs.
static __device__ __noinline__ bool drain_wait(uint32_t bar, uint32_t parity, unsigned int* flag) {
  const uint64_t t0 = now_ns();
  while (!try_parity(bar, parity)) {
    if (now_ns() - t0 > kDrainNs) {
      atomicExch(flag, 1u);
      return false;
    }
  }
  return true;
}

}  // namespace bw
}  // namespace wq
