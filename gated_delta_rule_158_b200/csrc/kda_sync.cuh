// kda_sync.cuh -- bounded waits used by libkda's kernels.
//
// No kernel in libkda waits without a limit.  A wait polls its condition;
// once it has polled kFastPolls times it starts reading the global
// nanosecond timer and gives up after a time limit, recording
// KDA_ERR_TIMEOUT in the workspace status word (read by
// kda_get_device_status) instead of trapping, so the context stays usable.
#pragma once

#include <stdint.h>

#include "kda_internal.cuh"

namespace kda {

constexpr long long kWaitLimitNs = 2000000000LL;  // 2 s: far above any real wait
constexpr int kFastPolls = 1 << 12;
constexpr uint32_t kSuspendNs = 1000;  // longest single suspension in a bounded wait

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits until *flag != 0.  Returns true on success, false on timeout (and
// records the timeout with `detail`).
__device__ __forceinline__ bool bounded_flag_wait(const volatile int32_t* flag,
                                                  long long limit_ns, StatusBlock* sb,
                                                  int32_t detail) {
  for (int i = 0; i < kFastPolls; ++i)
    if (*flag != 0) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (*flag != 0) return true;
    if ((long long)(global_ns() - t0) > limit_ns) {
      record_status(sb, KDA_ERR_TIMEOUT, detail);
      return false;
    }
    __nanosleep(256);
  }
}

// mbarrier helpers (shared::cta addresses as 32-bit integers)
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
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
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended for up to hint_ns until the
// phase completes (it is woken as soon as it does), instead of spinning.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity,
                                                   uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Non-blocking: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Barrier `id` over `count` threads that also ORs a predicate across them,
// so every participant gets the same answer.
__device__ __forceinline__ bool bar_red_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Waits for the phase with the given parity to complete.  On timeout sets
// *abort (shared), records the status and returns false.  The first
// try_wait (which may itself suspend the thread for a while) is inline; the
// polling loop is an out-of-line call, so the many call sites of a kernel
// stay small in the instruction cache.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity,
                                                   volatile int* abort_flag, StatusBlock* sb,
                                                   int32_t detail, uint32_t hint_ns,
                                                   long long limit_ns) {
  // suspended waits of up to kSuspendNs each: no issue slots spent while waiting
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, hint_ns)) return true;
    if (*abort_flag) return false;
    if ((long long)(global_ns() - t0) > limit_ns) {
      *abort_flag = 1;
      record_status(sb, KDA_ERR_TIMEOUT, detail);
      return false;
    }
  }
}

// limit_ns bounds the wait (kWaitLimitNs unless a caller lowers it to
// exercise the timeout path).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag, StatusBlock* sb,
                                                  int32_t detail,
                                                  long long limit_ns = kWaitLimitNs,
                                                  uint32_t hint_ns = kSuspendNs) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort_flag, sb, detail, hint_ns, limit_ns);
}

// Abort-path drain: waits (up to the time limit, whatever the abort flag says)
// for asynchronous work this CTA already issued to land before its shared
// memory or TMEM is released.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  for (int i = 0; i < kFastPolls; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((long long)(global_ns() - t0) > kWaitLimitNs) return false;
  }
}

}  // namespace kda
