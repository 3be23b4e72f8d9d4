// mbarrier.cuh -- shared-memory barrier and bulk-copy helpers of the kernels
// that stream through TMA (cp.async.bulk) rings.  Every wait is bounded in
// time: on time-out the waiter raises QSA_DEV_TIMEOUT in the caller's status
// word and sets the CTA's abort flag, and the other roles stop at their next
// wait, so no kernel of this library can hang its GPU.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {
namespace mbar {

constexpr unsigned long long kWaitLimitNs = 200ull * 1000 * 1000;  // 200 ms per wait

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes) : "memory");
}
// One try of a phase wait.  The thread is suspended until the phase completes
// or the hint (ns) runs out, so waiting warps leave the issue slots to the
// warps that have work; without a hint the wait loops spin hot.
constexpr uint32_t kSuspendHintNs = 10000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for the phase with the given parity; false (and the abort flag
// set, QSA_DEV_TIMEOUT raised) when it does not come.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status, unsigned long long limit_ns = kWaitLimitNs) {
  const unsigned long long t0 = gtimer();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(b, parity)) return true;
    if (*abort_flag) return false;
    if ((i & 15u) == 15u && gtimer() - t0 > limit_ns) break;
  }
  *abort_flag = 1;
  flag(status, QSA_DEV_TIMEOUT);
  return false;
}
// After an abort: wait, with its own bound and whatever the abort flag says,
// for a phase this thread armed, so that no copy or MMA still writes shared
// memory or TMEM when the CTA leaves.
__device__ __forceinline__ bool mbar_drain(uint64_t* b, uint32_t parity) {
  const unsigned long long t0 = gtimer();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(b, parity)) return true;
    if ((i & 15u) == 15u && gtimer() - t0 > kWaitLimitNs) return false;
  }
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size a multiple
// of 16), completing `bytes` of the transaction count of `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(saddr(dst)), "l"(src), "r"(bytes), "r"(saddr(bar))
      : "memory");
}

}  // namespace mbar
}  // namespace qsa
