// selftest.cu -- a self-test of the bounded mbarrier wait (mbarrier.cuh) that
// the TMA / tcgen05 kernels use for every phase: the wait runs out on a
// barrier that nothing arrives at, sets the CTA's abort flag and raises
// QSA_DEV_TIMEOUT; a second waiter is released by the abort flag; a bulk copy
// put in flight before the wait is drained before the CTA exits.  Nothing in
// it faults, traps or spins without a bound.
#include "qsa_internal.cuh"
#include "mbarrier.cuh"

namespace qsa {
namespace {

using namespace mbar;

// warp 1's own limit exceeds warp 0's by this much: released well before it,
// it can only have been the abort flag
constexpr unsigned long long kWarp1ExtraNs = 1000ull * 1000 * 1000;

// the bulk copy's source: 16 bytes with a known pattern, 16-byte aligned
__device__ __align__(16) uint32_t g_selftest_src[4] = {0x51a7e570u, 0x0badf00du, 0x7e57ab1eu, 0x00c0ffeeu};

__global__ void __launch_bounds__(64, 1) selftest_wait_kernel(unsigned long long limit_ns, uint32_t* status,
                                                              uint32_t* report) {
  __shared__ alignas(16) uint32_t dst[4];
  __shared__ alignas(8) uint64_t bar_never, bar_copy;
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar_never, 1);
    mbar_init(&bar_copy, 1);
    abort_word = 0;
    dst[0] = dst[1] = dst[2] = dst[3] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;\nfence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_tx(&bar_copy, 16);
      bulk_load(dst, g_selftest_src, 16, &bar_copy);
    }
    __syncwarp();
    const unsigned long long t0 = gtimer();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_never, 0, abort_flag, status, limit_ns));
    const unsigned long long t1 = gtimer();
    if (lane == 0) {
      const bool landed = mbar_drain(&bar_copy, 0);
      bool same = landed;
      for (int i = 0; i < 4; ++i) same = same && dst[i] == g_selftest_src[i];
      report[0] = ok ? 1u : 0u;
      report[2] = (uint32_t)((t1 - t0) / 1000ull);
      report[4] = landed ? 1u : 0u;
      report[5] = same ? 1u : 0u;
    }
  } else {
    const unsigned long long t0 = gtimer();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_never, 0, abort_flag, status, limit_ns + kWarp1ExtraNs));
    const unsigned long long t1 = gtimer();
    if (lane == 0) {
      report[1] = ok ? 1u : 0u;
      report[3] = (uint32_t)((t1 - t0) / 1000ull);
    }
  }
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t limit_us, uint32_t* status, uint32_t* report, cudaStream_t s) {
  selftest_wait_kernel<<<1, 64, 0, s>>>(1000ull * limit_us, status, report);
  return cudaGetLastError();
}

}  // namespace qsa
