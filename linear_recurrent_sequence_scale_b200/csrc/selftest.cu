// Self-test of the bounded device waits: one thread waits on an mbarrier that
// nothing arrives on.  The wait gives up after the given time, records its
// site code in this unit's error flag and the kernel returns normally, so the
// context stays usable; the host reads the code with ret_device_error().
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace ret {

constexpr int kSelftestSite = 901;

__global__ void bounded_wait_selftest(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  sm100::mbar_init(&bar, 1);
  sm100::fence_mbar_init();
  // no arrival ever comes: the wait must run out after limit_ns
  sm100::mbar_wait(&bar, 0, kSelftestSite, limit_ns);
}

int selftest_device_error() { return read_clear_device_error(); }

cudaError_t launch_bounded_wait_selftest(int limit_ms, cudaStream_t st) {
  bounded_wait_selftest<<<1, 1, 0, st>>>(static_cast<uint64_t>(limit_ms) * 1000000ull);
  return cudaPeekAtLastError();
}

}  // namespace ret
