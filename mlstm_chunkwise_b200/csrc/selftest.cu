// Failure-detection self-test: a bounded wait that nothing ever satisfies.
//
// One thread waits on a fresh mbarrier (expected arrival count 1, no arrival
// and no transaction ever posted) through the same bounded wait every kernel
// of the library uses.  After the watchdog limit the wait records the
// watchdog bit and the site kSelftestSite in the device error word and
// returns false; the kernel then exits normally, so the context stays usable
// and the host reads MLSTM_ERR_TIMEOUT.  No trap, no fault, no endless loop.
#include "tc.h"
#include "tc_ptx.cuh"

namespace mlstm {
namespace {

constexpr uint32_t kSelftestSite = 0xF7;

__global__ void watchdog_selftest_kernel(Problem p) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t a = tc::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(a, 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)tc::mbar_wait(a, 0, p, kSelftestSite);
  __syncthreads();
}

}  // namespace

cudaError_t launch_watchdog_selftest(uint32_t* err, unsigned long long max_polls,
                                     cudaStream_t st) {
  Problem p{};
  p.err = err;
  p.max_polls = max_polls;
  watchdog_selftest_kernel<<<1, 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace mlstm
