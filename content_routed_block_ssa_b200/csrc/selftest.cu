// Self-test of the failure path every kernel wait takes: one CTA waits on an
// mbarrier that nothing arrives at, through the same bounded wait the
// kernels use; the wait gives up after its limit, records its site code in
// the device failure word and the kernel returns, leaving the context usable.
#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

__global__ void __launch_bounds__(32) selftest_wait_kernel(uint32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, err, SITE_SELFTEST);   // no arrival: times out
}

}  // namespace

cudaError_t launch_selftest_wait(const LaunchCtx& c) {
  selftest_wait_kernel<<<1, 32, 0, c.stream>>>(c.err);
  note_launch();
  return cudaGetLastError();
}

}  // namespace ssa
