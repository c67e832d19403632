// Failure-path self-test of the device-side bounded waits (spattn_wait_selftest).
//
// One CTA waits on an mbarrier that nothing ever completes, through the same
// bounded-wait routine the tile kernels use: warp 0 with a short deadline,
// warp 1 with the tile kernels' deadline.  Warp 0 times out and records the
// timeout in the plan's error word; warp 1 sees the CTA abort flag and gives
// up.  Both return: no fault, no hang, the context stays usable.
#include "kernels.cuh"
#include "sm100.cuh"

namespace spattn {
namespace {

using namespace dev;

__global__ void __launch_bounds__(64, 1) wait_selftest_kernel(int* err, long long deadline) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const Abort ab{&abort_flag, err};
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x < 32)
    (void)__all_sync(0xffffffffu, mbar_wait(&bar, 0, ab, deadline));
  else
    (void)__all_sync(0xffffffffu, mbar_wait(&bar, 0, ab));
}

}  // namespace

cudaError_t launch_wait_selftest(int* err, long long deadline_cycles, cudaStream_t st) {
  wait_selftest_kernel<<<1, 64, 0, st>>>(err, deadline_cycles);
  return cudaGetLastError();
}

}  // namespace spattn
