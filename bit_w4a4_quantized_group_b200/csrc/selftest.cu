// Self-test of the failure path: a bounded wait that is meant to run out.
//
// One warp waits on an mbarrier that nothing arrives at.  The wait gives up after
// the given time, records kErrSiteSelftest in the device error word and the kernel
// returns normally, so the context stays usable.  This exercises, on the device,
// the same wait every kernel of the library uses, without any fault or hang.
#include <cuda_runtime.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_device.cuh"

namespace svdq {
namespace {

__global__ void selftest_bounded_wait_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncwarp();
  // phase 0 never completes: no thread arrives
  wait_bounded(&bar, 0, &abort_flag, err, kErrSiteSelftest, limit_ns);
}

}  // namespace

cudaError_t launch_selftest_bounded_wait(int* err, uint64_t limit_ns, cudaStream_t s) {
  selftest_bounded_wait_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace svdq
