// Self-test of the failure detection: the bounded mbarrier wait every kernel
// of the library uses, made to run out on purpose without faulting or
// hanging the GPU.
#pragma once
#include "tc_ptx.cuh"

namespace mla {
namespace tc {

// One CTA of one warp: lane 0 initializes an mbarrier that expects one
// arrival, which never comes, and waits on it through mbar_wait_for with
// `limit_ns`. The wait gives up after the limit, sets the CTA's abort flag and
// the device error word (kDevErrTimeout), and the kernel returns; nothing
// else is in flight. *gave_up records the wait's result (1 = it gave up).
__global__ void __launch_bounds__(32, 1) wait_timeout_selftest_kernel(uint64_t limit_ns, int* gave_up) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const bool arrived = mbar_wait_for(&bar, 0, &abort_flag, limit_ns);
    *gave_up = arrived ? 0 : 1;
  }
}

}  // namespace tc
}  // namespace mla
