// selftest.cuh -- exercises the library's bounded-wait failure path on the
// device without faulting, trapping or hanging it.
//
// One warp initialises an mbarrier that no thread arrives at and no copy
// completes (nothing is in flight), waits on it with the same bounded wait
// the kernels use, gives up after `polls` polls, records
// TBQ4_ERR_DEVICE_TIMEOUT in the device status word and returns.  The context
// stays usable; tbq4_get_device_status reads the code back.
#pragma once
#include "common.cuh"
#include "mbarrier.cuh"

namespace tbq4 {

__global__ void __launch_bounds__(32, 1) bounded_wait_selftest_kernel(uint32_t polls) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
    }
    __syncwarp();
    // phase 0 never completes: its one expected arrival never comes
    if (!mbar_wait_bounded(b, 0u, polls) && threadIdx.x == 0) record_status(7u);
}

}  // namespace tbq4
