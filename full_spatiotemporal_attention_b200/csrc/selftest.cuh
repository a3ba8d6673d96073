// Watchdog self-test: one CTA waits on an mbarrier whose arrival never
// comes.  Every wait in the kernels is bounded, so the wait must give up
// after its limit, raise the CTA's abort flag, record its code in the device
// error word and return; the kernel then exits normally and the context
// stays usable.  Nothing here traps or faults.
#pragma once

#include "ptx.cuh"

namespace va3d {

__global__ void watchdog_probe_kernel() {
    __shared__ __align__(8) uint64_t bar_storage;
    __shared__ int abort_word;
    const uint32_t bar = smem_u32(&bar_storage);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);          // expects one arrival; none is ever made
        abort_word = 0;
        mbar_init_fence();
    }
    __syncthreads();
    volatile int *abort_flag = &abort_word;
    mbar_wait(bar, 0, abort_flag, VA3D_DEVERR_TIMEOUT_SELFTEST);
}

}  // namespace va3d
