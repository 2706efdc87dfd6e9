// Self-test of the failure path every pipeline wait takes (ptx.cuh,
// mbar_wait): a bounded wait that runs out records BSMT_ERR_DEVICE_TIMEOUT in
// the device status word and raises the CTA's abort flag, and the CTA's other
// waits then return instead of spinning. The kernel makes that happen on
// purpose, with no fault: warp 0 waits on an mbarrier that nothing arrives
// on, warp 1 on a second one, and both return normally.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace bsmt {

// result[0] / result[1]: 1 if warp 0 / warp 1 saw its wait complete, 0 if the
// wait gave up; result[2]: warp 0's wait time in microseconds.
__global__ void __launch_bounds__(64) wait_timeout_selftest_kernel(int32_t* result) {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const uint64_t t0 = globaltimer_ns();
    // phase 0 of either barrier never completes: no thread arrives
    const bool ok = mbar_wait(smem_u32(&bars[warp]), 0, &abort_flag);
    const uint64_t t1 = globaltimer_ns();
    if (lane == 0) {
        result[warp] = ok ? 1 : 0;
        if (warp == 0) result[2] = static_cast<int32_t>((t1 - t0) / 1000u);
    }
}

}  // namespace bsmt
