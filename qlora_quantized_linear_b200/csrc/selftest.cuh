// selftest.cuh -- a kernel whose only job is to let its bounded waits run out,
// so that tests can check the timeout path of the library on a real device:
// each wait gives up after the given limit, records the timeout in the device
// status word and returns; nothing traps, faults or spins without a bound.
#pragma once

#include "common.cuh"

namespace lbq {

// A word that nothing ever writes: a wait for it to become nonzero can only
// end by its time limit.
__device__ uint32_t g_never_set;

// One CTA: thread 0 waits on an mbarrier phase that never completes (count 1,
// no arrivals), then on g_never_set, each bounded by limit_ns.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_wait(&bar, 0, &abort_flag, limit_ns);     // records kStatusTimeout when it gives up
        flag_wait_geq(&g_never_set, 1u, limit_ns);     // the same for the flag wait
    }
}

}  // namespace lbq
