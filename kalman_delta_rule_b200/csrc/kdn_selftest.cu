// Self-test of the failure-detection path: the bounded waits the kernels use (a poll of a
// global word, as in the decoupled look-backs, and an mbarrier phase wait, as in the tensor-core
// kernels) run out on conditions that never come true, record KDN_ERR_TIMEOUT in the device
// error word and return; the context stays usable.  Nothing faults, traps or hangs.
#include "kdn_common.cuh"
#include "kdn_launch.h"
#include "kdn_tc.cuh"

namespace kdn {

namespace {
__device__ unsigned g_never_set;   // zero-initialised; no kernel writes it

__global__ void bounded_wait_selftest_kernel(long long limit, unsigned *err) {
    if (threadIdx.x != 0) return;
    // 1. poll of a global word, bounded by SM clock cycles
    const long long t0 = clock64();
    bool gave_up = false;
    while (*(volatile unsigned *)&g_never_set == 0u) {
        if (clock64() - t0 > limit) {
            gave_up = true;
            break;
        }
        __nanosleep(64);
    }
    if (gave_up) raise_error(err, ERR_TIMEOUT);
    // 2. an mbarrier phase that nobody completes, through the kernels' own bounded wait
    __shared__ uint64_t bar;
    tc::mbar_init(&bar, 1);
    tc::mbar_fence_init();
    if (!tc::mbar_wait(&bar, 0, limit)) raise_error(err, ERR_TIMEOUT);
}
}  // namespace

cudaError_t launch_bounded_wait_selftest(long long limit_cycles, unsigned *err, cudaStream_t st) {
    bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(limit_cycles, err);
    return cudaGetLastError();
}

}  // namespace kdn
