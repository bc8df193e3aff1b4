// Diagnostic: exercises the time-out path of the bounded device-side waits.
#include "common.cuh"
#include "kernels.h"

namespace moedisp {

namespace {
// One thread waits on a barrier phase that nothing ever completes (no arrival, no
// transaction bytes), with the given limit: the wait must give up and report TIMEOUT.
__global__ void bounded_wait_kernel(uint64_t limit_ns, int32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    grid_dep_wait();
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_for(&bar, 0, limit_ns)) raise_status(status, MOEDISP_STATUS_TIMEOUT);
}
}  // namespace

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, int32_t* status, cudaStream_t stream) {
    return launch_pdl(bounded_wait_kernel, dim3(1), dim3(1), 0, stream, 1, limit_ns, status);
}

}  // namespace moedisp
