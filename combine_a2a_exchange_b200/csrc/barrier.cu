// Rank barrier for expert parallelism over W GPUs, on the GPUs themselves, with a time
// limit.
//
// The PyTorch symm_mem change orders its ranks with signal-pad barriers that spin without
// a limit (a rank that died leaves every other rank's GPU spinning). Here each rank owns a
// signal array of W words in peer-mapped memory; a barrier publishes this rank's epoch in
// word `rank` of every rank's array with a system-scope release store, then waits with
// acquire loads until every word of its own array has reached the epoch. Epochs only grow,
// so one word per peer serves every barrier and nothing is reset between them: a rank that
// already went on to the next barrier has, by then, passed this one, and its larger epoch
// satisfies the comparison (taken with wrap-around). A wait that runs out sets
// MOEDISP_STATUS_TIMEOUT and returns; nothing traps.
#include "common.cuh"
#include "kernels.h"

namespace moedisp {

namespace {
constexpr int kBarrierThreads = 128;

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__global__ void __launch_bounds__(kBarrierThreads)
ep_barrier_kernel(uint32_t* const* __restrict__ peers, int W, int rank, uint32_t epoch,
                  uint64_t limit_ns, int32_t* status) {
    // Every kernel before this one on the stream has completed and its writes (rows pushed
    // into the peers' buffers among them) are performed once the dependency wait returns;
    // the system-scope fence orders them before the arrival stores below.
    grid_dep_wait();
    __threadfence_system();
    __syncthreads();
    for (int q = threadIdx.x; q < W; q += blockDim.x) st_release_sys(peers[q] + rank, epoch);
    const uint32_t* own = peers[rank];
    bool late = false;
    const uint64_t t0 = global_timer_ns();
    for (int q = threadIdx.x; q < W && !late; q += blockDim.x) {
        for (uint32_t i = 1;; ++i) {
            if ((int32_t)(ld_acquire_sys(own + q) - epoch) >= 0) break;
            if ((i & 63u) == 0u && global_timer_ns() - t0 > limit_ns) {
                late = true;
                break;
            }
        }
    }
    if (late) raise_status(status, MOEDISP_STATUS_TIMEOUT);
    __syncthreads();
    grid_dep_launch_dependents();
}
}  // namespace

cudaError_t launch_ep_barrier(uint32_t* const* peer_signals, int W, int rank, uint32_t epoch,
                              uint64_t limit_ns, int32_t* status, cudaStream_t stream) {
    return launch_pdl(ep_barrier_kernel, dim3(1), dim3(kBarrierThreads), 0, stream, 1,
                      peer_signals, W, rank, epoch, limit_ns, status);
}

}  // namespace moedisp
