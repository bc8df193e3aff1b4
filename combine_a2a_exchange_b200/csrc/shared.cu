// Shared experts (Ascend aclnnMoeDistributeDispatchV2: sharedExpertNum, sharedExpertRankNum,
// expertShardType 0): the routing is widened so that the ordinary layout, dispatch and
// combine carry the shared experts too. The first S of the W ranks host shared-expert
// replicas (S / N of each of the N shared experts, grouped by shared expert), the other
// W - S ranks the E routed experts, ne = E / (W - S) each. In a uniform expert space of
// W * ne experts (ne per rank), routed expert e is S * ne + e and the shared replica on
// rank d is d * ne. Each token keeps its K routed slots and gets N more, one per shared
// expert, on replica (r mod (S / N)) of that expert's group, with weight 1.
//
// One elementwise pass over the G * (K + N) output slots; reads each input slot once.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace moedisp {

namespace {
constexpr int kSharedThreads = 256;

struct SharedArgs {
    const int32_t* ids;
    const float* w;
    int64_t G;
    int T, K, E, N, S, ne, W;
    int32_t* ext_ids;
    float* ext_w;
    int32_t* status;
};

__global__ void __launch_bounds__(kSharedThreads) shared_routing_kernel(SharedArgs a) {
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int KN = a.K + a.N;
    const int64_t n = a.G * KN;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    bool bad = false;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int64_t g = i / KN;
        const int k = (int)(i - g * KN);
        if (k < a.K) {
            const int32_t e = __ldg(a.ids + g * a.K + k);
            const bool ok = e >= 0 && e < a.E;
            bad |= !ok;
            a.ext_ids[i] = ok ? a.S * a.ne + e : a.W * a.ne;
            a.ext_w[i] = __ldg(a.w + g * a.K + k);
        } else {
            const int j = k - a.K;
            const int replicas = a.S / a.N;
            const int r = (int)(g / a.T);
            a.ext_ids[i] = (j * replicas + r % replicas) * a.ne;
            a.ext_w[i] = 1.0f;
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
        raise_status(a.status, MOEDISP_STATUS_BAD_EXPERT_ID);
}
}  // namespace

cudaError_t launch_shared_routing(const int32_t* expert_ids, const float* expert_scales, int W,
                                  int T, int K, int E, int N, int S, int32_t* ext_ids,
                                  float* ext_scales, int32_t* status, cudaStream_t stream) {
    SharedArgs a;
    a.ids = expert_ids;
    a.w = expert_scales;
    a.G = (int64_t)W * T;
    a.T = T;
    a.K = K;
    a.E = E;
    a.N = N;
    a.S = S;
    a.ne = E / (W - S);
    a.W = W;
    a.ext_ids = ext_ids;
    a.ext_w = ext_scales;
    a.status = status;
    const int64_t n = a.G * (K + N);
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)shared_routing_kernel, kSharedThreads, 0, &per_sm);
    if (err != cudaSuccess) return err;
    int64_t grid = (n + kSharedThreads - 1) / kSharedThreads;
    grid = std::min<int64_t>(grid, (int64_t)current_sm_count() * per_sm);
    grid = std::max<int64_t>(grid, 1);
    return launch_pdl(shared_routing_kernel, dim3((unsigned)grid), dim3(kSharedThreads), 0, stream,
                      1, a);
}

}  // namespace moedisp
