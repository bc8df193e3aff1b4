// Internal host-side launchers of libmoedisp (called by abi.cu after validation).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "moedisp.h"

namespace moedisp {

// Streaming-multiprocessor count of the current device (cached per device).
int current_sm_count();
int64_t current_l2_bytes();     // L2 cache size of the current device

// Lets `kernel` use the device's full opt-in dynamic shared memory (once per device).
cudaError_t allow_dynamic_smem(const void* kernel);

// Resident blocks per SM of `kernel` at this block size and dynamic shared memory
// (at least 1; cached per device). Also calls allow_dynamic_smem.
cudaError_t blocks_per_sm(const void* kernel, int threads, size_t smem, int* out);

// Grid for `items` equal work items spread by a grid-stride loop over at most `max_grid`
// resident blocks: the fewest items per block that fit, and the fewest blocks that then
// cover them, so that every block gets the same count (no last-wave tail).
inline int64_t balanced_grid(int64_t items, int64_t max_grid) {
    if (items <= 0 || max_grid <= 0) return 1;
    const int64_t per = (items + max_grid - 1) / max_grid;
    return (items + per - 1) / per;
}

// Launches `kernel` with programmatic stream serialization (and a 1-D cluster of
// `cluster` blocks when cluster > 1) and returns the launch status.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, int cluster, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)n;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

cudaError_t launch_a2a_plan(const int64_t* in_splits, int W, int64_t* src_offsets,
                            int64_t* out_splits, int64_t* dst_offsets, int32_t* status,
                            cudaStream_t stream);

cudaError_t launch_a2a_v(const void* in, int64_t in_rank_stride_rows, void* out,
                         int64_t out_cap_rows, int64_t row_bytes, int W,
                         const int64_t* src_offsets, const int64_t* out_splits,
                         const int64_t* dst_offsets, int32_t* status, cudaStream_t stream);

// Layout tiling, shared by the workspace-size query and the launcher.
struct LayoutGeometry {
    int64_t slots_per_rank;   // T*K
    int tiles_per_rank;
    int64_t tile_len;         // slots per tile
    int steps;                // 32-slot steps per warp (a power of two)
    int64_t n_tiles;
    size_t off_tile_hist, off_tile_prefix, total_bytes;
};
LayoutGeometry layout_geometry(const moedisp_dims& d);

cudaError_t launch_layout(const int32_t* expert_ids, const uint8_t* active, int active_dims,
                          int major_align, const moedisp_dims& dims, const moedisp_layout& layout,
                          void* workspace, int32_t* status, cudaStream_t stream);

// Allocation-free layout: the tiled path on the library's static scratch array.
size_t layout_noalloc_scratch_bytes();
cudaError_t launch_layout_noalloc(const int32_t* expert_ids, const uint8_t* active,
                                  int active_dims, int major_align, const moedisp_dims& dims, const moedisp_layout& layout,
                                  int32_t* status, cudaStream_t stream);

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, int32_t* status, cudaStream_t stream);

// Barrier across W ranks over peer-mapped signal words (bounded wait).
cudaError_t launch_ep_barrier(uint32_t* const* peer_signals, int W, int rank, uint32_t epoch,
                              uint64_t limit_ns, int32_t* status, cudaStream_t stream);

cudaError_t launch_a2a_token_rows(const int64_t* src_offsets, const int64_t* out_splits,
                                  const int64_t* dst_offsets, int W, int64_t T,
                                  int64_t in_rank_stride_rows, int64_t* token_rows,
                                  uint8_t* active, int32_t* status, cudaStream_t stream);

cudaError_t launch_dispatch(const void* x, int64_t x_rows, const int64_t* token_rows, int H,
                            const moedisp_dims& dims,
                            const moedisp_layout& layout, int quant_mode,
                            const float* smooth_scales, void* expand_x,
                            float* dynamic_scales, int64_t* expert_token_nums,
                            int expert_token_nums_type, int32_t* ep_recv_counts,
                            int32_t* status, cudaStream_t stream);

// Rank `rank`'s dispatch when the W ranks are separate GPUs: its T tokens' rows go to
// rows of the ranks' own buffers through a device table of W pointers (peer memory).
cudaError_t launch_dispatch_peers(const void* x, int H, const moedisp_dims& dims, int rank,
                                  const int32_t* expert_ids, const moedisp_layout& layout,
                                  int quant_mode, void* const* peer_out,
                                  float* const* peer_scales, int64_t peer_cap, int32_t* status,
                                  cudaStream_t stream);
cudaError_t launch_combine_peers(const void* const* peer_expert_out, int64_t peer_cap, int H,
                                 const moedisp_dims& dims, int rank, const int32_t* expert_ids,
                                 const moedisp_layout& layout, const float* expert_scales,
                                 void* y, int32_t* status, cudaStream_t stream);

// Exchange -> dispatch pipelined through per-segment ready words (set-up + one kernel).
size_t pipeline_workspace_bytes(int W);
cudaError_t launch_a2a_dispatch_pipelined(const void* in, int64_t in_rank_stride_rows,
                                          const int64_t* src_offsets, const int64_t* out_splits,
                                          const int64_t* dst_offsets, void* recv, int H,
                                          const moedisp_dims& dims, const moedisp_layout& L,
                                          int quant_mode, void* expand_x, float* dynamic_scales,
                                          int64_t* expert_token_nums, int expert_token_nums_type,
                                          int32_t* ep_recv_counts, uint32_t* ready, uint32_t epoch,
                                          int roles, uint64_t limit_ns, void* workspace,
                                          int32_t* status, cudaStream_t stream);

cudaError_t launch_combine(const void* expert_out, int H, const moedisp_dims& dims,
                           const moedisp_layout& layout, const float* expert_scales, void* y,
                           int32_t* status, cudaStream_t stream);

cudaError_t launch_shared_routing(const int32_t* expert_ids, const float* expert_scales, int W,
                                  int T, int K, int E, int N, int S, int32_t* ext_ids,
                                  float* ext_scales, int32_t* status, cudaStream_t stream);

cudaError_t launch_combine_rmsnorm(const void* expert_out, int H, const moedisp_dims& dims,
                                   const moedisp_layout& layout, const float* expert_scales,
                                   const void* residual, const float* gamma, float eps,
                                   void* residual_out, void* y, int32_t* status,
                                   cudaStream_t stream);

}  // namespace moedisp
