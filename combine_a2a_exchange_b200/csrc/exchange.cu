// All-to-all-v exchange plan and row exchange between W virtual ranks held in one GPU.
//
// Plan: the ExchangePlan of the PyTorch symm_mem change (make_a2a_exchange_plan). There
// every rank learns its row of the plan through NVSHMEM gets and a one-block prefix sum;
// here all W rows live in one HBM, so block b scans row b and column b of the send
// matrix directly.
//
// Row exchange: the get-style all_to_all_v of the same change, where each block copies
// one peer's contribution with a remote block get. Every (destination i, source j)
// segment is one contiguous byte range in both buffers, so a block streams it through
// shared memory with 1-D bulk (TMA) copies: one thread keeps kStages-1 loads in flight
// and writes each landed piece back out with a bulk store. Segments are visited in the
// rotated peer order the same change uses for its signalled variant, so that concurrent
// blocks read from different source ranks.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace moedisp {

namespace {
constexpr int kPlanThreads = 256;
constexpr int kA2AStages = 4;
constexpr uint32_t kA2APiece = 16384;                 // bytes per bulk copy
constexpr int kA2AThreads = 32;                        // one issuing lane per block
}  // namespace

__global__ void __launch_bounds__(kPlanThreads)
a2a_plan_kernel(const int64_t* __restrict__ S, int W, int64_t* __restrict__ src_offsets,
                int64_t* __restrict__ out_splits, int64_t* __restrict__ dst_offsets,
                int32_t* status) {
    __shared__ int64_t warp_tot[32];
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int b = blockIdx.x;
    bool bad = false;
    // Row b of S is what rank b sends; its exclusive scan at k is where rank k's rows
    // start inside rank b's input, i.e. src_offsets[k][b].
    int64_t carry = 0;
    for (int base = 0; base < W; base += blockDim.x) {
        const int k = base + threadIdx.x;
        const int64_t v = k < W ? S[(int64_t)b * W + k] : 0;
        bad |= v < 0;
        int64_t tot;
        const int64_t ex = block_exclusive_scan(v, warp_tot, tot);
        if (k < W) src_offsets[(int64_t)k * W + b] = carry + ex;
        carry += tot;
    }
    // Column b of S is what every rank sends to rank b: rank b's out_splits, whose
    // exclusive scan is rank b's dst_offsets.
    carry = 0;
    for (int base = 0; base < W; base += blockDim.x) {
        const int j = base + threadIdx.x;
        const int64_t v = j < W ? S[(int64_t)j * W + b] : 0;
        int64_t tot;
        const int64_t ex = block_exclusive_scan(v, warp_tot, tot);
        if (j < W) {
            out_splits[(int64_t)b * W + j] = v;
            dst_offsets[(int64_t)b * W + j] = carry + ex;
        }
        carry += tot;
    }
    if (bad) raise_status(status, MOEDISP_STATUS_BAD_SPLIT);
}

__global__ void __launch_bounds__(kA2AThreads)
a2a_v_kernel(const uint8_t* __restrict__ in, int64_t in_stride_rows, uint8_t* __restrict__ out,
             int64_t out_cap_rows, int64_t row_bytes, int W, const int64_t* __restrict__ src_off,
             const int64_t* __restrict__ out_splits, const int64_t* __restrict__ dst_off,
             int blocks_per_seg, int32_t* status) {
    extern __shared__ __align__(128) uint8_t stage_buf[];
    __shared__ __align__(8) uint64_t bars[kA2AStages];
    grid_dep_wait();
    grid_dep_launch_dependents();
    if (threadIdx.x != 0) return;

    const int64_t seg = blockIdx.x / blocks_per_seg;
    const int sub = blockIdx.x % blocks_per_seg;
    const int i = (int)(seg / W);                       // destination rank
    const int j = (int)((i + seg % W) % W);             // source rank, rotated by i
    const int64_t n = out_splits[(int64_t)i * W + j];
    if (n == 0) return;
    const int64_t so = src_off[(int64_t)i * W + j];
    const int64_t d0 = dst_off[(int64_t)i * W + j];
    if (n < 0 || so < 0 || d0 < 0 || so > in_stride_rows - n || d0 > out_cap_rows - n) {
        if (sub == 0) raise_status(status, MOEDISP_STATUS_BAD_SPLIT);
        return;
    }
    const uint8_t* src = in + ((int64_t)j * in_stride_rows + so) * row_bytes;
    uint8_t* dst = out + ((int64_t)i * out_cap_rows + d0) * row_bytes;
    const int64_t total = n * row_bytes;
    const int64_t n_pieces = (total + kA2APiece - 1) / kA2APiece;
    if (sub >= n_pieces) return;
    const int64_t mine = (n_pieces - sub + blocks_per_seg - 1) / blocks_per_seg;

    for (int s = 0; s < kA2AStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();

    auto piece_off = [&](int64_t q) { return (sub + q * blocks_per_seg) * (int64_t)kA2APiece; };
    auto piece_len = [&](int64_t q) {
        return (uint32_t)min64(kA2APiece, total - piece_off(q));
    };
    auto issue = [&](int64_t q) {
        const int st = (int)(q % kA2AStages);
        const uint32_t len = piece_len(q);
        mbar_arrive_expect_tx(&bars[st], len);
        bulk_load(stage_buf + st * kA2APiece, src + piece_off(q), len, &bars[st]);
    };

    const int64_t pro = min64(kA2AStages, mine);
    for (int64_t q = 0; q < pro; ++q) issue(q);
    int64_t issued = pro;                               // pieces whose loads were armed
    for (int64_t q = 0; q < mine; ++q) {
        const int st = (int)(q % kA2AStages);
        if (!mbar_wait(&bars[st], (uint32_t)((q / kA2AStages) & 1))) {
            // Stop issuing, and let the loads already armed land before the block exits.
            raise_status(status, MOEDISP_STATUS_TIMEOUT);
            (void)mbar_drain(bars, kA2AStages, q, issued);
            break;
        }
        bulk_store(dst + piece_off(q), stage_buf + st * kA2APiece, piece_len(q));
        bulk_commit();
        // Refill the stage the previous piece was stored from, once that store has
        // finished reading it.
        if (q >= 1 && q - 1 + kA2AStages < mine) {
            bulk_wait_read<1>();
            issue(q - 1 + kA2AStages);
            issued = q + kA2AStages;
        }
    }
    bulk_wait<0>();
}

// ------------------------------------------------------------------ launchers

// Source of every receive position, for a dispatch that reads the exchanged tokens in
// place (no receive buffer): position p of rank i (p < T, the receive capacity) holds,
// when it is one of the rows rank i receives, row src_offsets[i][j] + (p - dst_offsets[i][j])
// of source rank j, where j is the segment holding p (dst_offsets[i] is the exclusive scan
// of out_splits[i], so j is the last segment starting at or before p); that row is
// j * in_rank_stride_rows + ... of the concatenated input. Other positions get -1 (and,
// with an active mask, 0). A segment outside its sender's rows gives -1 and BAD_SPLIT; a
// rank that receives more than T rows in total (rows that have no position) sets
// CAPACITY, as a2a_v flags a receive buffer too small for its rows.
__global__ void __launch_bounds__(kPlanThreads)
a2a_token_rows_kernel(const int64_t* __restrict__ src_offsets,
                      const int64_t* __restrict__ out_splits,
                      const int64_t* __restrict__ dst_offsets, int W, int64_t T,
                      int64_t in_rank_stride_rows, int64_t* __restrict__ token_rows,
                      uint8_t* __restrict__ active, int32_t* status) {
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int64_t n = (int64_t)W * T;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t first = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // Rows received by rank i end at its last segment's end (dst_offsets[i] is the
    // exclusive scan of out_splits[i]); beyond T they have no receive position.
    for (int64_t i = first; i < W; i += stride) {
        const int64_t last = i * W + W - 1;
        if (__ldg(dst_offsets + last) + __ldg(out_splits + last) > T)
            raise_status(status, MOEDISP_STATUS_CAPACITY);
    }
    bool bad = false;
    for (int64_t g = first; g < n; g += stride) {
        const int i = (int)(g / T);
        const int64_t p = g - (int64_t)i * T;
        const int64_t* dst = dst_offsets + (int64_t)i * W;
        int lo = 0, hi = W;                      // last j with dst[j] <= p (or 0)
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(dst + mid) <= p) lo = mid; else hi = mid;
        }
        const int64_t q = p - __ldg(dst + lo);
        const int64_t len = __ldg(out_splits + (int64_t)i * W + lo);
        int64_t row = -1;
        if (q >= 0 && q < len) {
            const int64_t src = __ldg(src_offsets + (int64_t)i * W + lo) + q;
            if (src >= 0 && src < in_rank_stride_rows) row = (int64_t)lo * in_rank_stride_rows + src;
            else bad = true;
        }
        token_rows[g] = row;
        if (active != nullptr) active[g] = row >= 0 ? 1 : 0;
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
        raise_status(status, MOEDISP_STATUS_BAD_SPLIT);
}

cudaError_t launch_a2a_token_rows(const int64_t* src_offsets, const int64_t* out_splits,
                                  const int64_t* dst_offsets, int W, int64_t T,
                                  int64_t in_rank_stride_rows, int64_t* token_rows,
                                  uint8_t* active, int32_t* status, cudaStream_t stream) {
    const int64_t n = (int64_t)W * T;
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)a2a_token_rows_kernel, kPlanThreads, 0, &per_sm);
    if (err != cudaSuccess) return err;
    int64_t grid = std::max<int64_t>(1, (n + kPlanThreads - 1) / kPlanThreads);
    grid = std::min<int64_t>(grid, (int64_t)current_sm_count() * per_sm);
    return launch_pdl(a2a_token_rows_kernel, dim3((unsigned)grid), dim3(kPlanThreads), 0, stream, 1,
                      src_offsets, out_splits, dst_offsets, W, T, in_rank_stride_rows, token_rows,
                      active, status);
}

cudaError_t launch_a2a_plan(const int64_t* in_splits, int W, int64_t* src_offsets,
                            int64_t* out_splits, int64_t* dst_offsets, int32_t* status,
                            cudaStream_t stream) {
    return launch_pdl(a2a_plan_kernel, dim3(W), dim3(kPlanThreads), 0, stream, 1, in_splits, W,
                      src_offsets, out_splits, dst_offsets, status);
}

cudaError_t launch_a2a_v(const void* in, int64_t in_rank_stride_rows, void* out,
                         int64_t out_cap_rows, int64_t row_bytes, int W,
                         const int64_t* src_offsets, const int64_t* out_splits,
                         const int64_t* dst_offsets, int32_t* status, cudaStream_t stream) {
    const size_t smem = (size_t)kA2AStages * kA2APiece;
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)a2a_v_kernel, kA2AThreads, smem, &per_sm);
    if (err != cudaSuccess) return err;
    const int64_t segs = (int64_t)W * W;
    const int64_t target = (int64_t)current_sm_count() * per_sm * 2;
    // No segment holds more rows than either its source or its destination buffer.
    const int64_t max_rows = std::max<int64_t>(0, std::min(in_rank_stride_rows, out_cap_rows));
    const int64_t max_pieces = std::max<int64_t>(1, (max_rows * row_bytes + kA2APiece - 1) / kA2APiece);
    int64_t bps = std::max<int64_t>(1, (target + segs - 1) / segs);
    bps = std::min(bps, max_pieces);
    const int64_t grid = segs * bps;
    if (grid > 0x7fffffffll) return cudaErrorInvalidConfiguration;
    return launch_pdl(a2a_v_kernel, dim3((unsigned)grid), dim3(kA2AThreads), smem, stream, 1,
                      static_cast<const uint8_t*>(in), in_rank_stride_rows,
                      static_cast<uint8_t*>(out), out_cap_rows, row_bytes, W, src_offsets,
                      out_splits, dst_offsets, (int)bps, status);
}

}  // namespace moedisp
