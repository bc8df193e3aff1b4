// Exchange -> dispatch pipelined through per-segment ready words, in one kernel.
//
// The PyTorch symm_mem change overlaps its get-style all-to-all with the MoE index push:
// the exchange kernel publishes, with a release store, how many rows of a peer's segment
// have arrived, and the concurrently running push kernel spins on that word (acquire)
// before pushing the rows on to their experts. Kernels that wait on one another cannot
// share one GPU safely as separate launches, so here both roles live in one persistent
// kernel whose blocks draw work items from a ticket counter:
//
//   producer item  (segment s, piece k): copy a piece (<= 32 KB) of segment s = (receiving
//                  rank i, source rank j) from j's send rows into i's receive buffer; the
//                  block that lands the segment's last rows stores ready[s] = epoch
//                  (release, GPU scope);
//   consumer item  (segment s, chunk c): wait (acquire, bounded) until ready[s] == epoch,
//                  then dispatch a chunk of the segment's received tokens -- the receive
//                  row read back (from L2, written moments before), quantised or not, and
//                  written to the K rows the layout gave its slots.
//
// Tickets hand the items out in the order P(0), P(1), C(0), P(2), C(1), ...: consumers of
// segment s come after the producers of segment s + 1, so they rarely wait, and every item
// a consumer waits for carries a smaller ticket -- it was taken by a block that is running
// and never waits itself, so no wait can deadlock however many blocks are resident. A
// consumer wait that runs out sets MOEDISP_STATUS_TIMEOUT and raises a flag that makes the
// other blocks stop waiting too.
//
// A small set-up kernel first validates the segments (as a2a_v does), counts the items of
// every ticket slot, scans them into offsets and resets the ticket counter and the
// per-segment landed-row counters in the workspace.
#include "common.cuh"
#include "kernels.h"
#include "dispatch_common.cuh"

#include <algorithm>

namespace moedisp {

namespace {
constexpr int kPipeThreads = 256;
constexpr int kSetupThreads = 1024;
constexpr int64_t kPieceBytes = 32768;     // producer item: at most this many bytes
constexpr int kConsumerRounds = 4;         // consumer item: rounds of one token per group
constexpr int kCopyVecs = kPieceBytes / 16 / kPipeThreads;   // 16-byte vectors per thread

struct PipeArgs {
    const uint4* in;           // [W][in_stride][H8] send rows
    int64_t in_stride;
    const int64_t* src_off;
    const int64_t* out_splits;
    const int64_t* dst_off;
    uint4* recv;               // [W][T][H8] receive rows
    int W;
    int64_t T;
    int K, H8;
    int64_t rows_per_piece;
    int64_t tokens_per_item;
    int roles;
    uint32_t epoch;
    uint32_t* ready;           // [W*W] caller-owned, published epochs
    uint64_t limit_ns;
    // workspace
    unsigned long long* ticket;
    uint32_t* abort_flag;
    uint32_t* landed;          // [W*W]
    int64_t* item_off;         // [2*W*W + 2]
    bool offsets_in_smem;      // the main kernel keeps a 32-bit copy of item_off in shared memory
    // dispatch
    const int32_t* dst_row;
    int64_t rows_cap;
    uint8_t* expand_x;
    float* scales;
    int32_t* status;
};

// Ticket slot u (0 <= u <= 2S, S = W*W segments): producers of segment seg, or consumers.
__host__ __device__ __forceinline__ void slot_of(int64_t u, bool* producer, int64_t* seg) {
    if (u == 0) {
        *producer = true;
        *seg = 0;
    } else if (u & 1) {
        *producer = true;
        *seg = (u + 1) / 2;        // == S for the last odd slot: no such segment, no items
    } else {
        *producer = false;
        *seg = u / 2 - 1;
    }
}

__device__ __forceinline__ bool segment_valid(const PipeArgs& a, int64_t s, int64_t* n,
                                              int64_t* so, int64_t* d0) {
    *n = a.out_splits[s];
    *so = a.src_off[s];
    *d0 = a.dst_off[s];
    return *n >= 0 && *so >= 0 && *d0 >= 0 && *so <= a.in_stride - *n && *d0 <= a.T - *n;
}

__global__ void __launch_bounds__(kSetupThreads) pipe_setup_kernel(PipeArgs a) {
    __shared__ int64_t warp_tot[32];
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int64_t S = (int64_t)a.W * a.W;
    const int64_t U = 2 * S + 1;
    bool bad = false;
    int64_t carry = 0;
    for (int64_t base = 0; base < U; base += blockDim.x) {
        const int64_t u = base + threadIdx.x;
        int64_t cnt = 0;
        if (u < U) {
            bool prod;
            int64_t s;
            slot_of(u, &prod, &s);
            if (s < S) {
                int64_t n, so, d0;
                const bool ok = segment_valid(a, s, &n, &so, &d0);
                bad |= !ok && prod;                 // each segment has one producer slot
                if (ok && n > 0) {
                    if (prod && (a.roles & MOEDISP_PIPE_PRODUCE))
                        cnt = (n + a.rows_per_piece - 1) / a.rows_per_piece;
                    if (!prod && (a.roles & MOEDISP_PIPE_CONSUME))
                        cnt = (n + a.tokens_per_item - 1) / a.tokens_per_item;
                }
            }
        }
        int64_t tot;
        const int64_t ex = block_exclusive_scan(cnt, warp_tot, tot);
        if (u < U) a.item_off[u] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) {
        a.item_off[U] = carry;
        *a.ticket = 0ull;
        *a.abort_flag = 0u;
    }
    for (int64_t s = threadIdx.x; s < S; s += blockDim.x) a.landed[s] = 0u;
    if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(a.status, MOEDISP_STATUS_BAD_SPLIT);
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Producer item: rows [r0, r1) of segment s copied to the receive buffer, then counted.
__device__ void produce(const PipeArgs& a, int64_t s, int64_t k) {
    int64_t n, so, d0;
    (void)segment_valid(a, s, &n, &so, &d0);
    const int i = (int)(s / a.W), j = (int)(s - (int64_t)i * a.W);
    const int64_t r0 = k * a.rows_per_piece, r1 = min64(n, r0 + a.rows_per_piece);
    const uint4* src = a.in + ((int64_t)j * a.in_stride + so + r0) * a.H8;
    uint4* dst = a.recv + ((int64_t)i * a.T + d0 + r0) * a.H8;
    const int64_t nv = (r1 - r0) * a.H8;                 // <= kCopyVecs * kPipeThreads
    uint4 v[kCopyVecs];
#pragma unroll
    for (int q = 0; q < kCopyVecs; ++q) {
        const int64_t e = threadIdx.x + (int64_t)q * kPipeThreads;
        if (e < nv) v[q] = __ldcs(src + e);
    }
#pragma unroll
    for (int q = 0; q < kCopyVecs; ++q) {
        const int64_t e = threadIdx.x + (int64_t)q * kPipeThreads;
        if (e < nv) dst[e] = v[q];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t got = (uint32_t)(r1 - r0);
        if ((int64_t)atom_add_acq_rel_gpu(a.landed + s, got) + got == n)
            st_release_gpu(a.ready + s, a.epoch);
    }
}

// Waits until segment s is published for this epoch (thread 0; bounded). False if the
// wait ran out or another block already gave up.
__device__ bool wait_ready(const PipeArgs& a, int64_t s) {
    __shared__ int ok_sh;
    if (threadIdx.x == 0) {
        int ok = 1;
        if (ld_acquire_gpu(a.ready + s) != a.epoch) {
            const uint64_t t0 = global_timer_ns();
            for (uint32_t it = 1;; ++it) {
                if (ld_acquire_gpu(a.ready + s) == a.epoch) break;
                if ((it & 31u) == 0u) {
                    if (*(volatile uint32_t*)a.abort_flag != 0u) {
                        ok = 0;
                        break;
                    }
                    if (global_timer_ns() - t0 > a.limit_ns) {
                        raise_status(a.status, MOEDISP_STATUS_TIMEOUT);
                        atomicExch(a.abort_flag, 1u);
                        ok = 0;
                        break;
                    }
                }
                __nanosleep(64);
            }
        }
        ok_sh = ok;
    }
    __syncthreads();
    return ok_sh != 0;
}

// Consumer item: tokens [p0, p1) of receiving rank i, one per group of WPT warps per
// round; the group reads the received row into registers (L2: ld.global.cg) and writes
// it, copied or quantised, to the K rows of its slots.
template <int Q, int WPT, int CPT>
__device__ void consume(const PipeArgs& a, int64_t s, int64_t c, float (&red)[kPipeThreads / 32 / WPT][2][WPT],
                        int& parity) {
    constexpr int NG = kPipeThreads / 32 / WPT;
    constexpr int GT = WPT * 32;
    constexpr float kQmax = Q == MOEDISP_QUANT_INT8 ? 127.0f : 448.0f;
    if (!wait_ready(a, s)) return;
    int64_t n, so, d0;
    (void)segment_valid(a, s, &n, &so, &d0);
    const int i = (int)(s / a.W);
    const int64_t p0 = d0 + c * a.tokens_per_item, p1 = d0 + min64(n, (c + 1) * a.tokens_per_item);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = warp / WPT, gw = warp - grp * WPT, gt = tid - grp * GT;
    const int K = a.K;
    const uint32_t out_vec = Q == MOEDISP_QUANT_NONE ? 16u : 8u;     // bytes per 8 columns
    for (int64_t p = p0 + grp; p < p1; p += NG) {
        const int64_t g = (int64_t)i * a.T + p;                     // token of the layout
        int32_t d = lane < K ? __ldg(a.dst_row + g * K + lane) : -1;
        if (d >= a.rows_cap) {
            raise_status(a.status, MOEDISP_STATUS_CAPACITY);
            d = -1;
        }
        if (d < 0) d = -1;
        if (!__ballot_sync(0xffffffffu, d >= 0)) continue;          // same in every warp
        const uint4* xr = a.recv + g * a.H8;
        uint4 v[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int cc = gt + j * GT;
            v[j] = cc < a.H8 ? __ldcg(xr + cc) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (Q == MOEDISP_QUANT_NONE) {
            for (int k = 0; k < K; ++k) {
                const int32_t dk = __shfl_sync(0xffffffffu, d, k);
                if (dk < 0) continue;
                uint4* dst = reinterpret_cast<uint4*>(a.expand_x + (int64_t)dk * a.H8 * out_vec);
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    const int cc = gt + j * GT;
                    if (cc < a.H8) __stcs(dst + cc, v[j]);
                }
            }
            continue;
        }
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < CPT; ++j) m = fmaxf(m, absmax8(v[j]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (WPT > 1) {
            if (lane == 0) red[grp][parity][gw] = m;
            group_barrier(1 + grp, GT);
#pragma unroll
            for (int w = 0; w < WPT; ++w) m = fmaxf(m, red[grp][parity][w]);
            parity ^= 1;
        }
        const float scale = __fdiv_rn(m, kQmax);
        const float inv = __frcp_rn(scale);
        const bool zero = m == 0.0f;
        uint2 q[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) q[j] = quant8<Q == MOEDISP_QUANT_NONE ? MOEDISP_QUANT_INT8 : Q>(v[j], scale, inv, zero);
        for (int k = 0; k < K; ++k) {
            const int32_t dk = __shfl_sync(0xffffffffu, d, k);
            if (dk < 0) continue;
            uint2* dst = reinterpret_cast<uint2*>(a.expand_x + (int64_t)dk * a.H8 * out_vec);
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const int cc = gt + j * GT;
                if (cc < a.H8) __stcs(dst + cc, q[j]);
            }
            if (gt == 0) a.scales[dk] = scale;
        }
    }
}

template <int Q, int WPT, int CPT>
__global__ void __launch_bounds__(kPipeThreads, CPT > 4 ? 2 : 4) pipe_main_kernel(PipeArgs a, DispatchCounts rc) {
    constexpr int NG = kPipeThreads / 32 / WPT;
    extern __shared__ int32_t off_sh[];                  // [U + 1] the ticket-slot offsets
    __shared__ float red[NG][2][WPT];
    __shared__ long long t_sh;
    grid_dep_wait();
    grid_dep_launch_dependents();
    if (a.roles & MOEDISP_PIPE_CONSUME) write_dispatch_counts(rc);
    const int64_t S = (int64_t)a.W * a.W;
    const int64_t U = 2 * S + 1;
    // Every work item looks its ticket up among the slot offsets: unless W is large, a block
    // copies them into shared memory once (there are at most 2*W*T items, below 2^31 by the
    // host's bound on W*T*K), so the lookups are not chains of dependent global loads.
    const bool sh = a.offsets_in_smem;
    if (sh) {
        for (int64_t u = threadIdx.x; u <= U; u += blockDim.x) off_sh[u] = (int32_t)__ldcg(a.item_off + u);
        __syncthreads();
    }
    auto off = [&](int64_t u) -> int64_t { return sh ? (int64_t)off_sh[u] : __ldcg(a.item_off + u); };
    const int64_t total = off(U);
    int parity = 0;
    while (true) {
        __syncthreads();                                   // t_sh of the last item is read
        if (threadIdx.x == 0) t_sh = (long long)atomicAdd(a.ticket, 1ull);
        __syncthreads();
        const int64_t t = t_sh;
        if (t >= total) break;
        int64_t lo = 0, hi = U;                            // off(lo) <= t < off(hi)
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if (off(mid) <= t) lo = mid; else hi = mid;
        }
        bool prod;
        int64_t s;
        slot_of(lo, &prod, &s);
        const int64_t k = t - off(lo);
        if (prod) produce(a, s, k);
        else consume<Q, WPT, CPT>(a, s, k, red, parity);
    }
}

template <int Q, int WPT, int CPT>
cudaError_t launch_pipe_w(PipeArgs a, const DispatchCounts& rc, cudaStream_t stream) {
    constexpr int NG = kPipeThreads / 32 / WPT;
    a.tokens_per_item = (int64_t)NG * kConsumerRounds;
    int per_sm = 1;
    const size_t table = (size_t)(2 * (int64_t)a.W * a.W + 2) * sizeof(int32_t);
    a.offsets_in_smem = table <= 48 * 1024;                      // W <= 78
    const size_t smem = a.offsets_in_smem ? table : 0;
    cudaError_t err = blocks_per_sm((const void*)pipe_main_kernel<Q, WPT, CPT>, kPipeThreads, smem, &per_sm);
    if (err != cudaSuccess) return err;
    err = launch_pdl(pipe_setup_kernel, dim3(1), dim3(kSetupThreads), 0, stream, 1, a);
    if (err != cudaSuccess) return err;
    const int64_t grid = (int64_t)current_sm_count() * per_sm;
    return launch_pdl(pipe_main_kernel<Q, WPT, CPT>, dim3((unsigned)grid), dim3(kPipeThreads), smem,
                      stream, 1, a, rc);
}

template <int Q>
cudaError_t launch_pipe_q(const PipeArgs& a, const DispatchCounts& rc, cudaStream_t stream) {
    const int nvec = a.H8;
    if (nvec <= 32) return launch_pipe_w<Q, 1, 1>(a, rc, stream);
    if (nvec <= 64) return launch_pipe_w<Q, 1, 2>(a, rc, stream);
    if (nvec <= 128) return launch_pipe_w<Q, 1, 4>(a, rc, stream);
    if (nvec <= 256) return launch_pipe_w<Q, 2, 4>(a, rc, stream);
    if (nvec <= 512) return launch_pipe_w<Q, 4, 4>(a, rc, stream);
    if (nvec <= 1024) return launch_pipe_w<Q, 8, 4>(a, rc, stream);
    return launch_pipe_w<Q, 8, 8>(a, rc, stream);
}

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
}  // namespace

size_t pipeline_workspace_bytes(int W) {
    const size_t S = (size_t)W * W;
    return al256(16) + al256(S * 4) + al256((2 * S + 2) * 8);
}

cudaError_t launch_a2a_dispatch_pipelined(const void* in, int64_t in_rank_stride_rows,
                                          const int64_t* src_offsets, const int64_t* out_splits,
                                          const int64_t* dst_offsets, void* recv, int H,
                                          const moedisp_dims& dims, const moedisp_layout& L,
                                          int quant_mode, void* expand_x, float* dynamic_scales,
                                          int64_t* expert_token_nums, int expert_token_nums_type,
                                          int32_t* ep_recv_counts, uint32_t* ready, uint32_t epoch,
                                          int roles, uint64_t limit_ns, void* workspace,
                                          int32_t* status, cudaStream_t stream) {
    const size_t S = (size_t)dims.W * dims.W;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    PipeArgs a;
    a.in = static_cast<const uint4*>(in);
    a.in_stride = in_rank_stride_rows;
    a.src_off = src_offsets;
    a.out_splits = out_splits;
    a.dst_off = dst_offsets;
    a.recv = static_cast<uint4*>(recv);
    a.W = dims.W;
    a.T = dims.T;
    a.K = dims.K;
    a.H8 = H / 8;
    a.rows_per_piece = std::max<int64_t>(1, kPieceBytes / ((int64_t)H * 2));
    a.tokens_per_item = 1;
    a.offsets_in_smem = false;
    a.roles = roles;
    a.epoch = epoch;
    a.ready = ready;
    a.limit_ns = limit_ns;
    a.ticket = reinterpret_cast<unsigned long long*>(ws);
    a.abort_flag = reinterpret_cast<uint32_t*>(ws + 8);
    a.landed = reinterpret_cast<uint32_t*>(ws + al256(16));
    a.item_off = reinterpret_cast<int64_t*>(ws + al256(16) + al256(S * 4));
    a.dst_row = L.dst_row;
    a.rows_cap = L.rows_cap;
    a.expand_x = static_cast<uint8_t*>(expand_x);
    a.scales = dynamic_scales;
    a.status = status;
    DispatchCounts rc;
    rc.cnt = L.cnt;
    rc.expert_base = L.expert_base;
    rc.rank_base = L.rank_base;
    rc.W = dims.W;
    rc.E = dims.E;
    rc.ne = dims.E / dims.W;
    rc.etn = expert_token_nums;
    rc.etn_type = expert_token_nums_type;
    rc.erc = ep_recv_counts;
    switch (quant_mode) {
        case MOEDISP_QUANT_NONE: return launch_pipe_q<MOEDISP_QUANT_NONE>(a, rc, stream);
        case MOEDISP_QUANT_INT8: return launch_pipe_q<MOEDISP_QUANT_INT8>(a, rc, stream);
        case MOEDISP_QUANT_FP8_E4M3: return launch_pipe_q<MOEDISP_QUANT_FP8_E4M3>(a, rc, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moedisp
