// MoE dispatch layout: a stable counting sort of the G*K (token, expert) slots by expert.
//
// The PyTorch symm_mem change computes the same thing in three separate pieces: a
// per-rank histogram of the top-k ids (torch.histc), the 0-based occurrence number of
// every slot (get_occurrence_numbers, an n_unique x n indicator matrix and a cumsum) and
// a one-block 2-D exchange plan (make2dExchangePlan) whose per-expert destination offsets
// the index-push kernel adds to the occurrence number. Here one pass does all of it:
//
//  kernel 1 (layout_hist_kernel): slots are cut into tiles of kTile slots that never
//    straddle a source rank. Each block counts its tile per expert with a
//    warp-aggregated shared-memory histogram (the lanes that share an expert are found
//    with one ballot per bit of the expert id; the group's lowest lane adds the group
//    size), writes the tile's
//    counts and clears the tile's look-back words. The last block to finish (atomic
//    ticket after a fence) reduces the tiles to cnt[r][e], scans over source ranks
//    (colprefix) and over experts (expert_base, rank_base), and forms send_splits.
//  kernel 2 (layout_scatter_kernel): blocks take tiles in ticket order. Each warp ranks
//    its part of the tile by the popcount of its lower peers (same ballots), on top of
//    a per-warp running count; the warps' counts are scanned per expert; the tile's
//    per-expert offset among all earlier tiles comes from a decoupled look-back (each
//    tile publishes its aggregate, then walks back over predecessors' status words in
//    windows of kWindow until it meets an inclusive prefix); finally every slot is
//    scattered: dst_row, occ and assist_info.
//
// When the whole problem fits one thread-block cluster (at most 16 rank-aligned tiles of
// at most 16384 slots), a single kernel replaces both: one 1024-thread block per tile
// ranks its slots as above, the blocks exchange their per-expert tile counts through
// distributed shared memory across the cluster barrier, and every block derives its
// tile offsets, the expert bases and the per-rank counts from those counts directly --
// no global scratch, no second launch, no look-back.
#include "common.cuh"
#include "kernels.h"

#include <cooperative_groups.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

namespace cg = cooperative_groups;

namespace moedisp {

namespace {
constexpr int kTile = 2048;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSlotsPerWarp = kTile / kWarps;
constexpr int kSteps = kSlotsPerWarp / 32;
constexpr int kWindow = 16;
constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagInclusive = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1;
// Shared memory that kernel 1's last block may use to hold cnt while it scans.
constexpr size_t kFinalizeSmemLimit = 160 * 1024;
// Single-kernel cluster path.
constexpr int kCThreads = 1024;
constexpr int kCWarps = kCThreads / 32;
constexpr int kCMaxSteps = 16;                          // 32-slot steps per warp
constexpr int64_t kCMaxTile = (int64_t)kCWarps * 32 * kCMaxSteps;   // 16384 slots
constexpr int kCMaxCluster = 16;

struct LayoutArgs {
    const int32_t* ids;
    const uint8_t* active;
    int W, T, K, E, ne;
    int64_t P;                 // slots per source rank, T*K
    int tiles_per_rank;
    int n_tiles;
    int cnt_in_smem;
    int32_t* cnt;
    int32_t* occ;
    int32_t* dst_row;
    int32_t* assist;
    int64_t* expert_base;
    int64_t* rank_base;
    int64_t* send_splits;
    int64_t rows_cap;
    uint32_t* counters;        // [0] blocks done in kernel 1, [1] tile ticket of kernel 2
    int32_t* tile_hist;        // [n_tiles][E]
    uint32_t* lookback;        // [n_tiles][E]
    int32_t* colprefix;        // [W][E] slots of expert e in source ranks < r
    int32_t* status;
};

__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Expert of slot s if the slot is active, else -1. `bad` is set for an active token's
// out-of-range id.
__device__ __forceinline__ int slot_expert(const LayoutArgs& a, int64_t s, bool& bad) {
    const int e = __ldg(a.ids + s);
    // s < 2^30 (checked on the host), so a 32-bit division finds the token.
    if (a.active != nullptr && __ldg(a.active + (uint32_t)s / (uint32_t)a.K) == 0) return -1;
    if (e < 0 || e >= a.E) {
        bad = true;
        return -1;
    }
    return e;
}

// Lanes of the warp whose key equals this lane's key (0 <= key < 2^bits): the AND, over
// the key's bits, of the ballot of lanes agreeing with this lane on that bit. `bits` must
// be the same in every lane. One ballot per bit, no match instruction.
__device__ __forceinline__ unsigned peers_by_ballot(unsigned key, int bits) {
    unsigned m = 0xffffffffu;
#pragma unroll
    for (int b = 0; b < 11; ++b) {
        if (b < bits) {
            const unsigned bit = (key >> b) & 1u;
            const unsigned bal = __ballot_sync(0xffffffffu, bit);
            m &= bit ? bal : ~bal;
        }
    }
    return m;
}

// Bits needed for the keys 0..E (expert + 1, 0 = no expert).
__host__ __device__ __forceinline__ int key_bits(int E) {
    int b = 1;
    while ((1 << b) <= E) ++b;
    return b;
}

__device__ void layout_finalize(const LayoutArgs& a, int32_t* smem) {
    __shared__ int64_t warp_tot[32];
    const int W = a.W, E = a.E, tpr = a.tiles_per_rank;
    int64_t* ebase = reinterpret_cast<int64_t*>(smem);            // [E + 1]
    int32_t* cnt_s = reinterpret_cast<int32_t*>(ebase + E + 1);   // [W * E] if it fits
    int32_t* cnt_src = a.cnt_in_smem ? cnt_s : a.cnt;

    // cnt[r][e]: sum of the tile counts of rank r.
    for (int idx = threadIdx.x; idx < W * E; idx += blockDim.x) {
        const int r = idx / E, e = idx - r * E;
        const int32_t* th = a.tile_hist + (int64_t)r * tpr * E + e;
        int32_t sum = 0;
#pragma unroll 8
        for (int c = 0; c < tpr; ++c) sum += __ldcg(th + (int64_t)c * E);
        a.cnt[idx] = sum;
        if (a.cnt_in_smem) cnt_s[idx] = sum;
    }
    __syncthreads();
    // Per expert: prefix over source ranks, total; then exclusive scan over experts.
    int64_t carry = 0;
    for (int base = 0; base < E; base += blockDim.x) {
        const int e = base + threadIdx.x;
        int64_t tot = 0;
        if (e < E) {
            for (int r = 0; r < W; ++r) {
                a.colprefix[(int64_t)r * E + e] = (int32_t)tot;
                tot += a.cnt_in_smem ? cnt_s[r * E + e] : __ldcg(cnt_src + (int64_t)r * E + e);
            }
        }
        int64_t chunk;
        const int64_t ex = block_exclusive_scan(tot, warp_tot, chunk);
        if (e < E) ebase[e] = carry + ex;
        carry += chunk;
    }
    if (threadIdx.x == 0) ebase[E] = carry;
    __syncthreads();
    const int64_t R = ebase[E];
    for (int e = threadIdx.x; e <= E; e += blockDim.x) a.expert_base[e] = ebase[e];
    for (int d = threadIdx.x; d <= W; d += blockDim.x) a.rank_base[d] = d < W ? ebase[d * a.ne] : R;
    for (int idx = threadIdx.x; idx < W * W; idx += blockDim.x) {
        const int r = idx / W, d = idx - r * W;
        int64_t sum = 0;
        for (int le = 0; le < a.ne; ++le) {
            const int e = d * a.ne + le;
            sum += a.cnt_in_smem ? cnt_s[r * E + e] : __ldcg(cnt_src + (int64_t)r * E + e);
        }
        a.send_splits[idx] = sum;
    }
    if (threadIdx.x == 0) {
        if (R > a.rows_cap) raise_status(a.status, MOEDISP_STATUS_CAPACITY);
        a.counters[0] = 0;   // ready for the next call
        a.counters[1] = 0;   // tile ticket of kernel 2
    }
}

__global__ void __launch_bounds__(kThreads) layout_hist_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int32_t smem[];
    __shared__ int is_last;
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int tile = blockIdx.x;
    const int r = tile / a.tiles_per_rank, c = tile - r * a.tiles_per_rank;
    const int64_t base = (int64_t)r * a.P;
    const int64_t lo = (int64_t)c * kTile, hi = min64(lo + kTile, a.P);
    const int lane = threadIdx.x & 31;

    int32_t* hist = smem;
    const int kb = key_bits(a.E);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    bool bad = false;
    for (int64_t l0 = lo; l0 < hi; l0 += blockDim.x) {
        const int64_t l = l0 + threadIdx.x;
        const int e = l < hi ? slot_expert(a, base + l, bad) : -1;
        const unsigned peers = peers_by_ballot((unsigned)(e + 1), kb);
        if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[e], __popc(peers));
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(a.status, MOEDISP_STATUS_BAD_EXPERT_ID);
    __syncthreads();
    int32_t* th = a.tile_hist + (int64_t)tile * a.E;
    uint32_t* lb = a.lookback + (int64_t)tile * a.E;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        th[e] = hist[e];
        lb[e] = 0;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(&a.counters[0], 1u) == (unsigned)(a.n_tiles - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    layout_finalize(a, smem);
}

__global__ void __launch_bounds__(kThreads) layout_scatter_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int32_t smem[];
    __shared__ int tile_s;
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int E = a.E;
    int32_t* warp_cnt = smem;                    // [kWarps][E]
    int32_t* tile_off = smem + kWarps * E;       // [E]
    if (threadIdx.x == 0) tile_s = (int)atomicAdd(&a.counters[1], 1u);
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) warp_cnt[i] = 0;
    __syncthreads();
    const int tile = tile_s;
    const int r = tile / a.tiles_per_rank, c = tile - r * a.tiles_per_rank;
    const int64_t base = (int64_t)r * a.P;
    const int64_t lo = (int64_t)c * kTile, hi = min64(lo + kTile, a.P);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lower = (1u << lane) - 1u;
    int32_t* mine = warp_cnt + warp * E;
    const int64_t wlo = lo + (int64_t)warp * kSlotsPerWarp;

    int ev[kSteps];
    int rk[kSteps];
    bool bad = false;
#pragma unroll
    for (int st = 0; st < kSteps; ++st) {
        const int64_t l = wlo + st * 32 + lane;
        ev[st] = l < hi ? slot_expert(a, base + l, bad) : -1;
    }
    // Rank within the warp's part, in slot order, on top of the warp's running counts.
    const int kb = key_bits(E);
#pragma unroll
    for (int st = 0; st < kSteps; ++st) {
        const int e = ev[st];
        const unsigned peers = peers_by_ballot((unsigned)(e + 1), kb);
        const int before = e >= 0 ? mine[e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) mine[e] = before + __popc(peers);
        __syncwarp();
        rk[st] = before + __popc(peers & lower);
    }
    __syncthreads();
    // Exclusive scan of the warps' counts per expert; the tile's count per expert.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const int32_t t = warp_cnt[w * E + e];
            warp_cnt[w * E + e] = run;
            run += t;
        }
        tile_off[e] = run;
    }
    __syncthreads();
    // Decoupled look-back: the number of slots of expert e in all earlier tiles.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const uint32_t count = (uint32_t)tile_off[e];
        uint32_t* my_word = a.lookback + (int64_t)tile * E + e;
        uint32_t excl = 0;
        if (tile == 0) {
            st_relaxed(my_word, kFlagInclusive | count);
        } else {
            st_relaxed(my_word, kFlagAggregate | count);
            int p = tile - 1;
            uint64_t t0 = 0;
            while (p >= 0) {
                const int n = min(kWindow, p + 1);
                uint32_t w[kWindow];
#pragma unroll
                for (int i = 0; i < kWindow; ++i)
                    w[i] = i < n ? ld_relaxed(a.lookback + (int64_t)(p - i) * E + e) : 0u;
                int used = 0;
                bool stop = false, found = false;
#pragma unroll
                for (int i = 0; i < kWindow; ++i) {
                    if (!stop && i < n) {
                        const uint32_t f = w[i] & ~kValueMask;
                        if (f == 0) {
                            stop = true;
                        } else {
                            excl += w[i] & kValueMask;
                            used = i + 1;
                            if (f == kFlagInclusive) found = stop = true;
                        }
                    }
                }
                if (found) break;
                p -= used;
                if (used < n) {           // predecessor p has not published yet
                    const uint64_t now = global_timer_ns();
                    if (t0 == 0) t0 = now;
                    else if (now - t0 > kWaitLimitNs) {
                        raise_status(a.status, MOEDISP_STATUS_TIMEOUT);
                        break;
                    }
                    __nanosleep(64);
                }
            }
            st_relaxed(my_word, kFlagInclusive | ((excl + count) & kValueMask));
        }
        tile_off[e] = (int32_t)excl;
    }
    __syncthreads();
    // Stable scatter.
    const int32_t* colp = a.colprefix + (int64_t)r * E;
#pragma unroll
    for (int st = 0; st < kSteps; ++st) {
        const int64_t l = wlo + st * 32 + lane;
        if (l >= hi) continue;
        const int64_t s = base + l;
        const int e = ev[st];
        if (e < 0) {
            a.dst_row[s] = -1;
            a.occ[s] = -1;
            continue;
        }
        const int32_t within = tile_off[e] + mine[e] + rk[st];   // earlier slots of e, all ranks
        const int64_t row = __ldg(a.expert_base + e) + within;
        a.occ[s] = within - __ldg(colp + e);
        a.dst_row[s] = (int32_t)row;
        if (row < a.rows_cap) a.assist[row] = (int32_t)s;
    }
}


__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// STEPS = 32-slot steps per warp (a power of two, at most kCMaxSteps).
template <int STEPS>
__global__ void __launch_bounds__(kCThreads, 1)
layout_cluster_kernel(LayoutArgs a, int64_t tile_len) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int64_t warp_tot[32];
    cg::cluster_group cluster = cg::this_cluster();
    const int E = a.E, W = a.W, tpr = a.tiles_per_rank;
    const int ES = E | 1;                                        // odd row stride: no bank conflicts
    int64_t* ebase = reinterpret_cast<int64_t*>(smem_raw);      // [E + 1]
    int32_t* wc = reinterpret_cast<int32_t*>(ebase + E + 1);    // [kCWarps][ES]
    int32_t* tcnt = wc + kCWarps * ES;                           // [E] this tile's counts
    int32_t* tpre = tcnt + E;                                    // [E] counts in earlier tiles
    int32_t* colp = tpre + E;                                    // [E] counts in earlier ranks
    int32_t* cntr = colp + E;                                    // [E] counts of this rank

    const int tile = (int)cluster.block_rank();
    const int C = (int)cluster.num_blocks();
    const int r = tile / tpr, c = tile - r * tpr;
    const int64_t base = (int64_t)r * a.P;
    const int64_t lo = (int64_t)c * tile_len, hi = min64(lo + tile_len, a.P);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lower = (1u << lane) - 1u;
    for (int i = threadIdx.x; i < kCWarps * ES; i += blockDim.x) wc[i] = 0;
    grid_dep_wait();
    grid_dep_launch_dependents();

    // Each warp owns STEPS*32 consecutive slots of the tile.
    int32_t* mine = wc + warp * ES;
    const int64_t wlo = lo + (int64_t)warp * STEPS * 32;
    int ev[STEPS];
    bool bad = false;
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
        const int64_t l = wlo + st * 32 + lane;
        ev[st] = l < hi ? slot_expert(a, base + l, bad) : -1;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(a.status, MOEDISP_STATUS_BAD_EXPERT_ID);
    __syncthreads();
    // Rank within the warp's slots, in slot order: packed as (rank << 11) | (expert + 1).
    uint32_t pk[STEPS];
    const int kb = key_bits(E);
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
        const int e = ev[st];
        const unsigned peers = peers_by_ballot((unsigned)(e + 1), kb);
        const int before = e >= 0 ? mine[e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) mine[e] = before + __popc(peers);
        __syncwarp();
        pk[st] = e >= 0 ? ((uint32_t)(before + __popc(peers & lower)) << 11) | (uint32_t)(e + 1) : 0u;
    }
    __syncthreads();
    // Per expert, an exclusive scan over the 32 warps' counts: one warp per expert,
    // lane w holding warp w's count.
    for (int e = warp; e < E; e += kCWarps) {
        const int32_t v = wc[lane * ES + e];
        const int32_t inc = warp_inclusive_scan_i32(v);
        wc[lane * ES + e] = inc - v;
        if (lane == 31) tcnt[e] = inc;
    }
    cluster.sync();   // every tile's counts are final and visible across the cluster

    // Counts of every tile, read from the other blocks' shared memory (all reads issued
    // together): offsets of this tile and of this rank, this rank's row of cnt, and the
    // expert totals, scanned into expert bases.
    int64_t carry = 0;
    for (int b0 = 0; b0 < E; b0 += blockDim.x) {
        const int e = b0 + threadIdx.x;
        int64_t tot = 0;
        if (e < E) {
            int32_t v[kCMaxCluster];
#pragma unroll
            for (int t = 0; t < kCMaxCluster; ++t)
                v[t] = t < C ? cluster.map_shared_rank(tcnt, t)[e] : 0;
            int32_t pre = 0, cp = 0, cr = 0;
#pragma unroll
            for (int t = 0; t < kCMaxCluster; ++t) {
                tot += v[t];
                pre += t < tile ? v[t] : 0;
                cp += t < r * tpr ? v[t] : 0;
                cr += (t >= r * tpr && t < (r + 1) * tpr) ? v[t] : 0;
            }
            tpre[e] = pre;
            colp[e] = cp;
            cntr[e] = cr;
        }
        int64_t chunk;
        const int64_t ex = block_exclusive_scan(tot, warp_tot, chunk);
        if (e < E) ebase[e] = carry + ex;
        carry += chunk;
    }
    if (threadIdx.x == 0) ebase[E] = carry;
    // This block reads no other block's shared memory from here on; it keeps its own
    // (which the others may still be reading) until the matching wait at the end.
    cluster_arrive_release();
    __syncthreads();

    const int64_t R = ebase[E];
    if (tile == 0) {
        for (int e = threadIdx.x; e <= E; e += blockDim.x) a.expert_base[e] = ebase[e];
        for (int d = threadIdx.x; d <= W; d += blockDim.x) a.rank_base[d] = d < W ? ebase[d * a.ne] : R;
        if (threadIdx.x == 0 && R > a.rows_cap) raise_status(a.status, MOEDISP_STATUS_CAPACITY);
    }
    if (c == 0) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) a.cnt[(int64_t)r * E + e] = cntr[e];
        for (int d = threadIdx.x; d < W; d += blockDim.x) {
            int64_t sum = 0;
            for (int le = 0; le < a.ne; ++le) sum += cntr[d * a.ne + le];
            a.send_splits[(int64_t)r * W + d] = sum;
        }
    }
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
        const int64_t l = wlo + st * 32 + lane;
        if (l >= hi) continue;
        const int64_t s = base + l;
        if (pk[st] == 0u) {
            a.dst_row[s] = -1;
            a.occ[s] = -1;
            continue;
        }
        const int e = (int)(pk[st] & 2047u) - 1;
        const int32_t within = tpre[e] + mine[e] + (int32_t)(pk[st] >> 11);
        const int64_t row = ebase[e] + within;
        a.occ[s] = within - colp[e];
        a.dst_row[s] = (int32_t)row;
        if (row < a.rows_cap) a.assist[row] = (int32_t)s;
    }
    cluster_wait_acquire();
}

// Cluster path geometry: tiles per rank and slots per tile, or false if the problem does
// not fit one cluster.
bool cluster_geometry(const moedisp_dims& d, int* tpr, int64_t* tile_len, int* steps) {
    const int64_t P = (int64_t)d.T * d.K;
    const int64_t need = std::max<int64_t>(1, (P + kCMaxTile - 1) / kCMaxTile);
    const int64_t want = std::min<int64_t>((P + 1023) / 1024, kCMaxCluster / std::max(1, d.W));
    const int64_t t = std::max(need, want);
    if ((int64_t)d.W * t > kCMaxCluster) return false;
    *tpr = (int)t;
    *tile_len = (P + t - 1) / t;
    const int need_steps = (int)((*tile_len + kCThreads - 1) / kCThreads);
    int p2 = 1;
    while (p2 < need_steps) p2 <<= 1;
    *steps = p2;
    return p2 <= kCMaxSteps;
}

size_t cluster_smem(int E) {
    return (size_t)(E + 1) * sizeof(int64_t) + ((size_t)kCWarps * (E | 1) + 4 * (size_t)E) * sizeof(int32_t);
}

// Whether a cluster of C blocks of this kernel can be resident on the current device.
cudaError_t cluster_fits(const void* kernel, int C, size_t smem, bool* ok) {
    static std::mutex mu;
    static std::map<std::tuple<int, const void*, int, size_t>, bool> cache;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find({dev, kernel, C, smem});
        if (it != cache.end()) {
            *ok = it->second;
            return cudaSuccess;
        }
    }
    err = allow_dynamic_smem(kernel);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(C);
    cfg.blockDim = dim3(kCThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    err = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
    if (err != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    cache[{dev, kernel, C, smem}] = n > 0;
    *ok = n > 0;
    return cudaSuccess;
}

// Launches the two-kernel path (histogram, then ranking + look-back + scatter) on the
// workspace pointers already in `a`.
cudaError_t launch_tiled(LayoutArgs& a, const moedisp_dims& dims, const LayoutGeometry& g,
                         cudaStream_t stream) {
    const size_t fin_base = (size_t)(dims.E + 1) * sizeof(int64_t);
    const size_t fin_cnt = (size_t)dims.W * dims.E * sizeof(int32_t);
    a.cnt_in_smem = fin_base + fin_cnt <= kFinalizeSmemLimit;
    size_t smem1 = std::max((size_t)dims.E * sizeof(int32_t), fin_base + (a.cnt_in_smem ? fin_cnt : 0));
    smem1 = (smem1 + 15) & ~(size_t)15;
    const size_t smem2 = (size_t)(kWarps + 1) * dims.E * sizeof(int32_t);

    cudaError_t err = allow_dynamic_smem((const void*)layout_hist_kernel);
    if (err != cudaSuccess) return err;
    err = allow_dynamic_smem((const void*)layout_scatter_kernel);
    if (err != cudaSuccess) return err;
    err = launch_pdl(layout_hist_kernel, dim3((unsigned)g.n_tiles), dim3(kThreads), smem1, stream, 1, a);
    if (err != cudaSuccess) return err;
    return launch_pdl(layout_scatter_kernel, dim3((unsigned)g.n_tiles), dim3(kThreads), smem2, stream,
                      1, a);
}

}  // namespace

LayoutGeometry layout_geometry(const moedisp_dims& d) {
    LayoutGeometry g{};
    g.slots_per_rank = (int64_t)d.T * d.K;
    g.tiles_per_rank = (int)std::max<int64_t>(1, (g.slots_per_rank + kTile - 1) / kTile);
    g.n_tiles = (int64_t)d.W * g.tiles_per_rank;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t off = 256;                                       // counters
    g.off_tile_hist = off;
    off += al((size_t)g.n_tiles * d.E * sizeof(int32_t));
    g.off_lookback = off;
    off += al((size_t)g.n_tiles * d.E * sizeof(uint32_t));
    g.off_colprefix = off;
    off += al((size_t)d.W * d.E * sizeof(int32_t));
    g.total_bytes = off;
    return g;
}

namespace {
LayoutArgs make_args(const int32_t* expert_ids, const uint8_t* active, const moedisp_dims& dims,
                     const moedisp_layout& L, void* workspace, int32_t* status,
                     const LayoutGeometry& g) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    LayoutArgs a;
    a.ids = expert_ids;
    a.active = active;
    a.W = dims.W;
    a.T = dims.T;
    a.K = dims.K;
    a.E = dims.E;
    a.ne = dims.E / dims.W;
    a.P = g.slots_per_rank;
    a.tiles_per_rank = g.tiles_per_rank;
    a.n_tiles = (int)g.n_tiles;
    a.cnt = L.cnt;
    a.occ = L.occ;
    a.dst_row = L.dst_row;
    a.assist = L.assist_info;
    a.expert_base = L.expert_base;
    a.rank_base = L.rank_base;
    a.send_splits = L.send_splits;
    a.rows_cap = L.rows_cap;
    a.counters = reinterpret_cast<uint32_t*>(ws);
    a.tile_hist = reinterpret_cast<int32_t*>(ws + g.off_tile_hist);
    a.lookback = reinterpret_cast<uint32_t*>(ws + g.off_lookback);
    a.colprefix = reinterpret_cast<int32_t*>(ws + g.off_colprefix);
    a.status = status;
    return a;
}
}  // namespace

cudaError_t launch_layout(const int32_t* expert_ids, const uint8_t* active,
                          const moedisp_dims& dims, const moedisp_layout& L, void* workspace,
                          int32_t* status, cudaStream_t stream) {
    const LayoutGeometry g = layout_geometry(dims);
    LayoutArgs a = make_args(expert_ids, active, dims, L, workspace, status, g);

    int tpr_c = 0, steps_c = 0;
    int64_t tile_c = 0;
    if (cluster_geometry(dims, &tpr_c, &tile_c, &steps_c)) {
        const int C = dims.W * tpr_c;
        const size_t smem = cluster_smem(dims.E);
        void (*kernel)(LayoutArgs, int64_t) =
            steps_c == 1 ? layout_cluster_kernel<1> : steps_c == 2 ? layout_cluster_kernel<2>
            : steps_c == 4 ? layout_cluster_kernel<4> : steps_c == 8 ? layout_cluster_kernel<8>
                           : layout_cluster_kernel<16>;
        bool ok = false;
        cudaError_t err = cluster_fits((const void*)kernel, C, smem, &ok);
        if (err != cudaSuccess) return err;
        if (ok) {
            a.tiles_per_rank = tpr_c;
            a.n_tiles = C;
            return launch_pdl(kernel, dim3(C), dim3(kCThreads), smem, stream, C, a, tile_c);
        }
    }

    return launch_tiled(a, dims, g, stream);
}

// ------------------------------------------------------------ allocation-free variant
//
// Scratch of moedisp_moe_dispatch_layout_noalloc: the two-kernel path's workspace kept in
// this library's own device memory (present on every GPU that loads the library, until
// the process exits), so the caller passes no workspace and nothing is allocated.
static __device__ __align__(256) unsigned char g_layout_scratch[MOEDISP_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of g_layout_scratch on the current device. The host-side name of a
// __device__ array is only a stand-in, so the address is looked up once per device
// (with that device current) and cached.
cudaError_t layout_scratch_address(void** out) {
    static std::mutex mu;
    static std::map<int, void*> cache;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_layout_scratch);
    if (err != cudaSuccess) return err;
    cache[dev] = p;
    *out = p;
    return cudaSuccess;
}
}  // namespace

size_t layout_noalloc_scratch_bytes() { return MOEDISP_NOALLOC_SCRATCH_BYTES; }

cudaError_t launch_layout_noalloc(const int32_t* expert_ids, const uint8_t* active,
                                  const moedisp_dims& dims, const moedisp_layout& L,
                                  int32_t* status, cudaStream_t stream) {
    const LayoutGeometry g = layout_geometry(dims);
    void* scratch = nullptr;
    cudaError_t err = layout_scratch_address(&scratch);
    if (err != cudaSuccess) return err;
    // The array keeps whatever the previous call left: clear the two counters that must
    // start at zero (every other scratch word is written before it is read).
    err = cudaMemsetAsync(scratch, 0, 256, stream);
    if (err != cudaSuccess) return err;
    LayoutArgs a = make_args(expert_ids, active, dims, L, scratch, status, g);
    return launch_tiled(a, dims, g, stream);
}

}  // namespace moedisp
