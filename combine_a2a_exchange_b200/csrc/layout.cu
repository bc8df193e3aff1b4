// MoE dispatch layout: a stable counting sort of the G*K (token, expert) slots by expert.
//
// The PyTorch symm_mem change computes the same thing in separate pieces: a per-rank
// histogram of the top-k ids (torch.histc), the 0-based occurrence number of every slot
// (get_occurrence_numbers, an n_unique x n indicator matrix and a cumsum) and a one-block
// 2-D exchange plan (make2dExchangePlan) whose per-expert destination offsets the
// index-push kernel adds to the occurrence number. Here the slots are cut into tiles that
// never straddle a source rank, and:
//
//  * small problems (at most 16 tiles of at most 2048 slots): one kernel, one thread-block
//    cluster. Each 256-thread block ranks its tile (below) and pushes its per-expert tile
//    counts into every block's shared memory (distributed shared memory stores, before
//    the cluster barrier); every block then derives its tile offsets, the expert bases and
//    the per-rank counts from its local copy -- no global scratch, no second launch, no
//    remote read after the barrier.
//  * larger problems: three kernels, each spread over the whole GPU.
//      count: one block per tile; a warp-aggregated shared-memory histogram -> the tile's
//             counts per expert;
//      scan:  one block per 32 experts; exclusive scans down the tiles -> per (tile,
//             expert) offsets and the expert totals;
//      rank:  one block per tile; ranks its slots (this needs only the inputs, so it runs
//             before waiting for the scan), then reads four rows of offsets, scans the
//             totals into expert bases and scatters dst_row, occ and assist_info.
//
// Ranking: each warp owns consecutive slots and walks them 32 at a time. The lanes that
// share an expert are found with one ballot per bit of (expert + 1) (a warp-level
// multisplit); a slot's rank is the popcount of its lower peers plus the warp's running
// count of that expert in shared memory, which the group's lowest lane then advances.
// Per expert, the warps' counts are scanned in warp order. Everything is in slot order,
// so the sort is stable and the result deterministic.
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
// Tiled (three-kernel) path.
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int64_t kTargetTiles = 296;         // about two blocks per SM
constexpr int kScanThreads = 1024;            // 32 warps: one column of experts per lane
constexpr int kScanPer = 16;                  // tiles per warp per pass (512 tiles per pass)
// Single-kernel cluster path.
constexpr int kCThreads = 256;
constexpr int kCWarps = kCThreads / 32;
constexpr int kCMaxSteps = 8;                 // tiles <= 2048 slots
constexpr int64_t kCMaxTile = (int64_t)kCWarps * 32 * kCMaxSteps;
constexpr int kCMaxCluster = 16;

struct LayoutArgs {
    const int32_t* ids;
    const uint8_t* active;     // null, [G] (per token, active_dims 1) or [G*K] (per slot, 2)
    int active_dims;
    int W, T, K, E, ne;
    int64_t align;             // major_align: expert segments padded to multiples (>= 2)
    int64_t P;                 // slots per source rank, T*K
    int tiles_per_rank;
    int n_tiles;
    int64_t tile_len;          // slots per tile (the last tile of a rank may be shorter)
    int32_t* cnt;
    int32_t* occ;
    int32_t* dst_row;
    int32_t* assist;
    int64_t* expert_base;
    int64_t* rank_base;
    int64_t* send_splits;
    int64_t rows_cap;
    int32_t* tile_hist;        // [n_tiles][E]      counts of each tile
    int32_t* tile_prefix;      // [n_tiles + 1][E]  counts in earlier tiles; last row = totals
    int32_t* status;
};

// Expert of slot s if the slot is active, else -1. `bad` is set for an active token's
// out-of-range id.
__device__ __forceinline__ int slot_expert(const LayoutArgs& a, int64_t s, bool& bad) {
    const int e = __ldg(a.ids + s);
    // s < 2^30 (checked on the host), so a 32-bit division finds the token.
    if (a.active != nullptr &&
        __ldg(a.active + (a.active_dims == 1 ? (uint32_t)s / (uint32_t)a.K : (uint32_t)s)) == 0)
        return -1;
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

// Rows of an expert's segment holding n routed rows: n, or with major_align A >= 2 the
// next multiple of A, at least A (an expert never gets an empty segment).
__device__ __forceinline__ int64_t padded_rows(int64_t n, int64_t A) {
    if (A <= 1) return n;
    const int64_t p = (n + A - 1) / A * A;
    return p < A ? A : p;
}

// Marks the padding rows of experts part, part + parts, ... as holding no slot (below
// rows_cap): each expert's range [ebase[e] + etot[e], ebase[e + 1]) is written by the whole
// block, coalesced. A no-op without major_align.
__device__ __forceinline__ void mark_padding(const LayoutArgs& a, const int64_t* ebase,
                                             const int32_t* etot, int part, int parts) {
    if (a.align <= 1) return;
    for (int e = part; e < a.E; e += parts) {
        const int64_t end = min64(ebase[e + 1], a.rows_cap);
        for (int64_t row = ebase[e] + etot[e] + threadIdx.x; row < end; row += blockDim.x)
            a.assist[row] = -1;
    }
}

// Bits needed for the keys 0..E (expert + 1, 0 = no expert).
__host__ __device__ __forceinline__ int key_bits(int E) {
    int b = 1;
    while ((1 << b) <= E) ++b;
    return b;
}

// Loads the expert of each of this lane's STEPS slots (-1 where none) and ranks them
// within the warp: packed (rank << 11) | (expert + 1), 0 for no expert. `mine` is the
// warp's running count per expert (shared memory, zeroed by the caller).
template <int STEPS>
__device__ __forceinline__ void rank_in_warp(const LayoutArgs& a, int64_t base, int64_t wlo,
                                             int64_t hi, int32_t* mine, uint32_t (&pk)[STEPS]) {
    const int lane = threadIdx.x & 31;
    const unsigned lower = (1u << lane) - 1u;
    int ev[STEPS];
    bool bad = false;
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
        const int64_t l = wlo + st * 32 + lane;
        ev[st] = l < hi ? slot_expert(a, base + l, bad) : -1;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(a.status, MOEDISP_STATUS_BAD_EXPERT_ID);
    const int kb = key_bits(a.E);
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
}

// Writes dst_row, occ and assist_info of this lane's slots. `pre` = slots of each expert
// before this tile, `colp` = before this rank, `mine` = before this warp inside the tile.
template <int STEPS>
__device__ __forceinline__ void scatter_slots(const LayoutArgs& a, int64_t base, int64_t wlo,
                                              int64_t hi, const uint32_t (&pk)[STEPS],
                                              const int32_t* pre, const int32_t* colp,
                                              const int32_t* mine, const int64_t* ebase) {
    const int lane = threadIdx.x & 31;
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
        const int32_t within = pre[e] + mine[e] + (int32_t)(pk[st] >> 11);
        const int64_t row = ebase[e] + within;
        a.occ[s] = within - colp[e];
        a.dst_row[s] = (int32_t)row;
        if (row < a.rows_cap) a.assist[row] = (int32_t)s;
    }
}

// --------------------------------------------------------------- tiled path

template <int STEPS>
__global__ void __launch_bounds__(kThreads) layout_count_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int32_t hist[];          // [E]
    const int tile = blockIdx.x;
    const int r = tile / a.tiles_per_rank, c = tile - r * a.tiles_per_rank;
    const int64_t base = (int64_t)r * a.P;
    const int64_t lo = (int64_t)c * a.tile_len, hi = min64(lo + a.tile_len, a.P);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int64_t wlo = lo + (int64_t)warp * STEPS * 32;
    int ev[STEPS];
    bool bad = false;
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
        const int64_t l = wlo + st * 32 + lane;
        ev[st] = l < hi ? slot_expert(a, base + l, bad) : -1;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(a.status, MOEDISP_STATUS_BAD_EXPERT_ID);
    const int kb = key_bits(a.E);
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
        const int e = ev[st];
        const unsigned peers = peers_by_ballot((unsigned)(e + 1), kb);
        if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[e], __popc(peers));
    }
    __syncthreads();
    int32_t* th = a.tile_hist + (int64_t)tile * a.E;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) th[e] = hist[e];
}

// Exclusive scan of tile_hist down each column (expert), 32 columns per block (lane =
// expert). In passes of up to 32 * kScanPer tiles: warp w takes a contiguous run of the
// pass's tiles, loads them all at once (coalesced rows of 32 experts) and scans them in
// registers; the warps' run totals are scanned across warps through shared memory (warp w
// scans expert column w), and the offsets are added on the way out. One round of loads
// per pass instead of a shared-memory transposition per 32 tiles (cfg3: the scan 4-6 us
// -> 2.7 us after its dependency wait; the layout 21.4 -> 17.4 us). Releasing the rank
// kernel before this kernel's wait, so that it ranks during the count and the scan, lost:
// its 256 blocks then compete with the count kernel's and finish ranking later (20 us).
__global__ void __launch_bounds__(kScanThreads) layout_scan_kernel(LayoutArgs a) {
    __shared__ int32_t wtot[32][33];                         // [warp][expert]: warp totals
    __shared__ int32_t ptot[32];                             // [expert]: the pass's totals
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    const bool valid = e < a.E;
    const int n = a.n_tiles;
    int32_t carry = 0;                                       // expert e: tiles of earlier passes
    for (int t0 = 0; t0 < n; t0 += 32 * kScanPer) {
        const int rows = min(32 * kScanPer, n - t0);
        const int per = (rows + 31) / 32;                    // tiles per warp in this pass
        const int w0 = t0 + warp * per;                      // this warp's first tile
        const int w1 = min(w0 + per, t0 + rows);
        int32_t v[kScanPer];
#pragma unroll
        for (int k = 0; k < kScanPer; ++k)                  // all loads in flight
            v[k] = (valid && w0 + k < w1) ? __ldcg(a.tile_hist + (int64_t)(w0 + k) * a.E + e) : 0;
        int32_t run = 0;                                     // exclusive prefix in the warp's run
#pragma unroll
        for (int k = 0; k < kScanPer; ++k) {
            const int32_t x = v[k];
            v[k] = run;
            run += x;
        }
        wtot[warp][lane] = run;
        __syncthreads();
        {                                                    // warp w scans expert column w
            const int32_t x = wtot[lane][warp];
            const int32_t inc = warp_inclusive_scan_i32(x);
            wtot[lane][warp] = inc - x;
            if (lane == 31) ptot[warp] = inc;
        }
        __syncthreads();
        const int32_t off = carry + wtot[warp][lane];
#pragma unroll
        for (int k = 0; k < kScanPer; ++k)
            if (valid && w0 + k < w1) a.tile_prefix[(int64_t)(w0 + k) * a.E + e] = off + v[k];
        carry += ptot[lane];
        __syncthreads();                                     // wtot / ptot are rewritten next pass
    }
    if (warp == 0 && valid) a.tile_prefix[(int64_t)n * a.E + e] = carry;   // totals row
}

template <int STEPS>
__global__ void __launch_bounds__(kThreads) layout_rank_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int64_t warp_tot[32];
    const int E = a.E, W = a.W, tpr = a.tiles_per_rank;
    const int ES = E | 1;
    int64_t* ebase = reinterpret_cast<int64_t*>(smem_raw);      // [E + 1]
    int32_t* wc = reinterpret_cast<int32_t*>(ebase + E + 1);    // [kWarps][ES]
    int32_t* pre = wc + kWarps * ES;                             // [E]
    int32_t* colp = pre + E;                                     // [E]
    int32_t* cntr = colp + E;                                    // [E]
    int32_t* etot = cntr + E;                                    // [E] rows routed to e
    const int tile = blockIdx.x;
    const int r = tile / tpr, c = tile - r * tpr;
    const int64_t base = (int64_t)r * a.P;
    const int64_t lo = (int64_t)c * a.tile_len, hi = min64(lo + a.tile_len, a.P);
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kWarps * ES; i += blockDim.x) wc[i] = 0;
    __syncthreads();

    // Ranking reads only the layout's inputs. They were complete before the count kernel
    // passed its own dependency wait, which precedes this kernel's start, so this part
    // overlaps the count and scan kernels.
    int32_t* mine = wc + warp * ES;
    const int64_t wlo = lo + (int64_t)warp * STEPS * 32;
    uint32_t pk[STEPS];
    rank_in_warp<STEPS>(a, base, wlo, hi, mine, pk);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const int32_t t = wc[w * ES + e];
            wc[w * ES + e] = run;
            run += t;
        }
    }

    grid_dep_wait();
    grid_dep_launch_dependents();
    const int32_t* tp = a.tile_prefix;
    const int64_t row_tile = (int64_t)tile * E, row_rank = (int64_t)r * tpr * E;
    const int64_t row_next = (int64_t)(r + 1) * tpr * E, row_tot = (int64_t)a.n_tiles * E;
    int64_t carry = 0;
    for (int b0 = 0; b0 < E; b0 += blockDim.x) {
        const int e = b0 + threadIdx.x;
        int64_t tot = 0;
        if (e < E) {
            pre[e] = __ldcg(tp + row_tile + e);
            const int32_t cp = __ldcg(tp + row_rank + e);
            colp[e] = cp;
            cntr[e] = __ldcg(tp + row_next + e) - cp;
            tot = __ldcg(tp + row_tot + e);
        }
        const int64_t seg = e < E ? padded_rows(tot, a.align) : 0;
        int64_t chunk;
        const int64_t ex = block_exclusive_scan(seg, warp_tot, chunk);
        if (e < E) {
            ebase[e] = carry + ex;
            etot[e] = (int32_t)tot;
        }
        carry += chunk;
    }
    if (threadIdx.x == 0) ebase[E] = carry;
    __syncthreads();
    mark_padding(a, ebase, etot, tile, a.n_tiles);

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
    scatter_slots<STEPS>(a, base, wlo, hi, pk, pre, colp, mine, ebase);
}

// ------------------------------------------------------------ cluster path

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int STEPS>
__global__ void __launch_bounds__(kCThreads, 1)
layout_cluster_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int64_t warp_tot[32];
    cg::cluster_group cluster = cg::this_cluster();
    const int E = a.E, W = a.W, tpr = a.tiles_per_rank;
    const int ES = E | 1;                                        // odd row stride: no bank conflicts
    int64_t* ebase = reinterpret_cast<int64_t*>(smem_raw);      // [E + 1]
    int32_t* wc = reinterpret_cast<int32_t*>(ebase + E + 1);    // [kCWarps][ES]
    int32_t* tpre = wc + kCWarps * ES;                           // [E] counts in earlier tiles
    int32_t* colp = tpre + E;                                    // [E] counts in earlier ranks
    int32_t* cntr = colp + E;                                    // [E] counts of this rank
    int32_t* etot = cntr + E;                                    // [E] rows routed to e
    int32_t* allc = etot + E;                                    // [C][E] every tile's counts

    const int tile = (int)cluster.block_rank();
    const int C = (int)cluster.num_blocks();
    const int r = tile / tpr, c = tile - r * tpr;
    const int64_t base = (int64_t)r * a.P;
    const int64_t lo = (int64_t)c * a.tile_len, hi = min64(lo + a.tile_len, a.P);
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kCWarps * ES; i += blockDim.x) wc[i] = 0;
    grid_dep_wait();
    grid_dep_launch_dependents();
    __syncthreads();
    // Distributed shared memory of a block may be written only once that block runs: this
    // arrival is matched by the wait before the counts are pushed (long satisfied by then).
    cluster_arrive_relaxed();

    int32_t* mine = wc + warp * ES;
    const int64_t wlo = lo + (int64_t)warp * STEPS * 32;
    uint32_t pk[STEPS];
    rank_in_warp<STEPS>(a, base, wlo, hi, mine, pk);
    __syncthreads();
    cluster_wait_acquire();
    // Per expert, an exclusive scan over the warps' counts, in warp order.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = 0;
#pragma unroll
        for (int w = 0; w < kCWarps; ++w) {
            const int32_t t = wc[w * ES + e];
            wc[w * ES + e] = run;
            run += t;
        }
        // pushed into row `tile` of every block's copy (remote stores need no round trip)
        for (int t = 0; t < C; ++t) cluster.map_shared_rank(allc, t)[tile * E + e] = run;
    }
    cluster.sync();   // every tile's counts have landed in every block (release / acquire)

    // Counts of every tile, now local: offsets of this tile and of this rank, this rank's
    // row of cnt, and the expert totals, scanned into expert bases. No block reads another
    // block's shared memory after the barrier, so blocks may finish independently.
    int64_t carry = 0;
    for (int b0 = 0; b0 < E; b0 += blockDim.x) {
        const int e = b0 + threadIdx.x;
        int64_t tot = 0;
        if (e < E) {
            int32_t v[kCMaxCluster];
#pragma unroll
            for (int t = 0; t < kCMaxCluster; ++t)
                v[t] = t < C ? allc[t * E + e] : 0;
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
        const int64_t seg = e < E ? padded_rows(tot, a.align) : 0;
        int64_t chunk;
        const int64_t ex = block_exclusive_scan(seg, warp_tot, chunk);
        if (e < E) {
            ebase[e] = carry + ex;
            etot[e] = (int32_t)tot;
        }
        carry += chunk;
    }
    if (threadIdx.x == 0) ebase[E] = carry;
    __syncthreads();
    mark_padding(a, ebase, etot, tile, C);

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
    scatter_slots<STEPS>(a, base, wlo, hi, pk, tpre, colp, mine, ebase);
}

int pow2_at_least(int64_t x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
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
    *steps = pow2_at_least((*tile_len + kCThreads - 1) / kCThreads);
    return *steps <= kCMaxSteps;
}

// Dynamic shared memory of a cluster of C blocks: expert bases, the warps' counts, four
// per-expert rows and the C pushed rows of tile counts.
size_t cluster_smem(int E, int C) {
    return (size_t)(E + 1) * sizeof(int64_t) +
           ((size_t)kCWarps * (E | 1) + (4 + (size_t)C) * (size_t)E) * sizeof(int32_t);
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

// Launches the three-kernel path on the workspace pointers already in `a`.
cudaError_t launch_tiled(LayoutArgs& a, const moedisp_dims& dims, const LayoutGeometry& g,
                         cudaStream_t stream) {
    a.tiles_per_rank = g.tiles_per_rank;
    a.n_tiles = (int)g.n_tiles;
    a.tile_len = g.tile_len;
    const int E = dims.E;
    const size_t smem_count = (size_t)E * sizeof(int32_t);
    const size_t smem_rank = (size_t)(E + 1) * sizeof(int64_t) +
                             ((size_t)kWarps * (E | 1) + 4 * (size_t)E) * sizeof(int32_t);
    void (*count)(LayoutArgs) = nullptr;
    void (*rank)(LayoutArgs) = nullptr;
    switch (g.steps) {
        case 1: count = layout_count_kernel<1>; rank = layout_rank_kernel<1>; break;
        case 2: count = layout_count_kernel<2>; rank = layout_rank_kernel<2>; break;
        case 4: count = layout_count_kernel<4>; rank = layout_rank_kernel<4>; break;
        case 8: count = layout_count_kernel<8>; rank = layout_rank_kernel<8>; break;
        default: count = layout_count_kernel<16>; rank = layout_rank_kernel<16>; break;
    }
    cudaError_t err = allow_dynamic_smem((const void*)count);
    if (err != cudaSuccess) return err;
    err = allow_dynamic_smem((const void*)rank);
    if (err != cudaSuccess) return err;
    const unsigned tiles = (unsigned)g.n_tiles;
    err = launch_pdl(count, dim3(tiles), dim3(kThreads), smem_count, stream, 1, a);
    if (err != cudaSuccess) return err;
    err = launch_pdl(layout_scan_kernel, dim3((unsigned)((E + 31) / 32)), dim3(kScanThreads), 0,
                     stream, 1, a);
    if (err != cudaSuccess) return err;
    return launch_pdl(rank, dim3(tiles), dim3(kThreads), smem_rank, stream, 1, a);
}

}  // namespace

LayoutGeometry layout_geometry(const moedisp_dims& d) {
    LayoutGeometry g{};
    g.slots_per_rank = (int64_t)d.T * d.K;
    const int64_t slots = (int64_t)d.W * g.slots_per_rank;
    // Tile size: a power of two between 512 and 4096 slots, aiming at kTargetTiles tiles;
    // tiles never straddle a rank, so a rank's last tile may be shorter.
    const int64_t want = std::min<int64_t>(4096, std::max<int64_t>(512, pow2_at_least((slots + kTargetTiles - 1) / kTargetTiles)));
    g.tiles_per_rank = (int)std::max<int64_t>(1, (g.slots_per_rank + want - 1) / want);
    g.tile_len = (g.slots_per_rank + g.tiles_per_rank - 1) / g.tiles_per_rank;
    g.steps = pow2_at_least(std::max<int64_t>(1, (g.tile_len + kThreads - 1) / kThreads));  // <= 16
    g.n_tiles = (int64_t)d.W * g.tiles_per_rank;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    g.off_tile_hist = 0;
    size_t off = al((size_t)g.n_tiles * d.E * sizeof(int32_t));
    g.off_tile_prefix = off;
    off += al((size_t)(g.n_tiles + 1) * d.E * sizeof(int32_t));
    g.total_bytes = off;
    return g;
}

namespace {
LayoutArgs make_args(const int32_t* expert_ids, const uint8_t* active, int active_dims,
                     int major_align, const moedisp_dims& dims, const moedisp_layout& L,
                     void* workspace, int32_t* status, const LayoutGeometry& g) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    LayoutArgs a;
    a.ids = expert_ids;
    a.active = active;
    a.active_dims = active_dims;
    a.align = major_align;
    a.W = dims.W;
    a.T = dims.T;
    a.K = dims.K;
    a.E = dims.E;
    a.ne = dims.E / dims.W;
    a.P = g.slots_per_rank;
    a.tiles_per_rank = g.tiles_per_rank;
    a.n_tiles = (int)g.n_tiles;
    a.tile_len = g.tile_len;
    a.cnt = L.cnt;
    a.occ = L.occ;
    a.dst_row = L.dst_row;
    a.assist = L.assist_info;
    a.expert_base = L.expert_base;
    a.rank_base = L.rank_base;
    a.send_splits = L.send_splits;
    a.rows_cap = L.rows_cap;
    a.tile_hist = reinterpret_cast<int32_t*>(ws + g.off_tile_hist);
    a.tile_prefix = reinterpret_cast<int32_t*>(ws + g.off_tile_prefix);
    a.status = status;
    return a;
}
}  // namespace

cudaError_t launch_layout(const int32_t* expert_ids, const uint8_t* active, int active_dims,
                          int major_align, const moedisp_dims& dims, const moedisp_layout& L,
                          void* workspace, int32_t* status, cudaStream_t stream) {
    const LayoutGeometry g = layout_geometry(dims);
    LayoutArgs a = make_args(expert_ids, active, active_dims, major_align, dims, L, workspace,
                             status, g);

    int tpr_c = 0, steps_c = 0;
    int64_t tile_c = 0;
    if (cluster_geometry(dims, &tpr_c, &tile_c, &steps_c)) {
        const int C = dims.W * tpr_c;
        const size_t smem = cluster_smem(dims.E, C);
        void (*kernel)(LayoutArgs) =
            steps_c == 1 ? layout_cluster_kernel<1> : steps_c == 2 ? layout_cluster_kernel<2>
            : steps_c == 4 ? layout_cluster_kernel<4> : layout_cluster_kernel<8>;
        bool ok = false;
        cudaError_t err = cluster_fits((const void*)kernel, C, smem, &ok);
        if (err != cudaSuccess) return err;
        if (ok) {
            a.tiles_per_rank = tpr_c;
            a.n_tiles = C;
            a.tile_len = tile_c;
            return launch_pdl(kernel, dim3(C), dim3(kCThreads), smem, stream, C, a);
        }
    }
    return launch_tiled(a, dims, g, stream);
}

// ------------------------------------------------------------ allocation-free variant
//
// Scratch of moedisp_moe_dispatch_layout_noalloc: the tiled path's workspace kept in
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
                                  int active_dims, int major_align, const moedisp_dims& dims,
                                  const moedisp_layout& L,
                                  int32_t* status, cudaStream_t stream) {
    const LayoutGeometry g = layout_geometry(dims);
    void* scratch = nullptr;
    cudaError_t err = layout_scratch_address(&scratch);
    if (err != cudaSuccess) return err;
    // The array keeps whatever the previous call left; nothing in it has to start at
    // zero: every scratch word is written (tile counts, then offsets) before it is read.
    LayoutArgs a = make_args(expert_ids, active, active_dims, major_align, dims, L, scratch,
                             status, g);
    return launch_tiled(a, dims, g, stream);
}

}  // namespace moedisp
