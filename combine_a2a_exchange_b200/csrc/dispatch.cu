// MoE dispatch copy: every token row goes to the K rows its active slots were given by
// the layout, optionally quantised per token (int8 or fp8-e4m3, dynamic scale).
//
// The PyTorch symm_mem index push sends one row per (token, expert) with a remote put
// from the source buffer. On one GPU the K destinations are rows of one expand_x buffer,
// so each token row is read from HBM exactly once. Unquantised, a persistent block brings
// the row into shared memory with a 1-D bulk (TMA) load and the K copies leave as K bulk
// stores issued by K lanes in parallel; each warp runs its own pipeline, looking ahead
// through its tokens (skipping tokens with no active slot), keeping up to stages-1 row
// loads in flight and reusing a stage only after the bulk stores that read it have
// drained. Quantised, a group of warps gathers the row into registers, quantises it once
// and writes the codes to the K rows. With per-expert smoothing every output row is
// quantised on its own, in expand_x's row order.
#include "common.cuh"
#include "kernels.h"
#include "dispatch_common.cuh"

#include <algorithm>

namespace moedisp {

namespace {
constexpr int kMaxStages = 8;

struct DispatchArgs {
    const uint8_t* x;
    int64_t G;
    int K, H;
    const int32_t* dst_row;
    int64_t rows_cap;
    uint8_t* expand_x;
    float* scales;
    const float* smooth;       // [E][H] per-expert smoothing (quantising modes) or null
    const int32_t* assist;     // [rows_cap] slot of each row (the smoothing kernel)
    const int64_t* rows;       // [G] row of x holding each token, -1 for none; null: row g
    int64_t x_rows;            // rows of x
    // Destination rows on W separate ranks (PEERS kernels): rank q's expand_x / scales are
    // peer_out[q] / peer_scales[q] (device pointers reachable from this GPU) with peer_cap
    // rows; global row d of expert e goes to rank e / ne, local row d - rank_base[e / ne].
    void* const* peer_out;
    float* const* peer_scales;
    int64_t peer_cap;
    const int32_t* ids;        // [G][K] expert ids of this rank's slots (PEERS)
    int stages;
    uint32_t in_bytes, out_bytes;
    // receive counts (optional)
    const int32_t* cnt;
    const int64_t* expert_base;
    const int64_t* rank_base;
    int W, E, ne;
    uint64_t kmagic;           // ceil(2^34 / K): slot / K = (slot * kmagic) >> 34 for slots < 2^30
    int64_t* etn;
    int etn_type;
    int32_t* erc;
    int32_t* status;
};

constexpr int kCopyThreads = 32;        // bf16 copy: one warp per block
constexpr int kQuantThreads = 256;      // quantising copy: block size

// PEERS: address of global destination row d of slot (g, k), or null (with
// MOEDISP_STATUS_CAPACITY raised) when it falls beyond its rank's peer_cap rows.
__device__ __forceinline__ uint8_t* peer_row(const DispatchArgs& a, int64_t g, int k, int32_t d,
                                             int64_t* local_out) {
    const int e = __ldg(a.ids + g * a.K + k);
    const int q = e / a.ne;
    const int64_t local = (int64_t)d - __ldg(a.rank_base + q);
    if (local < 0 || local >= a.peer_cap) {
        raise_status(a.status, MOEDISP_STATUS_CAPACITY);
        return nullptr;
    }
    *local_out = local;
    return static_cast<uint8_t*>(a.peer_out[q]) + local * a.out_bytes;
}

// Row of x that holds token g (g itself unless a gather map is given), -1 past the end.
__device__ __forceinline__ int64_t token_source(const DispatchArgs& a, int64_t g) {
    if (g >= a.G) return -1;
    return a.rows == nullptr ? g : __ldg(a.rows + g);
}

__device__ void write_recv_counts(const DispatchArgs& a) {
    DispatchCounts c;
    c.cnt = a.cnt;
    c.expert_base = a.expert_base;
    c.rank_base = a.rank_base;
    c.W = a.W;
    c.E = a.E;
    c.ne = a.ne;
    c.etn = a.etn;
    c.etn_type = a.etn_type;
    c.erc = a.erc;
    write_dispatch_counts(c);
}

// bf16 dispatch: one warp per block; lane 0 streams token rows in, lanes 0..K-1 write
// them out. PEERS: the K destinations are rows of the W ranks' own buffers (peer memory),
// each lane resolving its slot's address one fill ahead.
template <bool PEERS>
__global__ void __launch_bounds__(kCopyThreads) dispatch_copy_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[kMaxStages];
    __shared__ int64_t tok[kMaxStages];
    __shared__ int32_t drow[kMaxStages][MOEDISP_MAX_K];
    __shared__ uint8_t* dptr[PEERS ? kMaxStages : 1][MOEDISP_MAX_K];   // resolved (PEERS)
    const int lane = threadIdx.x & 31;
    const int S = a.stages, K = a.K;
    uint8_t* inbuf = smem;

    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    grid_dep_wait();
    grid_dep_launch_dependents();
    write_recv_counts(a);

    // Look-ahead over this block's tokens. The routing (K destination rows) of the token
    // after the one being armed is loaded one fill ahead, so arming a stage does not wait
    // for a dependent load.
    int64_t pf_g = blockIdx.x;
    int32_t pf_d = (pf_g < a.G && lane < K) ? __ldg(a.dst_row + pf_g * K + lane) : -1;
    int64_t pf_s = token_source(a, pf_g);
    auto fill = [&](int st) {
        while (true) {
            const int64_t g = pf_g;
            int32_t d = pf_d;
            const int64_t src = pf_s;
            pf_g = g + gridDim.x;
            pf_d = (pf_g < a.G && lane < K) ? __ldg(a.dst_row + pf_g * K + lane) : -1;
            pf_s = token_source(a, pf_g);
            if (g >= a.G) {
                if (lane == 0) {
                    tok[st] = -1;
                    mbar_arrive(&bars[st]);
                }
                return;
            }
            if (d >= a.rows_cap) {
                raise_status(a.status, MOEDISP_STATUS_CAPACITY);
                d = -1;
            }
            if (d < 0) d = -1;
            uint8_t* ptr = nullptr;
            if (PEERS && d >= 0) {
                int64_t local;
                ptr = peer_row(a, g, lane, d, &local);
                if (ptr == nullptr) d = -1;
            }
            if (__ballot_sync(0xffffffffu, d >= 0)) {
                if (src < 0 || src >= a.x_rows) {      // routed, but no row of x holds it
                    if (lane == 0) raise_status(a.status, MOEDISP_STATUS_BAD_SPLIT);
                    continue;
                }
                if (PEERS && lane < K) dptr[PEERS ? st : 0][lane] = ptr;   // read back by this lane
                int32_t dk[MOEDISP_MAX_K];
#pragma unroll
                for (int k = 0; k < MOEDISP_MAX_K; ++k) dk[k] = __shfl_sync(0xffffffffu, d, k);
                if (lane == 0) {
#pragma unroll
                    for (int k = 0; k < MOEDISP_MAX_K; ++k)
                        if (k < K) drow[st][k] = dk[k];
                    tok[st] = g;
                    mbar_arrive_expect_tx(&bars[st], a.in_bytes);
                    bulk_load(inbuf + (size_t)st * a.in_bytes, a.x + src * a.in_bytes, a.in_bytes,
                              &bars[st]);
                }
                return;
            }
        }
    };

    for (int st = 0; st < S; ++st) fill(st);
    int64_t filled = S;                 // pipeline iterations whose stage has been filled

    const bool issuer = lane < K;
    for (int it = 0;; ++it) {
        const int st = it % S;
        const uint32_t par = (uint32_t)((it / S) & 1);
        // Lane 0 waits with a time limit and shares the outcome; then every lane observes
        // the already completed phase itself.
        int ok = 1;
        if (lane == 0) ok = mbar_wait(&bars[st], par) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            // Stop filling, and let the row loads already armed land before the block
            // exits (a stage filled with the end-of-work marker completes at once).
            if (lane == 0) {
                raise_status(a.status, MOEDISP_STATUS_TIMEOUT);
                (void)mbar_drain(bars, S, it, filled);
            }
            break;
        }
        (void)mbar_wait(&bars[st], par);
        const int64_t g = tok[st];
        if (g < 0) break;
        const uint8_t* row_in = inbuf + (size_t)st * a.in_bytes;

        if (issuer) {
            const int32_t d = drow[st][lane];
            if (d >= 0) {
                uint8_t* dst = PEERS ? dptr[PEERS ? st : 0][lane] : a.expand_x + (int64_t)d * a.out_bytes;
                bulk_store(dst, row_in, a.in_bytes);
            }
            bulk_commit();
        }
        // Refill the stage of the previous token once its stores have read it.
        if (it >= 1) {
            if (issuer) bulk_wait_read<1>();
            __syncwarp();
            fill((it - 1) % S);
            filled = it - 1 + S + 1;
        }
    }
    if (issuer) bulk_wait<0>();
}

// max(|a|, |b|, |c|) in one instruction (the three-input form of max, sm_100 and later);
// like fmaxf, a NaN input is passed over in favour of the others.
__device__ __forceinline__ float fmax3_abs(float a, float b, float c) {
    float r;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Quantising dispatch with per-expert smoothing. The copy of token g for expert e is
// x[g] * smooth[e] quantised on its own, so the work is per row of expand_x, not per
// token, and it is arithmetic-heavy (a product, a maximum and a quantisation per output
// element). A block takes chunks of rows of one expert at a time: it copies smooth[e] into
// shared memory once per run of rows, and its token groups (WPT warps each) share the
// rows. A group gathers its row's token x[assist_info[row] / K] straight into registers
// (CPT 16-byte chunks per thread, all loads issued before the first use), reduces
// max |x * smooth[e]| (shuffles, plus a named barrier across the group's warps), and
// stores the codes (window quantisation, 8 bytes per chunk, coalesced) and the row's
// scale. No staging buffers; nothing waits on another block.
//
// Order of the rows. Within an expert's segment the rows are in slot order, hence grouped
// by source rank: rank r's rows of expert e start at expert_base[e] + sum_{r'<r} cnt[r'][e].
// RANK_ORDER walks the rows rank by rank (for each rank, its part of every expert's
// segment), so that all K copies of a token are quantised while its x row is still in L2:
// the whole grid works on one or two ranks' tokens at a time instead of on every token
// (each row of x is then read from DRAM about once rather than up to K times). Without
// RANK_ORDER (x within twice the L2, cnt absent or the tables too large) the rows go in
// expand_x order.

// Rows [row, seg_end) of expert e; smooth[e] is loaded into sbuf first.
template <int Q, int WPT, int CPT, bool EXACT>
__device__ __forceinline__ void smooth_rows(const DispatchArgs& a, float4* sbuf, float (*red)[2][WPT],
                                            int e, int32_t row, int32_t seg_end, int& parity) {
    constexpr int NG = kQuantThreads / 32 / WPT;     // groups per block
    constexpr int GT = WPT * 32;                     // threads per group
    constexpr float kQmax = Q == MOEDISP_QUANT_INT8 ? 127.0f : 448.0f;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = warp / WPT, gw = warp - grp * WPT, gt = tid - grp * GT;
    // an exact fit (nvec == CPT * GT) makes every bounds test below a compile-time true
    const int nvec = EXACT ? CPT * GT : a.H >> 3, n4 = 2 * nvec;
    const int64_t slots = a.G * a.K;
    const uint4* x4 = reinterpret_cast<const uint4*>(a.x);
    // smooth[e] in two planes: chunk c's first four values at sbuf[c], its last four at
    // sbuf[nvec + c], so that a warp's 16-byte reads of consecutive chunks are contiguous
    // (interleaved, they would span twice the banks' width: two wavefronts per read)
    __syncthreads();                                 // every group is done with the last rows
    const float4* src = reinterpret_cast<const float4*>(a.smooth + (int64_t)e * a.H);
    for (int i = tid; i < n4; i += kQuantThreads) sbuf[(i & 1) * nvec + (i >> 1)] = __ldg(src + i);
    __syncthreads();
    for (row += grp; row < seg_end; row += NG) {
        const int32_t slot = __ldg(a.assist + row);          // same for the group
        if (slot == -1) continue;                            // a padding row
        if (slot < 0 || (int64_t)slot >= slots) {
            if (gt == 0) raise_status(a.status, MOEDISP_STATUS_BAD_EXPERT_ID);
            continue;
        }
        const int64_t xrow = token_source(a, (int64_t)(((uint64_t)(uint32_t)slot * a.kmagic) >> 34));
        if (xrow < 0 || xrow >= a.x_rows) {
            if (gt == 0) raise_status(a.status, MOEDISP_STATUS_BAD_SPLIT);
            continue;
        }
        const uint4* xr = x4 + xrow * nvec;
        uint4 v[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = gt + j * GT;
            v[j] = c < nvec ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        float mq[2] = {0.0f, 0.0f};                 // independent partial maxima
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = gt + j * GT;
            if (c < nvec) {
                float xs[8];
                smooth8(v[j], sbuf[c], sbuf[nvec + c], xs);
#pragma unroll
                for (int q = 0; q < 4; ++q) mq[q & 1] = fmax3_abs(mq[q & 1], xs[2 * q], xs[2 * q + 1]);
            }
        }
        float m = fmaxf(mq[0], mq[1]);
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
        uint2* dst = reinterpret_cast<uint2*>(a.expand_x + (int64_t)row * a.out_bytes);
        // the window decides (nearly) every code; a thread with an undecided one rewrites
        // its chunks element by element (same thread, same addresses: the later stores are
        // the ones that stay)
        uint32_t amb = window_ok(scale) ? 0u : 1u;
        if (amb == 0u) {
            const float2 lo = window_lo(inv), hi = window_hi(inv);
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const int c = gt + j * GT;
                if (c < nvec) {
                    float xs[8];
                    smooth8(v[j], sbuf[c], sbuf[nvec + c], xs);
                    __stcs(dst + c, quant8w<Q>(xs, lo, hi, amb));
                }
            }
        }
        if (amb != 0u) {
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const int c = gt + j * GT;
                if (c < nvec) {
                    float xs[8];
                    smooth8(v[j], sbuf[c], sbuf[nvec + c], xs);
                    __stcs(dst + c, quant8f<Q>(xs, scale, inv, m == 0.0f));
                }
            }
        }
        if (gt == 0) a.scales[row] = scale;
    }
}

template <int Q, int WPT, int CPT, bool RANK_ORDER, bool EXACT>
__global__ void __launch_bounds__(kQuantThreads, EXACT && WPT == 1 ? 2 : (CPT > 4 ? 3 : 4))
dispatch_smooth_kernel(DispatchArgs a) {
    constexpr int NG = kQuantThreads / 32 / WPT;
    extern __shared__ __align__(16) float4 sbuf[];   // [H / 4]: smooth[e]; then the tables
    __shared__ float red[NG][2][WPT];
    __shared__ int64_t warp_tot[32];
    const int tid = threadIdx.x;
    grid_dep_wait();
    grid_dep_launch_dependents();
    write_recv_counts(a);

    const int64_t r_all = a.expert_base[a.E];
    if (blockIdx.x == 0 && tid == 0 && r_all > a.rows_cap)
        raise_status(a.status, MOEDISP_STATUS_CAPACITY);
    // rows and slots are below 2^31 (checked on the host): 32-bit row arithmetic here,
    // which keeps registers for the row's data (cfg3, 80 registers: spills 96 -> 44 bytes,
    // 989 -> 948 us)
    const int32_t R = (int32_t)min64(r_all, a.rows_cap);
    int parity = 0;

    if (!RANK_ORDER) {
        const int32_t RC = max(64, (int32_t)(((int64_t)R + 4 * (int64_t)gridDim.x - 1) / (4 * (int64_t)gridDim.x)));
        for (int32_t ch = blockIdx.x; (int64_t)ch * RC < R; ch += gridDim.x) {
            int32_t r = ch * RC;
            const int32_t end = min(R, r + RC);
            int lo = 0, hi = a.E;                   // expert_base[lo] <= r < expert_base[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (a.expert_base[mid] <= r) lo = mid; else hi = mid;
            }
            for (int e = lo; r < end; ++e) {
                const int32_t seg_end = (int32_t)min64(end, a.expert_base[e + 1]);
                if (seg_end <= r) continue;
                smooth_rows<Q, WPT, CPT, EXACT>(a, sbuf, red, e, r, seg_end, parity);
                r = seg_end;
            }
        }
        return;
    }

    // Tables over the W*E (rank, expert) parts, rank-major: vpre[i] = routed rows of the
    // parts before part i (vpre[W*E] = all of them), cpre[i] = offset of part i in its
    // expert's segment (sum of cnt over the lower ranks).
    const int WE = a.W * a.E;
    int32_t* vpre = reinterpret_cast<int32_t*>(sbuf + (a.H >> 2));
    int32_t* cpre = vpre + WE + 1;
    for (int e = tid; e < a.E; e += kQuantThreads) {
        int32_t run = 0;
        for (int q = 0; q < a.W; ++q) {
            const int32_t c = __ldg(a.cnt + (int64_t)q * a.E + e);
            cpre[q * a.E + e] = run;
            vpre[q * a.E + e + 1] = c;
            run += c;
        }
    }
    __syncthreads();
    {
        const int per = (WE + kQuantThreads - 1) / kQuantThreads;
        const int i0 = min(WE, tid * per), i1 = min(WE, i0 + per);
        int64_t part = 0;
        for (int i = i0; i < i1; ++i) part += vpre[i + 1];
        int64_t total;
        int64_t run = block_exclusive_scan(part, warp_tot, total);
        for (int i = i0; i < i1; ++i) {
            run += vpre[i + 1];
            vpre[i + 1] = (int32_t)run;
        }
        if (tid == 0) vpre[0] = 0;
    }
    __syncthreads();
    const int32_t Rv = vpre[WE];
    const int32_t RC = max(64, (int32_t)(((int64_t)Rv + 4 * (int64_t)gridDim.x - 1) / (4 * (int64_t)gridDim.x)));
    for (int32_t ch = blockIdx.x; (int64_t)ch * RC < Rv; ch += gridDim.x) {
        int32_t v = ch * RC;
        const int32_t vend = min(Rv, v + RC);
        int lo = 0, hi = WE;                        // vpre[lo] <= v < vpre[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (vpre[mid] <= v) lo = mid; else hi = mid;
        }
        for (int i = lo; v < vend; ++i) {
            const int32_t part_end = min(vend, vpre[i + 1]);
            if (part_end <= v) continue;
            const int e = i % a.E;
            const int32_t row = (int32_t)__ldg(a.expert_base + e) + cpre[i] + (v - vpre[i]);
            const int32_t row_end = min(R, row + (part_end - v));
            // (a layout whose counts disagree with its bases yields rows outside [0, R):
            // none of them is touched)
            if (row >= 0 && row < row_end)
                smooth_rows<Q, WPT, CPT, EXACT>(a, sbuf, red, e, row, row_end, parity);
            v = part_end;
        }
    }
}

// Quantising dispatch: token order, each row read once and quantised once. A group of
// WPT warps gathers its token's row straight into registers (CPT 16-byte chunks per
// thread, all issued together): no shared-memory staging, so that nothing but registers
// limits the warps per SM (a bulk-copy-staged version was measured 5 % slower on cfg3 and
// cfg4: its stages capped an SM at ~24 warps). Groups take tokens g = group, group +
// groups, ...; per token: the K destination rows (lanes 0..K-1, shuffled), skip if none
// is routed, max |x| (shuffles + a named barrier across the group), then the codes are
// written to the K rows (8 bytes per chunk, coalesced) with the scale.
template <int Q, int WPT, int CPT, bool PEERS>
__global__ void __launch_bounds__(kQuantThreads, CPT > 4 ? 2 : 4) dispatch_quant_kernel(DispatchArgs a) {
    constexpr int NG = kQuantThreads / 32 / WPT;
    constexpr int GT = WPT * 32;
    constexpr float kQmax = Q == MOEDISP_QUANT_INT8 ? 127.0f : 448.0f;
    __shared__ float red[NG][2][WPT];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = warp / WPT, gw = warp - grp * WPT, gt = tid - grp * GT;
    grid_dep_wait();
    grid_dep_launch_dependents();
    write_recv_counts(a);
    const int K = a.K, nvec = a.H >> 3;
    const int64_t groups = (int64_t)gridDim.x * NG;
    int parity = 0;
    for (int64_t g = (int64_t)blockIdx.x * NG + grp; g < a.G; g += groups) {
        int32_t d = lane < K ? __ldg(a.dst_row + g * K + lane) : -1;
        if (d >= a.rows_cap) {
            raise_status(a.status, MOEDISP_STATUS_CAPACITY);
            d = -1;
        }
        if (d < 0) d = -1;
        if (!__ballot_sync(0xffffffffu, d >= 0)) continue;          // same in every warp
        const int64_t src = token_source(a, g);
        if (src < 0 || src >= a.x_rows) {
            if (gt == 0) raise_status(a.status, MOEDISP_STATUS_BAD_SPLIT);
            continue;
        }
        const uint4* xr = reinterpret_cast<const uint4*>(a.x) + src * nvec;
        uint4 v[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = gt + j * GT;
            v[j] = c < nvec ? __ldcs(xr + c) : make_uint4(0u, 0u, 0u, 0u);
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
        uint2 q[CPT];
        // e4m3: the window of the smoothing kernel (cfg4 fp8 96.7 -> 94.4 us); int8 keeps
        // the element-by-element decision, which measured faster here (400 vs 436 us on
        // cfg3) although the window wins in the smoothing kernel
        uint32_t amb = Q == MOEDISP_QUANT_FP8_E4M3 && window_ok(scale) ? 0u : 1u;
        if (amb == 0u) {
            const float2 lo = window_lo(inv), hi = window_hi(inv);
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                float f[8];
                unpack8(v[j], f);
                q[j] = quant8w<Q>(f, lo, hi, amb);
            }
        }
        if (amb != 0u) {
#pragma unroll
            for (int j = 0; j < CPT; ++j) q[j] = quant8<Q>(v[j], scale, inv, m == 0.0f);
        }
        // PEERS: lane k resolves slot k's rank and local row (and scale address)
        uint8_t* myrow = nullptr;
        float* mysc = nullptr;
        if (PEERS && d >= 0) {
            int64_t local = 0;
            myrow = peer_row(a, g, lane, d, &local);
            if (myrow != nullptr) mysc = a.peer_scales[__ldg(a.ids + g * K + lane) / a.ne] + local;
        }
        for (int k = 0; k < K; ++k) {
            const int32_t dk = __shfl_sync(0xffffffffu, d, k);
            uint2* dst;
            if (PEERS) {
                dst = reinterpret_cast<uint2*>(__shfl_sync(0xffffffffu, (unsigned long long)myrow, k));
                if (dst == nullptr) continue;
            } else {
                if (dk < 0) continue;
                dst = reinterpret_cast<uint2*>(a.expand_x + (int64_t)dk * a.out_bytes);
            }
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const int c = gt + j * GT;
                if (c < nvec) __stcs(dst + c, q[j]);
            }
            if (PEERS) {
                float* sp = reinterpret_cast<float*>(__shfl_sync(0xffffffffu, (unsigned long long)mysc, k));
                if (gt == 0) *sp = scale;
            } else if (gt == 0) {
                a.scales[dk] = scale;
            }
        }
    }
}

cudaError_t launch_copy(DispatchArgs a, cudaStream_t stream) {
    // Few tokens per block keep the pipeline's serial start short: use the fewest stages
    // (2, 4 or 8) with which one wave of resident blocks gives each block at most about
    // two tokens per stage... i.e. prefer many shallow blocks while the tokens are few.
    const int sms = current_sm_count();
    int S = 8, per_sm = 1;
    for (int cand : {2, 4, 8}) {
        if ((size_t)cand * a.in_bytes > 64 * 1024 && cand > 2) break;
        int n = 1;
        cudaError_t err = blocks_per_sm((const void*)dispatch_copy_kernel<false>, kCopyThreads,
                                        (size_t)cand * a.in_bytes, &n);
        if (err != cudaSuccess) return err;
        S = cand;
        per_sm = n;
        if ((int64_t)sms * n * cand * 2 >= a.G) break;     // one wave covers the tokens
    }
    a.stages = S;
    const size_t smem = (size_t)S * a.in_bytes;
    int64_t grid = (int64_t)sms * per_sm;
    grid = std::min<int64_t>(grid, std::max<int64_t>(a.G, 1));
    return launch_pdl(a.peer_out != nullptr ? dispatch_copy_kernel<true> : dispatch_copy_kernel<false>,
                      dim3((unsigned)grid), dim3(kCopyThreads), smem, stream, 1, a);
}

// Smoothing kernel geometry: CPT chunks of the row per thread and WPT warps per row. Each
// warp of a row's group repeats the row's own work (its routing and token lookups, checks,
// the scale's division and reciprocal, the group maximum), so few warps per row with many
// chunks each (up to 8; 80 registers, 3 blocks per SM) beat many warps with few chunks:
// cfg3 (H = 7168: 4 warps x 7 chunks, an exact fit) 1430 -> 1083 us against 8 x 4; cfg4
// (H = 2048: 1 warp x 8) 282 -> 248 us against 2 x 4; 2 blocks per SM (105 registers)
// measured in between. When the row fits the group exactly (H / 8 == CPT * WPT * 32) the
// kernel is built with every bounds test resolved at compile time (EXACT), which lets the
// compiler overlap the chunks' loads and arithmetic freely: cfg3 1089 -> 997 us (with a
// few spilled registers at 80, still the faster), cfg4 237 -> 218 us, and 202 us with one
// warp per row at 2 blocks per SM (no spills); with 4-warp rows 2 blocks per SM lost
// (1153 us).
//
// Rank order (see the kernel) when x is well beyond the L2 (up to about twice its size
// most of the K re-reads of a row hit it anyway, and the tables cost more than they save:
// cfg4, 134 MB of x, 250 vs 235 us; cfg3, 470 MB, 1085 vs 1161 us), the layout's counts
// are given, their tables fit in shared memory beside the smoothing row and the row
// counts fit in 32 bits.
constexpr int kSmoothMaxParts = 4096;

template <int Q, int WPT, int CPT, bool EXACT>
cudaError_t launch_smooth_x(DispatchArgs a, cudaStream_t stream) {
    const int64_t WE = (int64_t)a.W * a.E;
    const bool ranked = a.cnt != nullptr && WE <= kSmoothMaxParts && a.G * a.K < (int64_t)INT32_MAX &&
                        a.x_rows * (int64_t)a.in_bytes > 2 * current_l2_bytes();
    const size_t smem = (size_t)a.H * 4 + (ranked ? (size_t)(2 * WE + 1) * 4 : 0);
    const void* fn = ranked ? (const void*)dispatch_smooth_kernel<Q, WPT, CPT, true, EXACT>
                            : (const void*)dispatch_smooth_kernel<Q, WPT, CPT, false, EXACT>;
    int per_sm = 1;
    cudaError_t err = blocks_per_sm(fn, kQuantThreads, smem, &per_sm);
    if (err != cudaSuccess) return err;
    const int64_t grid = (int64_t)current_sm_count() * per_sm;
    if (ranked)
        return launch_pdl(dispatch_smooth_kernel<Q, WPT, CPT, true, EXACT>, dim3((unsigned)grid),
                          dim3(kQuantThreads), smem, stream, 1, a);
    return launch_pdl(dispatch_smooth_kernel<Q, WPT, CPT, false, EXACT>, dim3((unsigned)grid),
                      dim3(kQuantThreads), smem, stream, 1, a);
}

template <int Q, int WPT, int CPT>
cudaError_t launch_smooth_w(DispatchArgs a, cudaStream_t stream) {
    if (a.H / 8 == CPT * WPT * 32) return launch_smooth_x<Q, WPT, CPT, true>(a, stream);
    return launch_smooth_x<Q, WPT, CPT, false>(a, stream);
}

template <int Q>
cudaError_t launch_smooth(const DispatchArgs& a, cudaStream_t stream) {
    const int nvec = a.H / 8;
    if (nvec <= 32) return launch_smooth_w<Q, 1, 1>(a, stream);
    if (nvec <= 64) return launch_smooth_w<Q, 1, 2>(a, stream);
    if (nvec <= 128) return launch_smooth_w<Q, 1, 4>(a, stream);
    if (nvec <= 256) return launch_smooth_w<Q, 1, 8>(a, stream);
    if (nvec <= 512) return launch_smooth_w<Q, 2, 8>(a, stream);
    if (nvec <= 896) return launch_smooth_w<Q, 4, 7>(a, stream);
    if (nvec <= 1024) return launch_smooth_w<Q, 4, 8>(a, stream);
    return launch_smooth_w<Q, 8, 8>(a, stream);
}

template <int Q, int WPT, int CPT>
cudaError_t launch_quant_w(DispatchArgs a, cudaStream_t stream) {
    void (*kernel)(DispatchArgs) = a.peer_out != nullptr ? dispatch_quant_kernel<Q, WPT, CPT, true>
                                                         : dispatch_quant_kernel<Q, WPT, CPT, false>;
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)kernel, kQuantThreads, 0, &per_sm);
    if (err != cudaSuccess) return err;
    constexpr int NG = kQuantThreads / 32 / WPT;
    int64_t grid = (int64_t)current_sm_count() * per_sm;
    grid = std::min<int64_t>(grid, std::max<int64_t>((a.G + NG - 1) / NG, 1));
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kQuantThreads), 0, stream, 1, a);
}

// Token-order quantising geometry: as the smoothing kernel's (chunks per thread up to four,
// then eight for the widest rows).
template <int Q>
cudaError_t launch_quant_tok(const DispatchArgs& a, cudaStream_t stream) {
    const int nvec = a.H / 8;
    if (nvec <= 32) return launch_quant_w<Q, 1, 1>(a, stream);
    if (nvec <= 64) return launch_quant_w<Q, 1, 2>(a, stream);
    if (nvec <= 128) return launch_quant_w<Q, 1, 4>(a, stream);
    if (nvec <= 256) return launch_quant_w<Q, 2, 4>(a, stream);
    if (nvec <= 512) return launch_quant_w<Q, 4, 4>(a, stream);
    if (nvec <= 1024) return launch_quant_w<Q, 8, 4>(a, stream);
    return launch_quant_w<Q, 8, 8>(a, stream);
}

template <int Q>
cudaError_t launch_quant(const DispatchArgs& a, cudaStream_t stream) {
    if (a.smooth != nullptr) return launch_smooth<Q>(a, stream);
    return launch_quant_tok<Q>(a, stream);
}

}  // namespace

cudaError_t launch_dispatch(const void* x, int64_t x_rows, const int64_t* token_rows, int H,
                            const moedisp_dims& dims, const moedisp_layout& L, int quant_mode,
                            const float* smooth_scales, void* expand_x,
                            float* dynamic_scales, int64_t* expert_token_nums,
                            int expert_token_nums_type, int32_t* ep_recv_counts,
                            int32_t* status, cudaStream_t stream) {
    DispatchArgs a;
    a.x = static_cast<const uint8_t*>(x);
    a.G = (int64_t)dims.W * dims.T;
    a.K = dims.K;
    a.H = H;
    a.dst_row = L.dst_row;
    a.rows_cap = L.rows_cap;
    a.expand_x = static_cast<uint8_t*>(expand_x);
    a.scales = dynamic_scales;
    a.smooth = smooth_scales;
    a.assist = L.assist_info;
    a.rows = token_rows;
    a.x_rows = x_rows;
    a.stages = 2;
    a.in_bytes = (uint32_t)H * 2u;
    a.out_bytes = quant_mode == MOEDISP_QUANT_NONE ? (uint32_t)H * 2u : (uint32_t)H;
    a.cnt = L.cnt;
    a.kmagic = ((uint64_t(1) << 34) + (uint64_t)dims.K - 1) / (uint64_t)dims.K;
    a.expert_base = L.expert_base;
    a.rank_base = L.rank_base;
    a.W = dims.W;
    a.E = dims.E;
    a.ne = dims.E / dims.W;
    a.etn = expert_token_nums;
    a.etn_type = expert_token_nums_type;
    a.erc = ep_recv_counts;
    a.status = status;
    a.peer_out = nullptr;
    a.peer_scales = nullptr;
    a.peer_cap = 0;
    a.ids = nullptr;
    switch (quant_mode) {
        case MOEDISP_QUANT_NONE: return launch_copy(a, stream);
        case MOEDISP_QUANT_INT8: return launch_quant<MOEDISP_QUANT_INT8>(a, stream);
        case MOEDISP_QUANT_FP8_E4M3: return launch_quant<MOEDISP_QUANT_FP8_E4M3>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_dispatch_peers(const void* x, int H, const moedisp_dims& dims, int rank,
                                  const int32_t* expert_ids, const moedisp_layout& L,
                                  int quant_mode, void* const* peer_out,
                                  float* const* peer_scales, int64_t peer_cap, int32_t* status,
                                  cudaStream_t stream) {
    const int64_t slot0 = (int64_t)rank * dims.T * dims.K;     // this rank's first slot
    DispatchArgs a;
    a.x = static_cast<const uint8_t*>(x);
    a.G = dims.T;
    a.K = dims.K;
    a.H = H;
    a.dst_row = L.dst_row + slot0;
    a.rows_cap = L.rows_cap;
    a.expand_x = nullptr;
    a.scales = nullptr;
    a.smooth = nullptr;
    a.assist = nullptr;
    a.rows = nullptr;
    a.x_rows = dims.T;
    a.stages = 2;
    a.in_bytes = (uint32_t)H * 2u;
    a.out_bytes = quant_mode == MOEDISP_QUANT_NONE ? (uint32_t)H * 2u : (uint32_t)H;
    a.cnt = nullptr;
    a.kmagic = ((uint64_t(1) << 34) + (uint64_t)dims.K - 1) / (uint64_t)dims.K;
    a.expert_base = L.expert_base;
    a.rank_base = L.rank_base;
    a.W = dims.W;
    a.E = dims.E;
    a.ne = dims.E / dims.W;
    a.etn = nullptr;
    a.etn_type = 1;
    a.erc = nullptr;
    a.status = status;
    a.peer_out = peer_out;
    a.peer_scales = peer_scales;
    a.peer_cap = peer_cap;
    a.ids = expert_ids + slot0;
    switch (quant_mode) {
        case MOEDISP_QUANT_NONE: return launch_copy(a, stream);
        case MOEDISP_QUANT_INT8: return launch_quant<MOEDISP_QUANT_INT8>(a, stream);
        case MOEDISP_QUANT_FP8_E4M3: return launch_quant<MOEDISP_QUANT_FP8_E4M3>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moedisp
