// MoE dispatch copy: every token row goes to the K rows its active slots were given by
// the layout, optionally quantised per token (int8 or fp8-e4m3, dynamic scale).
//
// The PyTorch symm_mem index push sends one row per (token, expert) with a remote put
// from the source buffer. On one GPU the K destinations are rows of one expand_x buffer,
// so each token row is read from HBM exactly once: a persistent block brings the row
// into shared memory with a 1-D bulk (TMA) load, quantises it there if asked, and the
// K copies leave shared memory as K bulk stores issued by K lanes in parallel. Each warp
// runs its own pipeline: it looks ahead through its tokens (skipping tokens with no
// active slot), keeps up to stages-1 row loads in flight, and reuses a stage only after
// the bulk stores that read it have drained.
#include "common.cuh"
#include "kernels.h"

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
    int stages;
    uint32_t in_bytes, out_bytes;
    // receive counts (optional)
    const int32_t* cnt;
    const int64_t* expert_base;
    const int64_t* rank_base;
    int W, E, ne;
    int64_t* etn;
    int etn_type;
    int32_t* erc;
    int32_t* status;
};

constexpr int kCopyThreads = 32;        // bf16 copy: one warp per block
constexpr int kQuantMaxWarps = 8;       // quantising copy: up to 8 independent warps per block

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float absmax8(const uint4& v) {
    float m = fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x)));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w))));
    return m;
}

// q = clamp(rint(x / scale), -127, 127), x / scale an IEEE fp32 divide.
__device__ __forceinline__ uint32_t q_int8_pair(uint32_t w, float scale) {
    int a = __float2int_rn(__fdiv_rn(bf16_lo(w), scale));
    int b = __float2int_rn(__fdiv_rn(bf16_hi(w), scale));
    a = max(-127, min(127, a));
    b = max(-127, min(127, b));
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8);
}

// e4m3(x / scale), round to nearest even, saturating to +-448 (hardware conversion).
__device__ __forceinline__ uint32_t q_e4m3_pair(uint32_t w, float scale) {
    const float2 f = make_float2(__fdiv_rn(bf16_lo(w), scale), __fdiv_rn(bf16_hi(w), scale));
    return (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
}

template <int Q>
__device__ __forceinline__ uint2 quant8(const uint4& v, float scale, bool zero) {
    if (zero) return make_uint2(0u, 0u);
    uint32_t p0, p1, p2, p3;
    if (Q == MOEDISP_QUANT_INT8) {
        p0 = q_int8_pair(v.x, scale); p1 = q_int8_pair(v.y, scale);
        p2 = q_int8_pair(v.z, scale); p3 = q_int8_pair(v.w, scale);
    } else {
        p0 = q_e4m3_pair(v.x, scale); p1 = q_e4m3_pair(v.y, scale);
        p2 = q_e4m3_pair(v.z, scale); p3 = q_e4m3_pair(v.w, scale);
    }
    return make_uint2(p0 | (p1 << 16), p2 | (p3 << 16));
}

__device__ void write_recv_counts(const DispatchArgs& a) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t first = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (a.erc != nullptr) {
        const int64_t n = (int64_t)a.W * a.ne * a.W;
        for (int64_t idx = first; idx < n; idx += stride) {
            const int64_t e = idx / a.W;                  // = d*ne + le
            const int r = (int)(idx - e * a.W);
            a.erc[idx] = a.cnt[(int64_t)r * a.E + e];
        }
    }
    if (a.etn != nullptr) {
        for (int64_t e = first; e < a.E; e += stride) {
            const int d = (int)(e / a.ne);
            a.etn[e] = a.etn_type == 0 ? a.expert_base[e + 1] - a.rank_base[d]
                                       : a.expert_base[e + 1] - a.expert_base[e];
        }
    }
}

// bf16 dispatch: one warp per block; lane 0 streams token rows in, lanes 0..K-1 write
// them out.
__global__ void __launch_bounds__(kCopyThreads) dispatch_copy_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[kMaxStages];
    __shared__ int64_t tok[kMaxStages];
    __shared__ int32_t drow[kMaxStages][MOEDISP_MAX_K];
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

    int64_t next_g = blockIdx.x;     // look-ahead cursor over this block's tokens
    // Arm stage `st` with the next token that has an active slot (or the end).
    auto fill = [&](int st) {
        while (true) {
            if (next_g >= a.G) {
                if (lane == 0) {
                    tok[st] = -1;
                    mbar_arrive(&bars[st]);
                }
                return;
            }
            int32_t d = -1;
            if (lane < K) {
                d = __ldg(a.dst_row + next_g * K + lane);
                if (d >= a.rows_cap) {
                    raise_status(a.status, MOEDISP_STATUS_CAPACITY);
                    d = -1;
                }
                if (d < 0) d = -1;
            }
            const unsigned any = __ballot_sync(0xffffffffu, d >= 0);
            if (any) {
                int32_t dk[MOEDISP_MAX_K];
#pragma unroll
                for (int k = 0; k < MOEDISP_MAX_K; ++k) dk[k] = __shfl_sync(0xffffffffu, d, k);
                if (lane == 0) {
#pragma unroll
                    for (int k = 0; k < MOEDISP_MAX_K; ++k)
                        if (k < K) drow[st][k] = dk[k];
                    tok[st] = next_g;
                    mbar_arrive_expect_tx(&bars[st], a.in_bytes);
                    bulk_load(inbuf + (size_t)st * a.in_bytes, a.x + next_g * a.in_bytes, a.in_bytes,
                              &bars[st]);
                }
                next_g += gridDim.x;
                return;
            }
            next_g += gridDim.x;
        }
    };

    for (int st = 0; st < S; ++st) fill(st);

    const bool issuer = lane < K;
    for (int it = 0;; ++it) {
        const int st = it % S;
        const uint32_t par = (uint32_t)((it / S) & 1);
        // Lane 0 waits with a time limit and shares the verdict; then every lane observes
        // the already completed phase itself.
        int ok = 1;
        if (lane == 0) ok = mbar_wait(&bars[st], par) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            if (lane == 0) raise_status(a.status, MOEDISP_STATUS_TIMEOUT);
            break;
        }
        (void)mbar_wait(&bars[st], par);
        const int64_t g = tok[st];
        if (g < 0) break;
        const uint8_t* row_in = inbuf + (size_t)st * a.in_bytes;

        if (issuer) {
            const int32_t d = drow[st][lane];
            if (d >= 0) bulk_store(a.expand_x + (int64_t)d * a.out_bytes, row_in, a.in_bytes);
            bulk_commit();
        }
        // Refill the stage of the previous token once its stores have read it.
        if (it >= 1) {
            if (issuer) bulk_wait_read<1>();
            __syncwarp();
            fill((it - 1) % S);
        }
    }
    if (issuer) bulk_wait<0>();
}

// Quantising dispatch: every warp is an independent pipeline over its own tokens, with
// its own stages, barriers and output buffers, so no block-wide barrier is needed per
// token. Lane 0 streams token rows in; the warp reduces the row's max |x| with
// shuffles, quantises the row into one of its two output buffers, and lanes 0..K-1
// write the quantised row (and the scale) to the token's K rows.
template <int Q>
__global__ void __launch_bounds__(kQuantMaxWarps * 32) dispatch_quant_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[kQuantMaxWarps][kMaxStages];
    __shared__ int64_t tok[kQuantMaxWarps][kMaxStages];
    __shared__ int32_t drow[kQuantMaxWarps][kMaxStages][MOEDISP_MAX_K];
    constexpr float kQmax = Q == MOEDISP_QUANT_INT8 ? 127.0f : 448.0f;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int S = a.stages, K = a.K;
    uint8_t* inbuf = smem + (size_t)warp * (S * a.in_bytes + 2 * a.out_bytes);
    uint8_t* outbuf = inbuf + (size_t)S * a.in_bytes;
    uint64_t* wbar = bars[warp];

    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&wbar[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    grid_dep_wait();
    grid_dep_launch_dependents();
    write_recv_counts(a);

    const int wpb = blockDim.x >> 5;
    const int64_t n_warps = (int64_t)gridDim.x * wpb;
    int64_t next_g = (int64_t)blockIdx.x * wpb + warp;
    auto fill = [&](int st) {
        while (true) {
            if (next_g >= a.G) {
                if (lane == 0) {
                    tok[warp][st] = -1;
                    mbar_arrive(&wbar[st]);
                }
                return;
            }
            int32_t d = -1;
            if (lane < K) {
                d = __ldg(a.dst_row + next_g * K + lane);
                if (d >= a.rows_cap) {
                    raise_status(a.status, MOEDISP_STATUS_CAPACITY);
                    d = -1;
                }
                if (d < 0) d = -1;
            }
            if (__ballot_sync(0xffffffffu, d >= 0)) {
                int32_t dk[MOEDISP_MAX_K];
#pragma unroll
                for (int k = 0; k < MOEDISP_MAX_K; ++k) dk[k] = __shfl_sync(0xffffffffu, d, k);
                if (lane == 0) {
#pragma unroll
                    for (int k = 0; k < MOEDISP_MAX_K; ++k)
                        if (k < K) drow[warp][st][k] = dk[k];
                    tok[warp][st] = next_g;
                    mbar_arrive_expect_tx(&wbar[st], a.in_bytes);
                    bulk_load(inbuf + (size_t)st * a.in_bytes, a.x + next_g * a.in_bytes,
                              a.in_bytes, &wbar[st]);
                }
                next_g += n_warps;
                return;
            }
            next_g += n_warps;
        }
    };

    for (int st = 0; st < S; ++st) fill(st);
    const bool issuer = lane < K;
    const int nvec = a.H >> 3;
    for (int it = 0;; ++it) {
        const int st = it % S;
        const uint32_t par = (uint32_t)((it / S) & 1);
        int ok = 1;
        if (lane == 0) ok = mbar_wait(&wbar[st], par) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            if (lane == 0) raise_status(a.status, MOEDISP_STATUS_TIMEOUT);
            break;
        }
        (void)mbar_wait(&wbar[st], par);
        const int64_t g = tok[warp][st];
        if (g < 0) break;
        const uint4* v = reinterpret_cast<const uint4*>(inbuf + (size_t)st * a.in_bytes);
        float m = 0.0f;
        for (int c = lane; c < nvec; c += 32) m = fmaxf(m, absmax8(v[c]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float scale = __fdiv_rn(m, kQmax);
        const bool zero = m == 0.0f;
        if (issuer) bulk_wait_read<1>();      // output buffer it % 2 is free again
        __syncwarp();
        uint8_t* ob = outbuf + (size_t)(it & 1) * a.out_bytes;
        uint2* o2 = reinterpret_cast<uint2*>(ob);
        for (int c = lane; c < nvec; c += 32) o2[c] = quant8<Q>(v[c], scale, zero);
        fence_proxy_async_smem();
        __syncwarp();
        if (issuer) {
            const int32_t d = drow[warp][st][lane];
            if (d >= 0) {
                bulk_store(a.expand_x + (int64_t)d * a.out_bytes, ob, a.out_bytes);
                a.scales[d] = scale;
            }
            bulk_commit();
        }
        __syncwarp();
        fill(st);                               // the warp is done reading stage st
    }
    if (issuer) bulk_wait<0>();
}

cudaError_t launch_copy(DispatchArgs a, cudaStream_t stream) {
    const size_t budget = 64 * 1024;
    const int S = (int)std::max<size_t>(2, std::min<size_t>(kMaxStages, budget / a.in_bytes));
    a.stages = S;
    const size_t smem = (size_t)S * a.in_bytes;
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)dispatch_copy_kernel, kCopyThreads, smem, &per_sm);
    if (err != cudaSuccess) return err;
    int64_t grid = (int64_t)current_sm_count() * per_sm;
    grid = std::min<int64_t>(grid, std::max<int64_t>(a.G, 1));
    return launch_pdl(dispatch_copy_kernel, dim3((unsigned)grid), dim3(kCopyThreads), smem, stream,
                      1, a);
}

template <int Q>
cudaError_t launch_quant(DispatchArgs a, cudaStream_t stream) {
    // Per warp: S input stages and two output buffers. Two stages when a row is large,
    // up to four when it is small; then as many warps per block as fit about 200 KB.
    const size_t fixed = 2 * (size_t)a.out_bytes;
    const size_t small = 25 * 1024;
    int S = 2;
    if (2 * (size_t)a.in_bytes + fixed <= small)
        S = (int)std::min<size_t>(4, (small - fixed) / a.in_bytes);
    a.stages = S;
    const size_t per_warp = (size_t)S * a.in_bytes + fixed;
    const int wpb = (int)std::max<size_t>(1, std::min<size_t>(kQuantMaxWarps, (200 * 1024) / per_warp));
    const size_t smem = (size_t)wpb * per_warp;
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)dispatch_quant_kernel<Q>, wpb * 32, smem, &per_sm);
    if (err != cudaSuccess) return err;
    int64_t grid = (int64_t)current_sm_count() * per_sm;
    grid = std::min<int64_t>(grid, std::max<int64_t>((a.G + wpb - 1) / wpb, 1));
    return launch_pdl(dispatch_quant_kernel<Q>, dim3((unsigned)grid), dim3(wpb * 32), smem, stream,
                      1, a);
}

}  // namespace

cudaError_t launch_dispatch(const void* x, int H, const moedisp_dims& dims,
                            const moedisp_layout& L, int quant_mode, void* expand_x,
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
    a.stages = 2;
    a.in_bytes = (uint32_t)H * 2u;
    a.out_bytes = quant_mode == MOEDISP_QUANT_NONE ? (uint32_t)H * 2u : (uint32_t)H;
    a.cnt = L.cnt;
    a.expert_base = L.expert_base;
    a.rank_base = L.rank_base;
    a.W = dims.W;
    a.E = dims.E;
    a.ne = dims.E / dims.W;
    a.etn = expert_token_nums;
    a.etn_type = expert_token_nums_type;
    a.erc = ep_recv_counts;
    a.status = status;
    switch (quant_mode) {
        case MOEDISP_QUANT_NONE: return launch_copy(a, stream);
        case MOEDISP_QUANT_INT8: return launch_quant<MOEDISP_QUANT_INT8>(a, stream);
        case MOEDISP_QUANT_FP8_E4M3: return launch_quant<MOEDISP_QUANT_FP8_E4M3>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moedisp
