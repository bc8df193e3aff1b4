// MoE combine: y[g] = bf16_rn(sum_k w[g,k] * expert_out[dst_row[g*K+k]]), the sum taken
// in fp32 with fused multiply-adds in ascending k (a fixed order, so the result is
// deterministic and reproducible bit for bit), skipping slots that were not routed.
//
// A block combines one token at a time: each thread owns 16-byte vectors (8 columns) of
// the token's row and issues the loads of two of them from all K rows before the first
// multiply-add, so 2K independent 16-byte loads per thread are in flight; the K rows are
// read front to back. Rows are read exactly once (streaming loads), y is written once
// (streaming stores). The gate weight, the fp32 accumulation and the bf16 cast are fused
// into the gather.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace moedisp {

namespace {
constexpr int kThreads = 128;

struct CombineArgs {
    const uint4* eo;          // expert_out rows, 16-byte vectors
    int64_t G;
    int H8;                   // vectors per row
    const int32_t* dst_row;
    const float* w;
    int64_t rows_cap;
    uint4* y;
    int32_t* status;
    // Rows on W separate ranks (PEERS): expert e's rows live in rank e / ne's buffer
    // peer_eo[e / ne] (peer memory), local row = global row - rank_base[e / ne].
    const uint4* const* peer_eo;
    int64_t peer_cap;
    const int32_t* ids;
    const int64_t* rank_base;
    int ne;
};

__device__ __forceinline__ float lo_f(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_f(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // a -> low half
    return *reinterpret_cast<const uint32_t*>(&h);
}

// FMA chain of one 16-byte vector (8 columns) over the K rows, in ascending k; rows that
// were not routed (d[k] < 0) are skipped.
template <int K>
__device__ __forceinline__ uint4 combine_vec(const uint4 (&v)[K], const int32_t (&d)[K],
                                             const float (&w)[K]) {
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
    for (int k = 0; k < K; ++k) {
        if (d[k] < 0) continue;
        const float wk = w[k];
        acc[0] = __fmaf_rn(wk, lo_f(v[k].x), acc[0]);
        acc[1] = __fmaf_rn(wk, hi_f(v[k].x), acc[1]);
        acc[2] = __fmaf_rn(wk, lo_f(v[k].y), acc[2]);
        acc[3] = __fmaf_rn(wk, hi_f(v[k].y), acc[3]);
        acc[4] = __fmaf_rn(wk, lo_f(v[k].z), acc[4]);
        acc[5] = __fmaf_rn(wk, hi_f(v[k].z), acc[5]);
        acc[6] = __fmaf_rn(wk, lo_f(v[k].w), acc[6]);
        acc[7] = __fmaf_rn(wk, hi_f(v[k].w), acc[7]);
    }
    uint4 o;
    o.x = pack_bf16(acc[0], acc[1]);
    o.y = pack_bf16(acc[2], acc[3]);
    o.z = pack_bf16(acc[4], acc[5]);
    o.w = pack_bf16(acc[6], acc[7]);
    return o;
}

// One token per block at a time (persistent grid-stride over tokens): its routing (K rows
// and weights; PEERS: each row's base address in its rank's buffer) is loaded once, one
// token ahead, and the block walks the token's columns in passes of two 16-byte vectors
// per thread, so 2K row loads per thread are in flight; each of the K rows is read front
// to back by one block.
template <int K, bool PEERS>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a) {
    grid_dep_wait();
    grid_dep_launch_dependents();
    int32_t nd[K];
    float nw[K];
    const uint4* np[PEERS ? K : 1];
    auto load_routing = [&](int64_t g) {
        if (g >= a.G) return;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            nd[k] = __ldg(a.dst_row + g * K + k);
            nw[k] = __ldg(a.w + g * K + k);
            if (PEERS) {
                np[PEERS ? k : 0] = nullptr;
                if (nd[k] >= 0 && nd[k] < a.rows_cap) {
                    const int q = __ldg(a.ids + g * K + k) / a.ne;
                    const int64_t local = (int64_t)nd[k] - __ldg(a.rank_base + q);
                    if (local >= 0 && local < a.peer_cap) np[PEERS ? k : 0] = a.peer_eo[q] + local * a.H8;
                    else nd[k] = a.rows_cap;                 // flagged as beyond capacity below
                }
            }
        }
    };
    load_routing(blockIdx.x);
    for (int64_t g = blockIdx.x; g < a.G; g += gridDim.x) {
        int32_t d[K];
        float w[K];
        const uint4* p[PEERS ? K : 1];
        bool over = false;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            d[k] = nd[k];
            w[k] = nw[k];
            if (PEERS) p[PEERS ? k : 0] = np[PEERS ? k : 0];
            if (d[k] >= a.rows_cap) {
                over = true;
                d[k] = -1;
            }
        }
        load_routing(g + gridDim.x);
        if (over && threadIdx.x == 0) raise_status(a.status, MOEDISP_STATUS_CAPACITY);
        uint4* yr = a.y + g * a.H8;
        for (int c0 = threadIdx.x; c0 < a.H8; c0 += 2 * kThreads) {
            const int c1 = c0 + kThreads;
            const bool two = c1 < a.H8;
            uint4 v0[K], v1[K];
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const uint4* row = PEERS ? p[PEERS ? k : 0] : a.eo + (int64_t)d[k] * a.H8;
                v0[k] = d[k] >= 0 ? __ldcs(row + c0) : make_uint4(0, 0, 0, 0);
                v1[k] = (d[k] >= 0 && two) ? __ldcs(row + c1) : make_uint4(0, 0, 0, 0);
            }
            __stcs(yr + c0, combine_vec<K>(v0, d, w));
            if (two) __stcs(yr + c1, combine_vec<K>(v1, d, w));
        }
    }
}

template <int K>
cudaError_t launch_k(const CombineArgs& a, cudaStream_t stream) {
    void (*kernel)(CombineArgs) = a.peer_eo != nullptr ? combine_kernel<K, true> : combine_kernel<K, false>;
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)kernel, kThreads, 0, &per_sm);
    if (err != cudaSuccess) return err;
    // All resident blocks (more bytes in flight beat an even last round of tokens).
    int64_t grid = (int64_t)current_sm_count() * per_sm;
    grid = std::min<int64_t>(grid, std::max<int64_t>(1, a.G));
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kThreads), 0, stream, 1, a);
}


// ------------------------------------------------- fused tail: + residual, RMSNorm
// MoE finalize followed by the residual add and RMSNorm, in one pass over HBM: per token,
// the combined row (fp32 FMA chain in k order, as above) plus the residual row (one fp32
// add) is rounded to bf16 -- the prenorm row, written to residual_out when asked -- and
// kept in shared memory while the block reduces its sum of squares; then every element
// is scaled by 1/sqrt(mean + eps) and gamma and stored as bf16. One block per token at a
// time (persistent grid); the prenorm buffer and the partial sums are double-buffered so
// one block barrier per token suffices.
constexpr int kRmsThreads = 256;

struct RmsArgs {
    const uint4* eo;
    int64_t G;
    int H8;
    const int32_t* dst_row;
    const float* w;
    int64_t rows_cap;
    const uint4* residual;
    const float4* gamma;
    float eps;
    uint4* residual_out;       // may be null
    uint4* y;
    int32_t* status;
};

template <int K>
__global__ void __launch_bounds__(kRmsThreads) combine_rmsnorm_kernel(RmsArgs a) {
    extern __shared__ __align__(16) uint4 prenorm[];          // [2][H8]
    __shared__ float red[2][kRmsThreads / 32];
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int it = 0;
    for (int64_t g = blockIdx.x; g < a.G; g += gridDim.x, ++it) {
        uint4* pb = prenorm + (size_t)(it & 1) * a.H8;
        int32_t d[K];
        float w[K];
        bool over = false;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            d[k] = __ldg(a.dst_row + g * K + k);
            w[k] = __ldg(a.w + g * K + k);
            if (d[k] >= a.rows_cap) {
                over = true;
                d[k] = -1;
            }
        }
        if (over && threadIdx.x == 0) raise_status(a.status, MOEDISP_STATUS_CAPACITY);
        float ss = 0.0f;
        for (int c = threadIdx.x; c < a.H8; c += kRmsThreads) {
            uint4 v[K];
#pragma unroll
            for (int k = 0; k < K; ++k)
                v[k] = d[k] >= 0 ? __ldcs(a.eo + (int64_t)d[k] * a.H8 + c) : make_uint4(0, 0, 0, 0);
            const uint4 res = __ldcs(a.residual + g * a.H8 + c);
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
            for (int k = 0; k < K; ++k) {
                if (d[k] < 0) continue;
                const float wk = w[k];
                acc[0] = __fmaf_rn(wk, lo_f(v[k].x), acc[0]);
                acc[1] = __fmaf_rn(wk, hi_f(v[k].x), acc[1]);
                acc[2] = __fmaf_rn(wk, lo_f(v[k].y), acc[2]);
                acc[3] = __fmaf_rn(wk, hi_f(v[k].y), acc[3]);
                acc[4] = __fmaf_rn(wk, lo_f(v[k].z), acc[4]);
                acc[5] = __fmaf_rn(wk, hi_f(v[k].z), acc[5]);
                acc[6] = __fmaf_rn(wk, lo_f(v[k].w), acc[6]);
                acc[7] = __fmaf_rn(wk, hi_f(v[k].w), acc[7]);
            }
            uint4 r;
            r.x = pack_bf16(__fadd_rn(acc[0], lo_f(res.x)), __fadd_rn(acc[1], hi_f(res.x)));
            r.y = pack_bf16(__fadd_rn(acc[2], lo_f(res.y)), __fadd_rn(acc[3], hi_f(res.y)));
            r.z = pack_bf16(__fadd_rn(acc[4], lo_f(res.z)), __fadd_rn(acc[5], hi_f(res.z)));
            r.w = pack_bf16(__fadd_rn(acc[6], lo_f(res.w)), __fadd_rn(acc[7], hi_f(res.w)));
            pb[c] = r;
            if (a.residual_out != nullptr) __stcs(a.residual_out + g * a.H8 + c, r);
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                ss = __fmaf_rn(lo_f(rw[j]), lo_f(rw[j]), ss);
                ss = __fmaf_rn(hi_f(rw[j]), hi_f(rw[j]), ss);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) red[it & 1][warp] = ss;
        __syncthreads();
        float tot = 0.0f;
#pragma unroll
        for (int i = 0; i < kRmsThreads / 32; ++i) tot += red[it & 1][i];
        const float inv = __frsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)(a.H8 * 8)), a.eps));
        for (int c = threadIdx.x; c < a.H8; c += kRmsThreads) {
            const uint4 r = pb[c];
            const float4 g0 = __ldg(a.gamma + 2 * c), g1 = __ldg(a.gamma + 2 * c + 1);
            uint4 o;
            o.x = pack_bf16(__fmul_rn(__fmul_rn(lo_f(r.x), inv), g0.x), __fmul_rn(__fmul_rn(hi_f(r.x), inv), g0.y));
            o.y = pack_bf16(__fmul_rn(__fmul_rn(lo_f(r.y), inv), g0.z), __fmul_rn(__fmul_rn(hi_f(r.y), inv), g0.w));
            o.z = pack_bf16(__fmul_rn(__fmul_rn(lo_f(r.z), inv), g1.x), __fmul_rn(__fmul_rn(hi_f(r.z), inv), g1.y));
            o.w = pack_bf16(__fmul_rn(__fmul_rn(lo_f(r.w), inv), g1.z), __fmul_rn(__fmul_rn(hi_f(r.w), inv), g1.w));
            __stcs(a.y + g * a.H8 + c, o);
        }
    }
}

template <int K>
cudaError_t launch_rms_k(const RmsArgs& a, cudaStream_t stream) {
    const size_t smem = 2 * (size_t)a.H8 * sizeof(uint4);
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)combine_rmsnorm_kernel<K>, kRmsThreads, smem, &per_sm);
    if (err != cudaSuccess) return err;
    const int64_t grid = balanced_grid(a.G, (int64_t)current_sm_count() * per_sm);
    return launch_pdl(combine_rmsnorm_kernel<K>, dim3((unsigned)grid), dim3(kRmsThreads), smem,
                      stream, 1, a);
}

}  // namespace

namespace {
cudaError_t launch_combine_args(const CombineArgs& a, int K, cudaStream_t stream) {
    switch (K) {
#define MOEDISP_K(n) \
    case n: return launch_k<n>(a, stream);
        MOEDISP_K(1) MOEDISP_K(2) MOEDISP_K(3) MOEDISP_K(4) MOEDISP_K(5) MOEDISP_K(6)
        MOEDISP_K(7) MOEDISP_K(8) MOEDISP_K(9) MOEDISP_K(10) MOEDISP_K(11) MOEDISP_K(12)
        MOEDISP_K(13) MOEDISP_K(14) MOEDISP_K(15) MOEDISP_K(16)
#undef MOEDISP_K
        default: return cudaErrorInvalidValue;
    }
}
}  // namespace

cudaError_t launch_combine(const void* expert_out, int H, const moedisp_dims& dims,
                           const moedisp_layout& L, const float* expert_scales, void* y,
                           int32_t* status, cudaStream_t stream) {
    CombineArgs a;
    a.eo = static_cast<const uint4*>(expert_out);
    a.G = (int64_t)dims.W * dims.T;
    a.H8 = H / 8;
    a.dst_row = L.dst_row;
    a.w = expert_scales;
    a.rows_cap = L.rows_cap;
    a.y = static_cast<uint4*>(y);
    a.status = status;
    a.peer_eo = nullptr;
    a.peer_cap = 0;
    a.ids = nullptr;
    a.rank_base = nullptr;
    a.ne = 1;
    return launch_combine_args(a, dims.K, stream);
}

cudaError_t launch_combine_peers(const void* const* peer_expert_out, int64_t peer_cap, int H,
                                 const moedisp_dims& dims, int rank, const int32_t* expert_ids,
                                 const moedisp_layout& L, const float* expert_scales, void* y,
                                 int32_t* status, cudaStream_t stream) {
    const int64_t slot0 = (int64_t)rank * dims.T * dims.K;
    CombineArgs a;
    a.eo = nullptr;
    a.G = dims.T;
    a.H8 = H / 8;
    a.dst_row = L.dst_row + slot0;
    a.w = expert_scales;
    a.rows_cap = L.rows_cap;
    a.y = static_cast<uint4*>(y);
    a.status = status;
    a.peer_eo = reinterpret_cast<const uint4* const*>(peer_expert_out);
    a.peer_cap = peer_cap;
    a.ids = expert_ids + slot0;
    a.rank_base = L.rank_base;
    a.ne = dims.E / dims.W;
    return launch_combine_args(a, dims.K, stream);
}

}  // namespace moedisp

namespace moedisp {

cudaError_t launch_combine_rmsnorm(const void* expert_out, int H, const moedisp_dims& dims,
                                   const moedisp_layout& L, const float* expert_scales,
                                   const void* residual, const float* gamma, float eps,
                                   void* residual_out, void* y, int32_t* status,
                                   cudaStream_t stream) {
    RmsArgs a;
    a.eo = static_cast<const uint4*>(expert_out);
    a.G = (int64_t)dims.W * dims.T;
    a.H8 = H / 8;
    a.dst_row = L.dst_row;
    a.w = expert_scales;
    a.rows_cap = L.rows_cap;
    a.residual = static_cast<const uint4*>(residual);
    a.gamma = reinterpret_cast<const float4*>(gamma);
    a.eps = eps;
    a.residual_out = static_cast<uint4*>(residual_out);
    a.y = static_cast<uint4*>(y);
    a.status = status;
    switch (dims.K) {
#define MOEDISP_K(n) \
    case n: return launch_rms_k<n>(a, stream);
        MOEDISP_K(1) MOEDISP_K(2) MOEDISP_K(3) MOEDISP_K(4) MOEDISP_K(5) MOEDISP_K(6)
        MOEDISP_K(7) MOEDISP_K(8) MOEDISP_K(9) MOEDISP_K(10) MOEDISP_K(11) MOEDISP_K(12)
        MOEDISP_K(13) MOEDISP_K(14) MOEDISP_K(15) MOEDISP_K(16)
#undef MOEDISP_K
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moedisp
