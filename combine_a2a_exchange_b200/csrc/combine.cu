// MoE combine: y[g] = bf16_rn(sum_k w[g,k] * expert_out[dst_row[g*K+k]]), the sum taken
// in fp32 with fused multiply-adds in ascending k (a fixed order, so the result is
// deterministic and reproducible bit for bit), skipping slots that were not routed.
//
// A thread owns 8 columns (one 16-byte vector) of one token: it issues all K row loads
// before the first multiply-add, so K independent 16-byte loads per thread are in
// flight; a warp covers 512 contiguous bytes of each row. Rows are read exactly once
// (streaming loads), y is written once (streaming stores). The gate weight, the fp32
// accumulation and the bf16 cast are fused into the gather.
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
};

__device__ __forceinline__ float lo_f(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_f(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // a -> low half
    return *reinterpret_cast<const uint32_t*>(&h);
}

template <int K>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a) {
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int chunks = (a.H8 + kThreads - 1) / kThreads;
    const int64_t items = a.G * chunks;
    // The next item's routing (rows and weights) is loaded while this item's rows are in
    // flight, so each item costs one dependent round trip instead of two.
    int32_t nd[K];
    float nw[K];
    auto load_routing = [&](int64_t item) {
        if (item >= items) return;
        const int64_t g = item / chunks;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            nd[k] = __ldg(a.dst_row + g * K + k);
            nw[k] = __ldg(a.w + g * K + k);
        }
    };
    load_routing(blockIdx.x);
    for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
        const int64_t g = item / chunks;
        const int vec = (int)(item - g * chunks) * kThreads + threadIdx.x;
        int32_t d[K];
        float w[K];
        bool over = false;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            d[k] = nd[k];
            w[k] = nw[k];
            if (d[k] >= a.rows_cap) {
                over = true;
                d[k] = -1;
            }
        }
        load_routing(item + gridDim.x);
        if (over && threadIdx.x == 0) raise_status(a.status, MOEDISP_STATUS_CAPACITY);
        if (vec >= a.H8) continue;
        uint4 v[K];
#pragma unroll
        for (int k = 0; k < K; ++k)
            v[k] = d[k] >= 0 ? __ldcs(a.eo + (int64_t)d[k] * a.H8 + vec) : make_uint4(0, 0, 0, 0);
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
        __stcs(a.y + g * a.H8 + vec, o);
    }
}

template <int K>
cudaError_t launch_k(const CombineArgs& a, cudaStream_t stream) {
    int per_sm = 1;
    cudaError_t err = blocks_per_sm((const void*)combine_kernel<K>, kThreads, 0, &per_sm);
    if (err != cudaSuccess) return err;
    const int chunks = (a.H8 + kThreads - 1) / kThreads;
    int64_t grid = (int64_t)current_sm_count() * per_sm;
    grid = std::min<int64_t>(grid, std::max<int64_t>(1, a.G * chunks));
    return launch_pdl(combine_kernel<K>, dim3((unsigned)grid), dim3(kThreads), 0, stream, 1, a);
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
    switch (dims.K) {
#define MOEDISP_K(n) \
    case n: return launch_k<n>(a, stream);
        MOEDISP_K(1) MOEDISP_K(2) MOEDISP_K(3) MOEDISP_K(4) MOEDISP_K(5) MOEDISP_K(6)
        MOEDISP_K(7) MOEDISP_K(8) MOEDISP_K(9) MOEDISP_K(10) MOEDISP_K(11) MOEDISP_K(12)
        MOEDISP_K(13) MOEDISP_K(14) MOEDISP_K(15) MOEDISP_K(16)
#undef MOEDISP_K
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moedisp
