// Helpers shared by the dispatch kernels: per-token dynamic quantisation of bf16 rows
// (int8 and fp8-e4m3: bf16 unpacking, the row maximum, the exact-but-fast code decision,
// code packing), named barriers for groups of warps, and the receive counts
// (expert_token_nums, ep_recv_counts) derived from the layout.
#pragma once

#include "common.cuh"

namespace moedisp {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ float absmax8(const uint4& v) {
    float m = fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x)));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w))));
    return m;
}

// Quantisation. The definition is q = clamp(rint(x / scale), -127, 127) for int8 and
// q = e4m3_rn_satfinite(x / scale) for fp8, with x / scale one IEEE fp32 division. The
// quotient is only needed near a rounding boundary of q, so it is first approximated
// by r = x * inv, inv = 1 / scale (both correctly rounded): then
//   |r - x/scale| <= |x/scale| * (2^-23 + 2^-48)  and  |fl(x/scale) - x/scale| <= |x/scale| * 2^-24,
// i.e. r and the IEEE quotient differ by at most ~3 units in the last place of fp32.
// When r is farther than that from every rounding boundary of q, both round to the same
// q; otherwise (and for inv or r not finite) the IEEE quotient is computed. The result
// is the definition's bit for bit; the fast test only decides which path gives it.

// int8 boundaries are the half-integers; |x/scale| <= ~127, so the bound above is below
// 2.3e-5 and a margin of 2^-14 from k + 0.5 is safe. Rounding to an integer uses the
// floating-point adder: for |v| < 2^22, rr = v + 1.5*2^23 rounds v's fraction away to the
// nearest integer, ties to even, and rr's bit pattern is that of 1.5*2^23 plus the
// integer. Two exact formulations are used, each where it measured faster: q_int8 below
// (the clamped integer, token-order dispatch) and, in quant8f, rr's own bits as a word
// whose low byte is the code when |r| < 127.5 (where the clamp cannot act: the low byte
// of 1.5*2^23 + q is q's two's-complement low byte), else the IEEE quotient, clamped.
//
// q_int8: the integer, clamped to +-127 (the clamp acts only when the scale itself is
// inexact far beyond fp32 rounding, i.e. subnormal).
__device__ __forceinline__ int q_int8(float x, float scale, float inv) {
    constexpr float kMagic = 12582912.0f;                    // 1.5 * 2^23
    float v = __fmul_rn(x, inv);
    float rr = __fadd_rn(v, kMagic);
    const float t = __fsub_rn(v, __fsub_rn(rr, kMagic));      // v - round(v), in [-0.5, 0.5]
    if (!(0.5f - fabsf(t) >= 0.00006103515625f)) {            // near k + 0.5, or not finite
        v = __fdiv_rn(x, scale);
        if (!(fabsf(v) < 4194304.0f)) return v > 0.0f ? 127 : -127;   // |v| >= 2^22 or NaN
        rr = __fadd_rn(v, kMagic);
    }
    const int q = (int)(__float_as_uint(rr) - __float_as_uint(kMagic));
    return max(-127, min(127, q));
}

// E4M3 keeps 3 mantissa bits: for 2^-6 <= |v| < 448 its rounding boundaries are the fp32
// values whose 20 low mantissa bits are exactly 0x80000. A shortcut quotient r that lies in
// that range and more than 16 fp32 ulps from such a boundary rounds like the IEEE quotient
// (the unsigned tests below); elsewhere (near a boundary, in E4M3's subnormal range, at
// the saturation edge, not finite) the IEEE quotient is used. Two codes come from one
// hardware conversion of the pair (round to nearest even, saturating to +-448), x0's in
// the low byte; r0, r1 are the shortcut quotients x * inv.
__device__ __forceinline__ bool e4m3_shortcut_ok(float r) {
    const uint32_t u = __float_as_uint(r) & 0x7fffffffu;
    return u - 0x3c800000u < 0x43e00000u - 0x3c800000u && (u & 0xfffffu) - 0x7fff0u > 32u;
}

__device__ __forceinline__ uint32_t q_e4m3_pair(float x0, float x1, float r0, float r1, float scale) {
    if (!e4m3_shortcut_ok(r0)) r0 = __fdiv_rn(x0, scale);
    if (!e4m3_shortcut_ok(r1)) r1 = __fdiv_rn(x1, scale);
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(r0, r1), __NV_SATFINITE, __NV_E4M3);
}

// The low bytes of four words, in order, in one word (three byte permutes).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Eight fp32 values (a smoothed row chunk) to eight codes. The floating-point steps of the
// shortcut run on pairs with the packed fp32x2 instructions (each lane an IEEE
// round-to-nearest operation, the same result as the scalar one): for int8 r = x * inv,
// rr = r + 1.5*2^23, t = r - (rr - 1.5*2^23), then the code word or the IEEE quotient
// element by element; for e4m3 the product r, then q_e4m3_pair.
template <int Q>
__device__ __forceinline__ uint2 quant8f(const float (&v)[8], float scale, float inv, bool zero) {
    if (zero) return make_uint2(0u, 0u);
    constexpr float kMagic = 12582912.0f;                    // 1.5 * 2^23
    const float2 inv2 = make_float2(inv, inv);
    uint32_t b[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float x0 = v[2 * p], x1 = v[2 * p + 1];
        const float2 r = __fmul2_rn(make_float2(x0, x1), inv2);
        if (Q == MOEDISP_QUANT_INT8) {
            const float2 rr = __fadd2_rn(r, make_float2(kMagic, kMagic));
            const float2 back = __fadd2_rn(rr, make_float2(-kMagic, -kMagic));
            const float2 t = __fadd2_rn(r, make_float2(-back.x, -back.y));
            const float xs[2] = {x0, x1};
            const float rs[2] = {r.x, r.y};
            const float rrs[2] = {rr.x, rr.y};
            const float ts[2] = {t.x, t.y};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (0.5f - fabsf(ts[h]) >= 0.00006103515625f && fabsf(rs[h]) < 127.5f) {
                    b[2 * p + h] = __float_as_uint(rrs[h]);
                } else {
                    const float q = fminf(fmaxf(__fdiv_rn(xs[h], scale), -127.0f), 127.0f);
                    b[2 * p + h] = __float_as_uint(__fadd_rn(q, kMagic));
                }
            }
        } else {
            const uint32_t pr = q_e4m3_pair(x0, x1, r.x, r.y, scale);
            b[2 * p] = pr & 0xffu;
            b[2 * p + 1] = pr >> 8;
        }
    }
    return make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
}

// Window quantisation: the code of every element of a row at once, for a row whose scale
// is a normal number. With inv = RN(1/scale), lo = RN(inv * (1 - 2^-22)) and
// hi = RN(inv * (1 + 2^-22)) satisfy
//   lo <= (1/scale) (1 + 2^-24)^2 (1 - 2^-22) < (1/scale) (1 - 2^-24)   and
//   hi >= (1/scale) (1 - 2^-24)^2 (1 + 2^-22) > (1/scale) (1 + 2^-24),
// while the IEEE quotient RN(x/scale) lies within (x/scale) (1 +- 2^-24) (or is below
// every rounding boundary, when it is subnormal). So the exact products x*lo and x*hi
// bracket RN(x/scale); both encodings are monotone (non-decreasing) functions of their
// input, so where the two ends give the same code, that code is RN(x/scale)'s. For int8
// an end is one fused multiply-add, RN(x*lo + 1.5*2^23), whose bits are those of
// 1.5*2^23 + rint(x*lo) (|x*lo| <= 127.0001 with a normal scale, so no clamp can act; the
// low byte is the code); for E4M3 an end is the rounded product RN(x*lo) (rounding is
// monotone too) converted by the hardware pair conversion. `amb` collects the bits in
// which the two ends differ: zero when every code was decided. An end's rounding
// window is |v| * 2^-21 wide, so a code is left undecided about once per 10^5 elements.
template <int Q>
__device__ __forceinline__ uint2 quant8w(const float (&v)[8], float2 lo, float2 hi, uint32_t& amb) {
    if constexpr (Q == MOEDISP_QUANT_INT8) {
        constexpr float kMagic = 12582912.0f;                    // 1.5 * 2^23
        const float2 mg = make_float2(kMagic, kMagic);
        uint32_t b[8];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 x = make_float2(v[2 * p], v[2 * p + 1]);
            const float2 a = __ffma2_rn(x, lo, mg);
            const float2 c = __ffma2_rn(x, hi, mg);
            b[2 * p] = __float_as_uint(a.x);
            b[2 * p + 1] = __float_as_uint(a.y);
            amb |= (b[2 * p] ^ __float_as_uint(c.x)) | (b[2 * p + 1] ^ __float_as_uint(c.y));
        }
        return make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
    } else {
        uint32_t h[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 x = make_float2(v[2 * p], v[2 * p + 1]);
            const uint32_t a = (uint32_t)__nv_cvt_float2_to_fp8x2(__fmul2_rn(x, lo), __NV_SATFINITE, __NV_E4M3);
            const uint32_t c = (uint32_t)__nv_cvt_float2_to_fp8x2(__fmul2_rn(x, hi), __NV_SATFINITE, __NV_E4M3);
            h[p] = a;
            amb |= a ^ c;
        }
        return make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
    }
}

// Whether a row's codes can come from the window (its scale a normal, finite number), and
// the two ends of the window.
__device__ __forceinline__ bool window_ok(float scale) {
    return scale >= 1.17549435e-38f && scale <= 3.40282347e38f;
}
__device__ __forceinline__ float2 window_lo(float inv) {
    const float t = __fmul_rn(inv, 0.999999761581420898f);    // 1 - 2^-22
    return make_float2(t, t);
}
__device__ __forceinline__ float2 window_hi(float inv) {
    const float t = __fmul_rn(inv, 1.00000023841857910f);     // 1 + 2^-22
    return make_float2(t, t);
}

// x chunk (8 bf16) times a smoothing chunk (8 fp32: s0 its first four, s1 its last four),
// one correctly rounded product each (four packed fp32x2 multiplies).
__device__ __forceinline__ void smooth8(const uint4& v, const float4& s0, const float4& s1, float (&o)[8]) {
    const float2 p0 = __fmul2_rn(make_float2(bf16_lo(v.x), bf16_hi(v.x)), make_float2(s0.x, s0.y));
    const float2 p1 = __fmul2_rn(make_float2(bf16_lo(v.y), bf16_hi(v.y)), make_float2(s0.z, s0.w));
    const float2 p2 = __fmul2_rn(make_float2(bf16_lo(v.z), bf16_hi(v.z)), make_float2(s1.x, s1.y));
    const float2 p3 = __fmul2_rn(make_float2(bf16_lo(v.w), bf16_hi(v.w)), make_float2(s1.z, s1.w));
    o[0] = p0.x; o[1] = p0.y; o[2] = p1.x; o[3] = p1.y;
    o[4] = p2.x; o[5] = p2.y; o[6] = p3.x; o[7] = p3.y;
}

__device__ __forceinline__ uint32_t q_int8_pair(uint32_t w, float scale, float inv) {
    const int a = q_int8(bf16_lo(w), scale, inv);
    const int b = q_int8(bf16_hi(w), scale, inv);
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8);
}

// Eight bf16 values (a row chunk) to eight codes: int8 as pairs of clamped integers (each
// formulation measured the faster in the token-order kernel), e4m3 two by two.
template <int Q>
__device__ __forceinline__ uint2 quant8(const uint4& v, float scale, float inv, bool zero) {
    if (zero) return make_uint2(0u, 0u);
    if (Q == MOEDISP_QUANT_INT8) {
        const uint32_t p0 = q_int8_pair(v.x, scale, inv), p1 = q_int8_pair(v.y, scale, inv);
        const uint32_t p2 = q_int8_pair(v.z, scale, inv), p3 = q_int8_pair(v.w, scale, inv);
        return make_uint2(p0 | (p1 << 16), p2 | (p3 << 16));
    }
    const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    uint32_t h[4];
#pragma unroll
    for (int p = 0; p < 4; ++p)
        h[p] = q_e4m3_pair(f[2 * p], f[2 * p + 1], __fmul_rn(f[2 * p], inv), __fmul_rn(f[2 * p + 1], inv),
                           scale);
    return make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
}

__device__ __forceinline__ void group_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Receive counts of one layout, written by whichever dispatch kernel runs it.
struct DispatchCounts {
    const int32_t* cnt;            // [W][E]
    const int64_t* expert_base;    // [E + 1]
    const int64_t* rank_base;      // [W + 1]
    int W, E, ne;
    int64_t* etn;                  // [W][ne] or null
    int etn_type;                  // 0: running sum over the rank's experts, 1: counts
    int32_t* erc;                  // [W][ne][W] or null
};

// Grid-stride over the whole grid: ep_recv_counts[d][le][r] = cnt[r][d*ne + le] (the last
// source rank's entry also holds the expert's padding rows under major_align), and
// expert_token_nums per destination rank and local expert.
__device__ __forceinline__ void write_dispatch_counts(const DispatchCounts& a) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t first = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (a.erc != nullptr) {
        const int64_t n = (int64_t)a.W * a.ne * a.W;
        for (int64_t idx = first; idx < n; idx += stride) {
            const int64_t e = idx / a.W;                  // = d*ne + le
            const int r = (int)(idx - e * a.W);
            int32_t v = a.cnt[(int64_t)r * a.E + e];
            if (r == a.W - 1) {
                // the last source rank's entry absorbs the expert's padding (major_align):
                // segment rows minus the rows routed to the expert
                int64_t routed = 0;
                for (int q = 0; q < a.W; ++q) routed += a.cnt[(int64_t)q * a.E + e];
                v += (int32_t)(a.expert_base[e + 1] - a.expert_base[e] - routed);
            }
            a.erc[idx] = v;
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

}  // namespace moedisp
