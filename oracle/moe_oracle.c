/*
 * moe_oracle.c -- plain CPU oracle (TEST INFRASTRUCTURE ONLY; see moe_oracle.h).
 *
 * Built with -O2 -ffp-contract=off and no fast-math, so every float operation below
 * is the single IEEE operation it is written as; the only fused multiply-adds are the
 * explicit fmaf()/fma() calls of the combine.
 *
 * Sources (web pages on expert-parallel MoE all-to-all):
 *  [P1] PyTorch "symm_mem" all-to-all exchange plan change: ExchangePlan doc comment,
 *       test_make_a2a_exchange_plan, test_a2a_with_exchange_plan, make2dExchangePlan,
 *       get_occurrence_numbers, _allToAllV_2d_index_push_kernel.
 *  [P3] torch-neuronx PR "Fix all_to_all_single lowering for uneven split sizes",
 *       section Motivation and Context / Testing (pad, even all-to-all, trim).
 *  [P4] Ascend aclnnMoeDistributeDispatchV2, sections Function, Parameters
 *       (quantMode, expertTokenNumsType, epRecvCountsOut) and Constraints.
 *  [P5] FlashInfer MNNVL all-reduce fusion PR: MoE finalize = weighted sum of each
 *       token's top-k expert rows, a routed index of -1 meaning "not routed".
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ conversions */

static uint32_t f32_bits(float v) { uint32_t u; memcpy(&u, &v, 4); return u; }
static float bits_f32(uint32_t u) { float v; memcpy(&v, &u, 4); return v; }

/* bf16 keeps the top 16 bits of an fp32; the cut is rounded to nearest, ties to even. */
uint16_t orc_bf16_from_f32(float v)
{
    uint32_t u = f32_bits(v);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u); /* NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

float orc_bf16_to_f32(uint16_t b) { return bits_f32((uint32_t)b << 16); }

/* OCP OFP8 E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; no infinity;
 * S.1111.111 is NaN; largest finite 448 = 1.75 * 2^8; smallest normal 2^-6;
 * subnormals m * 2^-9, m = 1..7. */
float orc_e4m3_to_f32(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xf, m = c & 7;
    double v;
    if (e == 0xf && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* Round to nearest even on the E4M3 grid, then saturate to the largest finite value. */
uint8_t orc_e4m3_from_f32(float v)
{
    if (isnan(v)) return 0x7f;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);            /* a = f * 2^ex, f in [0.5, 1): floor(log2 a) = ex - 1 */
    int e = ex - 1;
    if (e < -6) e = -6;       /* subnormal range shares the 2^-9 quantum */
    double quantum = ldexp(1.0, e - 3);
    double n = a / quantum;   /* exact: quantum is a power of two */
    double r = nearbyint(n);  /* default rounding mode: nearest, ties to even */
    double val = r * quantum;
    if (val > 448.0) val = 448.0;
    /* encode val */
    if (val == 0.0) return sign;
    int ve;
    frexp(val, &ve);
    int E = ve - 1;
    if (E < -6) {             /* subnormal: val = m * 2^-9 */
        int m = (int)(val / ldexp(1.0, -9));
        return (uint8_t)(sign | m);
    }
    int m = (int)((val / ldexp(1.0, E) - 1.0) * 8.0);
    return (uint8_t)(sign | ((E + 7) << 3) | m);
}

/* ------------------------------------------------------------- O1 exchange plan */

/* [P1] ExchangePlan: out_splits = what each peer sends me (the exchanged in_splits);
 * src_offsets = where in each peer's input my rows start (the exchanged exclusive scan
 * of the peer's in_splits); dst_offsets = exclusive scan of my out_splits. */
int orc_a2a_exchange_plan(int W, const int64_t *S, int64_t *src_offsets,
                          int64_t *out_splits, int64_t *dst_offsets)
{
    int flags = 0;
    if (W < 0) return ORC_BAD_ARG;
    for (int i = 0; i < W * W; i++)
        if (S[i] < 0) flags |= ORC_BAD_SPLIT;
    for (int i = 0; i < W; i++) {
        for (int j = 0; j < W; j++) {
            out_splits[(int64_t)i * W + j] = S[(int64_t)j * W + i];
            int64_t acc = 0;                       /* exclusive scan of peer j's splits */
            for (int k = 0; k < i; k++) acc += S[(int64_t)j * W + k];
            src_offsets[(int64_t)i * W + j] = acc;
        }
        int64_t acc = 0;
        for (int j = 0; j < W; j++) {
            dst_offsets[(int64_t)i * W + j] = acc;
            acc += out_splits[(int64_t)i * W + j];
        }
    }
    return flags;
}

/* ------------------------------------------------------------------- O2 a2a_v */

/* [P1] get-style all-to-all-v: rank i fetches out_splits[i][j] rows of peer j from
 * row src_offsets[i][j] of j's input into its output at row dst_offsets[i][j].
 * A segment that would leave either buffer is skipped and flagged. */
int orc_a2a_v(int W, const uint8_t *in, int64_t in_rank_stride_rows, uint8_t *out,
              int64_t out_cap_rows, int64_t row_bytes, const int64_t *src_offsets,
              const int64_t *out_splits, const int64_t *dst_offsets)
{
    int flags = 0;
    for (int i = 0; i < W; i++) {
        for (int j = 0; j < W; j++) {
            int64_t n = out_splits[(int64_t)i * W + j];
            int64_t so = src_offsets[(int64_t)i * W + j];
            int64_t d0 = dst_offsets[(int64_t)i * W + j];
            if (n == 0) continue;
            if (n < 0 || so < 0 || d0 < 0 || so + n > in_rank_stride_rows ||
                d0 + n > out_cap_rows) {
                flags |= ORC_BAD_SPLIT;
                continue;
            }
            for (int64_t q = 0; q < n; q++) {
                const uint8_t *src = in + ((int64_t)j * in_rank_stride_rows + so + q) * row_bytes;
                uint8_t *dst = out + ((int64_t)i * out_cap_rows + d0 + q) * row_bytes;
                memcpy(dst, src, (size_t)row_bytes);
            }
        }
    }
    return flags;
}

/* ----------------------------------------------------------------- O3 layout */

/* Steps in the order of [P1]:
 *  1. per source rank r: bincount of its (token, k) expert ids -> cnt[r][e]
 *     (the 2-D plan's in_splits) and the 0-based occurrence number of every slot
 *     among the earlier slots of r with the same expert (get_occurrence_numbers:
 *     running count minus self);
 *  2. the 2-D (expert-major) plan, make2dExchangePlan: for destination rank d and its
 *     local expert le (expert = d*ne + le):
 *        cusum_per_expert[r][expert] = sum_{r' < r} cnt[r'][expert]
 *        aggregate[d][le]            = sum_r cnt[r][expert]
 *        cusum_per_rank[d][le]       = sum_{le' < le} aggregate[d][le']
 *        dst_offsets[r][expert]      = cusum_per_expert[r][expert] + cusum_per_rank[d][le]
 *  3. the index push: slot s of rank r with expert e goes to row
 *        dst_offsets[r][e] + occ[s] of rank owner(e) = e / ne  ([P1]
 *        _allToAllV_2d_index_push_kernel), i.e. global row rank_base[d] + that.
 * Inactive slots ([P4] xActiveMask: a 1-D mask [G] of tokens, read as any pattern, or a
 * 2-D mask [G][K] of slots, where a token whose K flags are all false sends nothing) and
 * expert ids outside [0, E) contribute no slot; both get occ = dst_row = -1.
 * major_align ([P1] all_to_all_vdev_2d major_align, the padding rule of the 2-D plan
 * test): 0 or 1, no padding; A >= 2, each expert's segment of aggregate[e] rows is
 * padded to max(A, ceil(aggregate[e] / A) * A) rows, so every expert starts on a multiple
 * of A; the padding rows follow the expert's real rows and get assist_info -1. */
static int64_t padded_rows(int64_t n, int64_t A)
{
    if (A <= 1) return n;
    int64_t p = (n + A - 1) / A * A;
    return p < A ? A : p;
}

int orc_moe_dispatch_layout(int W, int T, int K, int E, const int32_t *expert_ids,
                            const uint8_t *active, int active_dims, int64_t major_align,
                            int64_t rows_cap, int32_t *cnt,
                            int32_t *occ, int32_t *dst_row, int32_t *assist_info,
                            int64_t *expert_base, int64_t *rank_base, int64_t *send_splits)
{
    if (W <= 0 || T < 0 || K <= 0 || E <= 0 || E % W != 0) return ORC_BAD_ARG;
    if (active && active_dims != 1 && active_dims != 2) return ORC_BAD_ARG;
    if (major_align < 0) return ORC_BAD_ARG;
    int flags = 0;
    int ne = E / W;
    int64_t G = (int64_t)W * T;
    int64_t *cusum_per_expert = (int64_t *)calloc((size_t)W * E, sizeof(int64_t));
    int64_t *aggregate = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *cusum_per_rank = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *dst2d = (int64_t *)calloc((size_t)W * E, sizeof(int64_t));
    int64_t *running = (int64_t *)calloc((size_t)E, sizeof(int64_t));

    /* step 1 */
    for (int r = 0; r < W; r++) {
        memset(running, 0, sizeof(int64_t) * E);
        for (int t = 0; t < T; t++) {
            int64_t g = (int64_t)r * T + t;
            for (int k = 0; k < K; k++) {
                int64_t s = g * K + k;
                int act = !active ? 1 : active_dims == 1 ? (active[g] != 0) : (active[s] != 0);
                int32_t e = expert_ids[s];
                if (act && (e < 0 || e >= E)) flags |= ORC_BAD_EXPERT;
                if (!act || e < 0 || e >= E) { occ[s] = -1; continue; }
                occ[s] = (int32_t)running[e];
                running[e] += 1;
            }
        }
        for (int e = 0; e < E; e++) cnt[(int64_t)r * E + e] = (int32_t)running[e];
    }

    /* step 2 */
    for (int e = 0; e < E; e++) {
        int64_t c = 0;
        for (int r = 0; r < W; r++) {
            cusum_per_expert[(int64_t)r * E + e] = c;
            c += cnt[(int64_t)r * E + e];
        }
        aggregate[e] = c;
    }
    for (int d = 0; d < W; d++) {
        int64_t c = 0;
        for (int le = 0; le < ne; le++) {
            cusum_per_rank[d * ne + le] = c;
            c += padded_rows(aggregate[d * ne + le], major_align);
        }
    }
    for (int r = 0; r < W; r++)
        for (int e = 0; e < E; e++)
            dst2d[(int64_t)r * E + e] = cusum_per_expert[(int64_t)r * E + e] + cusum_per_rank[e];

    int64_t acc = 0;
    for (int d = 0; d < W; d++) {
        rank_base[d] = acc;
        for (int le = 0; le < ne; le++) acc += padded_rows(aggregate[d * ne + le], major_align);
    }
    rank_base[W] = acc;
    for (int e = 0; e < E; e++) expert_base[e] = rank_base[e / ne] + cusum_per_rank[e];
    expert_base[E] = acc;
    if (acc > rows_cap) flags |= ORC_CAPACITY;

    for (int r = 0; r < W; r++)
        for (int d = 0; d < W; d++) {
            int64_t c = 0;
            for (int le = 0; le < ne; le++) c += cnt[(int64_t)r * E + d * ne + le];
            send_splits[(int64_t)r * W + d] = c;
        }

    /* step 3 */
    for (int64_t g = 0; g < G; g++) {
        int r = (int)(g / (T > 0 ? T : 1));
        for (int k = 0; k < K; k++) {
            int64_t s = g * K + k;
            if (occ[s] < 0) { dst_row[s] = -1; continue; }
            int32_t e = expert_ids[s];
            int64_t row = rank_base[e / ne] + dst2d[(int64_t)r * E + e] + occ[s];
            dst_row[s] = (int32_t)row;
            if (row < rows_cap) assist_info[row] = (int32_t)s;
        }
    }
    for (int e = 0; e < E; e++)
        for (int64_t row = expert_base[e] + aggregate[e]; row < expert_base[e + 1]; row++)
            if (row < rows_cap) assist_info[row] = -1;

    free(cusum_per_expert); free(aggregate); free(cusum_per_rank); free(dst2d); free(running);
    return flags;
}

/* [P4] expertTokenNumsOut (per local expert: count, or with type 0 the running sum over
 * the rank's local experts, read as inclusive) and epRecvCountsOut (rows received from
 * each source rank, ordered expert-major like [P1]'s 2-D out_splits). With major_align,
 * as in [P1]'s 2-D plan, the last source rank's entry absorbs the expert's padding, so
 * both count the padded segment. */
int orc_moe_recv_counts(int W, int E, const int32_t *cnt, int64_t major_align,
                        int expert_token_nums_type, int64_t *expert_token_nums,
                        int32_t *ep_recv_counts)
{
    if (W <= 0 || E <= 0 || E % W != 0 || major_align < 0) return ORC_BAD_ARG;
    int ne = E / W;
    for (int d = 0; d < W; d++) {
        int64_t run = 0;
        for (int le = 0; le < ne; le++) {
            int e = d * ne + le;
            int64_t tot = 0;
            for (int r = 0; r < W; r++) {
                int32_t c = cnt[(int64_t)r * E + e];
                ep_recv_counts[((int64_t)d * ne + le) * W + r] = c;
                tot += c;
            }
            int64_t pad = padded_rows(tot, major_align) - tot;
            ep_recv_counts[((int64_t)d * ne + le) * W + (W - 1)] += (int32_t)pad;
            tot += pad;
            run += tot;
            expert_token_nums[(int64_t)d * ne + le] = expert_token_nums_type == 0 ? run : tot;
        }
    }
    return 0;
}

/* ---------------------------------------------------------------- O4 dispatch */

/* Per-token dynamic quantisation ([P4] quantMode 2): scale = max|x| / QMAX in fp32
 * (QMAX = 127 for int8, 448 for e4m3), q = round(x / scale) with one IEEE fp32 divide;
 * int8 rounds half to even and clamps to [-127, 127]; e4m3 rounds to nearest even and
 * saturates. An all-zero row has scale 0 and q = 0. */
float orc_quant_row_f32(int H, const float *x, int quant_mode, uint8_t *q)
{
    float amax = 0.0f;
    for (int h = 0; h < H; h++) {
        float a = fabsf(x[h]);
        if (a > amax) amax = a;
    }
    float qmax = quant_mode == 2 ? 127.0f : 448.0f;
    float scale = amax / qmax;
    for (int h = 0; h < H; h++) {
        if (amax == 0.0f) { q[h] = 0; continue; }
        float v = x[h] / scale;
        if (quant_mode == 2) {
            float r = rintf(v);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q[h] = (uint8_t)(int8_t)r;
        } else {
            q[h] = orc_e4m3_from_f32(v);
        }
    }
    return scale;
}

float orc_quant_row(int H, const uint16_t *x, int quant_mode, uint8_t *q)
{
    float *v = (float *)malloc(sizeof(float) * (size_t)(H > 0 ? H : 1));
    for (int h = 0; h < H; h++) v[h] = orc_bf16_to_f32(x[h]);
    float scale = orc_quant_row_f32(H, v, quant_mode, q);
    free(v);
    return scale;
}

/* [P1] index push / [P4] expandXOut: every active slot s writes its token's row
 * (quantised or not) to row dst_row[s]. Rows at or beyond rows_cap are skipped and
 * flagged. With smooth ([P4] scalesOptional, [E][H]; quantising modes only) the row sent
 * to expert e = expert_ids[s] is first multiplied element-wise by smooth[e] (one fp32
 * product per element) and quantised on its own, so each copy has its own scale. */
int orc_moe_dispatch(int G, int K, int H, const uint16_t *x, const int32_t *dst_row,
                     int64_t rows_cap, int quant_mode, void *expand_x, float *dynamic_scales,
                     const float *smooth, int E, const int32_t *expert_ids)
{
    if (quant_mode != 0 && quant_mode != 2 && quant_mode != 3) return ORC_BAD_ARG;
    if (smooth && (quant_mode == 0 || !expert_ids || E <= 0)) return ORC_BAD_ARG;
    int flags = 0;
    size_t out_row = quant_mode == 0 ? (size_t)H * 2 : (size_t)H;
    uint8_t *q = (uint8_t *)malloc((size_t)H > 0 ? (size_t)H : 1);
    float *xs = (float *)malloc(sizeof(float) * (size_t)(H > 0 ? H : 1));
    for (int64_t g = 0; g < G; g++) {
        const uint16_t *xr = x + g * (int64_t)H;
        float scale = 0.0f;
        int have_q = 0;
        for (int k = 0; k < K; k++) {
            int32_t row = dst_row[g * K + k];
            if (row < 0) continue;
            if (row >= rows_cap) { flags |= ORC_CAPACITY; continue; }
            uint8_t *dst = (uint8_t *)expand_x + (size_t)row * out_row;
            if (quant_mode == 0) {
                memcpy(dst, xr, out_row);
            } else if (smooth) {
                int32_t e = expert_ids[g * K + k];
                if (e < 0 || e >= E) { flags |= ORC_BAD_EXPERT; continue; }
                for (int h = 0; h < H; h++)
                    xs[h] = orc_bf16_to_f32(xr[h]) * smooth[(int64_t)e * H + h];
                dynamic_scales[row] = orc_quant_row_f32(H, xs, quant_mode, q);
                memcpy(dst, q, out_row);
            } else {
                if (!have_q) { scale = orc_quant_row(H, xr, quant_mode, q); have_q = 1; }
                memcpy(dst, q, out_row);
                dynamic_scales[row] = scale;
            }
        }
    }
    free(q);
    free(xs);
    return flags;
}

/* ----------------------------------------------------------------- O5 combine */

/* [P4] CombineV2 / [P5] MoE finalize: y[g] = sum_k w[g,k] * expert_out[dst_row[g*K+k]];
 * a slot with dst_row -1 (not routed) contributes nothing; a token with no routed slot
 * gives 0. O5a accumulates in double. */
int orc_moe_combine_f64(int G, int K, int H, const uint16_t *expert_out, int64_t rows_cap,
                        const int32_t *dst_row, const float *w, double *y64)
{
    int flags = 0;
    for (int64_t g = 0; g < G; g++) {
        double *y = y64 + g * (int64_t)H;
        for (int h = 0; h < H; h++) y[h] = 0.0;
        for (int k = 0; k < K; k++) {
            int32_t row = dst_row[g * K + k];
            if (row < 0) continue;
            if (row >= rows_cap) { flags |= ORC_CAPACITY; continue; }
            const uint16_t *v = expert_out + (int64_t)row * H;
            double wk = (double)w[g * K + k];
            for (int h = 0; h < H; h++) y[h] += wk * (double)orc_bf16_to_f32(v[h]);
        }
    }
    return flags;
}

/* O5b: acc = 0; for k = 0..K-1 in order: acc = fmaf(w[g,k], v_k, acc); y = bf16(acc). */
int orc_moe_combine_f32(int G, int K, int H, const uint16_t *expert_out, int64_t rows_cap,
                        const int32_t *dst_row, const float *w, uint16_t *y)
{
    int flags = 0;
    float *acc = (float *)malloc(sizeof(float) * (size_t)(H > 0 ? H : 1));
    for (int64_t g = 0; g < G; g++) {
        for (int h = 0; h < H; h++) acc[h] = 0.0f;
        for (int k = 0; k < K; k++) {
            int32_t row = dst_row[g * K + k];
            if (row < 0) continue;
            if (row >= rows_cap) { flags |= ORC_CAPACITY; continue; }
            const uint16_t *v = expert_out + (int64_t)row * H;
            float wk = w[g * K + k];
            for (int h = 0; h < H; h++) acc[h] = fmaf(wk, orc_bf16_to_f32(v[h]), acc[h]);
        }
        for (int h = 0; h < H; h++) y[g * (int64_t)H + h] = orc_bf16_from_f32(acc[h]);
    }
    free(acc);
    return flags;
}

/* ------------------------------------------------------- fused tail (RMSNorm) */

/* [P5] MoE finalize followed by the residual add and RMSNorm: the prenorm row is the
 * token's combined row plus its residual (kept as residual_out in bf16), normalised by
 * the root mean square of that bf16 row (plus eps) and scaled by gamma. */
int orc_moe_combine_rmsnorm_f64(int G, int K, int H, const uint16_t *expert_out,
                                int64_t rows_cap, const int32_t *dst_row, const float *w,
                                const uint16_t *residual, const float *gamma, float eps,
                                uint16_t *residual_out, double *y64)
{
    int flags = 0;
    double *s = (double *)malloc(sizeof(double) * (size_t)(H > 0 ? H : 1));
    for (int64_t g = 0; g < G; g++) {
        for (int h = 0; h < H; h++) s[h] = (double)orc_bf16_to_f32(residual[g * (int64_t)H + h]);
        for (int k = 0; k < K; k++) {
            int32_t row = dst_row[g * K + k];
            if (row < 0) continue;
            if (row >= rows_cap) { flags |= ORC_CAPACITY; continue; }
            const uint16_t *v = expert_out + (int64_t)row * H;
            double wk = (double)w[g * K + k];
            for (int h = 0; h < H; h++) s[h] += wk * (double)orc_bf16_to_f32(v[h]);
        }
        double ss = 0.0;
        for (int h = 0; h < H; h++) {
            uint16_t r = orc_bf16_from_f32((float)s[h]);
            residual_out[g * (int64_t)H + h] = r;
            double rv = (double)orc_bf16_to_f32(r);
            ss += rv * rv;
        }
        double inv = 1.0 / sqrt(ss / H + (double)eps);
        for (int h = 0; h < H; h++)
            y64[g * (int64_t)H + h] = (double)orc_bf16_to_f32(residual_out[g * (int64_t)H + h]) * inv *
                                      (double)gamma[h];
    }
    free(s);
    return flags;
}

int orc_moe_combine_rmsnorm_f32(int G, int K, int H, const uint16_t *expert_out,
                                int64_t rows_cap, const int32_t *dst_row, const float *w,
                                const uint16_t *residual, const float *gamma, float eps,
                                uint16_t *residual_out, uint16_t *y)
{
    int flags = 0;
    float *acc = (float *)malloc(sizeof(float) * (size_t)(H > 0 ? H : 1));
    for (int64_t g = 0; g < G; g++) {
        for (int h = 0; h < H; h++) acc[h] = 0.0f;
        for (int k = 0; k < K; k++) {
            int32_t row = dst_row[g * K + k];
            if (row < 0) continue;
            if (row >= rows_cap) { flags |= ORC_CAPACITY; continue; }
            const uint16_t *v = expert_out + (int64_t)row * H;
            float wk = w[g * K + k];
            for (int h = 0; h < H; h++) acc[h] = fmaf(wk, orc_bf16_to_f32(v[h]), acc[h]);
        }
        float ss = 0.0f;
        for (int h = 0; h < H; h++) {
            float sv = acc[h] + orc_bf16_to_f32(residual[g * (int64_t)H + h]);
            uint16_t r = orc_bf16_from_f32(sv);
            residual_out[g * (int64_t)H + h] = r;
            float rv = orc_bf16_to_f32(r);
            ss = fmaf(rv, rv, ss);
        }
        float inv = 1.0f / sqrtf(ss / (float)H + eps);
        for (int h = 0; h < H; h++)
            y[g * (int64_t)H + h] =
                orc_bf16_from_f32(orc_bf16_to_f32(residual_out[g * (int64_t)H + h]) * inv * gamma[h]);
    }
    free(acc);
    return flags;
}

/* ------------------------------------------------------ shared experts ([P4]) */

/* [P4] sharedExpertNum N, sharedExpertRankNum S, expertShardType 0: the first S of the W
 * ranks host shared experts (one replica each, S / N replicas of each of the N shared
 * experts, replica groups in shared-expert order), the other W - S ranks host the
 * E routed experts, ne = E / (W - S) each. Every token also goes to each shared expert.
 * Reading of the pages (which fix only the counts: a shared rank receives
 * Bs * W * N / S tokens): source rank r's tokens go to replica (r mod (S / N)) of each
 * shared expert, i.e. rank j * (S / N) + r mod (S / N) for shared expert j.
 * The result is a routing over a uniform expert space of W * ne experts, ne per rank:
 * routed expert e becomes S * ne + e; shared expert j's replica on rank d is expert d * ne
 * (the rank's other ne - 1 expert ids stay unused). ext_ids / ext_w are [G][K + N]: the
 * K routed slots (weights as given; an id outside [0, E) is mapped to W * ne, still out of
 * range), then the N shared slots with weight 1. */
int orc_shared_expert_routing(int W, int T, int K, int E, int N, int S,
                              const int32_t *expert_ids, const float *w,
                              int32_t *ext_ids, float *ext_w)
{
    if (W <= 0 || T < 0 || K <= 0 || E <= 0 || N < 0 || S < 0 || S >= W) return ORC_BAD_ARG;
    if ((S == 0) != (N == 0)) return ORC_BAD_ARG;
    if (S > 0 && (W % S != 0 || S % N != 0)) return ORC_BAD_ARG;
    if (E % (W - S) != 0) return ORC_BAD_ARG;
    int ne = E / (W - S);
    int KN = K + N;
    int flags = 0;
    for (int r = 0; r < W; r++)
        for (int t = 0; t < T; t++) {
            int64_t g = (int64_t)r * T + t;
            for (int k = 0; k < K; k++) {
                int32_t e = expert_ids[g * K + k];
                if (e < 0 || e >= E) {
                    flags |= ORC_BAD_EXPERT;
                    ext_ids[g * KN + k] = W * ne;
                } else {
                    ext_ids[g * KN + k] = S * ne + e;
                }
                ext_w[g * KN + k] = w[g * K + k];
            }
            for (int j = 0; j < N; j++) {
                int replicas = S / N;
                int d = j * replicas + r % replicas;
                ext_ids[g * KN + K + j] = d * ne;
                ext_w[g * KN + K + j] = 1.0f;
            }
        }
    return flags;
}
