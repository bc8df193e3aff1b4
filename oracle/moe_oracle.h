/*
 * moe_oracle.h -- plain, slow CPU oracle for expert-parallel MoE dispatch / combine
 * and the all-to-all-v exchange plan.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU
 * baseline may call it. It shares no code, header, table or helper with the CUDA
 * library; the two are compared on the same seeded inputs.
 *
 * Layouts (row-major, plain host memory, caller-owned):
 *   in_splits[W][W]          S[i][j] = rows rank i sends to rank j
 *   expert_ids[G][K] int32   slot s = g*K + k, token g = r*T + t on source rank r
 *   x[G][H] bf16 bits, expand_x[rows_cap][H] (bf16 bits, int8 or e4m3 bytes)
 *
 * Return values: 0 or a bitwise OR of ORC_* flags describing invalid input that was
 * skipped (never an out-of-bounds access).
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    ORC_CAPACITY = 1,      /* more rows than the receive capacity */
    ORC_BAD_EXPERT = 2,    /* an expert id outside [0, E) */
    ORC_BAD_SPLIT = 8,     /* a negative split or a segment outside its buffer */
    ORC_BAD_ARG = 16       /* unusable dimensions */
};

/* bf16 / OCP-OFP8 E4M3 conversions written from the formats' definitions. */
uint16_t orc_bf16_from_f32(float v);                 /* round to nearest even */
float orc_bf16_to_f32(uint16_t b);
uint8_t orc_e4m3_from_f32(float v);                  /* RNE, saturate to +-448 */
float orc_e4m3_to_f32(uint8_t c);

/* O1: exchange plan. Outputs are [W][W]; row i is what rank i holds. */
int orc_a2a_exchange_plan(int W, const int64_t *in_splits, int64_t *src_offsets,
                          int64_t *out_splits, int64_t *dst_offsets);

/* O2: all-to-all-v of byte rows. Rank j's send rows start at in + j*in_rank_stride_rows
 * rows; rank i's receive rows at out + i*out_cap_rows rows. */
int orc_a2a_v(int W, const uint8_t *in, int64_t in_rank_stride_rows, uint8_t *out,
              int64_t out_cap_rows, int64_t row_bytes, const int64_t *src_offsets,
              const int64_t *out_splits, const int64_t *dst_offsets);

/* O3: dispatch layout. active may be NULL (all active); active_dims 1: active[G] per
 * token, 2: active[G][K] per slot. Inactive slots get occ = -1, dst_row = -1. major_align
 * 0/1: none, A >= 2: expert segments padded to multiples of A (at least A rows), padding
 * rows get assist_info -1. assist_info entries at or beyond R = expert_base[E] are left
 * untouched. */
int orc_moe_dispatch_layout(int W, int T, int K, int E, const int32_t *expert_ids,
                            const uint8_t *active, int active_dims, int64_t major_align,
                            int64_t rows_cap, int32_t *cnt,
                            int32_t *occ, int32_t *dst_row, int32_t *assist_info,
                            int64_t *expert_base, int64_t *rank_base, int64_t *send_splits);

/* Per-destination-rank outputs of dispatch, derived from cnt:
 * expert_token_nums[W][ne] (type 1 counts, type 0 inclusive prefix sum over local
 * experts); ep_recv_counts[W][ne][W] = rows that local expert le of rank d receives
 * from source rank r. */
int orc_moe_recv_counts(int W, int E, const int32_t *cnt, int64_t major_align,
                        int expert_token_nums_type, int64_t *expert_token_nums,
                        int32_t *ep_recv_counts);

/* O4: dispatch copy with optional per-token dynamic quantisation (0 none, 2 int8,
 * 3 fp8-e4m3). dynamic_scales may be NULL for mode 0. smooth ([E][H] fp32, quantising
 * modes only; needs expert_ids [G][K]) or NULL: per-expert smoothing before quantisation. */
int orc_moe_dispatch(int G, int K, int H, const uint16_t *x, const int32_t *dst_row,
                     int64_t rows_cap, int quant_mode, void *expand_x, float *dynamic_scales,
                     const float *smooth, int E, const int32_t *expert_ids);

/* Per-token quantisation of one row (exposed for pins). Returns the scale. */
float orc_quant_row(int H, const uint16_t *x, int quant_mode, uint8_t *q);
float orc_quant_row_f32(int H, const float *x, int quant_mode, uint8_t *q);

/* O5a: combine in double precision; y64[G][H]. */
int orc_moe_combine_f64(int G, int K, int H, const uint16_t *expert_out, int64_t rows_cap,
                        const int32_t *dst_row, const float *w, double *y64);
/* O5b: combine with a fixed-order fp32 fused multiply-add chain, then bf16 (RNE). */
int orc_moe_combine_f32(int G, int K, int H, const uint16_t *expert_out, int64_t rows_cap,
                        const int32_t *dst_row, const float *w, uint16_t *y);

/* Fused tail, MoE finalize + residual + RMSNorm ([P5]), on one GPU:
 *   s      = combine(g) + residual[g]           (the combine as in O5)
 *   res    = bf16(s)                            residual_out
 *   y[g,h] = bf16( res[h] / sqrt(mean_h res^2 + eps) * gamma[h] )
 * _f64: every step in double (res rounded to bf16 as defined); _f32: the fixed-order fp32
 * FMA chain, one fp32 add of the residual, the sum of squares in ascending h. */
int orc_moe_combine_rmsnorm_f64(int G, int K, int H, const uint16_t *expert_out,
                                int64_t rows_cap, const int32_t *dst_row, const float *w,
                                const uint16_t *residual, const float *gamma, float eps,
                                uint16_t *residual_out, double *y64);
int orc_moe_combine_rmsnorm_f32(int G, int K, int H, const uint16_t *expert_out,
                                int64_t rows_cap, const int32_t *dst_row, const float *w,
                                const uint16_t *residual, const float *gamma, float eps,
                                uint16_t *residual_out, uint16_t *y);

/* Shared experts ([P4] sharedExpertNum N, sharedExpertRankNum S, expertShardType 0): the
 * routing widened to K + N slots over W * (E / (W - S)) experts, shared-expert ranks
 * first; ext_ids / ext_w are [G][K + N]. */
int orc_shared_expert_routing(int W, int T, int K, int E, int N, int S,
                              const int32_t *expert_ids, const float *w,
                              int32_t *ext_ids, float *ext_w);

#ifdef __cplusplus
}
#endif
#endif
