// extern "C" entry points of libmoedisp: argument validation on the host, then the
// kernel launchers. Validation never touches the GPU, so every rejection path works on
// a machine without one. Conventions are documented in include/moedisp.h.
#include <stdio.h>
#include <string.h>

#include <initializer_list>
#include <mutex>

#include "kernels.h"

namespace {

struct Span {
    const void* p;
    size_t bytes;
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const Span& a, const Span& b) {
    if (a.p == nullptr || b.p == nullptr || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a.p), y = reinterpret_cast<uintptr_t>(b.p);
    return x < y + b.bytes && y < x + a.bytes;
}

// True when any output span overlaps another output or any input span.
bool any_alias(std::initializer_list<Span> outs, std::initializer_list<Span> ins) {
    for (auto o = outs.begin(); o != outs.end(); ++o) {
        for (auto o2 = o + 1; o2 != outs.end(); ++o2)
            if (overlaps(*o, *o2)) return true;
        for (const Span& i : ins)
            if (overlaps(*o, i)) return true;
    }
    return false;
}

int rc(cudaError_t e) { return e == cudaSuccess ? MOEDISP_OK : MOEDISP_ERR_CUDA; }

int check_dims(const moedisp_dims& d) {
    if (d.W < 1 || d.T < 0 || d.K < 1 || d.E < 1) return MOEDISP_ERR_INVALID;
    if (d.E % d.W != 0) return MOEDISP_ERR_INVALID;
    if (d.K > MOEDISP_MAX_K || d.E > MOEDISP_MAX_E) return MOEDISP_ERR_UNSUPPORTED;
    if ((int64_t)d.W * d.T * d.K >= (int64_t(1) << 30)) return MOEDISP_ERR_UNSUPPORTED;
    return MOEDISP_OK;
}

// major_align: 0 or 1 (no padding) up to MOEDISP_MAX_ALIGN; the padded row count
// (at most G*K + E*align) must stay an int32 row index.
int check_major_align(int major_align, const moedisp_dims& d) {
    if (major_align < 0) return MOEDISP_ERR_INVALID;
    if (major_align > MOEDISP_MAX_ALIGN) return MOEDISP_ERR_UNSUPPORTED;
    const int64_t worst = (int64_t)d.W * d.T * d.K + (major_align > 1 ? (int64_t)d.E * major_align : 0);
    if (worst >= (int64_t(1) << 31)) return MOEDISP_ERR_UNSUPPORTED;
    return MOEDISP_OK;
}

int check_rows_cap(int64_t rows_cap) {
    if (rows_cap < 0) return MOEDISP_ERR_INVALID;
    if (rows_cap > 0x7fffffffll) return MOEDISP_ERR_UNSUPPORTED;
    return MOEDISP_OK;
}

const char* const kStatusNames[16] = {
    "ok",
    "capacity",
    "bad expert id",
    "capacity | bad expert id",
    "timeout",
    "capacity | timeout",
    "bad expert id | timeout",
    "capacity | bad expert id | timeout",
    "bad split",
    "capacity | bad split",
    "bad expert id | bad split",
    "capacity | bad expert id | bad split",
    "timeout | bad split",
    "capacity | timeout | bad split",
    "bad expert id | timeout | bad split",
    "capacity | bad expert id | timeout | bad split",
};

}  // namespace

namespace {
// moe_dispatch and moe_dispatch_gather: token g's row is token_rows[g] of x (x_rows rows),
// or row g when token_rows is null (x_rows = G).
int dispatch_impl(const void* x, int64_t x_rows, const int64_t* token_rows, int H, moedisp_dims dims,
                         const moedisp_layout* layout, int quant_mode,
                         const float* smooth_scales, void* expand_x,
                         float* dynamic_scales, int64_t* expert_token_nums,
                         int expert_token_nums_type, int32_t* ep_recv_counts,
                         int32_t* status, moedisp_stream_t stream) {
    if (!layout || !status) return MOEDISP_ERR_NULLPTR;
    int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    const moedisp_layout& L = *layout;
    if ((c = check_rows_cap(L.rows_cap)) != MOEDISP_OK) return c;
    if (quant_mode != MOEDISP_QUANT_NONE && quant_mode != MOEDISP_QUANT_INT8 &&
        quant_mode != MOEDISP_QUANT_FP8_E4M3)
        return MOEDISP_ERR_INVALID;
    if (expert_token_nums && expert_token_nums_type != 0 && expert_token_nums_type != 1)
        return MOEDISP_ERR_INVALID;
    if (smooth_scales && quant_mode == MOEDISP_QUANT_NONE) return MOEDISP_ERR_INVALID;
    if (H <= 0) return MOEDISP_ERR_INVALID;
    if (H > MOEDISP_MAX_H) return MOEDISP_ERR_UNSUPPORTED;
    if (H % (quant_mode == MOEDISP_QUANT_NONE ? 8 : 16) != 0) return MOEDISP_ERR_MISALIGNED;
    const int64_t G = (int64_t)dims.W * dims.T;
    const int64_t slots = G * dims.K;
    if (G > 0 && (!x || !L.dst_row)) return MOEDISP_ERR_NULLPTR;
    if (x_rows < 0) return MOEDISP_ERR_INVALID;
    if (smooth_scales && L.rows_cap > 0 && (!L.assist_info || !L.expert_base))
        return MOEDISP_ERR_NULLPTR;
    if (L.rows_cap > 0 && !expand_x) return MOEDISP_ERR_NULLPTR;
    if (quant_mode != MOEDISP_QUANT_NONE && L.rows_cap > 0 && !dynamic_scales)
        return MOEDISP_ERR_NULLPTR;
    if (expert_token_nums && (!L.expert_base || !L.rank_base)) return MOEDISP_ERR_NULLPTR;
    if (ep_recv_counts && (!L.cnt || !L.expert_base)) return MOEDISP_ERR_NULLPTR;
    if (!aligned(x, 16) || !aligned(expand_x, 16) || !aligned(L.dst_row, 4) ||
        !aligned(dynamic_scales, 4) || !aligned(expert_token_nums, 8) ||
        !aligned(ep_recv_counts, 4) || !aligned(status, 4) || !aligned(smooth_scales, 16) ||
        !aligned(L.assist_info, 4) || !aligned(L.expert_base, 8) || !aligned(token_rows, 8))
        return MOEDISP_ERR_MISALIGNED;
    const size_t out_row = quant_mode == MOEDISP_QUANT_NONE ? (size_t)H * 2 : (size_t)H;
    const int ne = dims.E / dims.W;
    const Span scales{quant_mode == MOEDISP_QUANT_NONE ? nullptr : dynamic_scales,
                      (size_t)L.rows_cap * 4};
    if (any_alias({{expand_x, (size_t)L.rows_cap * out_row},
                   scales,
                   {expert_token_nums, (size_t)dims.E * 8},
                   {ep_recv_counts, (size_t)dims.W * ne * dims.W * 4},
                   {status, 4}},
                  {{x, (size_t)x_rows * H * 2},
                   {token_rows, (size_t)G * 8},
                   {L.dst_row, (size_t)slots * 4},
                   {smooth_scales, (size_t)dims.E * H * 4},
                   {smooth_scales ? L.assist_info : nullptr, (size_t)L.rows_cap * 4},
                   {L.cnt, (size_t)dims.W * dims.E * 4},
                   {L.expert_base, (size_t)(dims.E + 1) * 8},
                   {L.rank_base, (size_t)(dims.W + 1) * 8}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_dispatch(x, x_rows, token_rows, H, dims, L, quant_mode, smooth_scales,
                                       expand_x,
                                       dynamic_scales,
                                       expert_token_nums, expert_token_nums_type, ep_recv_counts,
                                       status, stream));
}
}  // namespace

extern "C" {

const char* moedisp_status_string(int code) {
    switch (code) {
        case MOEDISP_ERR_NULLPTR: return "null pointer";
        case MOEDISP_ERR_INVALID: return "invalid argument";
        case MOEDISP_ERR_MISALIGNED: return "misaligned pointer or row size";
        case MOEDISP_ERR_ALIASED: return "output overlaps another buffer";
        case MOEDISP_ERR_UNSUPPORTED: return "unsupported size or mode";
        case MOEDISP_ERR_WORKSPACE: return "workspace missing or too small";
        case MOEDISP_ERR_CUDA: return "CUDA runtime error";
        default: break;
    }
    if (code >= 0 && code < 16) return kStatusNames[code];
    return "unknown code";
}

int moedisp_version(void) { return 3; }

int moedisp_selftest_bounded_wait(uint32_t limit_us, int32_t* status, moedisp_stream_t stream) {
    if (!status) return MOEDISP_ERR_NULLPTR;
    if (!aligned(status, 4)) return MOEDISP_ERR_MISALIGNED;
    if (limit_us < 1 || limit_us > 10000000u) return MOEDISP_ERR_INVALID;
    return rc(moedisp::launch_bounded_wait_selftest((uint64_t)limit_us * 1000ull, status, stream));
}

int moedisp_ep_barrier(uint32_t* const* peer_signals, int W, int rank, uint32_t epoch,
                       uint32_t timeout_us, int32_t* status, moedisp_stream_t stream) {
    if (!peer_signals || !status) return MOEDISP_ERR_NULLPTR;
    if (W < 1 || rank < 0 || rank >= W || epoch == 0) return MOEDISP_ERR_INVALID;
    if (W > MOEDISP_MAX_W) return MOEDISP_ERR_UNSUPPORTED;
    if (timeout_us < 1 || timeout_us > 10000000u) return MOEDISP_ERR_INVALID;
    if (!aligned(peer_signals, 8) || !aligned(status, 4)) return MOEDISP_ERR_MISALIGNED;
    return rc(moedisp::launch_ep_barrier(peer_signals, W, rank, epoch,
                                         (uint64_t)timeout_us * 1000ull, status, stream));
}

int moedisp_a2a_exchange_plan(const int64_t* in_splits, int W, int64_t* src_offsets,
                              int64_t* out_splits, int64_t* dst_offsets, int32_t* status,
                              moedisp_stream_t stream) {
    if (!in_splits || !src_offsets || !out_splits || !dst_offsets || !status)
        return MOEDISP_ERR_NULLPTR;
    if (W < 1) return MOEDISP_ERR_INVALID;
    if (W > MOEDISP_MAX_W) return MOEDISP_ERR_UNSUPPORTED;
    if (!aligned(in_splits, 8) || !aligned(src_offsets, 8) || !aligned(out_splits, 8) ||
        !aligned(dst_offsets, 8) || !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const size_t n = (size_t)W * W * sizeof(int64_t);
    if (any_alias({{src_offsets, n}, {out_splits, n}, {dst_offsets, n}, {status, 4}},
                  {{in_splits, n}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_a2a_plan(in_splits, W, src_offsets, out_splits, dst_offsets, status,
                                       stream));
}

int moedisp_a2a_v(const void* in, int64_t in_rank_stride_rows, void* out,
                  int64_t out_cap_rows, int64_t row_bytes, int W,
                  const int64_t* src_offsets, const int64_t* out_splits,
                  const int64_t* dst_offsets, int32_t* status, moedisp_stream_t stream) {
    if (!src_offsets || !out_splits || !dst_offsets || !status) return MOEDISP_ERR_NULLPTR;
    if (W < 1 || in_rank_stride_rows < 0 || out_cap_rows < 0 || row_bytes <= 0)
        return MOEDISP_ERR_INVALID;
    if (W > MOEDISP_MAX_W) return MOEDISP_ERR_UNSUPPORTED;
    if ((in_rank_stride_rows > 0 && !in) || (out_cap_rows > 0 && !out)) return MOEDISP_ERR_NULLPTR;
    if (row_bytes % 16 != 0 || !aligned(in, 16) || !aligned(out, 16) || !aligned(src_offsets, 8) ||
        !aligned(out_splits, 8) || !aligned(dst_offsets, 8) || !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const double in_total = (double)W * (double)in_rank_stride_rows * (double)row_bytes;
    const double out_total = (double)W * (double)out_cap_rows * (double)row_bytes;
    if (in_total > 4.0e18 || out_total > 4.0e18) return MOEDISP_ERR_UNSUPPORTED;
    const size_t nin = (size_t)W * in_rank_stride_rows * row_bytes;
    const size_t nout = (size_t)W * out_cap_rows * row_bytes;
    const size_t np = (size_t)W * W * sizeof(int64_t);
    if (any_alias({{out, nout}, {status, 4}},
                  {{in, nin}, {src_offsets, np}, {out_splits, np}, {dst_offsets, np}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_a2a_v(in, in_rank_stride_rows, out, out_cap_rows, row_bytes, W,
                                    src_offsets, out_splits, dst_offsets, status, stream));
}

int moedisp_layout_workspace_size(moedisp_dims dims, size_t* bytes) {
    if (!bytes) return MOEDISP_ERR_NULLPTR;
    const int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    *bytes = moedisp::layout_geometry(dims).total_bytes;
    return MOEDISP_OK;
}

int moedisp_moe_dispatch_layout(const int32_t* expert_ids, const uint8_t* active_mask,
                                int active_mask_dims, int major_align, moedisp_dims dims, const moedisp_layout* layout,
                                void* workspace, size_t workspace_bytes, int32_t* status,
                                moedisp_stream_t stream) {
    if (!layout || !status) return MOEDISP_ERR_NULLPTR;
    int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    const moedisp_layout& L = *layout;
    if ((c = check_rows_cap(L.rows_cap)) != MOEDISP_OK) return c;
    const int64_t slots = (int64_t)dims.W * dims.T * dims.K;
    if (!L.cnt || !L.expert_base || !L.rank_base || !L.send_splits) return MOEDISP_ERR_NULLPTR;
    if (slots > 0 && (!expert_ids || !L.occ || !L.dst_row)) return MOEDISP_ERR_NULLPTR;
    if (L.rows_cap > 0 && !L.assist_info) return MOEDISP_ERR_NULLPTR;
    if (active_mask && active_mask_dims != 1 && active_mask_dims != 2) return MOEDISP_ERR_INVALID;
    if ((c = check_major_align(major_align, dims)) != MOEDISP_OK) return c;
    if (!workspace) return MOEDISP_ERR_WORKSPACE;
    const moedisp::LayoutGeometry g = moedisp::layout_geometry(dims);
    if (workspace_bytes < g.total_bytes) return MOEDISP_ERR_WORKSPACE;
    if (!aligned(expert_ids, 4) || !aligned(L.cnt, 4) || !aligned(L.occ, 4) ||
        !aligned(L.dst_row, 4) || !aligned(L.assist_info, 4) || !aligned(L.expert_base, 8) ||
        !aligned(L.rank_base, 8) || !aligned(L.send_splits, 8) || !aligned(workspace, 16) ||
        !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const int64_t G = (int64_t)dims.W * dims.T;
    if (any_alias({{L.cnt, (size_t)dims.W * dims.E * 4},
                   {L.occ, (size_t)slots * 4},
                   {L.dst_row, (size_t)slots * 4},
                   {L.assist_info, (size_t)L.rows_cap * 4},
                   {L.expert_base, (size_t)(dims.E + 1) * 8},
                   {L.rank_base, (size_t)(dims.W + 1) * 8},
                   {L.send_splits, (size_t)dims.W * dims.W * 8},
                   {workspace, g.total_bytes},
                   {status, 4}},
                  {{expert_ids, (size_t)slots * 4},
                   {active_mask, (size_t)(active_mask_dims == 2 ? slots : G)}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_layout(expert_ids, active_mask, active_mask_dims, major_align, dims,
                                     L, workspace, status, stream));
}

int moedisp_moe_dispatch_layout_noalloc(const int32_t* expert_ids, const uint8_t* active_mask,
                                        int active_mask_dims, int major_align, moedisp_dims dims, const moedisp_layout* layout,
                                        int32_t* status, moedisp_stream_t stream) {
    if (!layout || !status) return MOEDISP_ERR_NULLPTR;
    int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    const moedisp_layout& L = *layout;
    if ((c = check_rows_cap(L.rows_cap)) != MOEDISP_OK) return c;
    const int64_t slots = (int64_t)dims.W * dims.T * dims.K;
    if (!L.cnt || !L.expert_base || !L.rank_base || !L.send_splits) return MOEDISP_ERR_NULLPTR;
    if (slots > 0 && (!expert_ids || !L.occ || !L.dst_row)) return MOEDISP_ERR_NULLPTR;
    if (L.rows_cap > 0 && !L.assist_info) return MOEDISP_ERR_NULLPTR;
    if (active_mask && active_mask_dims != 1 && active_mask_dims != 2) return MOEDISP_ERR_INVALID;
    if ((c = check_major_align(major_align, dims)) != MOEDISP_OK) return c;
    if (moedisp::layout_geometry(dims).total_bytes > moedisp::layout_noalloc_scratch_bytes())
        return MOEDISP_ERR_UNSUPPORTED;
    if (!aligned(expert_ids, 4) || !aligned(L.cnt, 4) || !aligned(L.occ, 4) ||
        !aligned(L.dst_row, 4) || !aligned(L.assist_info, 4) || !aligned(L.expert_base, 8) ||
        !aligned(L.rank_base, 8) || !aligned(L.send_splits, 8) || !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const int64_t G = (int64_t)dims.W * dims.T;
    if (any_alias({{L.cnt, (size_t)dims.W * dims.E * 4},
                   {L.occ, (size_t)slots * 4},
                   {L.dst_row, (size_t)slots * 4},
                   {L.assist_info, (size_t)L.rows_cap * 4},
                   {L.expert_base, (size_t)(dims.E + 1) * 8},
                   {L.rank_base, (size_t)(dims.W + 1) * 8},
                   {L.send_splits, (size_t)dims.W * dims.W * 8},
                   {status, 4}},
                  {{expert_ids, (size_t)slots * 4},
                   {active_mask, (size_t)(active_mask_dims == 2 ? slots : G)}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_layout_noalloc(expert_ids, active_mask, active_mask_dims,
                                             major_align, dims, L, status, stream));
}

int moedisp_moe_dispatch(const void* x, int H, moedisp_dims dims,
                         const moedisp_layout* layout, int quant_mode,
                         const float* smooth_scales, void* expand_x,
                         float* dynamic_scales, int64_t* expert_token_nums,
                         int expert_token_nums_type, int32_t* ep_recv_counts,
                         int32_t* status, moedisp_stream_t stream) {
    return dispatch_impl(x, (int64_t)dims.W * dims.T, nullptr, H, dims, layout, quant_mode,
                         smooth_scales, expand_x, dynamic_scales, expert_token_nums,
                         expert_token_nums_type, ep_recv_counts, status, stream);
}

int moedisp_moe_dispatch_gather(const void* x, int64_t x_rows, const int64_t* token_rows, int H,
                                moedisp_dims dims, const moedisp_layout* layout, int quant_mode,
                                const float* smooth_scales, void* expand_x,
                                float* dynamic_scales, int64_t* expert_token_nums,
                                int expert_token_nums_type, int32_t* ep_recv_counts,
                                int32_t* status, moedisp_stream_t stream) {
    if ((int64_t)dims.W * dims.T > 0 && !token_rows) return MOEDISP_ERR_NULLPTR;
    return dispatch_impl(x, x_rows, token_rows, H, dims, layout, quant_mode, smooth_scales,
                         expand_x, dynamic_scales, expert_token_nums, expert_token_nums_type,
                         ep_recv_counts, status, stream);
}

int moedisp_a2a_dispatch_pipelined_workspace_size(int W, size_t* bytes) {
    if (!bytes) return MOEDISP_ERR_NULLPTR;
    if (W < 1) return MOEDISP_ERR_INVALID;
    if (W > MOEDISP_MAX_W) return MOEDISP_ERR_UNSUPPORTED;
    *bytes = moedisp::pipeline_workspace_bytes(W);
    return MOEDISP_OK;
}

int moedisp_a2a_dispatch_pipelined(const void* in, int64_t in_rank_stride_rows,
                                   const int64_t* src_offsets, const int64_t* out_splits,
                                   const int64_t* dst_offsets, void* recv, int H,
                                   moedisp_dims dims, const moedisp_layout* layout,
                                   int quant_mode, void* expand_x, float* dynamic_scales,
                                   int64_t* expert_token_nums, int expert_token_nums_type,
                                   int32_t* ep_recv_counts, uint32_t* ready, uint32_t epoch,
                                   int roles, uint32_t wait_limit_us, void* workspace,
                                   size_t workspace_bytes, int32_t* status,
                                   moedisp_stream_t stream) {
    if (!layout || !status) return MOEDISP_ERR_NULLPTR;
    int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    const moedisp_layout& L = *layout;
    if ((c = check_rows_cap(L.rows_cap)) != MOEDISP_OK) return c;
    if (quant_mode != MOEDISP_QUANT_NONE && quant_mode != MOEDISP_QUANT_INT8 &&
        quant_mode != MOEDISP_QUANT_FP8_E4M3)
        return MOEDISP_ERR_INVALID;
    if (expert_token_nums && expert_token_nums_type != 0 && expert_token_nums_type != 1)
        return MOEDISP_ERR_INVALID;
    if (roles != MOEDISP_PIPE_PRODUCE && roles != MOEDISP_PIPE_CONSUME && roles != MOEDISP_PIPE_BOTH)
        return MOEDISP_ERR_INVALID;
    if (wait_limit_us < 1 || wait_limit_us > 10000000u) return MOEDISP_ERR_INVALID;
    if (epoch == 0) return MOEDISP_ERR_INVALID;        // zeroed words would read as published
    if (H <= 0 || in_rank_stride_rows < 0) return MOEDISP_ERR_INVALID;
    if (H > MOEDISP_MAX_H) return MOEDISP_ERR_UNSUPPORTED;
    if (H % (quant_mode == MOEDISP_QUANT_NONE ? 8 : 16) != 0) return MOEDISP_ERR_MISALIGNED;
    const int64_t G = (int64_t)dims.W * dims.T;
    if (G == 0 && (!src_offsets || !out_splits || !dst_offsets)) return MOEDISP_OK;
    if (!src_offsets || !out_splits || !dst_offsets || !ready || !workspace)
        return MOEDISP_ERR_NULLPTR;
    if (G > 0 && (!recv || !L.dst_row)) return MOEDISP_ERR_NULLPTR;
    if (in_rank_stride_rows > 0 && !in) return MOEDISP_ERR_NULLPTR;
    if (L.rows_cap > 0 && !expand_x) return MOEDISP_ERR_NULLPTR;
    if (quant_mode != MOEDISP_QUANT_NONE && L.rows_cap > 0 && !dynamic_scales)
        return MOEDISP_ERR_NULLPTR;
    if (expert_token_nums && (!L.expert_base || !L.rank_base)) return MOEDISP_ERR_NULLPTR;
    if (ep_recv_counts && (!L.cnt || !L.expert_base)) return MOEDISP_ERR_NULLPTR;
    if (workspace_bytes < moedisp::pipeline_workspace_bytes(dims.W)) return MOEDISP_ERR_WORKSPACE;
    if (!aligned(in, 16) || !aligned(recv, 16) || !aligned(expand_x, 16) ||
        !aligned(src_offsets, 8) || !aligned(out_splits, 8) || !aligned(dst_offsets, 8) ||
        !aligned(L.dst_row, 4) || !aligned(dynamic_scales, 4) || !aligned(expert_token_nums, 8) ||
        !aligned(ep_recv_counts, 4) || !aligned(ready, 4) || !aligned(workspace, 16) ||
        !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const size_t row = (size_t)H * 2;
    const size_t out_row = quant_mode == MOEDISP_QUANT_NONE ? row : (size_t)H;
    const size_t plan = (size_t)dims.W * dims.W * 8;
    const int ne = dims.E / dims.W;
    const Span scales{quant_mode == MOEDISP_QUANT_NONE ? nullptr : dynamic_scales,
                      (size_t)L.rows_cap * 4};
    if (any_alias({{recv, (size_t)G * row},
                   {expand_x, (size_t)L.rows_cap * out_row},
                   scales,
                   {expert_token_nums, (size_t)dims.E * 8},
                   {ep_recv_counts, (size_t)dims.W * ne * dims.W * 4},
                   {ready, (size_t)dims.W * dims.W * 4},
                   {workspace, moedisp::pipeline_workspace_bytes(dims.W)},
                   {status, 4}},
                  {{in, (size_t)dims.W * in_rank_stride_rows * row},
                   {src_offsets, plan}, {out_splits, plan}, {dst_offsets, plan},
                   {L.dst_row, (size_t)G * dims.K * 4},
                   {L.cnt, (size_t)dims.W * dims.E * 4},
                   {L.expert_base, (size_t)(dims.E + 1) * 8},
                   {L.rank_base, (size_t)(dims.W + 1) * 8}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_a2a_dispatch_pipelined(
        in, in_rank_stride_rows, src_offsets, out_splits, dst_offsets, recv, H, dims, L,
        quant_mode, expand_x, dynamic_scales, expert_token_nums, expert_token_nums_type,
        ep_recv_counts, ready, epoch, roles, (uint64_t)wait_limit_us * 1000ull, workspace, status,
        stream));
}

int moedisp_a2a_token_rows(const int64_t* src_offsets, const int64_t* out_splits,
                           const int64_t* dst_offsets, int W, int64_t T,
                           int64_t in_rank_stride_rows, int64_t* token_rows, uint8_t* active,
                           int32_t* status, moedisp_stream_t stream) {
    if (!status) return MOEDISP_ERR_NULLPTR;
    if (W < 1 || T < 0 || in_rank_stride_rows < 0) return MOEDISP_ERR_INVALID;
    if (W > MOEDISP_MAX_W) return MOEDISP_ERR_UNSUPPORTED;
    // With T = 0 there are no positions, but a given plan is still checked for rows that
    // would need one (CAPACITY).
    if (T == 0 && (!src_offsets || !out_splits || !dst_offsets)) return MOEDISP_OK;
    if (!src_offsets || !out_splits || !dst_offsets || (T > 0 && !token_rows))
        return MOEDISP_ERR_NULLPTR;
    if (!aligned(src_offsets, 8) || !aligned(out_splits, 8) || !aligned(dst_offsets, 8) ||
        !aligned(token_rows, 8) || !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const size_t plan = (size_t)W * W * 8, n = (size_t)W * T;
    if (any_alias({{token_rows, n * 8}, {active, n}, {status, 4}},
                  {{src_offsets, plan}, {out_splits, plan}, {dst_offsets, plan}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_a2a_token_rows(src_offsets, out_splits, dst_offsets, W, T,
                                             in_rank_stride_rows, token_rows, active, status,
                                             stream));
}

int moedisp_moe_combine(const void* expert_out, int H, moedisp_dims dims,
                        const moedisp_layout* layout, const float* expert_scales, void* y,
                        int32_t* status, moedisp_stream_t stream) {
    if (!layout || !status) return MOEDISP_ERR_NULLPTR;
    int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    const moedisp_layout& L = *layout;
    if ((c = check_rows_cap(L.rows_cap)) != MOEDISP_OK) return c;
    if (H <= 0) return MOEDISP_ERR_INVALID;
    if (H % 8 != 0) return MOEDISP_ERR_MISALIGNED;
    const int64_t G = (int64_t)dims.W * dims.T;
    if (G == 0) return MOEDISP_OK;
    if (!y || !expert_scales || !L.dst_row) return MOEDISP_ERR_NULLPTR;
    if (L.rows_cap > 0 && !expert_out) return MOEDISP_ERR_NULLPTR;
    if (!aligned(expert_out, 16) || !aligned(y, 16) || !aligned(expert_scales, 4) ||
        !aligned(L.dst_row, 4) || !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    if (any_alias({{y, (size_t)G * H * 2}, {status, 4}},
                  {{expert_out, (size_t)L.rows_cap * H * 2},
                   {expert_scales, (size_t)G * dims.K * 4},
                   {L.dst_row, (size_t)G * dims.K * 4}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_combine(expert_out, H, dims, L, expert_scales, y, status, stream));
}

int moedisp_moe_dispatch_peers(const void* x, int H, moedisp_dims dims, int rank,
                               const int32_t* expert_ids, const moedisp_layout* layout,
                               int quant_mode, void* const* peer_expand_x,
                               float* const* peer_scales, int64_t peer_rows_cap, int32_t* status,
                               moedisp_stream_t stream) {
    if (!layout || !status) return MOEDISP_ERR_NULLPTR;
    int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    const moedisp_layout& L = *layout;
    if ((c = check_rows_cap(L.rows_cap)) != MOEDISP_OK) return c;
    if (rank < 0 || rank >= dims.W || peer_rows_cap < 0) return MOEDISP_ERR_INVALID;
    if (quant_mode != MOEDISP_QUANT_NONE && quant_mode != MOEDISP_QUANT_INT8 &&
        quant_mode != MOEDISP_QUANT_FP8_E4M3)
        return MOEDISP_ERR_INVALID;
    if (H <= 0) return MOEDISP_ERR_INVALID;
    if (H > MOEDISP_MAX_H) return MOEDISP_ERR_UNSUPPORTED;
    if (H % (quant_mode == MOEDISP_QUANT_NONE ? 8 : 16) != 0) return MOEDISP_ERR_MISALIGNED;
    if (dims.T == 0) return MOEDISP_OK;
    if (!x || !expert_ids || !L.dst_row || !L.rank_base || !peer_expand_x) return MOEDISP_ERR_NULLPTR;
    if (quant_mode != MOEDISP_QUANT_NONE && !peer_scales) return MOEDISP_ERR_NULLPTR;
    if (!aligned(x, 16) || !aligned(expert_ids, 4) || !aligned(L.dst_row, 4) ||
        !aligned(L.rank_base, 8) || !aligned(peer_expand_x, 8) || !aligned(peer_scales, 8) ||
        !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    return rc(moedisp::launch_dispatch_peers(x, H, dims, rank, expert_ids, L, quant_mode,
                                             peer_expand_x, peer_scales, peer_rows_cap, status,
                                             stream));
}

int moedisp_moe_combine_peers(const void* const* peer_expert_out, int64_t peer_rows_cap, int H,
                              moedisp_dims dims, int rank, const int32_t* expert_ids,
                              const moedisp_layout* layout, const float* expert_scales, void* y,
                              int32_t* status, moedisp_stream_t stream) {
    if (!layout || !status) return MOEDISP_ERR_NULLPTR;
    int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    const moedisp_layout& L = *layout;
    if ((c = check_rows_cap(L.rows_cap)) != MOEDISP_OK) return c;
    if (rank < 0 || rank >= dims.W || peer_rows_cap < 0 || H <= 0) return MOEDISP_ERR_INVALID;
    if (H % 8 != 0) return MOEDISP_ERR_MISALIGNED;
    if (dims.T == 0) return MOEDISP_OK;
    if (!peer_expert_out || !expert_ids || !L.dst_row || !L.rank_base || !expert_scales || !y)
        return MOEDISP_ERR_NULLPTR;
    if (!aligned(peer_expert_out, 8) || !aligned(expert_ids, 4) || !aligned(L.dst_row, 4) ||
        !aligned(L.rank_base, 8) || !aligned(expert_scales, 4) || !aligned(y, 16) ||
        !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const size_t slots = (size_t)dims.W * dims.T * dims.K;
    if (any_alias({{y, (size_t)dims.T * H * 2}, {status, 4}},
                  {{expert_ids, slots * 4}, {L.dst_row, slots * 4},
                   {expert_scales, (size_t)dims.T * dims.K * 4}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_combine_peers(peer_expert_out, peer_rows_cap, H, dims, rank,
                                            expert_ids, L, expert_scales, y, status, stream));
}

int moedisp_shared_expert_routing(const int32_t* expert_ids, const float* expert_scales, int W,
                                  int T, int K, int E, int shared_expert_num,
                                  int shared_expert_rank_num, int32_t* ext_ids, float* ext_scales,
                                  int32_t* status, moedisp_stream_t stream) {
    const int N = shared_expert_num, S = shared_expert_rank_num;
    if (!status) return MOEDISP_ERR_NULLPTR;
    if (W < 1 || T < 0 || K < 1 || E < 1 || N < 0 || S < 0 || S >= W) return MOEDISP_ERR_INVALID;
    if ((S == 0) != (N == 0)) return MOEDISP_ERR_INVALID;
    if (S > 0 && (W % S != 0 || S % N != 0)) return MOEDISP_ERR_INVALID;
    if (E % (W - S) != 0) return MOEDISP_ERR_INVALID;
    if (K + N > MOEDISP_MAX_K) return MOEDISP_ERR_UNSUPPORTED;
    if ((int64_t)W * (E / (W - S)) > MOEDISP_MAX_E) return MOEDISP_ERR_UNSUPPORTED;
    const int64_t G = (int64_t)W * T;
    if (G * (K + N) >= (int64_t(1) << 30)) return MOEDISP_ERR_UNSUPPORTED;
    if (G == 0) return MOEDISP_OK;
    if (!expert_ids || !expert_scales || !ext_ids || !ext_scales) return MOEDISP_ERR_NULLPTR;
    if (!aligned(expert_ids, 4) || !aligned(expert_scales, 4) || !aligned(ext_ids, 4) ||
        !aligned(ext_scales, 4) || !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const size_t nin = (size_t)G * K * 4, nout = (size_t)G * (K + N) * 4;
    if (any_alias({{ext_ids, nout}, {ext_scales, nout}, {status, 4}},
                  {{expert_ids, nin}, {expert_scales, nin}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_shared_routing(expert_ids, expert_scales, W, T, K, E, N, S, ext_ids,
                                             ext_scales, status, stream));
}

int moedisp_moe_combine_rmsnorm(const void* expert_out, int H, moedisp_dims dims,
                                const moedisp_layout* layout, const float* expert_scales,
                                const void* residual, const float* gamma, float eps,
                                void* residual_out, void* y, int32_t* status,
                                moedisp_stream_t stream) {
    if (!layout || !status) return MOEDISP_ERR_NULLPTR;
    int c = check_dims(dims);
    if (c != MOEDISP_OK) return c;
    const moedisp_layout& L = *layout;
    if ((c = check_rows_cap(L.rows_cap)) != MOEDISP_OK) return c;
    if (H <= 0 || !(eps >= 0.0f) || eps > 1.0e30f) return MOEDISP_ERR_INVALID;
    if (H % 8 != 0) return MOEDISP_ERR_MISALIGNED;
    if (H > MOEDISP_MAX_H) return MOEDISP_ERR_UNSUPPORTED;
    const int64_t G = (int64_t)dims.W * dims.T;
    if (G == 0) return MOEDISP_OK;
    if (!y || !expert_scales || !L.dst_row || !residual || !gamma) return MOEDISP_ERR_NULLPTR;
    if (L.rows_cap > 0 && !expert_out) return MOEDISP_ERR_NULLPTR;
    if (!aligned(expert_out, 16) || !aligned(y, 16) || !aligned(residual, 16) ||
        !aligned(residual_out, 16) || !aligned(gamma, 16) || !aligned(expert_scales, 4) ||
        !aligned(L.dst_row, 4) || !aligned(status, 4))
        return MOEDISP_ERR_MISALIGNED;
    const size_t rowb = (size_t)G * H * 2;
    if (any_alias({{y, rowb}, {residual_out, rowb}, {status, 4}},
                  {{expert_out, (size_t)L.rows_cap * H * 2},
                   {residual, rowb},
                   {gamma, (size_t)H * 4},
                   {expert_scales, (size_t)G * dims.K * 4},
                   {L.dst_row, (size_t)G * dims.K * 4}}))
        return MOEDISP_ERR_ALIASED;
    return rc(moedisp::launch_combine_rmsnorm(expert_out, H, dims, L, expert_scales, residual, gamma,
                                              eps, residual_out, y, status, stream));
}

}  // extern "C"
