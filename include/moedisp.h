/*
 * moedisp.h -- C ABI of libmoedisp: expert-parallel (EP) MoE token dispatch / combine
 * and the uneven all-to-all-v exchange, for NVIDIA B200 (sm_100a).
 *
 * The W EP ranks of the exchange are "virtual ranks": slices of one GPU's memory --
 * except in moe_dispatch_peers / moe_combine_peers, where they are W GPUs and the rows
 * move through a table of the ranks' buffer addresses (peer memory).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Ownership: the caller allocates and owns every buffer. All pointers named
 *    "device" point to device memory of the current CUDA device. The library never
 *    allocates, frees or synchronises; each call validates its arguments on the host,
 *    enqueues its kernels on `stream` and returns.
 *  - Host-detected errors return a negative MOEDISP_ERR_* code and enqueue nothing.
 *  - Device-detected errors are OR-ed into `*status` (an int32 in device memory that the
 *    caller zeroes) as MOEDISP_STATUS_* bits; read it after the stream completes. No
 *    kernel traps, asserts or waits without bound: every device-side wait gives up after
 *    about two seconds and sets MOEDISP_STATUS_TIMEOUT. A kernel that times out stops
 *    issuing copies and waits (again with a limit) for the ones in flight before it
 *    exits; the outputs of a call that reported MOEDISP_STATUS_TIMEOUT are undefined.
 *  - Empty inputs (no rows, no tokens, all splits 0) are valid no-ops.
 *  - Integer, index, copy and quantisation outputs are deterministic and bit-exact
 *    against a plain CPU implementation; combine sums each token's K rows in fp32 in
 *    ascending k with fused multiply-adds, so it is deterministic too.
 *
 * Notation: W ranks, T tokens per rank, G = W*T global tokens (token g = r*T + t lives on
 * source rank r), K experts per token, E experts, ne = E/W experts per rank,
 * owner(e) = e / ne. Slot s = g*K + k is the k-th expert choice of token g.
 */
#ifndef MOEDISP_H
#define MOEDISP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st *moedisp_stream_t;

/* Host-side return codes. The error classes follow the status-code convention of the
 * Ascend aclnnMoeDistributeDispatchV2 API (Returns: null pointer, invalid parameter,
 * unsupported shape or value). */
#define MOEDISP_OK                0
#define MOEDISP_ERR_NULLPTR      -1  /* a required pointer is NULL */
#define MOEDISP_ERR_INVALID      -2  /* a size, count or mode is out of range */
#define MOEDISP_ERR_MISALIGNED   -3  /* a pointer or row size breaks the 16-byte rule */
#define MOEDISP_ERR_ALIASED      -4  /* an output overlaps an input or another output */
#define MOEDISP_ERR_UNSUPPORTED  -5  /* valid but outside this build's limits */
#define MOEDISP_ERR_WORKSPACE    -6  /* workspace missing or too small */
#define MOEDISP_ERR_CUDA         -7  /* a CUDA runtime call or kernel launch failed */

/* Device-side status bits (OR-ed into *status). */
#define MOEDISP_STATUS_CAPACITY      1  /* rows beyond the receive capacity were dropped */
#define MOEDISP_STATUS_BAD_EXPERT_ID 2  /* an active slot named an expert outside [0, E) */
#define MOEDISP_STATUS_TIMEOUT       4  /* a bounded device-side wait gave up */
#define MOEDISP_STATUS_BAD_SPLIT     8  /* a negative split or a segment outside its buffer */

/* Limits of this build. */
#define MOEDISP_MAX_K        16      /* Ascend dispatch: 0 < K <= 16 */
#define MOEDISP_MAX_E        1024    /* Ascend A3: moeExpertNum <= 1024 */
#define MOEDISP_MAX_H        16384   /* hidden size (elements) for dispatch staging */
#define MOEDISP_MAX_W        65536   /* ranks of an exchange plan */
#define MOEDISP_MAX_ALIGN    65536   /* major_align of the layout */

/* Returns a static, human-readable name for a return code (< 0) or status bits (> 0). */
const char *moedisp_status_string(int code);

/* ABI version, currently 3 (2: active_mask_dims in the layout calls, smoothing scales in
 * moe_dispatch; 3: major_align in the layout calls). */
int moedisp_version(void);

/* Diagnostic for the time-out path of the device-side waits (this library's own
 * addition; the pages' kernels spin without a limit). Enqueues a one-thread kernel that
 * waits, through the same bounded-wait helper every kernel uses, on a barrier phase that
 * nothing completes; after limit_us microseconds (1..10^7) it must give up and OR
 * MOEDISP_STATUS_TIMEOUT into *status (device memory). No fault, trap or hang: the
 * context stays usable. */
int moedisp_selftest_bounded_wait(uint32_t limit_us, int32_t *status, moedisp_stream_t stream);

/* ------------------------------------------------------------------------------------
 * a2a_exchange_plan
 *
 * The all-to-all-v exchange plan of the PyTorch symm_mem change ("ExchangePlan" doc
 * comment, make_a2a_exchange_plan, and the checks in test_make_a2a_exchange_plan), for
 * all W virtual ranks at once. With S = in_splits (S[i][j] = rows rank i sends to j):
 *     out_splits[i][j]  = S[j][i]                  rows rank i receives from j
 *     src_offsets[i][j] = sum_{k<i} S[j][k]        where i's rows start in j's input
 *     dst_offsets[i][j] = sum_{k<j} out_splits[i][k]   where j's rows land in i's output
 * All five arrays are int64 [W][W], row-major, device memory; the three outputs must not
 * overlap each other or in_splits. A negative split sets MOEDISP_STATUS_BAD_SPLIT (the
 * outputs are then computed from the values as given). One kernel, W blocks.
 * ---------------------------------------------------------------------------------- */
int moedisp_a2a_exchange_plan(const int64_t *in_splits, int W, int64_t *src_offsets,
                              int64_t *out_splits, int64_t *dst_offsets, int32_t *status,
                              moedisp_stream_t stream);

/* ------------------------------------------------------------------------------------
 * a2a_v
 *
 * The uneven all-to-all-v row exchange driven by a plan (PyTorch symm_mem all_to_all_v,
 * get style: rank i fetches its rows from each peer j), between W virtual ranks:
 *     for every i, j and q < out_splits[i][j]:
 *       out row (i*out_cap_rows + dst_offsets[i][j] + q) =
 *       in  row (j*in_rank_stride_rows + src_offsets[i][j] + q)
 * `in` holds W send buffers of in_rank_stride_rows rows each, `out` W receive buffers of
 * out_cap_rows rows each; rows are `row_bytes` opaque bytes (the copy is dtype-agnostic).
 * Output rows no segment covers are left untouched. A segment whose source or
 * destination range leaves its rank's buffer (or has a negative size/offset) is skipped
 * and sets MOEDISP_STATUS_BAD_SPLIT.
 * Requirements: row_bytes > 0 and a multiple of 16; in and out 16-byte aligned and not
 * overlapping; plan arrays int64 [W][W] device memory (e.g. from a2a_exchange_plan).
 * ---------------------------------------------------------------------------------- */
int moedisp_a2a_v(const void *in, int64_t in_rank_stride_rows, void *out,
                  int64_t out_cap_rows, int64_t row_bytes, int W,
                  const int64_t *src_offsets, const int64_t *out_splits,
                  const int64_t *dst_offsets, int32_t *status, moedisp_stream_t stream);

/* ------------------------------------------------------------------------------------
 * MoE dispatch layout
 * ---------------------------------------------------------------------------------- */
typedef struct {
    int W;   /* EP ranks, >= 1 */
    int T;   /* tokens per rank, >= 0 */
    int K;   /* experts per token, 1..MOEDISP_MAX_K */
    int E;   /* experts, 1..MOEDISP_MAX_E, E % W == 0 */
} moedisp_dims;

/* Caller-owned device buffers that one moe_dispatch_layout call fills and that
 * moe_dispatch / moe_combine read. */
typedef struct {
    int32_t *cnt;          /* [W][E]   active slots of source rank r choosing expert e   */
    int32_t *occ;          /* [G*K]    0-based occurrence of slot s among the earlier
                                       active slots of its source rank with its expert;
                                       -1 for an inactive slot                           */
    int32_t *dst_row;      /* [G*K]    row of expand_x that slot s is dispatched to; -1
                                       for an inactive slot                              */
    int32_t *assist_info;  /* [rows_cap] slot s = g*K + k that row r holds (r < R)        */
    int64_t *expert_base;  /* [E+1]    first row of expert e; expert_base[E] = R         */
    int64_t *rank_base;    /* [W+1]    first row of destination rank d; rank_base[W] = R */
    int64_t *send_splits;  /* [W][W]   rows source rank r sends to destination rank d
                                       (the in_splits of a 1-D exchange plan)            */
    int64_t  rows_cap;     /* rows that expand_x / assist_info hold                       */
} moedisp_layout;

/* Bytes of device workspace moe_dispatch_layout needs for `dims`. */
int moedisp_layout_workspace_size(moedisp_dims dims, size_t *bytes);

/* moe_dispatch_layout
 *
 * Routes the G*K (token, expert) slots into an expert-grouped layout, following the
 * PyTorch symm_mem 2-D exchange plan and index-push dispatch (get_occurrence_numbers,
 * make2dExchangePlan, _allToAllV_2d_index_push_kernel) and the Ascend
 * aclnnMoeDistributeDispatchV2 inputs (expertIds int32 [Bs][K], xActiveMask of shape
 * (Bs,) or (Bs, K)):
 *   cnt[r][e]   = active slots of rank r with expert e (the 2-D plan's in_splits);
 *   occ[s]      = earlier active slots of s's rank with s's expert (0-based);
 *   rows of expand_x are ordered by destination rank, then local expert, then source
 *   rank, then token, then k -- i.e. dst_row[s] is the position of s in a stable sort of
 *   all active slots by expert id:
 *     dst_row[s] = expert_base[e] + sum_{r' < r} cnt[r'][e] + occ[s];
 *   assist_info[dst_row[s]] = s.
 * expert_ids: int32 [G][K] device; active_mask: uint8 device or NULL (all active), with
 * active_mask_dims 1: [G], one flag per token (any pattern of active tokens is
 * accepted), or 2: [G][K], one flag per slot (a token whose K flags are all zero sends
 * nothing); active_mask_dims is ignored when active_mask is NULL, else anything but 1 or 2
 * is MOEDISP_ERR_INVALID. A slot is active when its flag (or its token's) is nonzero and
 * its expert id lies in [0, E); an active slot's out-of-range id sets
 * MOEDISP_STATUS_BAD_EXPERT_ID and that slot is dropped. If R > rows_cap,
 * MOEDISP_STATUS_CAPACITY is set, every output is still computed, and assist_info is
 * written only below rows_cap.
 * major_align (the PyTorch symm_mem all_to_all_vdev_2d major_align, with the padding rule
 * of its 2-D exchange-plan test): 0 or 1, no padding; A in [2, MOEDISP_MAX_ALIGN], every
 * expert's segment of n routed rows is padded to max(A, ceil(n / A) * A) rows, so every
 * expert starts on a multiple of A and none is empty (as grouped-GEMM kernels want):
 * expert_base and rank_base then count padded segments, R = expert_base[E] includes the
 * padding, the padding rows follow each expert's routed rows and get assist_info -1 (below
 * rows_cap), and moe_dispatch leaves them untouched. Negative: MOEDISP_ERR_INVALID; above
 * MOEDISP_MAX_ALIGN: MOEDISP_ERR_UNSUPPORTED.
 * workspace: device memory of at least moedisp_layout_workspace_size() bytes, 16-byte
 * aligned; its contents need no initialisation (every word is written before it is
 * read). Calls sharing one workspace must not run concurrently.
 * Kernels: for up to 16 tiles of up to 2048 slots, one thread-block cluster that ranks
 * the tiles and exchanges their counts through distributed shared memory; otherwise
 * three: per-tile warp-aggregated histograms, per-expert scans down the tiles, and a
 * per-tile ranking + scatter. */
int moedisp_moe_dispatch_layout(const int32_t *expert_ids, const uint8_t *active_mask,
                                int active_mask_dims, int major_align, moedisp_dims dims, const moedisp_layout *layout,
                                void *workspace, size_t workspace_bytes, int32_t *status,
                                moedisp_stream_t stream);

/* moe_dispatch_layout_noalloc
 *
 * The same computation and outputs as moe_dispatch_layout, for callers that cannot
 * allocate device memory for the workspace: code running under an allocator that owns
 * all device memory and forbids side allocations, code inside a region where
 * allocation is not allowed (for example while a stream is being captured), or embedded
 * and real-time callers that must not allocate after start-up. (The source pages have no
 * counterpart; their APIs always take a caller-allocated workspace.)
 * Instead of a workspace argument it uses a scratch array of
 * MOEDISP_NOALLOC_SCRATCH_BYTES that lives in this library's own device memory: every
 * GPU that loads the library holds it until the process exits. It always runs the
 * three-kernel tiled path (histograms, scans, ranking + scatter) on that array.
 *  - Dims whose workspace (moedisp_layout_workspace_size) exceeds
 *    MOEDISP_NOALLOC_SCRATCH_BYTES are rejected with MOEDISP_ERR_UNSUPPORTED.
 *  - It calls no allocating routine. The first call on a device looks up the array's
 *    device address (once per device, with that device current); make that first call
 *    before any stream capture.
 *  - All calls share the one array, which keeps the last call's contents; nothing in it
 *    needs to start at zero (every word is written before it is read). Calls that
 *    overlap on the GPU (on different streams, or from different threads) race on the
 *    array and must not be made.
 * Other arguments and errors are those of moedisp_moe_dispatch_layout. */
#define MOEDISP_NOALLOC_SCRATCH_BYTES (2u << 20)
int moedisp_moe_dispatch_layout_noalloc(const int32_t *expert_ids, const uint8_t *active_mask,
                                        int active_mask_dims, int major_align, moedisp_dims dims, const moedisp_layout *layout,
                                        int32_t *status, moedisp_stream_t stream);

/* Quantisation modes of moe_dispatch (the Ascend quantMode values; 3 is this library's
 * fp8 variant of the same per-token dynamic scheme). */
#define MOEDISP_QUANT_NONE      0
#define MOEDISP_QUANT_INT8      2
#define MOEDISP_QUANT_FP8_E4M3  3

/* moe_dispatch
 *
 * Copies every token row to the rows its active slots were given by
 * moe_dispatch_layout (Ascend expandXOut; PyTorch symm_mem index push), optionally
 * quantised per token (Ascend quantMode 2, per-token dynamic):
 *   NONE: expand_x[dst_row[s]] = x[g]                            (bf16, H*2 bytes/row)
 *   INT8: a = max_h |x[g,h]|, scale = a / 127 (fp32, IEEE divide),
 *         q = a == 0 ? 0 : clamp(rint(x / scale), -127, 127)     (int8, H bytes/row)
 *   FP8_E4M3: scale = a / 448, q = a == 0 ? 0 : e4m3(x / scale), round to nearest even,
 *         saturating to +-448                                    (e4m3, H bytes/row)
 *   dynamic_scales[dst_row[s]] = scale (quant modes).
 * smooth_scales (Ascend scalesOptional, the per-expert quantisation smoothing factors):
 * fp32 [E][H] device, 16-byte aligned, or NULL; quant modes only (with NONE it is
 * MOEDISP_ERR_INVALID). When given, the copy for slot s = (g, k) routed to expert e
 * quantises x[g] * smooth_scales[e] (one fp32 product per element) instead of x[g], with
 * its own a and scale. The rows are then produced from the layout's expert_base,
 * assist_info and, when it is given, cnt (which orders the work rank by rank when x is
 * large; a row whose assist_info is outside [0, G*K) is skipped and sets
 * MOEDISP_STATUS_BAD_EXPERT_ID); dst_row is not read.
 * x: bf16 [G][H] device, 16-byte aligned; expand_x: [layout->rows_cap][H] elements of
 * the output type, 16-byte aligned, not overlapping x; dynamic_scales: fp32
 * [rows_cap] (required for quant modes, ignored otherwise). H % 8 == 0 (NONE) or
 * H % 16 == 0 (quant), H <= MOEDISP_MAX_H.
 * Optional (NULL to skip), per destination rank d and local expert le:
 *   expert_token_nums int64 [W][ne]: rows of expert d*ne+le (type 1), or the running sum
 *     over the rank's local experts up to and including le (type 0);
 *   ep_recv_counts int32 [W][ne][W]: rows expert d*ne+le receives from source rank r; with
 *     major_align the last source rank's entry also counts the expert's padding rows (as
 *     the 2-D plan's out_splits do), and expert_token_nums counts padded segments.
 * Rows at or beyond rows_cap are not written (MOEDISP_STATUS_CAPACITY).
 * One persistent kernel: an unquantised token row is brought into shared memory once by
 * a bulk (TMA) copy and leaves it as K bulk copies; a quantised one is read once into
 * registers and its codes leave as 8-byte streaming stores to the K rows. With smoothing
 * each block walks runs of rows of one expert, holding that expert's smoothing row in
 * shared memory and gathering each row's token into registers. The codes are those of the
 * IEEE quotient x / scale bit for bit (a faster decision is used only where it provably
 * agrees). */
int moedisp_moe_dispatch(const void *x, int H, moedisp_dims dims,
                         const moedisp_layout *layout, int quant_mode,
                         const float *smooth_scales, void *expand_x,
                         float *dynamic_scales, int64_t *expert_token_nums,
                         int expert_token_nums_type, int32_t *ep_recv_counts,
                         int32_t *status, moedisp_stream_t stream);

/* moe_combine
 *
 * The weighted combine back (Ascend aclnnMoeDistributeCombineV2 inputs expandX,
 * expertIds / assist info, expertScales; FlashInfer MoE finalize, where a routed index
 * of -1 means "not routed"):
 *   y[g] = bf16_rn( acc ),  acc = 0; for k = 0..K-1 with a routed slot:
 *                                    acc = fmaf(expert_scales[g,k], expert_out[dst_row[g*K+k]], acc)
 * A token with no routed slot gets y[g] = 0.
 * expert_out: bf16 [layout->rows_cap][H] device (the experts' outputs, rows in the
 * dispatch layout); expert_scales: fp32 [G][K] device; y: bf16 [G][H] device, not
 * overlapping expert_out. H % 8 == 0; all row pointers 16-byte aligned. */
int moedisp_moe_combine(const void *expert_out, int H, moedisp_dims dims,
                        const moedisp_layout *layout, const float *expert_scales, void *y,
                        int32_t *status, moedisp_stream_t stream);

/* moe_dispatch_gather
 *
 * moe_dispatch for tokens that stay where they are: token g's row is row token_rows[g]
 * of x (x: bf16 [x_rows][H]); token_rows int64 [G] device, 8-byte aligned. A routed token
 * whose token_rows entry is outside [0, x_rows) is skipped and sets
 * MOEDISP_STATUS_BAD_SPLIT. Everything else is moe_dispatch's (x rows read once, in
 * place). With a2a_token_rows this is the exchange and the dispatch in one pass: the
 * PyTorch symm_mem change pipelines its get-style exchange into the index push through
 * per-block ready counters; on one GPU the received rows need not be materialised at
 * all, and each row streams from its sender's buffer straight to its K expert rows
 * (the kernel's own stage barriers are the ready signals). */
int moedisp_moe_dispatch_gather(const void *x, int64_t x_rows, const int64_t *token_rows, int H,
                                moedisp_dims dims, const moedisp_layout *layout, int quant_mode,
                                const float *smooth_scales, void *expand_x,
                                float *dynamic_scales, int64_t *expert_token_nums,
                                int expert_token_nums_type, int32_t *ep_recv_counts,
                                int32_t *status, moedisp_stream_t stream);

/* a2a_dispatch_pipelined
 *
 * The exchange and the dispatch of the exchanged tokens overlapped through per-segment
 * ready words, after the PyTorch symm_mem change's get-style exchange that publishes
 * (release) how many rows of each peer have arrived while the index-push kernel spins on
 * those words (acquire) before pushing the rows on to their experts. One call does what
 * a2a_v followed by moe_dispatch does:
 *   recv row (i*T + dst_offsets[i][j] + q) = in row (j*in_rank_stride_rows +
 *       src_offsets[i][j] + q)                         for q < out_splits[i][j]  (a2a_v)
 *   expand_x / dynamic_scales of every received token, dispatched as moe_dispatch does
 *       with `layout` (the layout of the W*T receive positions: token g = i*T + p)
 * but in one persistent kernel: blocks take exchange pieces of segment (i, j) and
 * dispatch chunks of already received segments from one ticket counter (the pieces of
 * segment s+1 come before the tokens of segment s), the block landing a segment's last
 * rows stores ready[i*W + j] = epoch (release), and the tokens of a segment are
 * dispatched once an acquire load sees it -- each received row is read back from L2
 * moments after it was written.
 * in: bf16 [W][in_rank_stride_rows][H]; recv: bf16 [W][T][H] (T = dims.T, the receive
 * capacity), both 16-byte aligned and not overlapping; plan arrays as for a2a_v; layout,
 * quant_mode, expand_x, dynamic_scales, expert_token_nums(_type), ep_recv_counts as for
 * moe_dispatch (no smoothing).
 * ready: uint32 [W][W] device, zeroed once when allocated and then left to this call;
 * epoch: 1, 2, 3, ... a new value for every exchange (the ready words keep the last one;
 * compared for equality, so after 2^32 - 1 the sequence goes on with 1).
 * Equally valid, and the form a CUDA graph can replay: zero the ready words in stream
 * order before every call and pass the same epoch each time (say 1). epoch 0 is rejected
 * (MOEDISP_ERR_INVALID): zeroed words would read as already published.
 * roles: MOEDISP_PIPE_BOTH (the normal case); MOEDISP_PIPE_PRODUCE, the exchange alone,
 * publishing the ready words; MOEDISP_PIPE_CONSUME, the dispatch alone, for rows that
 * another party delivered into recv and published with this epoch (a PRODUCE call of
 * the same epoch before it, or a peer). wait_limit_us (1..10^7): a dispatch chunk whose
 * segment is not published within this time sets MOEDISP_STATUS_TIMEOUT, and the
 * kernel stops waiting for any segment (the outputs are then incomplete).
 * A segment whose ranges leave their buffers (or has a negative size/offset) is neither
 * exchanged nor dispatched and sets MOEDISP_STATUS_BAD_SPLIT. Tokens are dispatched segment
 * by segment: a receive position that no valid segment covers is not dispatched even if
 * the layout routes it (build the layout with the received positions as its mask, e.g.
 * from a2a_token_rows, and the two agree).
 * workspace: device memory of moedisp_a2a_dispatch_pipelined_workspace_size(W) bytes,
 * 16-byte aligned, no initialisation needed; calls sharing a workspace or ready words
 * must not run concurrently. H % 8 == 0 (NONE) or H % 16 == 0, H <= MOEDISP_MAX_H.
 * Two kernels: a one-block set-up (segment checks, ticket offsets), then the pipeline. */
#define MOEDISP_PIPE_PRODUCE 1
#define MOEDISP_PIPE_CONSUME 2
#define MOEDISP_PIPE_BOTH    3
int moedisp_a2a_dispatch_pipelined_workspace_size(int W, size_t *bytes);
int moedisp_a2a_dispatch_pipelined(const void *in, int64_t in_rank_stride_rows,
                                   const int64_t *src_offsets, const int64_t *out_splits,
                                   const int64_t *dst_offsets, void *recv, int H,
                                   moedisp_dims dims, const moedisp_layout *layout,
                                   int quant_mode, void *expand_x, float *dynamic_scales,
                                   int64_t *expert_token_nums, int expert_token_nums_type,
                                   int32_t *ep_recv_counts, uint32_t *ready, uint32_t epoch,
                                   int roles, uint32_t wait_limit_us, void *workspace,
                                   size_t workspace_bytes, int32_t *status,
                                   moedisp_stream_t stream);

/* a2a_token_rows
 *
 * The source of every receive position of an exchange plan (a2a_exchange_plan's outputs
 * src_offsets, out_splits, dst_offsets, [W][W] int64 device), for moe_dispatch_gather over
 * the received tokens without a receive buffer: position p < T of rank i (T = the
 * per-rank receive capacity, the dispatch's T) that a2a_v would fill from source rank j
 * gets row j * in_rank_stride_rows + src_offsets[i][j] + (p - dst_offsets[i][j]) of the
 * senders' concatenated input (a2a_v's `in`); other positions get -1.
 * token_rows: int64 [W][T] device; active: uint8 [W][T] device (1 where a row is received,
 * the layout's per-token mask) or NULL. A segment leaving its sender's rows gives -1 and
 * MOEDISP_STATUS_BAD_SPLIT. A rank that receives more than T rows in total (its last
 * segment ends beyond T) sets MOEDISP_STATUS_CAPACITY: the rows past T have no position
 * and are not dispatched. */
int moedisp_a2a_token_rows(const int64_t *src_offsets, const int64_t *out_splits,
                           const int64_t *dst_offsets, int W, int64_t T,
                           int64_t in_rank_stride_rows, int64_t *token_rows, uint8_t *active,
                           int32_t *status, moedisp_stream_t stream);

/* moe_dispatch_peers / moe_combine_peers
 *
 * Expert parallelism over W separate GPUs (one rank each). Every rank all-gathers the
 * routing (expert_ids [W*T][K], the active mask) -- a few bytes per token -- and computes
 * the global layout of all W ranks with moe_dispatch_layout (dims {W, T, K, E}); then:
 *   moe_dispatch_peers: rank `rank` writes its T token rows (x: bf16 [T][H]) straight to
 *     their K destination rows in the owning ranks' buffers: global row d of expert e
 *     lands in rank q = e / ne's expand_x, local row d - rank_base[q], through
 *     peer_expand_x (a device array of W pointers to the ranks' expand_x buffers, each
 *     [peer_rows_cap][H] of the output type, mapped into this GPU -- its own included),
 *     with the scales through peer_scales (device array of W float pointers; quant modes)
 *     -- the dispatch and the exchange in one kernel, each row read from HBM once and sent
 *     over NVLink once per destination;
 *   moe_combine_peers: rank `rank` computes y[t] (bf16 [T][H]) of its own tokens by
 *     gathering each slot's expert-output row from the owning rank's buffer through
 *     peer_expert_out (device array of W pointers, each [peer_rows_cap][H] bf16), with
 *     this rank's weights (expert_scales fp32 [T][K]) -- the exchange back and the
 *     weighted sum in one kernel.
 * expert_ids: the all-gathered ids the layout was computed from (the owner of each slot).
 * Results equal moe_dispatch / moe_combine of the single-buffer layout, row for row (local
 * row = global row - rank_base[q]). A slot whose local row is at or beyond peer_rows_cap
 * is skipped and sets MOEDISP_STATUS_CAPACITY. Ordering between ranks (expand_x rows
 * complete before the experts run, expert outputs complete before the combine) is the
 * caller's: a barrier across the ranks' streams. Not supported with smoothing scales or a
 * gather map. The pointers in the tables are not checked against each other. */
int moedisp_moe_dispatch_peers(const void *x, int H, moedisp_dims dims, int rank,
                               const int32_t *expert_ids, const moedisp_layout *layout,
                               int quant_mode, void *const *peer_expand_x,
                               float *const *peer_scales, int64_t peer_rows_cap, int32_t *status,
                               moedisp_stream_t stream);
int moedisp_moe_combine_peers(const void *const *peer_expert_out, int64_t peer_rows_cap, int H,
                              moedisp_dims dims, int rank, const int32_t *expert_ids,
                              const moedisp_layout *layout, const float *expert_scales, void *y,
                              int32_t *status, moedisp_stream_t stream);

/* ipc_export / ipc_import / ipc_close
 *
 * Peer mappings for moe_dispatch_peers / moe_combine_peers / ep_barrier when the ranks are
 * processes (one per GPU, or several on one GPU): plain CUDA IPC mappings, so no memory is
 * bound to an NVLink multicast object (the PyTorch symm_mem change maps its buffers with
 * NVSHMEM instead). Host-side calls on the current device; no kernel, no allocation.
 *   ipc_export: for a device buffer of this process (any pointer into a cudaMalloc
 *     allocation, e.g. a caching allocator's segment), writes the allocation's IPC handle
 *     (MOEDISP_IPC_HANDLE_BYTES bytes, host memory) and the buffer's byte offset in it.
 *     Send both to the other ranks (they are plain bytes). Pointers that are not device
 *     memory of this process: MOEDISP_ERR_INVALID; a CUDA refusal: MOEDISP_ERR_CUDA
 *     (memory from a virtual-memory allocator cannot be exported this way).
 *   ipc_import: in another process, maps the allocation (once per process, shared by
 *     every buffer imported from it) and returns the buffer's address in this process.
 *     A handle of this same process cannot be opened (MOEDISP_ERR_CUDA): use the buffer
 *     itself. Importing one buffer twice: MOEDISP_ERR_INVALID.
 *   ipc_close: releases a pointer ipc_import returned (the mapping goes with its last
 *     buffer); the peer's buffers must not be used after it. */
#define MOEDISP_IPC_HANDLE_BYTES 64
int moedisp_ipc_export(const void *dev_ptr, void *handle, int64_t *offset);
int moedisp_ipc_import(const void *handle, int64_t offset, void **dev_ptr);
int moedisp_ipc_close(void *dev_ptr);

/* ep_barrier
 *
 * Orders the W ranks of moe_dispatch_peers / moe_combine_peers on the GPUs themselves,
 * with a time limit (this library's own addition: the PyTorch symm_mem change orders its
 * ranks with signal-pad barriers that wait without one). Each rank owns a signal array of
 * W uint32 words in peer-mappable device memory, zeroed once before the first barrier;
 * peer_signals is a device array of W pointers to the ranks' arrays as mapped into this
 * GPU (its own included), 8-byte aligned. Rank `rank`'s call, in stream order:
 *   - after every earlier kernel on the stream has completed (its writes into peers'
 *     buffers included), stores `epoch` into word `rank` of every rank's array (a
 *     system-scope release);
 *   - waits until every word of its own array has reached `epoch` (acquire loads, compared
 *     with wrap-around), so that no rank's later kernels start before every rank has
 *     finished its earlier ones.
 * epoch: 1, 2, 3, ... in the same sequence on every rank (one per barrier; words are never
 * reset); 0 is rejected (MOEDISP_ERR_INVALID: it would pass zeroed words), so after
 * 2^32 - 1 the sequence goes on with 1 (the wrap-around compare holds while no rank is
 * 2^31 barriers ahead of another). A wait longer than timeout_us (1..10^7 microseconds) gives up, ORs
 * MOEDISP_STATUS_TIMEOUT into *status and returns: a rank that died or fell behind is
 * reported, not waited for (the caller reads the status and stops). W = 1 only publishes.
 * One block. */
int moedisp_ep_barrier(uint32_t *const *peer_signals, int W, int rank, uint32_t epoch,
                       uint32_t timeout_us, int32_t *status, moedisp_stream_t stream);

/* shared_expert_routing
 *
 * Shared experts (Ascend aclnnMoeDistributeDispatchV2 sharedExpertNum N,
 * sharedExpertRankNum S, expertShardType 0: shared-expert ranks before the routed-expert
 * ranks), expressed as a wider routing that the layout, dispatch and combine take as is.
 * The first S of the W ranks each host one shared-expert replica (S / N replicas of each of
 * the N shared experts, grouped by shared expert); the other W - S ranks host the E routed
 * experts, ne = E / (W - S) each. In the uniform expert space of W * ne experts:
 *   routed expert e          -> S * ne + e    (an id outside [0, E) -> W * ne, still out
 *                                              of range: BAD_EXPERT_ID at the layout)
 *   shared expert j, token of source rank r -> (j * (S / N) + r mod (S / N)) * ne
 * (the pages fix only the counts -- a shared rank receives T * W * N / S tokens; the
 * replica of a source rank is this library's choice). Outputs, [G][K + N] each:
 * ext_ids int32 (the K routed slots, then the N shared ones) and ext_scales fp32 (the
 * given weights, then 1). Then call moe_dispatch_layout, moe_dispatch and moe_combine with
 * dims {W, T, K + N, W * ne}; a shared rank's ne - 1 other local experts stay empty.
 * Rules: N = 0 exactly when S = 0; S < W, W % S == 0, S % N == 0, E % (W - S) == 0
 * (else MOEDISP_ERR_INVALID); K + N <= MOEDISP_MAX_K and W * ne <= MOEDISP_MAX_E (else
 * MOEDISP_ERR_UNSUPPORTED). Out-of-range ids set MOEDISP_STATUS_BAD_EXPERT_ID. */
int moedisp_shared_expert_routing(const int32_t *expert_ids, const float *expert_scales, int W,
                                  int T, int K, int E, int shared_expert_num,
                                  int shared_expert_rank_num, int32_t *ext_ids,
                                  float *ext_scales, int32_t *status, moedisp_stream_t stream);

/* moe_combine_rmsnorm
 *
 * The combine fused with the residual add and RMSNorm that follow it (the FlashInfer
 * MNNVL PR's "MoE finalize + residual + RMSNorm" tail, without its tensor-parallel
 * all-reduce), one pass over HBM:
 *   prenorm[g] = bf16_rn( acc + residual[g] )        acc as in moe_combine (fp32, k order),
 *                                                    one fp32 add per element
 *   y[g,h]     = bf16_rn( (prenorm[g,h] * rs) * gamma[h] ),
 *                rs = 1/sqrt( sum_h prenorm[g,h]^2 / H + eps )   (fp32)
 * residual: bf16 [G][H]; gamma: fp32 [H]; residual_out: bf16 [G][H] receiving prenorm, or
 * NULL; y: bf16 [G][H]. Outputs must not overlap inputs. H % 8 == 0, H <= MOEDISP_MAX_H;
 * all row pointers and gamma 16-byte aligned; eps >= 0. prenorm is bit-exact; y depends on
 * the order of the sum of squares (a block reduction) within fp32 rounding. */
int moedisp_moe_combine_rmsnorm(const void *expert_out, int H, moedisp_dims dims,
                                const moedisp_layout *layout, const float *expert_scales,
                                const void *residual, const float *gamma, float eps,
                                void *residual_out, void *y, int32_t *status,
                                moedisp_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOEDISP_H */
