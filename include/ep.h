/*
 * ep.h -- MoE token layout, dispatch and combine on one B200 (sm_100a).
 *
 * C ABI of libep_b200.so.  All tensors are plain device pointers, row-major
 * and densely packed; all memory belongs to the caller.  Only ep_peer_alloc /
 * ep_peer_free (device memory other processes map) and ep_peer_open /
 * ep_peer_close (those mappings) allocate, free or map device memory, and no
 * entry point synchronises the host except ep_get_device_error() and a
 * layout call (or a one-call layout + dispatch) given a num_valid_host
 * pointer.  Every other call is asynchronous on `stream` (a cudaStream_t;
 * NULL = the legacy default stream).
 *
 * The operations follow these pages (title, section):
 *   [README] "DeepEP-Ascend" README (sgl-kernel-npu python/deep_ep),
 *            "API Overview" table: get_dispatch_layout, dispatch, combine,
 *            low_latency_dispatch, low_latency_combine; "Quantization Modes
 *            in Normal Dispatch"; "Environment Variables":
 *            MOE_EXPERT_TOKEN_NUMS_TYPE (count vs prefix-sum form),
 *            MOE_ENABLE_TOPK_NEG_ONE (-1 = not dispatched).
 *   [EC]     DeepEP issue #595, "Support Expert-Choice Routing via Native
 *            Expert-Centric API ([num_experts, capacity])": "Proposed
 *            Solutions", Solution 1 (token_indices [num_experts, capacity]
 *            and its dispatch/combine pair) and Solution 2 (skip -1 padding).
 *
 * Notation: T tokens, H hidden, K top-k width, E experts, R logical ranks
 * (rank r owns experts [r*E/R, (r+1)*E/R)), C expert capacity.
 *
 * Status and errors
 *   Argument problems found on the host return EP_ERR_INVALID_ARG (or
 *   EP_ERR_UNSUPPORTED / EP_ERR_WORKSPACE) before anything is launched.
 *   A failed launch returns EP_ERR_CUDA.  Problems only the device can see
 *   (an index out of range, a padded buffer that is full, a bounded wait
 *   that ran out) never fault: the offending element is skipped and a bit
 *   is OR-ed into the error word at the start of the layout workspace,
 *   read back by ep_get_device_error().
 */
#ifndef EP_B200_H_
#define EP_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EP_ABI_VERSION 3

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

typedef struct CUstream_st* ep_stream_t; /* same type as cudaStream_t */

typedef enum {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1, /* bad size, null or misaligned pointer, bad enum */
    EP_ERR_BAD_INDEX = 2,   /* device: routing id outside [-1, E) or [-1, T) */
    EP_ERR_OVERFLOW = 3,    /* device: destination row beyond the buffer */
    EP_ERR_WORKSPACE = 4,   /* workspace missing, misaligned or too small */
    EP_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
    EP_ERR_UNSUPPORTED = 6, /* valid request the library does not handle */
    EP_ERR_TIMEOUT = 7      /* device: a bounded wait gave up */
} ep_status_t;

/* Element formats.  EP_BF16 / EP_FP32 are plain arrays.  The others are the
 * quantised dispatch payloads of the [README] "Quantization Modes" table
 * ("int8", "pertoken_fp8_e4m3", "mx_fp8_e4m3", "mx_fp8_e5m2",
 * "mx_fp4_e2m1"; EP_FP8_E4M3 is the 128-channel FP8 of low_latency_dispatch):
 *   value               codes per row            scales per row
 *   EP_FP8_E4M3         H bytes, e4m3            H/128 fp32 (amax/448)
 *   EP_INT8_PER_TOKEN   H bytes, int8            1 fp32 (amax/127)
 *   EP_FP8_E4M3_PER_TOKEN H bytes, e4m3          1 fp32 (amax/448)
 *   EP_MXFP8_E4M3       H bytes, e4m3            H/32 e8m0 bytes
 *   EP_MXFP8_E5M2       H bytes, e5m2            H/32 e8m0 bytes
 *   EP_MXFP4_E2M1       H/2 bytes, two e2m1      H/32 e8m0 bytes
 *                       codes per byte, element
 *                       2i in the low nibble
 * Dynamic scales (fp32): scale = amax/qmax and code = encode(x * (qmax/amax))
 * with qmax/amax clamped to FLT_MAX, qmax = 448 (e4m3, nearest-even,
 * saturating) or 127 (int8, nearest-even, clamped to [-127, 127]); amax == 0
 * gives scale 0 and zero codes.  MX scales (OCP Microscaling v1.0): per block
 * of 32, X = floor(log2 amax) - emax (e4m3 8, e5m2 15, e2m1 2) clamped to
 * [-127, 127] (amax == 0 gives -127), scale byte X + 127, code =
 * encode(x * 2^-X), nearest-even and saturating to the format's largest
 * finite value (448, 57344, 6). */
typedef enum {
    EP_BF16 = 0,
    EP_FP32 = 1,
    EP_FP8_E4M3 = 2,
    EP_INT8_PER_TOKEN = 3,
    EP_FP8_E4M3_PER_TOKEN = 4,
    EP_MXFP8_E4M3 = 5,
    EP_MXFP8_E5M2 = 6,
    EP_MXFP4_E2M1 = 7
} ep_dtype_t;

/* COMPACT: expert e's rows are [expert_offsets[e], expert_offsets[e+1]) of
 *   one buffer (normal-mode dispatch); rank r's rows are the contiguous
 *   range [expert_offsets[r*E/R], expert_offsets[(r+1)*E/R]).
 * PADDED: expert e owns rows [e*max_tokens, (e+1)*max_tokens), as the
 *   low-latency per-expert receive buffers of num_max_dispatch_tokens rows;
 *   rows past num_tokens_per_expert[e] are never written. */
typedef enum { EP_LAYOUT_COMPACT = 0, EP_LAYOUT_PADDED = 1 } ep_buffer_mode_t;

typedef enum { EP_ROUTING_TOPK = 0, EP_ROUTING_EXPERT_CHOICE = 1 } ep_routing_t;

/* bits of the device error word */
#define EP_DEVERR_BAD_INDEX 0x1u
#define EP_DEVERR_OVERFLOW 0x2u
#define EP_DEVERR_TIMEOUT 0x4u

/* The routing decision, read-only.
 *   TOPK:          topk_idx  int64 [T, K]; entry -1 = slot not dispatched.
 *   EXPERT_CHOICE: token_indices int32 [E, C]; entry -1 = empty slot.
 * Ids outside [-1, E) (resp. [-1, T)) are treated as -1 and flagged
 * EP_DEVERR_BAD_INDEX.  Limits: T >= 0; K, E, C >= 1; 1 <= R <= 32;
 * E % R == 0; T*K and E*C below 2^31; token-choice layout needs E <= 1024. */
typedef struct {
    ep_routing_t routing;
    const int64_t* topk_idx;
    const int32_t* token_indices;
    int32_t num_tokens;
    int32_t num_topk;
    int32_t capacity;
    int32_t num_experts;
    int32_t num_ranks;
} ep_routing_desc_t;

/* Layout outputs (written by ep_get_layout) and the handle that dispatch
 * and combine read back.  Pointers not used by a routing kind may be NULL.
 *   num_tokens_per_expert int32 [E]    pairs (TOPK) or filled slots (EC) per expert
 *   expert_offsets        int32 [E+1]  TOPK: exclusive scan of the counts
 *   num_tokens_per_rank   int32 [R]    tokens with >= 1 expert in rank r
 *   is_token_in_rank      uint8 [T, R] 0/1
 *   slot                  int32 [T, K] TOPK: rank of pair (t,k) among the
 *                                      pairs of its expert in ascending
 *                                      (t, k) order; -1 if not routed
 *   token_offsets         int32 [T+1]  EC: exclusive scan of picks per token
 *   token_slots           int32 [E*C]  EC: slot ids s = e*C + c picking each
 *                                      token, ascending; [0, token_offsets[T])
 *                                      is written
 *   workspace             device scratch of ep_workspace_bytes() bytes,
 *                         256-byte aligned: the device error word, the
 *                         grid-barrier words of the token-choice layout and
 *                         its per-CTA expert totals, or the expert-choice
 *                         layout's per-token arrays.  Zero it once
 *                         (ep_workspace_init) before first use; calls leave
 *                         it reusable.  One workspace per stream: calls that
 *                         share one must not overlap on the GPU.
 *   num_valid_host        optional HOST pointer to one int32 (pinned or
 *                         pageable), NULL = not used.  When set, the layout
 *                         call copies the number of rows the routing fills
 *                         (TOPK: expert_offsets[E], the routed pairs; EC:
 *                         token_offsets[T], the filled slots) into it and
 *                         synchronises `stream` before returning, so the
 *                         caller can size its receive buffer without a read
 *                         of its own.  This is the only synchronisation a
 *                         layout call ever makes; leave it NULL while the
 *                         stream is being captured. */
typedef struct {
    int32_t* num_tokens_per_expert;
    int32_t* expert_offsets;
    int32_t* num_tokens_per_rank;
    uint8_t* is_token_in_rank;
    int32_t* slot;
    int32_t* token_offsets;
    int32_t* token_slots;
    void* workspace;
    size_t workspace_bytes;
    int32_t* num_valid_host;
} ep_layout_t;

/* Bytes of workspace the layout of this routing needs (>= 256; the first
 * 256 bytes hold the device error word).  Pure host function. */
EP_API size_t ep_workspace_bytes(const ep_routing_desc_t* routing);

/* Zero `bytes` of workspace on `stream` (a cudaMemsetAsync). */
EP_API ep_status_t ep_workspace_init(void* workspace, size_t bytes, ep_stream_t stream);

/* get_dispatch_layout ([README] API Overview; count and prefix-sum forms per
 * MOE_EXPERT_TOKEN_NUMS_TYPE; -1 per MOE_ENABLE_TOPK_NEG_ONE).
 * TOPK writes num_tokens_per_expert, expert_offsets, num_tokens_per_rank,
 * is_token_in_rank and slot.  EXPERT_CHOICE ([EC] Solution 1) writes
 * num_tokens_per_expert, num_tokens_per_rank, is_token_in_rank,
 * token_offsets and token_slots.  Deterministic: the same routing gives the
 * same bytes on every call.  With layout->num_valid_host set, the number of
 * filled rows is also copied to the host and the call returns after the
 * stream has caught up (the [README] dispatch returns the received-token
 * count to the host in the same way). */
EP_API ep_status_t ep_get_layout(const ep_routing_desc_t* routing, const ep_layout_t* layout, ep_stream_t stream);

/* Token-choice dispatch ([README] API Overview: dispatch; low_latency_dispatch
 * for PADDED).  For every routed pair (t,k) of expert e with slot s:
 *   row = expert_offsets[e] + s          (COMPACT)
 *   row = e * max_tokens_per_expert + s  (PADDED; s >= max_tokens -> skipped,
 *                                         EP_DEVERR_OVERFLOW)
 * and row >= num_recv_rows is skipped with EP_DEVERR_OVERFLOW.
 *   x            bf16 [T, H], 16-byte aligned, H % 8 == 0
 *   out_dtype    EP_BF16: recv_x bf16 [rows, H] receives x[t] bit for bit.
 *                A quantised format (see ep_dtype_t): recv_x receives the
 *                codes of x[t] and recv_scales (fp32, or e8m0 bytes for MX)
 *                its scales, both row-major with the row sizes listed at
 *                ep_dtype_t.  Needs H % 128 == 0 (EP_FP8_E4M3), H % 32 == 0
 *                (MX), H <= 32768, and recv_scales aligned to its element
 *                ([README] "Quantization Modes in Normal Dispatch").
 *   topk_weights fp32 [T, K], needed only when recv_weights != NULL
 *   recv_src     optional int32 [rows]: source token of each written row
 *   recv_weights optional fp32 [rows]: gate weight of each written row
 * Rows not named by any pair are left untouched. */
EP_API ep_status_t ep_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing, const ep_layout_t* layout,
                        ep_buffer_mode_t mode, int32_t max_tokens_per_expert, int64_t num_recv_rows,
                        ep_dtype_t out_dtype, const float* topk_weights, void* recv_x, void* recv_scales,
                        int32_t* recv_src, float* recv_weights, ep_stream_t stream);

/* Layout and dispatch in one call ([README] API Overview: get_dispatch_layout
 * followed by dispatch): exactly ep_get_layout(routing, layout) followed by
 * ep_dispatch(x, hidden, routing, layout, mode, ...), with the same outputs,
 * arguments and errors (nothing is launched unless both calls' arguments
 * pass).  Being the library's own back-to-back launches, the dispatch's
 * threads start while the layout kernel runs and load their source rows
 * before waiting for it; ep_dispatch alone must first wait for whatever
 * kernel precedes it on the stream, which may have written x.
 * layout->workspace must have ep_workspace_bytes() bytes;
 * layout->num_valid_host is honoured as by ep_get_layout. */
EP_API ep_status_t ep_layout_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                      const ep_layout_t* layout, ep_buffer_mode_t mode, int32_t max_tokens_per_expert,
                                      int64_t num_recv_rows, ep_dtype_t out_dtype, const float* topk_weights,
                                      void* recv_x, void* recv_scales, int32_t* recv_src, float* recv_weights,
                                      ep_stream_t stream);

/* Low-latency dispatch ([README] API Overview: low_latency_dispatch, which
 * takes topk_idx and num_max_dispatch_tokens_per_rank and needs no separate
 * layout call): exactly ep_get_layout(routing, layout) followed by
 * ep_dispatch(..., EP_LAYOUT_PADDED, max_tokens_per_expert,
 * num_recv_rows = E * max_tokens_per_expert, out_dtype, ...), with the same
 * outputs, arguments and errors, but in ONE launch when T * K <= 8192,
 * K <= 32 and E <= 1024 (each token's CTA counts the earlier pairs of its
 * experts itself; the last token's CTA forms the counts, offsets and
 * per-rank totals).  Larger batches take the two-call path.  out_dtype may
 * be EP_BF16 or any quantised format; layout->workspace must have
 * ep_workspace_bytes() bytes. */
EP_API ep_status_t ep_dispatch_low_latency(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                           const ep_layout_t* layout, int32_t max_tokens_per_expert,
                                           ep_dtype_t out_dtype, const float* topk_weights, void* recv_x,
                                           void* recv_scales, int32_t* recv_src, float* recv_weights,
                                           ep_stream_t stream);

/* Token-choice combine ([README] API Overview: combine / low_latency_combine,
 * the weighted reduce; [EC] Solution 2: -1 slots are skipped).
 *   out[t] = sum over k = 0..K-1 of topk_weights[t,k] * y[row(t,k)], over the
 *   routed pairs only, accumulated in fp32 as acc = fmaf(w, y, acc) from 0
 *   in ascending k; written as fp32 or rounded once (RNE) to bf16.  A token
 *   with no routed pair gets +0.  row(t,k) is the dispatch row above; rows
 *   >= num_y_rows are skipped with EP_DEVERR_OVERFLOW.
 *   y   bf16 [num_y_rows, H], 16-byte aligned;  out [T, H] (out_dtype BF16 or FP32). */
EP_API ep_status_t ep_combine(const void* y, int32_t hidden, int64_t num_y_rows, const ep_routing_desc_t* routing,
                       const ep_layout_t* layout, ep_buffer_mode_t mode, int32_t max_tokens_per_expert,
                       const float* topk_weights, void* out, ep_dtype_t out_dtype, ep_stream_t stream);

/* Expert-choice dispatch ([EC] Solution 1, dispatch_expert_choice):
 *   recv_x[e*C + c] = x[token_indices[e, c]] for every filled slot; rows of
 *   empty slots are untouched.  x bf16 [T, H]; recv_x bf16 [E*C, H]; both
 *   16-byte aligned, H % 8 == 0.  Needs only routing and layout->workspace. */
EP_API ep_status_t ep_dispatch_expert_choice(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                      const ep_layout_t* layout, void* recv_x, ep_stream_t stream);

/* ep_get_layout followed by ep_dispatch_expert_choice, in one call (same
 * arguments, results and checks; nothing is launched unless both calls can
 * run).  The copy reads no result of the layout, so it runs while the layout
 * kernel runs instead of after it; it still ends only after the layout has,
 * so work that the caller queues next on `stream` sees both.  The separate
 * calls cannot overlap this way: a dispatch alone must first wait for
 * whatever kernel precedes it, which may have written x or token_indices.
 * layout->num_valid_host is honoured as by ep_get_layout. */
EP_API ep_status_t ep_layout_dispatch_expert_choice(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                                    const ep_layout_t* layout, void* recv_x, ep_stream_t stream);

/* Expert-choice combine ([EC] Solution 1, the combine of the new API pair):
 *   out[t] = sum over the token's slots s in token_slots[token_offsets[t] ..
 *   token_offsets[t+1]) (ascending s) of expert_weights[s] * y[s], as an fmaf
 *   chain in fp32 from 0; unpicked tokens get +0.  y bf16 [E*C, H];
 *   expert_weights fp32 [E, C]; out [T, H] (BF16 or FP32).  Uses the CSR
 *   written by ep_get_layout for the same routing. */
EP_API ep_status_t ep_combine_expert_choice(const void* y, int32_t hidden, const ep_routing_desc_t* routing,
                                     const ep_layout_t* layout, const float* expert_weights, void* out,
                                     ep_dtype_t out_dtype, ep_stream_t stream);

/* ------------------------------------------------------------------------
 * Per-rank (deduplicated) path: [README] "API Overview", normal-mode
 * dispatch "to expert ranks" (received tokens plus their top-k information)
 * and combine "(reduce) tokens from dispatch" with the dispatch handle.
 * A token is copied once to every logical rank r with
 * is_token_in_rank[t, r] = 1, instead of once per (token, expert) pair.
 * Rank r's rows are its tokens in ascending token order; the ranks' row
 * ranges are laid end to end in one buffer of rank_offsets[R] rows.
 *   rank_offsets  int32 [R+1]  exclusive scan of num_tokens_per_rank
 *   rank_row      int32 [T, R] row of token t in rank r's range, -1 if the
 *                              token does not go to rank r
 * ---------------------------------------------------------------------- */
typedef struct {
    int32_t* rank_offsets;
    int32_t* rank_row;
} ep_rank_layout_t;

/* Rank layout from the is_token_in_rank and num_tokens_per_rank that
 * ep_get_layout wrote for the same routing (either routing kind). */
EP_API ep_status_t ep_get_rank_layout(const ep_routing_desc_t* routing, const ep_layout_t* layout,
                                      const ep_rank_layout_t* rank_layout, ep_stream_t stream);

/* Per-rank dispatch (TOPK routing): recv_x[rank_row[t, r]] = x[t] for every
 * rank of every token, and, per received row, the token's K entries as the
 * rank sees them:
 *   recv_topk_idx     optional int64 [rows, K]: e - r*E/R for an expert e of
 *                     rank r, else -1
 *   recv_topk_weights optional fp32 [rows, K]: topk_weights[t, k] for those
 *                     entries, else 0 (needs topk_weights when T > 0)
 *   recv_src          optional int32 [rows]: source token
 * x bf16 [T, H], recv_x bf16 [num_recv_rows, H], both 16-byte aligned,
 * H % 8 == 0.  Rows >= num_recv_rows are skipped with EP_DEVERR_OVERFLOW. */
EP_API ep_status_t ep_dispatch_ranks(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                     const ep_layout_t* layout, const ep_rank_layout_t* rank_layout,
                                     int64_t num_recv_rows, const float* topk_weights, void* recv_x,
                                     int64_t* recv_topk_idx, float* recv_topk_weights, int32_t* recv_src,
                                     ep_stream_t stream);

/* ep_get_layout, ep_get_rank_layout and ep_dispatch_ranks in one call (the
 * same arguments, results and checks; nothing is launched unless all three
 * can run).  The dispatch's CTAs load their source rows while the rank
 * layout kernel runs and wait for it only before they read rank_row; the
 * separate calls cannot overlap this way, since a dispatch alone must first
 * wait for whatever kernel precedes it (it may have written x). */
EP_API ep_status_t ep_layout_dispatch_ranks(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                            const ep_layout_t* layout, const ep_rank_layout_t* rank_layout,
                                            int64_t num_recv_rows, const float* topk_weights, void* recv_x,
                                            int64_t* recv_topk_idx, float* recv_topk_weights, int32_t* recv_src,
                                            ep_stream_t stream);

/* Rank-level combine: out[t] = sum over the token's ranks r in ascending
 * order of y[rank_row[t, r]], fp32 additions from 0 (the ranks have applied
 * the gate weights), written as fp32 or rounded once (RNE) to bf16; a token
 * with no rank gets +0.  y bf16 [num_y_rows, H]; out [T, H]. */
EP_API ep_status_t ep_combine_ranks(const void* y, int32_t hidden, int64_t num_y_rows, const ep_routing_desc_t* routing,
                                    const ep_layout_t* layout, const ep_rank_layout_t* rank_layout, void* out,
                                    ep_dtype_t out_dtype, ep_stream_t stream);

/* ------------------------------------------------------------------------
 * Per-rank path over peer memory: one process per GPU, the routing's R
 * logical ranks are the R processes of a group, and the all-to-all of the
 * per-rank path is fused into its kernels.  [README] "Normal Mode (Prefill /
 * Training)" (intranode transfer) and the strategy table's all-to-all: each
 * token goes once to every rank that holds one of its experts, and one
 * partial row per (token, rank) comes back and is reduced on the token's
 * rank.  Here the dispatch kernel stores each (token, rank) row straight
 * into that rank's receive buffer, and the combine kernel reads the partial
 * rows straight from the ranks' buffers: no staging buffer and no separate
 * transfer.
 *
 * Every rank r holds, in device memory that the other processes map
 * (ep_peer_alloc / ep_peer_open):
 *   recv_x             bf16  [capacity, H]  rows it receives
 *   recv_topk_idx      int64 [capacity, K]  their top-k entries as rank r
 *                                           sees them (local expert id or -1)
 *   recv_topk_weights  fp32  [capacity, K]  gate weight or 0
 *   recv_src           int32 [capacity]     source token on the source rank
 *   y                  bf16  [capacity, H]  partial rows it sends back, in
 *                                           the order of recv_x
 *   rank_counts        int32 [R, R]         row i = rank i's
 *                                           num_tokens_per_rank
 * Rank j's rows are those of source rank 0 first, each source's rows in
 * ascending token order; source i's block starts at row
 *   base(i, j) = sum over i' < i of rank_counts[i', j]
 * and token t of source i lands at base(i, j) + rank_row[t, j] -
 * rank_offsets[j] (its rank layout).  This is the order an all-to-all-v of
 * the ep_dispatch_ranks rows delivers, and the results equal that path's bit
 * for bit.
 *
 * ep_peers_t holds, per rank r, the address under which THIS process reaches
 * rank r's buffer (its own allocation for r == rank, a mapping made by
 * ep_peer_open otherwise), as device arrays of R addresses; each process
 * builds its own tables, since mappings differ between processes.
 *
 * These calls only move data: none of their kernels waits for another rank.
 * The caller separates the ranks' phases with a barrier that every rank
 * passes only after its own kernels of the phase before have completed (for
 * example: synchronise the stream, then a process-group barrier):
 *   1. ep_get_layout (R ranks) -> ep_get_rank_layout -> ep_peer_publish_counts
 *   2. barrier
 *   3. ep_dispatch_peers
 *   4. barrier; rank j's received rows: sum over i of its rank_counts[i, j]
 *   5. local experts: rank j writes its partial rows to y[0 .. received)
 *   6. barrier
 *   7. ep_combine_peers
 * and step 2 of the next round orders its writes after every rank's step 7.
 * Rows that would land at or past `capacity` are skipped with
 * EP_DEVERR_OVERFLOW in the calling rank's workspace error word.
 * ---------------------------------------------------------------------- */
typedef struct {
    int32_t num_ranks;                /* R: the routing's num_ranks */
    int32_t rank;                     /* this process's rank, 0 <= rank < R */
    int64_t capacity;                 /* rows of every rank's recv_x and y */
    void* const* recv_x;              /* device array of R addresses */
    int64_t* const* recv_topk_idx;    /* device array of R addresses, or NULL */
    float* const* recv_topk_weights;  /* device array of R addresses, or NULL */
    int32_t* const* recv_src;         /* device array of R addresses, or NULL */
    const void* const* y;             /* device array of R addresses */
    int32_t* const* rank_counts;      /* device array of R addresses */
} ep_peers_t;

/* Bytes of an IPC handle (cudaIpcMemHandle_t) as ep_peer_alloc writes it. */
#define EP_IPC_HANDLE_BYTES 64

/* Device memory that other processes can map: `bytes` (>= 1) allocated with
 * cudaMalloc on the current device (256-byte aligned) into *ptr, and its IPC
 * handle written to handle[0 .. EP_IPC_HANDLE_BYTES).  Release with
 * ep_peer_free after every process that opened it has closed it. */
EP_API ep_status_t ep_peer_alloc(size_t bytes, void** ptr, void* handle);
EP_API ep_status_t ep_peer_free(void* ptr);

/* Map another process's ep_peer_alloc buffer (its handle, received by any
 * host channel) into this process: *ptr is its address here (over NVLink
 * when it lives on another GPU; peer access is enabled on first use).  A
 * process cannot open its own handles: use the pointer it allocated.  Unmap
 * with ep_peer_close. */
EP_API ep_status_t ep_peer_open(const void* handle, void** ptr);
EP_API ep_status_t ep_peer_close(void* ptr);

/* Step 1: store layout->num_tokens_per_rank (written by ep_get_layout for
 * `routing`, R = peers->num_ranks) as row `rank` of every rank's
 * rank_counts. */
EP_API ep_status_t ep_peer_publish_counts(const ep_routing_desc_t* routing, const ep_layout_t* layout,
                                          const ep_peers_t* peers, ep_stream_t stream);

/* Step 3 (TOPK routing): for every token t and rank j with rank_row[t, j]
 * >= 0, row base(rank, j) + rank_row[t, j] - rank_offsets[j] of rank j's
 * recv_x gets x[t] (one read of x[t], one store per rank), and its
 * recv_topk_idx / recv_topk_weights / recv_src entries (when the tables are
 * given) the token's K entries as rank j sees them and t.  base() is read
 * from this rank's own rank_counts, which must hold every rank's row (step
 * 2).  x bf16 [T, H], 16-byte aligned, H % 8 == 0; topk_weights fp32 [T, K]
 * (needed with recv_topk_weights when T > 0).  Every recv_x must be
 * 16-byte aligned. */
EP_API ep_status_t ep_dispatch_peers(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                     const ep_layout_t* layout, const ep_rank_layout_t* rank_layout,
                                     const float* topk_weights, const ep_peers_t* peers, ep_stream_t stream);

/* Step 7: out[t] = sum over the token's ranks j in ascending order of row
 * base(rank, j) + rank_row[t, j] - rank_offsets[j] of rank j's y, fp32
 * additions from 0, written as fp32 or rounded once (RNE) to bf16; a token
 * with no rank gets +0 -- ep_combine_ranks with the rows read in place.
 * out [T, H] (out_dtype BF16 or FP32), 16-byte aligned; every y must be
 * 16-byte aligned. */
EP_API ep_status_t ep_combine_peers(int32_t hidden, const ep_routing_desc_t* routing, const ep_layout_t* layout,
                                    const ep_rank_layout_t* rank_layout, const ep_peers_t* peers, void* out,
                                    ep_dtype_t out_dtype, ep_stream_t stream);

/* ep_get_layout for callers that cannot allocate device memory.  The pages
 * have no counterpart: this is a deployment variant of the layout call.
 *
 * Who needs it: code that must not call cudaMalloc (or any allocator) when
 * it builds a layout -- a plugin inside an inference server or framework that
 * is handed only its input and output tensors while the host program owns
 * every other byte of device memory, or a decode loop where an allocation
 * could synchronise the device and stall the step.
 *
 * It computes exactly what ep_get_layout computes, writing the same outputs
 * in `layout`, but ignores layout->workspace / workspace_bytes: its scratch is
 * a fixed array of EP_STATIC_WORKSPACE_BYTES inside the library, held by
 * every GPU that loads the library until the process exits.  A routing whose
 * ep_workspace_bytes() exceeds that size is rejected with EP_ERR_WORKSPACE
 * before anything is launched (token choice needs 256 + 256*(E + 32) bytes,
 * at most 270 KB, and always fits; expert choice needs 256 + 4*(2*T + E*C)
 * bytes rounded up to 256).  Nothing is allocated or freed.
 *   device_error_flags  optional device pointer to one uint32: zeroed at the
 *                       start of the call, then receives the EP_DEVERR_* bits
 *                       the layout kernels raise (NULL: not reported).
 * layout->num_valid_host is honoured as by ep_get_layout.
 * The first call on a device looks up the array's device address (with that
 * device current), so make one call per device before any stream capture.
 * All calls share the array and it keeps the last call's contents: calls that
 * overlap on the GPU (other streams, other host threads) race on it and must
 * be serialised by the caller.  Every call first zeroes the array's 256-byte
 * header (error word and grid-barrier words) on `stream`, so a call that
 * follows one whose wait ran out (EP_DEVERR_TIMEOUT) starts clean: there is
 * nothing for the caller to reset. */
#define EP_STATIC_WORKSPACE_BYTES ((size_t)4 << 20)
EP_API ep_status_t ep_get_layout_no_alloc(const ep_routing_desc_t* routing, const ep_layout_t* layout,
                                          uint32_t* device_error_flags, ep_stream_t stream);

/* Synchronise `stream`, read the device error word of layout->workspace into
 * *flags (EP_DEVERR_* bits), clear it if `clear`, and return EP_OK when it is
 * zero, else the status of the lowest set bit (BAD_INDEX, OVERFLOW, TIMEOUT).
 * After EP_ERR_TIMEOUT re-run ep_workspace_init on the workspace (the
 * grid-barrier words may hold a partial count). */
EP_API ep_status_t ep_get_device_error(const ep_layout_t* layout, uint32_t* flags, int clear, ep_stream_t stream);

EP_API const char* ep_status_string(ep_status_t status);
EP_API int ep_version(void);

#ifdef __cplusplus
}
#endif
#endif /* EP_B200_H_ */
