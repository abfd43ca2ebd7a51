/*
 * ep.h -- C ABI of the B200 (sm_100a) MoE expert-parallel layout / dispatch /
 * combine library (libep_b200.so).
 *
 * The operations follow the interface the DeepEP pages describe:
 *   - "DeepEP (DeepEveryParallel) Documentation" (docsearch.algolia.com),
 *     item 10 "Perform MoE Dispatch and Combine for Training or Prefilling":
 *     dispatch takes the hidden states, the top-k expert ids and weights, the
 *     number of experts and the expert alignment, routes every token to its
 *     experts and returns the received rows plus a handle with the routing
 *     metadata; combine takes expert outputs and that handle and reduces them
 *     back to the source tokens.
 *   - the same page, item 3 "Perform MoE Dispatch and Combine for Inference
 *     Decoding": a cached handle is passed again when the gating decision has
 *     not changed, so the layout and its host synchronisation are skipped.
 *   - "DeepSeek publica DeepEP, una biblioteca open source para entrenamiento
 *     e inferencia MoE" (news.hada.io), section "Patrones de uso en
 *     entrenamiento, prefill y decoding": the handle carries the per-expert
 *     received-token counts the expert GEMMs need; section "Resultados de
 *     medición de rendimiento": FP8 dispatch, BF16 combine.
 *
 * On one GPU the expert-parallel ranks are virtual: rank r owns experts
 * [r*E/R, (r+1)*E/R) and the contiguous slice of receive rows of those
 * experts.  The calls at the end of this header run the same contract with
 * the ranks as real GPUs, one process each.
 *
 * Notation: T tokens, H hidden size, k top-k slots per token, E experts,
 * R virtual ranks.  A slot is a pair (t, j), 0 <= j < k.
 *
 * Definition of the layout (the pages do not spell it out; this library
 * fixes it so that results are bit-exact and independent of scheduling):
 *   receive rows are expert-major; inside an expert's segment rows follow
 *   (source token, slot) order.  Packed mode (capacity == 0): segment e
 *   starts at seg[e] = sum over e' < e of align_up(cnt[e'], expert_alignment).
 *   Padded mode (capacity > 0): segment e is rows [e*capacity, (e+1)*capacity).
 *   A slot whose id is -1 is unused: no row, no combine term.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device (or managed) memory of the
 *     current device; the caller allocates and owns them.  Pointers marked
 *     "host" are ordinary host memory.
 *   - Row-major, densely packed arrays.  x, recv_x, y and combined_x must be
 *     16-byte aligned; recv_scales, topk_weights 4-byte aligned.
 *   - All device work is enqueued on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and is asynchronous, unless a call says it
 *     synchronises.
 *   - Argument errors are detected on the host and returned at once with
 *     nothing enqueued.  Data errors found on the device set the handle's
 *     device error word instead, and the layout still completes: an id
 *     outside [-1, E) is taken as an unused slot, and in padded mode an
 *     expert named by more than `capacity` slots keeps its first `capacity`
 *     slots in (token, slot) order while the rest get no row (pos -1).
 *     Counts and is_token_in_rank count every slot that names an expert.
 *     ep_handle_check() reports the word (a bad id before an overflow).
 *     Every device write stays inside the buffers described here.  No call
 *     traps, aborts or throws across the ABI.
 *   - Limits: 1 <= k <= 32, 1 <= E <= 4096, 1 <= R <= E, E % R == 0,
 *     T * k < 2^31, 8 <= H <= 2^24, H % 8 == 0 (bf16) and H % 128 == 0 (FP8).
 */
#ifndef EP_B200_EP_H
#define EP_B200_EP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so that the header needs no CUDA include. */
typedef struct CUstream_st *ep_stream_t;

/* Opaque routing handle (the pages' EPHandle): owns device copies of the
 * slot positions, the source-token index of every receive row, the expert
 * segments, the rank slices, the per-expert counts and a device error word. */
typedef struct ep_handle ep_handle;

typedef enum ep_status {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1,   /* bad size, null or misaligned pointer, limits exceeded */
    EP_ERR_BAD_EXPERT_ID = 2, /* a top-k id outside [-1, E) (device-detected) */
    EP_ERR_CAPACITY = 3,      /* padded mode: an expert received more than `capacity` tokens */
    EP_ERR_CUDA = 4,          /* a CUDA runtime call failed */
    EP_ERR_OOM = 5,           /* device allocation failed */
    EP_ERR_TIMEOUT = 6,       /* reserved: a bounded device-side wait gave up (no kernel waits today) */
    EP_ERR_NO_DEVICE = 7,     /* no CUDA device, or the device is not sm_100 */
    EP_ERR_SCRATCH_LIMIT = 8  /* ep_layout_noalloc: the problem needs more than its fixed scratch */
} ep_status;

/* Human-readable name of a status.  Never NULL; static storage. */
const char *ep_status_str(ep_status status);

/* Upper bound on the receive rows a layout with these parameters can use:
 * E * capacity in padded mode, T*k + E*(expert_alignment-1) in packed mode.
 * recv_x / y must have at least this many rows.  This is the receive-buffer
 * bound the pages' dispatch takes as num_max_tokens_per_rank ("DeepEP
 * (DeepEveryParallel) Documentation", item 10: the per-rank receive capacity
 * is an argument of dispatch, so the buffers can be sized before any routing
 * is known); with `capacity` > 0 the bound is the padded per-expert layout of
 * the decoding case (item 3).  Host only, pure.  Returns 0 for invalid
 * arguments. */
size_t ep_max_recv_rows(int num_tokens, int num_topk, int num_experts,
                        int expert_alignment, int capacity);

/* Routing layout: the metadata part of the pages' dispatch (docsearch item
 * 10; news.hada.io "Patrones de uso ...").  Computes, bit-exactly:
 *   num_tokens_per_expert[e] = number of slots naming expert e       (device int32 [E], may be NULL)
 *   num_tokens_per_rank[r]   = tokens with >= 1 expert on rank r      (device int32 [R], may be NULL)
 *   is_token_in_rank[t][r]   = 1 if token t has an expert on rank r   (device uint8 [T, R], may be NULL)
 * and a new handle holding pos[T][k] (receive row of each slot, -1 for
 * unused or over-capacity slots), src_idx[rows] (source token of each
 * receive row, -1 for padding), seg[E+1] and rank_off[R+1].
 *   topk_idx: device int32 [T, k]; ids in [-1, E).
 *   expert_alignment >= 1: packed segments are rounded up to a multiple of it.
 *   capacity: 0 for packed mode, else rows per expert (a multiple of expert_alignment).
 * On success *out_handle receives a handle that the caller frees with
 * ep_handle_free().  The handle's device memory is allocated stream-ordered
 * on `stream` from a memory pool the library keeps per device (memory freed by
 * ep_handle_free returns to that pool for the next layout, not to the
 * driver).  T == 0 is allowed (empty handle). */
ep_status ep_layout(const int32_t *topk_idx, int num_tokens, int num_topk,
                    int num_experts, int num_ranks, int expert_alignment, int capacity,
                    int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                    uint8_t *is_token_in_rank, ep_handle **out_handle, ep_stream_t stream);

/* Dispatch (docsearch item 10, FP8 per "deepseek-ai/DeepEP" repolode
 * "Funciones clave"): scatter every token's hidden row to the receive row of
 * each of its valid slots.
 *   x: device bf16 [T, H].
 *   use_fp8 == 0: recv_x is device bf16 [recv_rows, H]; each row a bit copy of x[t].
 *   use_fp8 != 0: recv_x is device e4m3 (OCP FP8 E4M3, 1 byte) [recv_rows, H] and
 *     recv_scales device fp32 [recv_rows, H/128].  Per token and 128-channel
 *     group g: amax = max |x|; scale = amax/448 (fp32, round to nearest);
 *     codes = e4m3_rn_satfinite(x * (448/amax)) with 448/amax one rounded
 *     fp32 division; an all-zero group gives scale 0 and codes 0x00.  The
 *     same codes and scales go to all k rows of the token.
 *   recv_src_idx: device int32 [recv_rows] or NULL; receives a copy of the
 *     handle's src_idx (-1 on padding rows).
 *   recv_rows: rows allocated in recv_x / recv_scales / recv_src_idx; must be
 *     >= ep_max_recv_rows() of the handle's layout.
 * Only rows that slots map to are written; padding rows keep their contents.
 * No allocation, no host synchronisation: may be captured in a CUDA graph and
 * reused with the same handle for every decoding step (docsearch item 3). */
ep_status ep_dispatch(const ep_handle *handle, const void *x, int hidden, int use_fp8,
                      void *recv_x, float *recv_scales, int32_t *recv_src_idx,
                      size_t recv_rows, ep_stream_t stream);

/* Combine (docsearch items 3 and 10; BF16 per news.hada.io "Resultados ..."):
 *   combined_x[t][i] = bf16_rn( fma chain, j = 0..k-1 over slots with pos >= 0,
 *                               acc = fmaf(topk_weights[t][j], y[pos[t][j]][i], acc),
 *                               starting from acc = +0.0f )
 *   y: device bf16 [recv_rows, H] (expert outputs, rows in the handle's layout).
 *   topk_weights: device fp32 [T, k].
 *   combined_x: device bf16 [T, H].  A token with no valid slot gets +0.0.
 * No allocation, no host synchronisation; graph-capturable. */
ep_status ep_combine(const ep_handle *handle, const void *y, const float *topk_weights,
                     int hidden, size_t recv_rows, void *combined_x, ep_stream_t stream);

/* Dispatch backward.  The pages ("DeepEP (DeepEveryParallel) Documentation",
 * item 10; news.hada.io "Patrones de uso ...") carry out dispatch's backward
 * pass with a combine; here it is the combine definition with every weight 1:
 *   grad_x[t][i] = bf16_rn( fp32 chain over valid slots j in slot order of
 *                           acc = acc + grad_recv[pos[t][j]][i], from +0.0f )
 *   grad_recv: device bf16 [recv_rows, H] (gradients of the receive rows; for
 *     an FP8 dispatch the gradient passes the quantisation unchanged).
 *   grad_x: device bf16 [T, H].  A token with no valid slot gets +0.0.
 * No allocation, no host synchronisation. */
ep_status ep_dispatch_backward(const ep_handle *handle, const void *grad_recv, int hidden,
                               size_t recv_rows, void *grad_x, ep_stream_t stream);

/* Combine backward (combine's backward pass is a dispatch, same passages):
 * with g = grad_out[t],
 *   grad_y[pos[t][j]][i] = bf16_rn( fp32_rn( topk_weights[t][j] * g[i] ) )   (weighted dispatch)
 *   grad_weights[t][j]   = sum_i g[i] * y[pos[t][j]][i]  accumulated in fp32 (dot product)
 *   grad_out: device bf16 [T, H]; y: device bf16 [recv_rows, H] (the expert
 *     outputs combine read; may be NULL when grad_weights is NULL);
 *   topk_weights: device fp32 [T, k]; grad_y: device bf16 [recv_rows, H]
 *     (only rows that slots map to are written);
 *   grad_weights: device fp32 [T, k] or NULL; 0 for unused slots.
 * grad_y is exact to the stated roundings.  grad_weights is summed in a fixed
 * order (deterministic run to run): per-thread chains over ceil(H/2048)
 * groups of 16 products, an xor shuffle tree and a sum over the block's 4
 * warps, so its error from the exact dot product is at most about
 * (16*ceil(H/2048) + 37) * 2^-24 * sum_i |g[i]*y[i]|.
 * No allocation, no host synchronisation. */
ep_status ep_combine_backward(const ep_handle *handle, const void *grad_out, const void *y,
                              const float *topk_weights, int hidden, size_t recv_rows,
                              void *grad_y, float *grad_weights, ep_stream_t stream);

/* Element formats of ep_dispatch_ex. */
#define EP_FORMAT_BF16 0
#define EP_FORMAT_E4M3 1

/* Dispatch with the options of the pages' full dispatch call ("DeepEP
 * (DeepEveryParallel) Documentation", item 10: BF16 or FP8 input, the FP8
 * input given as data plus scale factors; the SM count the call may use, as
 * "DeepSeek publica DeepEP ..." (news.hada.io), "Interfaz centrada en
 * ElasticBuffer", lets num_sms be set per call) and a scale layout a grouped
 * FP8 GEMM can consume ([hada] "Cambios clave de la versión V2": a GEMM
 * layout).
 *   in_format / out_format: EP_FORMAT_BF16 -> BF16 (bit copy, as ep_dispatch),
 *     EP_FORMAT_BF16 -> EP_FORMAT_E4M3 (quantised here, as ep_dispatch), or
 *     EP_FORMAT_E4M3 -> EP_FORMAT_E4M3: x is device e4m3 [T, H] already
 *     quantised and x_scales device fp32 [T, H/128] row-major; codes and
 *     scales are copied to the k rows unchanged.
 *   recv_scales: scale of receive row p and group g stored at
 *     recv_scales[p * scale_row_stride + g * scale_group_stride].  Accepted
 *     layouts: row-major (group stride 1, row stride >= H/128; ep_dispatch
 *     uses H/128) and column-major (row stride 1, group stride >= recv_rows,
 *     e.g. recv_rows rounded up to a multiple of 4 for 16-byte aligned
 *     columns).  The buffer must hold (recv_rows-1)*row_stride +
 *     (H/128-1)*group_stride + 1 floats.  Column-major scales of e4m3 input
 *     are written by a second kernel from x_scales in receive-row order
 *     (contiguous runs per column); of quantised-here input, by the
 *     dispatch itself, one 4-byte store per row and group
 *     (ep_dispatch_fp8_colmajor is the faster call for that case).
 *   num_sms: 0 = no limit (one block per token chunk); n > 0 = at most the
 *     blocks n SMs can hold at once, looping over the work, so that
 *     concurrent kernels on other streams keep the remaining SMs' worth of
 *     resources (the hardware still places the blocks).
 * Other arguments and rules as ep_dispatch. */
ep_status ep_dispatch_ex(const ep_handle *handle, const void *x, const float *x_scales, int hidden,
                         int in_format, int out_format, void *recv_x, float *recv_scales,
                         int64_t scale_row_stride, int64_t scale_group_stride,
                         int32_t *recv_src_idx, size_t recv_rows, int num_sms, ep_stream_t stream);

/* FP8 dispatch with column-major scales, the layout a grouped FP8 GEMM reads
 * ([hada] "Cambios clave de la versión V2": a GEMM layout), written the fast
 * way.  Codes, scales and rules as ep_dispatch with use_fp8 != 0; the scale
 * of receive row p and group g goes to recv_scales[g * scale_ld + p].
 *   scale_ld: leading dimension of recv_scales, >= recv_rows (e.g. recv_rows
 *     rounded up to a multiple of 4 for 16-byte aligned columns); the buffer
 *     holds (H/128 - 1) * scale_ld + recv_rows floats.
 *   token_scales: device fp32 [T, H/128] row-major, written: the scale of every
 *     token and group (the values the token's receive rows get).  Besides
 *     being an output, it is the table the second kernel reads.
 * Two kernels: the dispatch writes the codes of every receive row and each
 * token's scales once, into token_scales; a second kernel walks the receive
 * rows in order and stores recv_scales column by column as contiguous runs.
 * (ep_dispatch_ex with a column-major layout gives the same values with one
 * scattered 4-byte store per row and group, which is slower.)  Padding rows
 * are not written.  num_sms as in ep_dispatch_ex.  No allocation, no host
 * synchronisation. */
ep_status ep_dispatch_fp8_colmajor(const ep_handle *handle, const void *x, int hidden, void *recv_x,
                                   float *recv_scales, int64_t scale_ld, float *token_scales,
                                   int32_t *recv_src_idx, size_t recv_rows, int num_sms, ep_stream_t stream);

/* Combine with an SM budget: as ep_combine, with num_sms as in ep_dispatch_ex. */
ep_status ep_combine_ex(const ep_handle *handle, const void *y, const float *topk_weights,
                        int hidden, size_t recv_rows, void *combined_x, int num_sms,
                        ep_stream_t stream);

/* Per-row routing outputs of dispatch: the pages' recv_topk_idx and
 * recv_topk_weights (docsearch item 10: dispatch returns them beside recv_x),
 * plus the slot each row came from.  Every receive row of this layout holds
 * one slot (t, j); for each row r < num_recv_rows of the handle:
 *   r filled by slot (t, j):  recv_topk_idx[r]     = topk_idx[t][j]  (the expert whose segment holds r)
 *                             recv_topk_weights[r] = topk_weights[t][j]  (bit copy)
 *                             recv_slot[r]         = t * k + j  (so t = recv_slot / k = src_idx[r])
 *   r filled by no slot:      -1, 0.0f, -1
 *   topk_weights: device fp32 [T, k]; read only when recv_topk_weights is
 *     not NULL (then it must not be NULL).
 *   recv_topk_idx, recv_topk_weights, recv_slot: device [recv_rows] int32 /
 *     fp32 / int32, 4-byte aligned, each may be NULL (nothing to do when all
 *     are).  All num_recv_rows rows are written, padding rows included; rows
 *     past num_recv_rows are not touched.
 *   recv_rows: length of those buffers, >= num_recv_rows of the handle.
 * Asynchronous, no allocation, no host synchronisation (capturable in a CUDA
 * graph with a kept handle).  After a data error the layout is still
 * complete (see the conventions at the top), and these values follow it:
 * an invalid id or an over-capacity slot fills no row. */
ep_status ep_dispatch_topk(const ep_handle *handle, const float *topk_weights,
                           int32_t *recv_topk_idx, float *recv_topk_weights, int32_t *recv_slot,
                           size_t recv_rows, ep_stream_t stream);

/* fp32 -> FP8 e4m3 encoding with the rounding FP8 dispatch uses (the
 * hardware's round-to-nearest-even, saturating conversion: OCP E4M3, no
 * infinities, values beyond +-448 and +-inf give +-448, NaN stays NaN), for
 * callers who pre-quantise (ep_dispatch_ex accepts e4m3 input with its
 * scales).  x: device fp32 [n]; codes: device uint8 [n]; both 16-byte
 * aligned.  Asynchronous on `stream`. */
ep_status ep_e4m3_encode(const float *x, uint8_t *codes, size_t n, ep_stream_t stream);

/* Release a handle: the end of the pages' EPHandle's life ("DeepEP
 * (DeepEveryParallel) Documentation", items 3 and 10: a handle returned by
 * dispatch is passed to combine and, while the routing does not change, to
 * later dispatches; here the caller says when it is no longer needed).  Its
 * device memory is freed stream-ordered on the stream that created it
 * (cudaFreeAsync); work that uses the handle on other streams must be ordered
 * before that stream's current position by the caller.  NULL is a no-op. */
void ep_handle_free(ep_handle *handle);

/* Handle geometry (host only, no device work). */
typedef struct ep_handle_info {
    int num_tokens, num_topk, num_experts, num_ranks, expert_alignment, capacity;
    size_t num_recv_rows; /* = ep_max_recv_rows(...) of this layout */
    int layout_kernels;   /* kernels the layout launched: 1 (one CTA, or T = 0) or 2 (tiled) */
    int layout_path;      /* EP_LAYOUT_PATH_*: how the layout ran */
} ep_handle_info;
#define EP_LAYOUT_PATH_EMPTY 0   /* T == 0 */
#define EP_LAYOUT_PATH_ONE_CTA 1 /* small problems: the whole layout in one CTA */
#define EP_LAYOUT_PATH_TILED 2   /* one CTA per tile of tokens, two kernels */
ep_status ep_handle_get_info(const ep_handle *handle, ep_handle_info *info);

/* Copy the handle's metadata into caller buffers (device-to-device, async on
 * `stream`).  Any destination may be NULL.
 *   pos: device int32 [T, k]; src_idx: device int32 [num_recv_rows];
 *   seg: device int32 [E+1]; rank_off: device int32 [R+1]. */
ep_status ep_handle_export(const ep_handle *handle, int32_t *pos, int32_t *src_idx,
                           int32_t *seg, int32_t *rank_off, ep_stream_t stream);

/* The pages' num_recv_tokens_per_expert_list: per-expert counts copied to
 * host int32 [E].  Synchronises `stream`. */
ep_status ep_handle_counts_host(const ep_handle *handle, int32_t *host_counts,
                                ep_stream_t stream);

/* Read the handle's device error word after the work enqueued on `stream`
 * so far.  The pages' dispatch checks its inputs and the receive capacity
 * (num_max_tokens_per_rank, docsearch item 10) inside its kernels; this
 * library records such data errors in the handle on the device instead of
 * stopping, and this call is where the caller learns of them.  Synchronises
 * `stream`.  Returns EP_OK, EP_ERR_BAD_EXPERT_ID, EP_ERR_CAPACITY or
 * EP_ERR_TIMEOUT (the first set, in that order). */
ep_status ep_handle_check(const ep_handle *handle, ep_stream_t stream);

/* Size, in 32-bit words, of the fixed device scratch array ep_layout_noalloc
 * uses (128 KiB).  Every GPU that loads the library holds it until the
 * process exits.  The library finds the array's device address on the first
 * call on a device and again after the device's CUDA context changes (e.g.
 * after cudaDeviceReset), so a reset device needs no action by the caller. */
#define EP_NOALLOC_SCRATCH_WORDS (1 << 15)

/* ep_layout_noalloc -- the routing layout of ep_layout, for callers that
 * cannot allocate device memory.  The pages have no counterpart: DeepEP's
 * buffer object allocates its own memory; this entry point exists for users
 * of this library whose device memory is planned up front (a static memory
 * planner in a serving loop), who run under another framework's allocator and
 * may not call the CUDA allocator themselves, or who cannot afford
 * cudaMalloc's implicit synchronisation on a latency-critical path.
 *
 * It computes exactly what ep_layout computes, bit for bit, but returns no
 * handle: the metadata a handle would own goes to caller buffers instead.
 *   pos:      device int32 [T, k]          (receive row of each slot, -1 if unused)
 *   src_idx:  device int32 [rows]          (rows = ep_max_recv_rows(...); -1 on padding)
 *   seg:      device int32 [E+1];  rank_off: device int32 [R+1]
 *   num_tokens_per_expert, num_tokens_per_rank, is_token_in_rank: as in
 *     ep_layout, each may be NULL.
 *   error_word: device uint32 [1] or NULL.  Cleared by the call, then set
 *     like a handle's error word (bit 1: id outside [-1, E); bit 2: padded
 *     expert over capacity).  With NULL, device-detected data errors are not
 *     reported.
 * Allocates nothing: no cudaMalloc / cudaMallocAsync / cudaFree and no
 * allocating library routine.  Its only device memory besides the caller's
 * buffers is a fixed scratch array of EP_NOALLOC_SCRATCH_WORDS words inside
 * the library; a problem that needs more is rejected.  The need is
 * align4(tiles*E) + align4(tiles*R) + align4(E) + align4(tiles) + 1 words,
 * with tiles = ceil(T / tile) and tile = 128 tokens, doubled until
 * tiles*(E + R) <= 24576.  Every problem with E + R >= 8 fits.  With very few
 * experts and millions of tokens the one flag word per tile can push the need
 * past the limit; such a problem is rejected with EP_ERR_SCRATCH_LIMIT before
 * anything is enqueued.  The first call on a device looks up the array's
 * device address (with that device current; again if the device's context
 * changed); make that first call before any stream capture.  All calls share
 * the array and it keeps the last call's contents: calls whose GPU work
 * overlaps (unordered streams) race on it; calls ordered on one stream do not.
 * EP_DEBUG logs one line per call, as for ep_layout, with the scratch words
 * the call uses.  Other limits and argument errors as for ep_layout. */
ep_status ep_layout_noalloc(const int32_t *topk_idx, int num_tokens, int num_topk,
                            int num_experts, int num_ranks, int expert_alignment, int capacity,
                            int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                            uint8_t *is_token_in_rank, int32_t *pos, int32_t *src_idx,
                            int32_t *seg, int32_t *rank_off, uint32_t *error_word,
                            ep_stream_t stream);

/* ========================================================================= *
 * Expert parallelism across GPUs (one process per GPU, W ranks)              *
 * ========================================================================= *
 *
 * The pages' dispatch sends every token to its experts on all ranks and
 * combine returns the expert outputs to the rank the token came from
 * (news.hada.io "Patrones de uso en entrenamiento, prefill y decoding";
 * docsearch item 10).  Here rank r of W owns experts [r*E/W, (r+1)*E/W), and
 * its receive buffer holds exactly the rows the single-GPU layout would give
 * rank r for all ranks' tokens concatenated in rank order: segment by
 * segment for its experts (packed with expert_alignment, or `capacity` rows
 * each), inside a segment by (source rank, source token, slot).
 *
 * One step, on every rank, all on one stream:
 *   1. ep_layout(local topk_idx, E, R = W, alignment 1, capacity 0) with
 *      num_tokens_per_expert -> counts[E];
 *   2. all-gather counts into all_counts[W][E] (e.g. NCCL; the caller's);
 *   3. ep_plan_create(...)  -- where each local slot goes, rank and row;
 *   4. ep_dispatch_peer(...) -- stores straight into the owners' buffers;
 *   5. a barrier collective (every rank's stores are complete before any
 *      rank reads its receive buffer), then the expert computation writes y;
 *   6. a barrier collective (every y complete), then ep_combine_peer(...),
 *      which reads the y rows from the owners' buffers.
 * The all-gather of the next step orders that step's stores after this
 * step's reads on every rank.  No kernel waits on another rank: ordering is
 * the caller's collectives (a rank that does not arrive shows up as a
 * collective timeout on the host, never as a spinning GPU).
 * A routing that does not change reuses the plan (cached handle, item 3).
 *
 * Peer memory: every rank's receive / scale / expert-output buffers must be
 * addressable from this process (ep_ipc_export / ep_ipc_import, or any other
 * mapping); only plain 16-byte loads and stores reach them. */

/* Rows a rank may receive: total_tokens (all ranks) * k, plus
 * (E/W) * (expert_alignment - 1) of alignment slack; (E/W) * capacity when
 * capacity > 0.  Host only, pure; 0 for invalid arguments. */
size_t ep_peer_max_recv_rows(int64_t total_tokens, int num_topk, int num_experts, int world,
                             int expert_alignment, int capacity);

typedef struct ep_plan ep_plan;

/* Plan of one rank for one routing.
 *   local: this rank's layout handle, made with num_ranks == world,
 *     expert_alignment 1 and capacity 0 (EP_ERR_INVALID_ARG otherwise); the
 *     plan reads its positions and segments now and keeps no reference.
 *   topk_idx: device int32 [T, k], the ids the local layout was made from.
 *   all_counts: device int32 [world, E]; row s = rank s's
 *     num_tokens_per_expert (every rank passes the same matrix).
 *   rank, world: this rank and the group size.
 *   expert_alignment, capacity: the receive layout, as in ep_layout (the same
 *     on every rank).
 *   recv_rows: rows of every rank's receive buffer (the same on every rank),
 *     < 2^31; ep_peer_max_recv_rows() rows always suffice.
 * Writes *out; the plan owns one stream-ordered device allocation, freed by
 * ep_plan_free.  A slot whose row would fall past recv_rows or past a padded
 * expert's capacity gets no row and sets the plan's error word
 * (ep_plan_check -> EP_ERR_CAPACITY); no call ever writes outside a buffer. */
ep_status ep_plan_create(const ep_handle *local, const int32_t *topk_idx, const int32_t *all_counts,
                         int rank, int world, int expert_alignment, int capacity, size_t recv_rows,
                         ep_plan **out, ep_stream_t stream);
void ep_plan_free(ep_plan *plan);

/* Copies of the plan (device-to-device, async; any destination may be NULL):
 *   dst: int32 [T, k, 2] (owner rank, row in the owner's receive buffer) of
 *     every local slot, (-1, -1) for a slot without a row;
 *   recv_seg: int32 [E/W + 1] segment starts of this rank's experts in its
 *     own receive buffer (recv_seg[E/W] = rows it receives);
 *   recv_counts: int32 [E/W] slots routed to each of this rank's experts by
 *     all ranks (the grouped GEMM's per-expert row counts). */
ep_status ep_plan_export(const ep_plan *plan, int32_t *dst, int32_t *recv_seg, int32_t *recv_counts,
                         ep_stream_t stream);
/* Rows this rank receives (host; synchronises the stream). */
ep_status ep_plan_recv_rows_host(const ep_plan *plan, int64_t *rows, ep_stream_t stream);
/* The plan's device error word (synchronises): EP_OK or EP_ERR_CAPACITY. */
ep_status ep_plan_check(const ep_plan *plan, ep_stream_t stream);

typedef struct ep_peers ep_peers;

/* Table of every rank's buffers as mapped in this process (host arrays of
 * `world` device pointers, entry r for rank r, this rank's own included):
 *   recv_x: receive buffers, [recv_rows, H] bf16 or e4m3, 16-byte aligned;
 *   recv_scales: FP8 scale buffers, fp32 [recv_rows, H/128] row-major, or
 *     NULL (BF16 dispatch only);
 *   y: expert-output buffers, bf16 [recv_rows, H] in receive-row order, or
 *     NULL (no combine);
 *   grad_y: buffers the combine backward writes the expert-output gradients
 *     into, bf16 [recv_rows, H] in receive-row order, or NULL.
 * Each pointer is checked on the host (non-NULL, 16-byte aligned) and the
 * tables are copied to device memory the object owns (ep_peers_free).  The
 * buffers themselves stay the caller's. */
ep_status ep_peers_create(int world, void *const *recv_x, float *const *recv_scales, void *const *y,
                          void *const *grad_y, size_t recv_rows, ep_peers **out);
void ep_peers_free(ep_peers *peers);

/* Per-row routing output tables of every rank (host arrays of `world`
 * device pointers, each [recv_rows], 4-byte aligned; any array may be NULL):
 * the expert id, the routing weight, the source rank and the source slot
 * (t * k + j on that rank) of each receive row.  Copied to device memory the
 * peer table owns; a second call replaces the first. */
ep_status ep_peers_set_topk(ep_peers *peers, int32_t *const *recv_topk_idx, float *const *recv_topk_weights,
                            int32_t *const *recv_src_rank, int32_t *const *recv_slot);

/* Per-row routing outputs across ranks: the pages' recv_topk_idx and
 * recv_topk_weights on the receiving side (docsearch item 10).  Every local
 * slot (t, j) with a row writes topk_idx[t][j], topk_weights[t][j], this
 * rank and t * k + j into the owner's tables at that row; this rank's own
 * rows that no slot fills (alignment or capacity padding inside its
 * received rows) get -1, 0.0f, -1, -1.  Rows past the received ones are not
 * touched.  topk_idx: device int32 [T, k] (the ids the plan was made from);
 * topk_weights: device fp32 [T, k], needed when a weight table is set.
 * Ordered like ep_dispatch_peer (the caller's collectives). */
ep_status ep_dispatch_topk_peer(const ep_plan *plan, const ep_peers *peers, const int32_t *topk_idx,
                                const float *topk_weights, ep_stream_t stream);

/* Dispatch across ranks: as ep_dispatch_ex, with row (d.y) of rank d.x's
 * buffers as the destination of each slot (d from the plan), written with
 * plain 16-byte stores through the peer mappings.  Scales of row p and group
 * g go to recv_scales[p * scale_row_stride + g * scale_group_stride] in the
 * owner's buffer, row-major (group stride 1, row stride >= H/128) or
 * column-major (row stride 1, group stride >= the peer table's recv_rows);
 * every rank's scale buffer must hold that layout.  The caller orders these
 * stores before the owners' reads with a collective. */
ep_status ep_dispatch_peer(const ep_plan *plan, const ep_peers *peers, const void *x, const float *x_scales,
                           int hidden, int in_format, int out_format, int64_t scale_row_stride,
                           int64_t scale_group_stride, int num_sms, ep_stream_t stream);

/* Combine across ranks: as ep_combine_ex, reading each slot's expert-output
 * row from its owner's y buffer through the peer mappings.  topk_weights
 * NULL means every weight 1, which is the backward of ep_dispatch_peer (the
 * pages: a dispatch's backward is a combine). */
ep_status ep_combine_peer(const ep_plan *plan, const ep_peers *peers, const float *topk_weights, int hidden,
                          void *combined_x, int num_sms, ep_stream_t stream);

/* Combine backward across ranks: as ep_combine_backward, with each slot's
 * gradient row bf16_rn(fp32_rn(w[t][j] * grad_out[t])) stored into its
 * owner's grad_y buffer and grad_w[t][j] = <grad_out[t], y row> read from
 * the owner's y buffer (the pages: a combine's backward is a dispatch).
 *   grad_out: device bf16 [T, H]; topk_weights: device fp32 [T, k];
 *   grad_w: device fp32 [T, k], or NULL to skip the dot products (then the
 *     peers' y table may be NULL).  Needs the peers' grad_y table.
 * Rows no slot fills are not written.  The caller orders the stores before
 * the owners' reads with a collective, as for ep_dispatch_peer. */
ep_status ep_combine_backward_peer(const ep_plan *plan, const ep_peers *peers, const void *grad_out,
                                   const float *topk_weights, int hidden, float *grad_w,
                                   ep_stream_t stream);

/* CUDA IPC for the peer table.  ep_ipc_export writes the 64-byte handle of
 * the cudaMalloc allocation that holds `ptr` and ptr's offset in it (host
 * outputs); another process on the same node opens it with ep_ipc_import
 * (peer access enabled lazily) and closes it with ep_ipc_release(ptr,
 * offset).  Allocations made through the virtual-memory API (e.g. an
 * expandable-segments allocator) cannot be exported: EP_ERR_CUDA. */
#define EP_IPC_HANDLE_BYTES 64
ep_status ep_ipc_export(const void *ptr, void *handle, uint64_t *offset);
ep_status ep_ipc_import(const void *handle, uint64_t offset, void **ptr);
ep_status ep_ipc_release(void *ptr, uint64_t offset);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_EP_H */
