// ep_internal.cuh -- shared definitions of the CUDA library (not part of the ABI).
//
// Kernels live in layout.cu, dispatch.cu and combine.cu; the C ABI in
// ep_api.cu validates arguments, owns the handle and launches them.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

// Launch-shape parameters, chosen by measurement on B200.  Each can be
// overridden with -D at build time to sweep it.
#ifndef EP_DISPATCH_MAX_CHUNK     // dispatch: at most this many channels per work unit
#define EP_DISPATCH_MAX_CHUNK 8192
#endif
#ifndef EP_DISPATCH_MIN_UNITS_PER_SM  // dispatch: split rows into more chunks until the grid has
#define EP_DISPATCH_MIN_UNITS_PER_SM 0  // this many blocks per SM (small batches; 0 = off)
#endif
#ifndef EP_DISPATCH_MIN_CHUNK     // dispatch: ... but never below this many channels per block
#define EP_DISPATCH_MIN_CHUNK 512
#endif
#ifndef EP_DISPATCH_STORE_CS      // dispatch: evict-first (.cs) stores of the receive rows
#define EP_DISPATCH_STORE_CS 0
#endif
#ifndef EP_DISPATCH_TABLE_KEEP_L2  // dispatch: per-token scale table stored with an evict-last L2 policy
#define EP_DISPATCH_TABLE_KEEP_L2 1
#endif
#ifndef EP_COMBINE_THREADS        // threads per combine block
#define EP_COMBINE_THREADS 128
#endif
#ifndef EP_COMBINE_VPT            // combine: 16-byte vectors per thread (1, 2 or 4)
#define EP_COMBINE_VPT 1
#endif
#ifndef EP_COMBINE_POS_BEFORE_WAIT  // combine (local, one unit per block, small grids) reads the token's
#define EP_COMBINE_POS_BEFORE_WAIT 1  // positions before its programmatic wait (the layout kernels then signal at exit)
#endif
#ifndef EP_COMBINE_EARLY_MAX_BLOCKS_PER_SM  // ... small grid: at most this many blocks per SM
#define EP_COMBINE_EARLY_MAX_BLOCKS_PER_SM 8
#endif
#ifndef EP_COMBINE_L2_PREFETCH    // combine: add the .L2::256B prefetch hint to the row loads
#define EP_COMBINE_L2_PREFETCH 0
#endif
#ifndef EP_COMBINE_STREAM_STORE   // combine: evict-first (.cs) stores of the output
#define EP_COMBINE_STREAM_STORE 0
#endif

#ifndef EP_BWD_BATCH              // combine backward: y rows loaded ahead per batch of slots
#define EP_BWD_BATCH 8
#endif
#ifndef EP_BWD_MAX_THREADS        // combine backward: threads per block (upper bound)
#define EP_BWD_MAX_THREADS 128
#endif
#ifndef EP_BWD_MIN_BLOCKS         // combine backward: resident blocks per SM to plan registers for
#define EP_BWD_MIN_BLOCKS 4
#endif
#ifndef EP_LAYOUT_LOAD_BATCH      // layout: 16-byte loads per thread in flight when staging counts
#define EP_LAYOUT_LOAD_BATCH 8
#endif
// Layout: the one-CTA path up to this many slots.  Measured on B200 (E = 256,
// k = 8): one CTA takes 12.3 / 16.2 / 21.4 / 29.7 us at 1K / 2K / 4K / 8K
// slots, the two tiled kernels (with the position kernel sized to its tile)
// about 15.3 us at every size from 2K slots up, so packed layouts switch at
// 1.5K slots.  Padded layouts stay on one CTA up to 8K: its helper CTAs
// spread the padding fill (decode shape: 12.5 us, tiled 21.5 us).
#ifndef EP_LAYOUT_SMALL_MAX_SLOTS
#define EP_LAYOUT_SMALL_MAX_SLOTS 1536
#endif
// Layout: the tiled kernels run about 2 tile slots per thread (rounded to
// whole warps, 256..EP_LAYOUT_TILE_MAX_THREADS).  Measured on B200 for the
// position kernel: 256 / 512 / 1024 threads gave 17.4 / 15.3 / 17.4 us at the
// metric shape (1024-slot tiles) and 21.5 / 21.5 / 19.4 us at large-skewed
// (2048-slot tiles); the count kernel at 1024 threads took large-skewed from
// 19.5 to 19.0 us and left the others unchanged.
#ifndef EP_LAYOUT_TILE_MAX_THREADS
#define EP_LAYOUT_TILE_MAX_THREADS 1024
#endif
#ifndef EP_LAYOUT_TILE_TOKENS     // layout: tokens per tile of the tiled path (doubled for large T)
#define EP_LAYOUT_TILE_TOKENS 128
#endif
#ifndef EP_LAYOUT_SMALL_MAX_SLOTS_PADDED
#define EP_LAYOUT_SMALL_MAX_SLOTS_PADDED 8192
#endif
#ifndef EP_LAYOUT_POS_EARLY_TRIGGER  // layout position kernel lets its dependents launch at its start
#define EP_LAYOUT_POS_EARLY_TRIGGER 0
#endif
#ifndef EP_LAYOUT_COUNT_EARLY_TRIGGER  // layout count kernel lets the position kernel launch at its start
#define EP_LAYOUT_COUNT_EARLY_TRIGGER 1
#endif
#ifndef EP_DISPATCH_EARLY_TRIGGER    // dispatch kernels let their dependents launch at their start
#define EP_DISPATCH_EARLY_TRIGGER 1
#endif
#if EP_COMBINE_POS_BEFORE_WAIT && EP_LAYOUT_POS_EARLY_TRIGGER
#error "the combine reads positions before its wait: the position kernel must signal at its exit"
#endif
#ifndef EP_FILL_EARLY_START          // fill pass from an input table starts before the copy kernel completes
#define EP_FILL_EARLY_START 1
#endif
#ifndef EP_USE_PDL                // launch kernels with programmatic dependent launch
#define EP_USE_PDL 1
#endif

namespace ep {

// Programmatic dependent launch (sm_90+).  Every kernel of the library is
// launched with programmatic stream serialisation, so the GPU may schedule it
// while the previous kernel in the stream is still finishing; the first thing
// each kernel does is pdl_wait(), which returns once the previous grid has
// completed and its memory is visible, so no input is read early.  It then
// lets its own dependents be scheduled.  The saving is the launch latency
// between back-to-back kernels.
// Wait only: the kernel's dependents launch when it exits (for kernels whose
// dependents can do nothing before it completes and whose early-launched
// blocks would only take resources from it).
__device__ __forceinline__ void pdl_wait() {
#if EP_USE_PDL
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}

__device__ __forceinline__ void pdl_trigger() {
#if EP_USE_PDL
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

__device__ __forceinline__ void pdl_wait_then_trigger() {
#if EP_USE_PDL
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

template <typename... Params, typename... Args>
cudaError_t launch_kernel(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = EP_USE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Bits of the handle's device error word.
constexpr uint32_t kErrBadExpertId = 1u;
constexpr uint32_t kErrCapacity = 2u;
constexpr uint32_t kErrTimeout = 4u;  // reserved: no kernel waits on another today

constexpr int kMaxTopk = 32;
constexpr int kMaxExperts = 4096;
constexpr int kMaxHidden = 1 << 24;  // channel offsets and per-row loops stay far inside int


}  // namespace ep

// The opaque handle of the ABI.  Host struct; the arrays are device memory
// carved out of one stream-ordered allocation.
struct ep_handle {
    int T, k, E, R, align, capacity, experts_per_rank;
    int tile_tokens, ntiles;
    int layout_kernels;      // kernels the layout launched (1 or 2)
    int layout_path;         // kLayoutPath*
    int64_t n_rows;          // receive rows the layout may use (ep_max_recv_rows)
    int device;
    cudaStream_t stream;     // the stream the handle was created (and is freed) on
    void *block;             // the allocation
    int32_t *pos;            // [T*k]
    int32_t *src_idx;        // [n_rows]
    int32_t *seg;            // [E+1]
    int32_t *rank_off;       // [R+1]
    int32_t *cnt;            // [E]
    int32_t *tile_cnt;       // [ntiles*E]  per-tile expert counts (scratch)
    int32_t *tile_rank;      // [ntiles*R]  per-tile token-in-rank counts (scratch)
    uint32_t *tile_err;      // [ntiles]    per-tile bad-id flags (scratch)
    uint32_t *err;           // [1] device error word
};

// The opaque multi-rank plan of the ABI: where every local slot goes on
// which rank, and this rank's receive segments.  Host struct; the arrays are
// device memory carved out of one stream-ordered allocation.
struct ep_plan {
    int T, k, E, world, rank, epr, align, capacity;
    int64_t recv_rows;       // rows of every rank's receive buffer
    int device;
    cudaStream_t stream;
    void *block;
    int2 *dst;               // [T*k] (owner rank, row in its receive buffer), (-1, -1) if none
    int32_t *pre;            // [E] slots of lower source ranks per expert (scratch)
    int32_t *offs;           // [E] row of this rank's first slot of each expert (scratch)
    int32_t *recv_seg;       // [epr+1] segment starts of this rank's experts in its receive buffer
    int32_t *recv_cnt;       // [epr] slots routed to each of this rank's experts (all sources)
    uint32_t *err;           // [1] device error word
};

namespace ep {

__host__ __device__ constexpr int align4(int n) { return (n + 3) & ~3; }

// Tile geometry of the layout.  Tiles of 128 tokens (doubled until the
// [tiles x (E + R)] count matrices fit the position kernel's shared memory);
// count-kernel rank-bitmask sub-blocks of at most 12288 words; position-kernel
// warps whose per-warp count rows fit 12288 words; the tile's ids staged in
// shared memory when they fit.
constexpr int kLayoutMatWords = 24576;
struct LayoutGeometry {
    int tile_tokens, ntiles, sub_tokens, pos_warps, tile_threads;
    bool ids_in_smem;  // the position kernel stages the tile's ids in shared memory
    bool small;        // the whole layout fits one CTA (layout_small_kernel)
};
// Shared-memory words of the one-CTA layout (32 warps).
inline int layout_small_smem_words(int T, int k, int E, int R) {
    return align4(T * k) + align4(E) + align4(E + 1) + align4(R) + 32 * (E + 1) + T * ((R + 31) / 32);
}
// Shared-memory words of the position kernel.
inline int layout_pos_smem_words(int ntiles, int E, int R, int pos_warps, int id_words) {
    return align4(ntiles * E) + align4(ntiles * R) + 2 * align4(E) + align4(E + 1) +
           align4(pos_warps * E) + id_words;
}
inline LayoutGeometry layout_geometry(int T, int k, int E, int R, int capacity) {
    LayoutGeometry g;
    g.tile_tokens = EP_LAYOUT_TILE_TOKENS;
    // 64-bit tile counts: T + tile_tokens - 1 overflows int for T near 2^31.
    while (((int64_t)T + g.tile_tokens - 1) / g.tile_tokens * (E + R) > kLayoutMatWords &&
           g.tile_tokens < (1 << 29))
        g.tile_tokens *= 2;
    g.ntiles = (int)(((int64_t)T + g.tile_tokens - 1) / g.tile_tokens);
    const int rw = (R + 31) / 32;
    g.sub_tokens = 12288 / rw < g.tile_tokens ? 12288 / rw : g.tile_tokens;
    int64_t pt = ((int64_t)g.tile_tokens * k / 2 + 31) / 32 * 32;
    g.tile_threads = (int)(pt < 256 ? 256 : pt > EP_LAYOUT_TILE_MAX_THREADS ? EP_LAYOUT_TILE_MAX_THREADS : pt);
    const int pos_warps = g.tile_threads / 32;
    g.pos_warps = 12288 / E >= pos_warps ? pos_warps : (12288 / E > 0 ? 12288 / E : 1);
    const int64_t id_words = (int64_t)g.tile_tokens * k;
    // (the position kernel keeps the slots' in-tile ranks beside the ids: twice the words)
    g.ids_in_smem = id_words <= 8192 &&
                    layout_pos_smem_words(g.ntiles, E, R, g.pos_warps, 2 * (int)id_words) <= 50000;
    const int64_t small_max = capacity > 0 ? EP_LAYOUT_SMALL_MAX_SLOTS_PADDED : EP_LAYOUT_SMALL_MAX_SLOTS;
    g.small = T > 0 && (int64_t)T * k <= small_max && E <= 512 &&
              layout_small_smem_words(T, k, E, R) <= 40000;
    return g;
}

struct LayoutArgs {
    const int32_t *topk_idx;
    int T, k, E, R, epr, align, capacity;
    int tile_tokens, ntiles, sub_tokens, pos_warps, tile_threads;
    bool ids_in_smem, small;
    // The position kernel ranks its slots inside the tile before waiting for
    // the count kernel (with the ids in shared memory).  Only when the two
    // kernels' CTAs need not share SMs (2 x tiles <= SMs): sharing, the extra
    // early work slows the count kernel more than it saves (measured).
    bool rank_early;
    int64_t n_rows;
    int32_t *pos, *src_idx, *seg, *rank_off, *cnt, *tile_cnt, *tile_rank;
    uint32_t *tile_err, *err;
    int32_t *out_cnt, *out_rank_tok;
    uint8_t *out_in_rank;
};

// Layout paths, as ep_handle_info reports them.
constexpr int kLayoutPathEmpty = 0;
constexpr int kLayoutPathOneCta = 1;
constexpr int kLayoutPathTiled = 2;  // layout_count_kernel + layout_pos_kernel

constexpr int kDispatchCopyBf16 = 0;  // bf16 in, bf16 rows out
constexpr int kDispatchQuantFp8 = 1;  // bf16 in, e4m3 rows + scales out (quantised here)
constexpr int kDispatchCopyFp8 = 2;   // e4m3 + scales in (already quantised), copied out

struct DispatchArgs {
    const uint8_t *x;        // bf16 [T, H], or e4m3 [T, H] for kDispatchCopyFp8
    const float *x_scales;   // [T, H/128] row-major, kDispatchCopyFp8 only
    const int32_t *pos;      // [T, k]
    uint8_t *recv;           // [rows, H] bf16 or e4m3
    float *scales;           // element (p, g) at p * s_row + g * s_grp (FP8 only)
    int64_t s_row, s_grp;
    int mode;                // kDispatch*
    int num_sms;             // 0: one block per unit; else grid capped to num_sms SMs' worth
    int T, k, H;
    int chunk;               // channels per work unit
    int nchunks;             // units per token
    int nunits;              // T * nchunks (< 2^31, checked on the host)
    // Multi-rank (peer) addressing, used instead of pos / recv / scales:
    const int2 *dst;                 // [T, k] (rank, row) of each slot, rank -1 if none
    uint8_t *const *peer_recv;       // [world] device pointers to every rank's receive buffer
    float *const *peer_scales;       // [world] ... scale buffers (FP8), or nullptr
    // Per-token scale table [T, H/128] row-major, written by the quantising
    // kernel when not null (kDispatchQuantFp8; local addressing only).  With
    // scales == nullptr no receive row gets a scale: a fill pass
    // (launch_scale_fill) writes them from the table afterwards.
    float *tok_scales;
};

// Column-order fill of column-major FP8 scales from a per-token table:
// scales[g * ld + p] = table[src_idx[p] * G + g] for every receive row p with
// src_idx[p] >= 0 (padding rows are not written).  Launched right after a
// dispatch kernel of the same handle: it reads src_idx before waiting for
// that kernel (the layout that wrote src_idx completed before it).
struct ScaleFillArgs {
    const int32_t *src_idx;  // [n_rows] (handle)
    const float *table;      // [T, G] row-major per-token scales
    float *scales;           // column-major: element (p, g) at g * ld + p
    int64_t ld;              // >= n_rows
    int64_t n_rows;
    int G;                   // H / 128
    int num_sms;             // 0: one block per tile; else grid capped
    bool vec_in;             // table rows read as 16-byte vectors (G % 4 == 0, table 16-byte aligned)
    // The table is the caller's input (pre-quantised scales), written before
    // the copy kernel this pass follows began, which writes no scale: the
    // pass starts without waiting for it, and waits only before it exits, so
    // that this grid completes after the copy kernel.  Not with num_sms.
    bool table_is_input;
};

struct CombineArgs {
    const uint8_t *y;        // bf16 [rows, H]
    const float *w;          // [T, k], or nullptr for unit weights (dispatch backward)
    const int32_t *pos;      // [T, k]
    uint8_t *out;            // bf16 [T, H]
    int T, k, H;
    int nvec;                // H / 8 (16-byte vectors per row)
    int vpt;                 // vectors per thread: 1, 2 or 4
    int blocks_per_token;    // ceil(nvec / (128 * vpt))
    int num_sms;             // 0: one block per (token, vector block); else grid capped
    bool pos_early;          // small grid: read the positions before the programmatic wait
    // Multi-rank (peer) addressing, used instead of pos / y:
    const int2 *src;                 // [T, k] (rank, row) of each slot's expert output, rank -1 if none
    const uint8_t *const *peer_y;    // [world] device pointers to every rank's expert outputs
};

struct CombineBwdArgs {
    const uint8_t *grad_out; // bf16 [T, H]
    const uint8_t *y;        // bf16 [rows, H] (only read when grad_w != nullptr)
    const float *w;          // [T, k]
    const int32_t *pos;      // [T, k]
    uint8_t *grad_y;         // bf16 [rows, H]
    float *grad_w;           // [T, k] or nullptr
    int T, k, H;
    // Multi-rank (peer) addressing, used instead of pos / y / grad_y:
    const int2 *dst;                 // [T, k] (rank, row) of each slot, rank -1 if none
    const uint8_t *const *peer_y;    // [world] every rank's expert outputs
    uint8_t *const *peer_grad_y;     // [world] every rank's grad_y buffer
};

struct RecvTopkArgs {
    const int32_t *src_idx;  // [n_rows] (handle)
    const int32_t *pos;      // [T, k] (handle)
    const int32_t *seg;      // [E + 1] (handle)
    const float *w;          // [T, k] or nullptr
    int32_t *out_idx;        // [n_rows] or nullptr
    float *out_w;            // [n_rows] or nullptr
    int32_t *out_slot;       // [n_rows] or nullptr
    int T, k, E;
    int64_t n_rows;
};

// Exclusive scan of one value per thread over the block (blockDim.x <= 1024);
// returns the exclusive prefix and writes the block total to *total.
// warp_s: 33 words of shared memory.  Every thread of the block must call it.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t *total, int32_t *warp_s) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
    int32_t incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += n;
    }
    if (lane == 31) warp_s[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int32_t w = (lane < nwarps) ? warp_s[lane] : 0;
        int32_t wi = w;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t n = __shfl_up_sync(0xffffffffu, wi, d);
            if (lane >= d) wi += n;
        }
        warp_s[lane] = wi - w;
        if (lane == 31) warp_s[32] = wi;
    }
    __syncthreads();
    const int32_t excl = warp_s[warp] + incl - v;
    *total = warp_s[32];
    __syncthreads();
    return excl;
}

struct RecvTopkPeerArgs {
    const int2 *dst;           // [T, k] plan: (owner rank, row) of each local slot
    const int32_t *topk_idx;   // [T, k]
    const float *w;            // [T, k] or nullptr
    int T, k, rank, epr, capacity;
    int32_t *const *p_idx;     // [world] per-row expert id tables, or nullptr
    float *const *p_w;         // [world] per-row weight tables, or nullptr
    int32_t *const *p_src;     // [world] per-row source rank tables, or nullptr
    int32_t *const *p_slot;    // [world] per-row source slot tables, or nullptr
    const int32_t *recv_seg;   // [epr + 1] this rank's segments (plan)
    const int32_t *recv_cnt;   // [epr] this rank's per-expert slot counts (plan)
};

struct PlanArgs {
    const int32_t *topk_idx;   // [T, k] this rank's ids
    const int32_t *pos;        // [T, k] local layout (packed, alignment 1)
    const int32_t *seg;        // [E + 1] local layout
    const int32_t *counts;     // [world, E] every rank's per-expert slot counts
    int T, k, E, world, rank, epr, align, capacity;
    int64_t recv_rows;
    int2 *dst;
    int32_t *pre, *offs, *recv_seg, *recv_cnt;
    uint32_t *err;
};

// Work units of a dispatch: each token's H channels split into nchunks
// chunks of `chunk` channels (a multiple of align_ch: 128 for FP8 groups, 8
// for BF16 vectors), at most EP_DISPATCH_MAX_CHUNK each.  A small batch is
// split further, down to EP_DISPATCH_MIN_CHUNK channels, until T * nchunks
// reaches EP_DISPATCH_MIN_UNITS_PER_SM blocks per SM.
inline void dispatch_chunking(int T, int H, int align_ch, int num_sms, int *chunk, int *nchunks) {
    int n = (H + EP_DISPATCH_MAX_CHUNK - 1) / EP_DISPATCH_MAX_CHUNK;
    const long long want_units = (long long)EP_DISPATCH_MIN_UNITS_PER_SM * num_sms;
    if (T > 0 && (long long)T * n < want_units) {
        const int min_chunk = EP_DISPATCH_MIN_CHUNK > align_ch ? EP_DISPATCH_MIN_CHUNK : align_ch;
        int max_n = H / min_chunk;
        if (max_n < 1) max_n = 1;
        long long want = (want_units + T - 1) / T;
        if (want > max_n) want = max_n;
        if (want > n) n = (int)want;
    }
    int c = (H + n - 1) / n;
    c = (c + align_ch - 1) / align_ch * align_ch;
    *chunk = c;
    *nchunks = (H + c - 1) / c;
}

// Launchers (return the cudaGetLastError() of the launch).
cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s);
size_t layout_count_smem(const LayoutArgs &a);
size_t layout_small_smem(const LayoutArgs &a);
size_t layout_pos_smem(const LayoutArgs &a);
cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s);
cudaError_t launch_scale_fill(const ScaleFillArgs &a, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s);
cudaError_t launch_combine_backward(const CombineBwdArgs &a, cudaStream_t s);
cudaError_t launch_recv_topk(const RecvTopkArgs &a, cudaStream_t s);
cudaError_t launch_e4m3_encode(const float *x, uint8_t *out, int64_t n, cudaStream_t s);
cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s);
cudaError_t launch_recv_topk_peer(const RecvTopkPeerArgs &a, cudaStream_t s);
// Peer-addressed variants of dispatch and combine (DispatchArgs::dst, CombineArgs::src).
cudaError_t launch_dispatch_peer(const DispatchArgs &a, cudaStream_t s);
cudaError_t launch_combine_peer(const CombineArgs &a, cudaStream_t s);
cudaError_t launch_combine_backward_peer(const CombineBwdArgs &a, cudaStream_t s);

// Per-device facts, cached.
struct DeviceInfo {
    int num_sms;
    int cc_major, cc_minor;
    int max_smem_optin;
};
cudaError_t device_info(int device, DeviceInfo *out);

}  // namespace ep
