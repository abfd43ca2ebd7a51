// layout.cu -- routing layout: per-expert / per-rank counts, is_token_in_rank,
// expert segments and the receive row of every slot.
//
// The layout is the metadata half of the pages' dispatch ("DeepEP
// (DeepEveryParallel) Documentation", item 10; "DeepSeek publica DeepEP ...",
// news.hada.io, "Patrones de uso en entrenamiento, prefill y decoding": the
// handle carries the routing metadata and the per-expert counts).  Receive
// rows are expert-major and, inside an expert, in (source token, slot) order,
// so every position is a pure function of topk_idx.  Two kernels, no
// inter-CTA waits, no atomics whose order could leak into a position:
//
//   1. layout_count_kernel (one CTA per tile of tokens): per-tile expert
//      histogram (shared-memory integer atomics: an integer sum does not
//      depend on the order), token-in-rank flags, per-tile rank counts and a
//      per-tile bad-id flag.
//   2. layout_pos_kernel (one CTA per tile): launched while the count
//      kernel runs, it first counts its tile's slots per warp
//      (__match_any_sync + popc; the ids predate the layout), then waits for
//      the count kernel, loads the whole [tiles x E] count matrix into shared
//      memory, derives its own tile base and the global segment offsets from
//      it (every CTA does this redundantly: a few tens of KB from L2 per CTA
//      instead of a serial single-CTA scan kernel), ranks its slots in slot
//      order with a prefix over its warps, and writes pos[t][j] and
//      src_idx[row].  CTAs 0, 1 and 2 publish the segments and error word, the
//      expert counts, and the rank slices and counts; the -1 fill of padding
//      rows is spread over all CTAs.
// Both run about two tile slots per thread (256..1024 threads; the rule and
// its measurements are in ep_internal.cuh).  The position kernel lets
// dispatch launch only when it exits: early-launched dispatch blocks would
// only wait beside it and take its registers and warp slots.
// Small problems take a third kernel instead, layout_small_kernel: the whole
// layout in one CTA (plus padding-fill helpers in padded mode).
#include <atomic>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kCountThreads = EP_LAYOUT_TILE_MAX_THREADS;  // launch bound; the launch uses a.tile_threads
constexpr int kPosThreads = EP_LAYOUT_TILE_MAX_THREADS;    // launch bound; the launch uses a.tile_threads

// Copy n int32 words global -> shared (16-byte vectors when both are aligned).
__device__ __forceinline__ void load_words(int32_t *dst, const int32_t *src, int n) {
    if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
        const int n4 = n >> 2;
        const int4 *s4 = reinterpret_cast<const int4 *>(src);
        int4 *d4 = reinterpret_cast<int4 *>(dst);
        // Batches of kBatch 16-byte loads per thread are all issued before any
        // is stored, so a CTA's copy takes a few L2 round trips, not one per vector.
        constexpr int kBatch = EP_LAYOUT_LOAD_BATCH;
        const int stride = blockDim.x;
        for (int i0 = threadIdx.x; i0 < n4; i0 += kBatch * stride) {
            int4 v[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int i = i0 + b * stride;
                if (i < n4) v[b] = __ldg(s4 + i);
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int i = i0 + b * stride;
                if (i < n4) d4[i] = v[b];
            }
        }
        for (int i = (n4 << 2) + threadIdx.x; i < n; i += blockDim.x) dst[i] = __ldg(src + i);
    } else {
        for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = __ldg(src + i);
    }
}

// is_token_in_rank rows of ntok consecutive tokens (one contiguous block of
// ntok * R bytes at dst) from their rank bitmasks in shared memory (RW =
// ceil(R / 32) words per token), by the whole CTA.  16-byte stores of 16
// flags when dst and R allow (16 rank bits never straddle a mask word), else
// 4-byte stores of 4 flags, else bytes.
__device__ __forceinline__ void write_in_rank_rows(uint8_t *dst, const uint32_t *mask_s, int ntok, int R) {
    const int RW = (R + 31) >> 5;
    const uintptr_t addr = reinterpret_cast<uintptr_t>(dst);
    if ((addr & 15u) == 0 && (R & 15) == 0) {
        const int per_row = R >> 4;
        uint4 *d16 = reinterpret_cast<uint4 *>(dst);
        for (int v = threadIdx.x; v < ntok * per_row; v += blockDim.x) {
            const int tl = v / per_row;
            const int f0 = (v - tl * per_row) * 16;
            const uint32_t m = mask_s[tl * RW + (f0 >> 5)] >> (f0 & 31);
            uint32_t q[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t b = m >> (4 * j);
                q[j] = (b & 1u) | ((b & 2u) << 7) | ((b & 4u) << 14) | ((b & 8u) << 21);
            }
            d16[v] = make_uint4(q[0], q[1], q[2], q[3]);
        }
    } else if ((addr & 3u) == 0 && (R & 3) == 0) {
        const int per_row = R >> 2;
        uint32_t *d4 = reinterpret_cast<uint32_t *>(dst);
        for (int v = threadIdx.x; v < ntok * per_row; v += blockDim.x) {
            const int tl = v / per_row;
            const int f0 = (v - tl * per_row) * 4;
            const uint32_t b = mask_s[tl * RW + (f0 >> 5)] >> (f0 & 31);
            d4[v] = (b & 1u) | ((b & 2u) << 7) | ((b & 4u) << 14) | ((b & 8u) << 21);
        }
    } else {
        for (int i = threadIdx.x; i < ntok * R; i += blockDim.x) {
            const int tl = i / R;
            const int r = i - tl * R;
            dst[i] = (uint8_t)((mask_s[tl * RW + (r >> 5)] >> (r & 31)) & 1u);
        }
    }
}

// Id of slot s of the tile (-1 for unused or invalid ids), from shared memory
// when the tile's ids were staged there.
__device__ __forceinline__ int tile_id(const LayoutArgs &a, const int32_t *ids_s, int64_t s0, int s) {
    int e = a.ids_in_smem ? ids_s[s] : __ldg(a.topk_idx + s0 + s);
    if (e < -1 || e >= a.E) e = -1;
    return e;
}

// ---------------------------------------------------------------------------
// 1. per-tile counts and token-in-rank flags
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kCountThreads) layout_count_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
#if EP_LAYOUT_COUNT_EARLY_TRIGGER
    pdl_wait_then_trigger();
#else
    pdl_wait();
#endif
    const int RW = (a.R + 31) >> 5;                                 // mask words per token
    int32_t *cnt_s = reinterpret_cast<int32_t *>(smem);             // [E]
    int32_t *rcnt_s = cnt_s + a.E;                                  // [R]
    uint32_t *mask_s = reinterpret_cast<uint32_t *>(rcnt_s + a.R);  // [sub_tokens][RW] rank bits
    int32_t *ids_s = reinterpret_cast<int32_t *>(mask_s) + align4(a.sub_tokens * RW);  // [tile ids]

    const int tile = blockIdx.x;
    const int t0 = tile * a.tile_tokens;
    const int nt = min(a.tile_tokens, a.T - t0);
    const int64_t s_tile = (int64_t)t0 * a.k;
    if (a.ids_in_smem) load_words(ids_s, a.topk_idx + s_tile, nt * a.k);
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) cnt_s[i] = 0;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) rcnt_s[i] = 0;
    int bad = 0;

    for (int sb = 0; sb < nt; sb += a.sub_tokens) {
        const int ns = min(a.sub_tokens, nt - sb);
        for (int i = threadIdx.x; i < ns * RW; i += blockDim.x) mask_s[i] = 0u;
        __syncthreads();

        const int sub0 = sb * a.k;  // first slot of the sub-block inside the tile
        const int nslots = ns * a.k;
        for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
            int e = a.ids_in_smem ? ids_s[sub0 + s] : __ldg(a.topk_idx + s_tile + sub0 + s);
            if (e < -1 || e >= a.E) e = -2;  // invalid id: counted as unused, flagged
            if (e < 0) {
                bad |= (e == -2);
                continue;
            }
            atomicAdd(&cnt_s[e], 1);
            const int r = e / a.epr;
            const uint32_t bit = 1u << (r & 31);
            // The slot that sets the token's bit for rank r counts the token.
            if (!(atomicOr(&mask_s[(s / a.k) * RW + (r >> 5)], bit) & bit)) atomicAdd(&rcnt_s[r], 1);
        }
        __syncthreads();

        if (a.out_in_rank != nullptr)
            write_in_rank_rows(a.out_in_rank + (int64_t)(t0 + sb) * a.R, mask_s, ns, a.R);
        __syncthreads();
    }

    bad = __syncthreads_or(bad);
    int32_t *tc = a.tile_cnt + (int64_t)tile * a.E;
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) tc[i] = cnt_s[i];
    int32_t *tr = a.tile_rank + (int64_t)tile * a.R;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) tr[i] = rcnt_s[i];
    if (threadIdx.x == 0) a.tile_err[tile] = bad ? kErrBadExpertId : 0u;
}

// ---------------------------------------------------------------------------
// 2. segments and positions
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPosThreads) layout_pos_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int E = a.E, R = a.R, W = a.pos_warps, NT = a.ntiles;
    int32_t *mat = reinterpret_cast<int32_t *>(smem);   // [NT][E] tile counts
    int32_t *rmat = mat + align4(NT * E);                // [NT][R] tile rank counts (CTA 0)
    int32_t *base_s = rmat + align4(NT * R);             // [E] rows of expert e before this tile
    int32_t *cnt_s = base_s + align4(E);                 // [E] expert totals
    int32_t *seg_s = cnt_s + align4(E);                  // [E+1] segment starts
    int32_t *wcnt = seg_s + align4(E + 1);               // [W][E]
    int32_t *ids_s = wcnt + align4(W * E);               // [tile_tokens * k] when a.ids_in_smem
    int32_t *rloc_s = ids_s + (a.ids_in_smem ? a.tile_tokens * a.k : 0);
                                                         // [tile_tokens * k] in-tile ranks (with ids_s)
    __shared__ int32_t warp_s[33];

    const int tile = blockIdx.x;
    const int t0 = tile * a.tile_tokens;
    const int nt = min(a.tile_tokens, a.T - t0);
    const int nslots = nt * a.k;
    const int64_t s0 = (int64_t)t0 * a.k;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    // The publishing is spread over up to three CTAs: CTA 0 the segments and
    // the error word, cnt_cta the expert counts, rank_cta the rank slices and
    // counts (it alone loads the tile rank counts).
    const int cnt_cta = NT > 1 ? 1 : 0;
    const int rank_cta = NT > 2 ? 2 : NT - 1;

    // Before waiting for the count kernel: the tile's ids and their per-warp
    // counts.  The ids were written before the layout began -- this kernel is
    // launched only when every count CTA has passed its own wait, so every
    // kernel that wrote them has completed -- and pass A touches shared memory
    // only, so it runs while the count kernel is still working.
    if (a.ids_in_smem) load_words(ids_s, a.topk_idx + s0, nslots);
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    // A: per-expert slot counts of each warp's contiguous range of the tile's slots.
    const int lo = (int)((int64_t)warp * nslots / W);
    const int hi = (int)((int64_t)(warp + 1) * nslots / W);
    const unsigned lt_mask = (1u << lane) - 1u;
    int32_t *my = wcnt + warp * E;
    if (warp < W) {
        for (int b = lo; b < hi; b += 32) {
            const int s = b + lane;
            const int e = (s < hi) ? tile_id(a, ids_s, s0, s) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
            __syncwarp();
        }
    }
    const bool rank_early = a.ids_in_smem && a.rank_early;
    if (rank_early) {
        // Still before the wait: each slot's rank among the tile's slots of
        // its expert (prefix over the warps, then the rank inside the warp),
        // so that after the wait only the tile base and the segment start
        // are left to add.
        __syncthreads();
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int32_t run = 0;
            for (int w = 0; w < W; ++w) {
                const int32_t v = wcnt[w * E + e];
                wcnt[w * E + e] = run;
                run += v;
            }
        }
        __syncthreads();
        if (warp < W) {
            for (int b = lo; b < hi; b += 32) {
                const int s = b + lane;
                const int e = (s < hi) ? tile_id(a, ids_s, s0, s) : -1;
                const unsigned peers = __match_any_sync(0xffffffffu, e);
                if (e >= 0) rloc_s[s] = my[e] + __popc(peers & lt_mask);
                __syncwarp();
                if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
                __syncwarp();
            }
        }
    }

#if EP_LAYOUT_POS_EARLY_TRIGGER
    pdl_wait_then_trigger();
#else
    pdl_wait();
#endif
    load_words(mat, a.tile_cnt, NT * E);
    if (tile == rank_cta && a.out_rank_tok != nullptr) load_words(rmat, a.tile_rank, NT * R);
    // CTA 0 also reads every tile's bad-id flag here, so the round trip
    // overlaps the matrix load instead of delaying its publish step.
    uint32_t tile_bad = 0u;
    if (tile == 0)
        for (int t = threadIdx.x; t < NT; t += blockDim.x) tile_bad |= __ldg(a.tile_err + t);
    __syncthreads();

    // Tile base and total of every expert.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t pre = 0, tot = 0;
        for (int t = 0; t < NT; ++t) {
            const int32_t v = mat[t * E + e];
            pre += (t < tile) ? v : 0;
            tot += v;
        }
        base_s[e] = pre;
        cnt_s[e] = tot;
    }
    __syncthreads();

    // Segment starts: exclusive scan of the segment sizes over experts.
    int32_t carry = 0;
    bool over = false;
    for (int base = 0; base < E; base += blockDim.x) {
        const int e = base + threadIdx.x;
        int32_t sz = 0;
        if (e < E) {
            const int32_t c = cnt_s[e];
            if (a.capacity > 0) {
                sz = a.capacity;
                over |= c > a.capacity;
            } else {
                sz = (c + a.align - 1) / a.align * a.align;
            }
        }
        int32_t total;
        const int32_t excl = block_exclusive_scan(sz, &total, warp_s);
        if (e < E) seg_s[e] = carry + excl;
        carry += total;
    }
    if (threadIdx.x == 0) seg_s[E] = carry;
    over = __syncthreads_or(over);

    if (tile == 0) {
        for (int e = threadIdx.x; e <= E; e += blockDim.x) a.seg[e] = seg_s[e];
        const uint32_t bad = __syncthreads_or(tile_bad != 0u) ? kErrBadExpertId : 0u;
        // The layout (re)initialises the handle's error word.
        if (threadIdx.x == 0) *a.err = bad | (over ? kErrCapacity : 0u);
    }
    if (tile == cnt_cta) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            a.cnt[e] = cnt_s[e];
            if (a.out_cnt != nullptr) a.out_cnt[e] = cnt_s[e];
        }
    }
    if (tile == rank_cta) {
        for (int r = threadIdx.x; r <= R; r += blockDim.x) a.rank_off[r] = seg_s[r * a.epr];
        if (a.out_rank_tok != nullptr) {
            for (int r = threadIdx.x; r < R; r += blockDim.x) {
                int32_t sum = 0;
                for (int t = 0; t < NT; ++t) sum += rmat[t * R + r];
                a.out_rank_tok[r] = sum;
            }
        }
    }

    // Padding rows get src_idx = -1: each CTA takes the experts e with
    // e % ntiles == tile and a share of the rows past the last segment.
    for (int e = tile + NT * warp; e < E; e += NT * nwarps) {
        int32_t used = cnt_s[e];
        if (a.capacity > 0) used = min(used, a.capacity);
        for (int64_t row = (int64_t)seg_s[e] + used + lane; row < seg_s[e + 1]; row += 32)
            a.src_idx[row] = -1;
    }
    for (int64_t row = (int64_t)seg_s[E] + (int64_t)tile * blockDim.x + threadIdx.x; row < a.n_rows;
         row += (int64_t)NT * blockDim.x)
        a.src_idx[row] = -1;

    if (rank_early) {
        // position = segment start + tile base + in-tile rank, slot by slot.
        for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
            const int e = tile_id(a, ids_s, s0, s);
            int32_t p = -1;
            if (e >= 0) {
                const int32_t rel = base_s[e] + rloc_s[s];
                if (a.capacity == 0 || rel < a.capacity) {
                    p = seg_s[e] + rel;
                    a.src_idx[p] = t0 + s / a.k;
                }
            }
            a.pos[s0 + s] = p;
        }
        return;
    }

    // B: exclusive prefix over the warps, starting from the tile base.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = base_s[e];
        for (int w = 0; w < W; ++w) {
            const int32_t v = wcnt[w * E + e];
            wcnt[w * E + e] = run;
            run += v;
        }
    }
    __syncthreads();

    // C: rank inside the expert in slot order; position = segment start + rank.
    if (warp < W) {
        for (int b = lo; b < hi; b += 32) {
            const int s = b + lane;
            const int e = (s < hi) ? tile_id(a, ids_s, s0, s) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            int32_t rel = 0;
            if (e >= 0) rel = my[e] + __popc(peers & lt_mask);
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
            __syncwarp();
            if (s < hi) {
                int32_t p = -1;
                if (e >= 0 && (a.capacity == 0 || rel < a.capacity)) {
                    p = seg_s[e] + rel;
                    a.src_idx[p] = t0 + s / a.k;
                }
                a.pos[s0 + s] = p;
            }
        }
    }
}

// dst[0, n) = -1 by the calling CTA, 16-byte stores where aligned.
__device__ __forceinline__ void fill_minus_one(int32_t *dst, int64_t n) {
    int64_t head = (int64_t)((16 - (reinterpret_cast<uintptr_t>(dst) & 15u)) & 15u) / 4;
    if (head > n) head = n;
    for (int64_t i = threadIdx.x; i < head; i += blockDim.x) dst[i] = -1;
    const int64_t n4 = (n - head) >> 2;
    int4 *d4 = reinterpret_cast<int4 *>(dst + head);
    for (int64_t i = threadIdx.x; i < n4; i += blockDim.x) d4[i] = make_int4(-1, -1, -1, -1);
    for (int64_t i = head + (n4 << 2) + threadIdx.x; i < n; i += blockDim.x) dst[i] = -1;
}

// ---------------------------------------------------------------------------
// Small problems: the whole layout in one CTA of 1024 threads
// ---------------------------------------------------------------------------
// With at most 1536 slots (8192 in padded mode; the thresholds and their
// measurements are in ep_internal.cuh), one CTA holds every id, the expert
// histogram, the per-warp counts and the rank bitmasks in shared memory, so
// counts, segments and positions need no second kernel and no count matrices
// in global memory.
// The 32 warps own contiguous slot ranges; ranks inside an expert come from
// __match_any_sync + popc plus a prefix over the warps, as in the tiled path.
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;

// Padded layouts (capacity > 0) have every padding row in a known place,
// [e*C + min(cnt[e], C), (e+1)*C), so helper CTAs fill them in parallel with
// CTA 0: each counts the ids of its share of experts and writes -1 to their
// tails.  The tails never overlap a valid row, so no ordering with CTA 0 is
// needed.
__device__ void small_fill_padding_tails(const LayoutArgs &a, int32_t *cnt_h) {
    const int nh = gridDim.x - 1;
    const int hb = blockIdx.x - 1;
    const int e0 = (int)((int64_t)hb * a.E / nh);
    const int e1 = (int)((int64_t)(hb + 1) * a.E / nh);
    for (int i = threadIdx.x; i < e1 - e0; i += blockDim.x) cnt_h[i] = 0;
    __syncthreads();
    const int nslots = a.T * a.k;
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int e = __ldg(a.topk_idx + s);
        if (e >= e0 && e < e1) atomicAdd(&cnt_h[e - e0], 1);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    for (int e = e0 + (threadIdx.x >> 5); e < e1; e += blockDim.x >> 5) {
        const int64_t start = (int64_t)e * a.capacity + min(cnt_h[e - e0], a.capacity);
        const int64_t end = (int64_t)(e + 1) * a.capacity;
        for (int64_t row = start + lane; row < end; row += 32) a.src_idx[row] = -1;
    }
}

// Kernels that write positions let their dependents launch only at their
// exit when the combine reads positions before its own wait.
__device__ __forceinline__ void layout_writer_wait() {
#if EP_COMBINE_POS_BEFORE_WAIT
    pdl_wait();
#else
    pdl_wait_then_trigger();
#endif
}

__global__ void __launch_bounds__(kSmallThreads) layout_small_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    layout_writer_wait();
    if (blockIdx.x > 0) {  // padding helper (padded mode only)
        small_fill_padding_tails(a, reinterpret_cast<int32_t *>(smem));
        return;
    }
    const int E = a.E, R = a.R;
    const int RW = (R + 31) >> 5;
    const int nslots = a.T * a.k;
    int32_t *ids_s = reinterpret_cast<int32_t *>(smem);      // [nslots]
    int32_t *cnt_s = ids_s + align4(nslots);                   // [E]
    int32_t *seg_s = cnt_s + align4(E);                        // [E+1]
    int32_t *rcnt_s = seg_s + align4(E + 1);                   // [R]
    // Per-warp counts, rows padded to an odd stride (E + 1 words) so that the
    // warp-parallel prefix below (lane = warp index) hits 32 different banks.
    const int ldw = E + 1;
    int32_t *wcnt = rcnt_s + align4(R);                        // [32][E + 1]
    uint32_t *mask_s = reinterpret_cast<uint32_t *>(wcnt + kSmallWarps * ldw);  // [T][RW]
    __shared__ int32_t warp_s[33];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    load_words(ids_s, a.topk_idx, nslots);
    for (int i = threadIdx.x; i < R; i += blockDim.x) rcnt_s[i] = 0;
    for (int i = threadIdx.x; i < kSmallWarps * ldw; i += blockDim.x) wcnt[i] = 0;
    for (int i = threadIdx.x; i < a.T * RW; i += blockDim.x) mask_s[i] = 0u;
    __syncthreads();

    // One pass over the slots: warp w owns the contiguous range [lo, hi) and
    // counts it per expert with __match_any_sync (leader lane adds popc);
    // every valid slot also sets its token's rank bit (the slot that sets it
    // counts the token for that rank).
    const int lo = (int)((int64_t)warp * nslots / kSmallWarps);
    const int hi = (int)((int64_t)(warp + 1) * nslots / kSmallWarps);
    int32_t *my = wcnt + warp * ldw;
    int bad = 0;
    for (int b = lo; b < hi; b += 32) {
        const int sidx = b + lane;
        int e = -1;
        if (sidx < hi) {
            e = ids_s[sidx];
            if (e < -1 || e >= E) {
                bad = 1;
                e = -1;
                ids_s[sidx] = -1;  // treated as unused from here on
            }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) {
            if (lane == __ffs(peers) - 1) my[e] += __popc(peers);
            const int r = e / a.epr;
            const uint32_t bit = 1u << (r & 31);
            if (!(atomicOr(&mask_s[(sidx / a.k) * RW + (r >> 5)], bit) & bit)) atomicAdd(&rcnt_s[r], 1);
        }
        __syncwarp();
    }
    bad = __syncthreads_or(bad);

    // Exclusive prefix over the 32 warps of every expert (one warp per expert,
    // lane = warp index) and the expert totals.
    for (int e = warp; e < E; e += kSmallWarps) {
        const int32_t v = wcnt[lane * ldw + e];
        int32_t incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t n = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += n;
        }
        wcnt[lane * ldw + e] = incl - v;
        if (lane == 31) cnt_s[e] = incl;
    }
    __syncthreads();

    // Segments.
    int32_t carry = 0;
    bool over = false;
    for (int base = 0; base < E; base += blockDim.x) {
        const int e = base + threadIdx.x;
        int32_t sz = 0;
        if (e < E) {
            const int32_t c = cnt_s[e];
            if (a.capacity > 0) {
                sz = a.capacity;
                over |= c > a.capacity;
            } else {
                sz = (c + a.align - 1) / a.align * a.align;
            }
        }
        int32_t total;
        const int32_t excl = block_exclusive_scan(sz, &total, warp_s);
        if (e < E) seg_s[e] = carry + excl;
        carry += total;
    }
    if (threadIdx.x == 0) seg_s[E] = carry;
    over = __syncthreads_or(over);

    // Publish counts, segments, rank slices and counts, the error word, the
    // token-in-rank rows; every row of src_idx starts as padding (-1).
    for (int e = threadIdx.x; e <= E; e += blockDim.x) a.seg[e] = seg_s[e];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        a.cnt[e] = cnt_s[e];
        if (a.out_cnt != nullptr) a.out_cnt[e] = cnt_s[e];
    }
    for (int r = threadIdx.x; r <= R; r += blockDim.x) a.rank_off[r] = seg_s[r * a.epr];
    if (a.out_rank_tok != nullptr)
        for (int r = threadIdx.x; r < R; r += blockDim.x) a.out_rank_tok[r] = rcnt_s[r];
    if (threadIdx.x == 0) *a.err = (bad ? kErrBadExpertId : 0u) | (over ? kErrCapacity : 0u);
    if (a.out_in_rank != nullptr) write_in_rank_rows(a.out_in_rank, mask_s, a.T, R);
    if (gridDim.x == 1) {
        // Packed mode: every row starts as padding (-1); the barrier orders
        // the fill before the valid rows are written over it below.
        fill_minus_one(a.src_idx, a.n_rows);
        __syncthreads();
    }

    // Positions: rank inside the expert in slot order.
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int b = lo; b < hi; b += 32) {
        const int sidx = b + lane;
        const int e = (sidx < hi) ? ids_s[sidx] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        int32_t rel = 0;
        if (e >= 0) rel = my[e] + __popc(peers & lt_mask);
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
        __syncwarp();
        if (sidx < hi) {
            int32_t p = -1;
            if (e >= 0 && (a.capacity == 0 || rel < a.capacity)) {
                p = seg_s[e] + rel;
                a.src_idx[p] = sidx / a.k;
            }
            a.pos[sidx] = p;
        }
    }
}

// T == 0: no tiles; one CTA writes the (empty or padded) segments, zero
// counts, -1 over every row and a clear error word.
__global__ void __launch_bounds__(kPosThreads) layout_empty_kernel(LayoutArgs a) {
    layout_writer_wait();
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x)
        a.seg[e] = a.capacity > 0 ? e * a.capacity : 0;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        a.cnt[e] = 0;
        if (a.out_cnt != nullptr) a.out_cnt[e] = 0;
    }
    for (int r = threadIdx.x; r <= a.R; r += blockDim.x)
        a.rank_off[r] = a.capacity > 0 ? r * a.epr * a.capacity : 0;
    if (a.out_rank_tok != nullptr)
        for (int r = threadIdx.x; r < a.R; r += blockDim.x) a.out_rank_tok[r] = 0;
    for (int64_t row = threadIdx.x; row < a.n_rows; row += blockDim.x) a.src_idx[row] = -1;
    if (threadIdx.x == 0) *a.err = 0u;
}

}  // namespace

size_t layout_small_smem(const LayoutArgs &a) {
    return (size_t)layout_small_smem_words(a.T, a.k, a.E, a.R) * 4;
}

size_t layout_count_smem(const LayoutArgs &a) {
    return (size_t)(a.E + a.R + align4(a.sub_tokens * ((a.R + 31) / 32)) +
                    (a.ids_in_smem ? a.tile_tokens * a.k : 0)) * 4;
}

size_t layout_pos_smem(const LayoutArgs &a) {
    // with the ids in shared memory, their in-tile ranks beside them
    return (size_t)layout_pos_smem_words(a.ntiles, a.E, a.R, a.pos_warps,
                                         a.ids_in_smem ? 2 * a.tile_tokens * a.k : 0) * 4;
}

// Raise a kernel's dynamic shared-memory limit when a launch needs more than
// the default (48 KiB including static shared memory; 32 KiB leaves room).
// Cached per device: the attribute is set once per size increase.
template <typename Kernel>
cudaError_t ensure_dyn_smem(Kernel kernel, size_t bytes, std::atomic<int> *cache) {
    if (bytes <= 32 * 1024) return cudaSuccess;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (cache[dev].load(std::memory_order_relaxed) >= (int)bytes) return cudaSuccess;
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (err == cudaSuccess) cache[dev].store((int)bytes, std::memory_order_relaxed);
    return err;
}

std::atomic<int> g_smem_small[64], g_smem_count[64], g_smem_pos[64];

cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s) {
    cudaError_t err;
    if (a.ntiles == 0) return launch_kernel(layout_empty_kernel, 1, kPosThreads, 0, s, a);
    if (a.small) {
        const size_t smem = layout_small_smem(a);
        if ((err = ensure_dyn_smem(layout_small_kernel, smem, g_smem_small)) != cudaSuccess) return err;
        // Padded mode: helper CTAs fill the padding tails, ~4096 rows each.
        int helpers = 0;
        if (a.capacity > 0) {
            helpers = (int)((a.n_rows + 4095) / 4096);
            helpers = helpers < 1 ? 1 : (helpers > 64 ? 64 : helpers);
            if (helpers > a.E) helpers = a.E;
        }
        return launch_kernel(layout_small_kernel, 1 + helpers, kSmallThreads, smem, s, a);
    }
    const size_t count_smem = layout_count_smem(a);
    const size_t pos_smem = layout_pos_smem(a);
    if ((err = ensure_dyn_smem(layout_count_kernel, count_smem, g_smem_count)) != cudaSuccess) return err;
    if ((err = ensure_dyn_smem(layout_pos_kernel, pos_smem, g_smem_pos)) != cudaSuccess) return err;
    if ((err = launch_kernel(layout_count_kernel, a.ntiles, a.tile_threads, count_smem, s, a)) != cudaSuccess)
        return err;
    return launch_kernel(layout_pos_kernel, a.ntiles, a.tile_threads, pos_smem, s, a);
}

}  // namespace ep
