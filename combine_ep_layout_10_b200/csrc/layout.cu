// layout.cu -- routing layout: per-expert / per-rank counts, is_token_in_rank,
// expert segments and the receive row of every slot.
//
// The layout is the metadata half of the pages' dispatch ("DeepEP
// (DeepEveryParallel) Documentation", item 10; "DeepSeek publica DeepEP ...",
// news.hada.io, "Patrones de uso en entrenamiento, prefill y decoding": the
// handle carries the routing metadata and the per-expert counts).  Receive
// rows are expert-major and, inside an expert, in (source token, slot) order,
// so every position is a pure function of topk_idx: three kernels, no
// inter-CTA waits and no atomics whose order could leak into a position.
//
//   1. layout_count_kernel (one CTA per tile of tokens): per-tile expert
//      histogram (shared-memory integer atomics: the result of an integer
//      sum does not depend on the order), token-in-rank flags and per-tile
//      rank counts.
//   2. layout_scan_kernel (one CTA): per-expert exclusive scan over tiles,
//      expert totals, segment offsets (block-wide scan), rank slices, rank
//      counts, capacity check, -1 fill of padding rows.
//   3. layout_pos_kernel (one CTA per tile): within-tile ranks in slot order
//      with warp __match_any_sync + popc, a prefix over the CTA's warps, and
//      the tile base from step 2; writes pos[t][j] and src_idx[row].
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kCountThreads = 256;
constexpr int kScanThreads = 1024;
constexpr int kPosThreads = 256;

__device__ __forceinline__ int load_id(const LayoutArgs &a, int64_t s, bool report) {
    int e = __ldg(a.topk_idx + s);
    if (e < -1 || e >= a.E) {
        if (report) atomicOr(a.err, kErrBadExpertId);
        e = -1;
    }
    return e;
}

// ---------------------------------------------------------------------------
// 1. per-tile counts and token-in-rank flags
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kCountThreads) layout_count_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    int32_t *cnt_s = reinterpret_cast<int32_t *>(smem);           // [E]
    int32_t *rcnt_s = cnt_s + a.E;                                // [R]
    uint32_t *flag_s = reinterpret_cast<uint32_t *>(rcnt_s + a.R);  // [sub_tokens * R]

    const int tile = blockIdx.x;
    const int t0 = tile * a.tile_tokens;
    const int nt = min(a.tile_tokens, a.T - t0);
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) cnt_s[i] = 0;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) rcnt_s[i] = 0;

    for (int sb = 0; sb < nt; sb += a.sub_tokens) {
        const int ns = min(a.sub_tokens, nt - sb);
        const int nflags = ns * a.R;
        for (int i = threadIdx.x; i < nflags; i += blockDim.x) flag_s[i] = 0u;
        __syncthreads();

        const int64_t s0 = (int64_t)(t0 + sb) * a.k;
        const int nslots = ns * a.k;
        for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
            const int e = load_id(a, s0 + s, true);
            if (e < 0) continue;
            atomicAdd(&cnt_s[e], 1);
            const int r = e / a.epr;
            // Only the first slot of a token that lands on rank r counts the token.
            if (atomicExch(&flag_s[(s / a.k) * a.R + r], 1u) == 0u) atomicAdd(&rcnt_s[r], 1);
        }
        __syncthreads();

        if (a.out_in_rank != nullptr) {
            uint8_t *dst = a.out_in_rank + (int64_t)(t0 + sb) * a.R;
            if ((reinterpret_cast<uintptr_t>(dst) & 3u) == 0 && (nflags & 3) == 0) {
                uint32_t *dw = reinterpret_cast<uint32_t *>(dst);
                for (int i = threadIdx.x; i < nflags / 4; i += blockDim.x) {
                    const uint32_t *f = flag_s + 4 * i;
                    dw[i] = f[0] | (f[1] << 8) | (f[2] << 16) | (f[3] << 24);
                }
            } else {
                for (int i = threadIdx.x; i < nflags; i += blockDim.x) dst[i] = (uint8_t)flag_s[i];
            }
        }
        __syncthreads();
    }

    int32_t *tc = a.tile_cnt + (int64_t)tile * a.E;
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) tc[i] = cnt_s[i];
    int32_t *tr = a.tile_rank + (int64_t)tile * a.R;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) tr[i] = rcnt_s[i];
}

// ---------------------------------------------------------------------------
// 2. scans
// ---------------------------------------------------------------------------

// Column partial sums of mat[ntiles][C] split into P contiguous tile ranges:
// part[p*C + c] = sum of mat[tile][c] over the p-th range.
__device__ void column_partials(const int32_t *mat, int ntiles, int C, int P, int32_t *part) {
    for (int item = threadIdx.x; item < P * C; item += blockDim.x) {
        const int c = item % C;
        const int p = item / C;
        const int lo = (int)((int64_t)p * ntiles / P);
        const int hi = (int)((int64_t)(p + 1) * ntiles / P);
        int32_t s = 0;
#pragma unroll 8
        for (int t = lo; t < hi; ++t) s += mat[(int64_t)t * C + c];
        part[p * C + c] = s;
    }
}

// Exclusive scan of v over the whole block (blockDim.x == kScanThreads);
// returns the exclusive prefix of this thread's value and the block total.
__device__ int32_t block_exclusive_scan(int32_t v, int32_t *total, int32_t *warp_s) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    int32_t incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += n;
    }
    if (lane == 31) warp_s[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t w = warp_s[lane];  // kScanThreads / 32 == 32 warps
        int32_t wi = w;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t n = __shfl_up_sync(0xffffffffu, wi, d);
            if (lane >= d) wi += n;
        }
        warp_s[lane] = wi - w;      // exclusive warp offsets
        if (lane == 31) warp_s[32] = wi;
    }
    __syncthreads();
    const int32_t excl = warp_s[warp] + incl - v;
    *total = warp_s[32];
    __syncthreads();
    return excl;
}

__global__ void __launch_bounds__(kScanThreads) layout_scan_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int E = a.E, R = a.R;
    const int partE = a.scan_parts_e * E;
    const int partR = a.scan_parts_r * R;
    int32_t *part = reinterpret_cast<int32_t *>(smem);        // [max(partE, partR)]
    int32_t *cnt_s = part + max(partE, partR);                 // [E]
    int32_t *seg_s = cnt_s + E;                                // [E+1]
    __shared__ int32_t warp_s[33];

    // Expert totals and exclusive per-tile bases.
    column_partials(a.tile_cnt, a.ntiles, E, a.scan_parts_e, part);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = 0;
        for (int p = 0; p < a.scan_parts_e; ++p) {
            const int32_t v = part[p * E + e];
            part[p * E + e] = run;
            run += v;
        }
        cnt_s[e] = run;
    }
    __syncthreads();
    for (int item = threadIdx.x; item < partE; item += blockDim.x) {
        const int e = item % E;
        const int p = item / E;
        const int lo = (int)((int64_t)p * a.ntiles / a.scan_parts_e);
        const int hi = (int)((int64_t)(p + 1) * a.ntiles / a.scan_parts_e);
        int32_t run = part[item];
        for (int t = lo; t < hi; ++t) {
            int32_t *cell = a.tile_cnt + (int64_t)t * E + e;
            const int32_t v = *cell;
            *cell = run;
            run += v;
        }
    }

    // Segment offsets: exclusive scan of the segment sizes over experts.
    int32_t carry = 0;
    for (int base = 0; base < E; base += blockDim.x) {
        const int e = base + threadIdx.x;
        int32_t sz = 0;
        if (e < E) {
            const int32_t c = cnt_s[e];
            if (a.capacity > 0) {
                sz = a.capacity;
                if (c > a.capacity) atomicOr(a.err, kErrCapacity);
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
    __syncthreads();

    for (int e = threadIdx.x; e <= E; e += blockDim.x) a.seg[e] = seg_s[e];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        a.cnt[e] = cnt_s[e];
        if (a.out_cnt != nullptr) a.out_cnt[e] = cnt_s[e];
    }
    for (int r = threadIdx.x; r <= R; r += blockDim.x) a.rank_off[r] = seg_s[r * a.epr];
    __syncthreads();  // part[] is reused below

    // Rank token counts.
    column_partials(a.tile_rank, a.ntiles, R, a.scan_parts_r, part);
    __syncthreads();
    if (a.out_rank_tok != nullptr) {
        for (int r = threadIdx.x; r < R; r += blockDim.x) {
            int32_t s = 0;
            for (int p = 0; p < a.scan_parts_r; ++p) s += part[p * R + r];
            a.out_rank_tok[r] = s;
        }
    }

    // Padding rows get src_idx = -1: the tail of every segment past its
    // (capacity-clamped) count, and the rows past the last segment.
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    for (int e = warp; e < E; e += nwarps) {
        int32_t used = cnt_s[e];
        if (a.capacity > 0) used = min(used, a.capacity);
        for (int64_t row = (int64_t)seg_s[e] + used + lane; row < seg_s[e + 1]; row += 32)
            a.src_idx[row] = -1;
    }
    for (int64_t row = (int64_t)seg_s[E] + threadIdx.x; row < a.n_rows; row += blockDim.x)
        a.src_idx[row] = -1;
}

// ---------------------------------------------------------------------------
// 3. positions
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPosThreads) layout_pos_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int E = a.E;
    const int W = a.pos_warps;
    int32_t *base_s = reinterpret_cast<int32_t *>(smem);  // [E] tile base inside each expert
    int32_t *seg_s = base_s + E;                          // [E]
    int32_t *wcnt = seg_s + E;                            // [W][E]

    const int tile = blockIdx.x;
    const int t0 = tile * a.tile_tokens;
    const int nt = min(a.tile_tokens, a.T - t0);
    const int nslots = nt * a.k;
    const int64_t s0 = (int64_t)t0 * a.k;

    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        base_s[e] = a.tile_cnt[(int64_t)tile * E + e];
        seg_s[e] = a.seg[e];
    }
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int lo = (int)((int64_t)warp * nslots / W);
    const int hi = (int)((int64_t)(warp + 1) * nslots / W);
    const unsigned lt_mask = (1u << lane) - 1u;
    int32_t *my = wcnt + warp * E;

    // A: slots of this warp's contiguous range, counted per expert.
    if (warp < W) {
        for (int b = lo; b < hi; b += 32) {
            const int s = b + lane;
            const int e = (s < hi) ? load_id(a, s0 + s, false) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && lane == __ffs(peers) - 1) my[e] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();

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

    // C: ranks in slot order; position = segment start + rank inside the expert.
    if (warp < W) {
        for (int b = lo; b < hi; b += 32) {
            const int s = b + lane;
            const int e = (s < hi) ? load_id(a, s0 + s, false) : -1;
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

}  // namespace

cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s) {
    const size_t count_smem = (size_t)(a.E + a.R) * 4 + (size_t)a.sub_tokens * a.R * 4;
    const size_t scan_smem =
        (size_t)(max(a.scan_parts_e * a.E, a.scan_parts_r * a.R) + a.E + a.E + 1) * 4;
    const size_t pos_smem = (size_t)(2 + a.pos_warps) * a.E * 4;
    cudaError_t err;
    if (count_smem > 48 * 1024 &&
        (err = cudaFuncSetAttribute(layout_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)count_smem)) != cudaSuccess)
        return err;
    if (scan_smem > 48 * 1024 &&
        (err = cudaFuncSetAttribute(layout_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)scan_smem)) != cudaSuccess)
        return err;
    if (pos_smem > 48 * 1024 &&
        (err = cudaFuncSetAttribute(layout_pos_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)pos_smem)) != cudaSuccess)
        return err;
    if (a.ntiles > 0) {
        layout_count_kernel<<<a.ntiles, kCountThreads, count_smem, s>>>(a);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    // The scan also runs for T == 0: it writes the (empty or padded) segments,
    // zero counts and the -1 fill of every row.
    layout_scan_kernel<<<1, kScanThreads, scan_smem, s>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (a.ntiles > 0) {
        layout_pos_kernel<<<a.ntiles, kPosThreads, pos_smem, s>>>(a);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace ep
