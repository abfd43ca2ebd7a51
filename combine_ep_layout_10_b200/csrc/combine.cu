// combine.cu -- top-k weighted reduction of expert outputs back to source
// token order, in BF16.
//
// Combine as the pages describe it ("DeepEP (DeepEveryParallel)
// Documentation", items 3 and 10: expert outputs are reduced back to the
// tokens they came from; BF16 combine in "DeepSeek publica DeepEP ...",
// news.hada.io, "Resultados de medición de rendimiento").  This library
// fixes the arithmetic: for every token t and channel i,
//     acc = +0.0f;  for j = 0..k-1 with pos[t][j] >= 0:
//         acc = fmaf(w[t][j], y[pos[t][j]][i], acc);
//     out[t][i] = bf16 round-to-nearest-even(acc).
// A gather of k rows per token plus FMAs: HBM bound (k*H*2 bytes read and H*2
// written per token).  Each thread owns one 16-byte vector (8 channels) of
// one token, issues all k row loads of a batch before it accumulates (k
// independent 16-byte loads in flight per thread, read-only non-coherent path
// without L1 allocation: y is never written during the kernel), then runs the
// FMA chain in slot order and stores 16 bytes.  With no weights (w == nullptr)
// every weight is 1: fmaf(1, y, acc) is the correctly rounded acc + y, which
// makes the same kernel the backward of dispatch (sum of the k row gradients).
// Threads j < k resolve the token's k source rows to pointers first: row
// pos[t][j] of the local y, or, when the ranks are real GPUs (PEER), row d.y
// of rank d.x's expert outputs, d = dst[t][j] of the plan, read through that
// rank's mapping in this process (NVLink peer loads; y is not written by
// anyone while the combine runs).
#include <cuda_bf16.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kCombineThreads = EP_COMBINE_THREADS;
constexpr int kLoadBatch = 8;  // row loads issued back to back before accumulating

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
#if EP_COMBINE_L2_PREFETCH
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
#else
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
#endif
    return r;
}

__device__ __forceinline__ void st_out_v4(void *p, const uint4 &v) {
#if EP_COMBINE_STREAM_STORE
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
#else
    *reinterpret_cast<uint4 *>(p) = v;
#endif
}

__device__ __forceinline__ void fma8(float (&acc)[8], float w, const uint4 &v) {
    acc[0] = __fmaf_rn(w, __uint_as_float(v.x << 16), acc[0]);
    acc[1] = __fmaf_rn(w, __uint_as_float(v.x & 0xffff0000u), acc[1]);
    acc[2] = __fmaf_rn(w, __uint_as_float(v.y << 16), acc[2]);
    acc[3] = __fmaf_rn(w, __uint_as_float(v.y & 0xffff0000u), acc[3]);
    acc[4] = __fmaf_rn(w, __uint_as_float(v.z << 16), acc[4]);
    acc[5] = __fmaf_rn(w, __uint_as_float(v.z & 0xffff0000u), acc[5]);
    acc[6] = __fmaf_rn(w, __uint_as_float(v.w << 16), acc[6]);
    acc[7] = __fmaf_rn(w, __uint_as_float(v.w & 0xffff0000u), acc[7]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

template <int VPT, bool LOOP, bool PEER, bool EARLY = false>
__global__ void __launch_bounds__(kCombineThreads, LOOP ? 8 : 1) combine_kernel(CombineArgs a) {
    __shared__ const uint8_t *src_s[kMaxTopk];
    __shared__ float w_s[kMaxTopk];
    const size_t row_bytes = (size_t)a.H * 2;
#if EP_COMBINE_POS_BEFORE_WAIT
    // EARLY (small grids, one unit per block, local addressing): a separate
    // instantiation, because its extra weight registers would cost the
    // bandwidth-bound large grids resident blocks (measured: metric combine
    // 166.8 -> 168.0 us).
    if (EARLY && !LOOP && !PEER) {
        // The token's k row pointers are read before the wait for the previous
        // kernel: pos belongs to the handle and only its layout writes it, and
        // no layout kernel lets a later kernel launch before it has finished
        // (the count kernel, which does, writes no position), so by the time
        // this kernel is launched the positions are complete.  The weights and
        // the expert outputs are read only after the wait, together.
        const int t = blockIdx.x / a.blocks_per_token;
        const int cb = blockIdx.x - t * a.blocks_per_token;
        if (threadIdx.x < a.k) {
            const int p = __ldg(a.pos + (int64_t)t * a.k + threadIdx.x);
            src_s[threadIdx.x] = p >= 0 ? a.y + (size_t)p * row_bytes : nullptr;
        }
        __syncthreads();
        pdl_wait_then_trigger();
#pragma unroll
        for (int vi = 0; vi < VPT; ++vi) {
            const int v = (cb * VPT + vi) * kCombineThreads + threadIdx.x;
            if (v >= a.nvec) break;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int j0 = 0; j0 < a.k; j0 += kLoadBatch) {
                uint4 r[kLoadBatch];
                float wr[kLoadBatch];
#pragma unroll
                for (int jj = 0; jj < kLoadBatch; ++jj) {
                    const int j = j0 + jj;
                    const uint8_t *src = (j < a.k) ? src_s[j] : nullptr;
                    if (src != nullptr) {
                        r[jj] = ld_stream_v4(src + (size_t)v * 16);
                        wr[jj] = a.w != nullptr ? __ldg(a.w + (int64_t)t * a.k + j) : 1.0f;
                    }
                }
#pragma unroll
                for (int jj = 0; jj < kLoadBatch; ++jj) {
                    const int j = j0 + jj;
                    const uint8_t *src = (j < a.k) ? src_s[j] : nullptr;
                    if (src != nullptr) fma8(acc, wr[jj], r[jj]);
                }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            st_out_v4(a.out + (size_t)t * row_bytes + (size_t)v * 16, o);
        }
        return;
    }
#endif
    pdl_wait_then_trigger();
    const int nblocks = a.T * a.blocks_per_token;  // < 2^31, checked on the host
    // One (token, vector block) pair per block unless the grid is capped
    // (LOOP): then a grid stride over the pairs.
#pragma unroll 1
    for (int b = blockIdx.x; b < nblocks; b += gridDim.x) {
    const int t = b / a.blocks_per_token;
    const int cb = b - t * a.blocks_per_token;
    if (threadIdx.x < a.k) {
        const int64_t s = (int64_t)t * a.k + threadIdx.x;
        const uint8_t *src = nullptr;
        if (PEER) {
            const int2 d = __ldg(a.src + s);
            if (d.x >= 0) src = a.peer_y[d.x] + (size_t)d.y * row_bytes;
        } else {
            const int p = __ldg(a.pos + s);
            if (p >= 0) src = a.y + (size_t)p * row_bytes;
        }
        src_s[threadIdx.x] = src;
        w_s[threadIdx.x] = a.w != nullptr ? __ldg(a.w + s) : 1.0f;
    }
    __syncthreads();

#pragma unroll
    for (int vi = 0; vi < VPT; ++vi) {
        const int v = (cb * VPT + vi) * kCombineThreads + threadIdx.x;
        if (v >= a.nvec) break;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < a.k; j0 += kLoadBatch) {
            uint4 r[kLoadBatch];
#pragma unroll
            for (int jj = 0; jj < kLoadBatch; ++jj) {
                const int j = j0 + jj;
                const uint8_t *src = (j < a.k) ? src_s[j] : nullptr;
                if (src != nullptr) r[jj] = ld_stream_v4(src + (size_t)v * 16);
            }
#pragma unroll
            for (int jj = 0; jj < kLoadBatch; ++jj) {
                const int j = j0 + jj;
                const uint8_t *src = (j < a.k) ? src_s[j] : nullptr;
                if (src != nullptr) fma8(acc, w_s[j], r[jj]);
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        st_out_v4(a.out + (size_t)t * row_bytes + (size_t)v * 16, o);
    }
    if (!LOOP) break;
    __syncthreads();  // src_s / w_s are rewritten for the next pair
    }
}

// Row pointer and weight of slot j of token t (thread j < k of a unit).
template <bool PEER>
__device__ __forceinline__ void combine_slot(const CombineArgs &a, int t, int j, size_t row_bytes,
                                             const uint8_t *&src, float &wt) {
    const int64_t s = (int64_t)t * a.k + j;
    src = nullptr;
    if (PEER) {
        const int2 d = __ldg(a.src + s);
        if (d.x >= 0) src = a.peer_y[d.x] + (size_t)d.y * row_bytes;
    } else {
        const int p = __ldg(a.pos + s);
        if (p >= 0) src = a.y + (size_t)p * row_bytes;
    }
    wt = a.w != nullptr ? __ldg(a.w + s) : 1.0f;
}

// The grid-capped form (an SM budget): a block walks the (token, vector
// block) units with a grid stride, one vector per thread, and the next
// unit's row pointers and weights are loaded (threads j < k) before this
// unit's row loads are issued and published to the other half of a double
// buffer after them, so that a unit costs one memory round trip, not two.
// Same arithmetic as combine_kernel.
template <bool PEER>
__global__ void __launch_bounds__(kCombineThreads, 8) combine_loop_kernel(CombineArgs a) {
    __shared__ const uint8_t *src_s[2][kMaxTopk];
    __shared__ float w_s[2][kMaxTopk];
    const size_t row_bytes = (size_t)a.H * 2;
    pdl_wait_then_trigger();
    const int nblocks = a.T * a.blocks_per_token;  // < 2^31, checked on the host
    const int tid = threadIdx.x;
    int b = blockIdx.x;
    if (b >= nblocks) return;
    if (tid < a.k) {
        const uint8_t *src;
        float wt;
        combine_slot<PEER>(a, b / a.blocks_per_token, tid, row_bytes, src, wt);
        src_s[0][tid] = src;
        w_s[0][tid] = wt;
    }
    int cur = 0;
#pragma unroll 1
    for (; b < nblocks; b += gridDim.x) {
        __syncthreads();  // buffer cur is published; nobody reads buffer cur ^ 1 any more
        // The next unit's slot: only the loads here; the pointer is formed
        // after this unit's row loads, so nothing waits on them early.
        const int bn = b + gridDim.x;
        int2 nd = make_int2(-1, -1);  // (rank, row) of the slot; rank 0 when local
        float nw = 0.0f;
        if (tid < a.k && bn < nblocks) {
            const int64_t s = (int64_t)(bn / a.blocks_per_token) * a.k + tid;
            if (PEER)
                nd = __ldg(a.src + s);
            else
                nd = make_int2(0, __ldg(a.pos + s));
            nw = a.w != nullptr ? __ldg(a.w + s) : 1.0f;
        }
        const int t = b / a.blocks_per_token;
        const int cb = b - t * a.blocks_per_token;
        const int v = cb * kCombineThreads + tid;
        if (v < a.nvec) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int j0 = 0; j0 < a.k; j0 += kLoadBatch) {
                uint4 r[kLoadBatch];
#pragma unroll
                for (int jj = 0; jj < kLoadBatch; ++jj) {
                    const int j = j0 + jj;
                    const uint8_t *src = (j < a.k) ? src_s[cur][j] : nullptr;
                    if (src != nullptr) r[jj] = ld_stream_v4(src + (size_t)v * 16);
                }
#pragma unroll
                for (int jj = 0; jj < kLoadBatch; ++jj) {
                    const int j = j0 + jj;
                    const uint8_t *src = (j < a.k) ? src_s[cur][j] : nullptr;
                    if (src != nullptr) fma8(acc, w_s[cur][j], r[jj]);
                }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            st_out_v4(a.out + (size_t)t * row_bytes + (size_t)v * 16, o);
        }
        if (tid < a.k) {
            const bool ok = PEER ? nd.x >= 0 : nd.y >= 0;
            src_s[cur ^ 1][tid] = !ok ? nullptr : (PEER ? a.peer_y[nd.x] : a.y) + (size_t)nd.y * row_bytes;
            w_s[cur ^ 1][tid] = nw;
        }
        cur ^= 1;
    }
}

template <bool PEER>
cudaError_t launch_combine_impl(const CombineArgs &a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    long long blocks = (long long)a.T * a.blocks_per_token;
    if ((long long)a.blocks_per_token * a.vpt * kCombineThreads < a.nvec)
        return cudaErrorInvalidConfiguration;
    const bool loop = a.num_sms > 0;
    void (*kernel)(CombineArgs) = nullptr;
    if (a.vpt == 1) kernel = loop ? combine_loop_kernel<PEER> : combine_kernel<1, false, PEER>;
#if EP_COMBINE_POS_BEFORE_WAIT
    if (!PEER && !loop && a.vpt == 1 && a.pos_early) kernel = combine_kernel<1, false, false, true>;
#endif
    if (!PEER) {  // wider vectors per thread: a tuning option of the local path only
        if (a.vpt == 2) kernel = loop ? combine_kernel<2, true, false> : combine_kernel<2, false, false>;
        if (a.vpt == 4) kernel = loop ? combine_kernel<4, true, false> : combine_kernel<4, false, false>;
    }
    if (kernel == nullptr) return cudaErrorInvalidConfiguration;
    if (loop) {
        int per_sm = 0;
        cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kCombineThreads, 0);
        if (err != cudaSuccess) return err;
        const long long cap = (long long)a.num_sms * (per_sm > 0 ? per_sm : 1);
        if (cap < blocks) blocks = cap;
    }
    return launch_kernel(kernel, (unsigned)blocks, kCombineThreads, 0, s, a);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s) { return launch_combine_impl<false>(a, s); }

cudaError_t launch_combine_peer(const CombineArgs &a, cudaStream_t s) { return launch_combine_impl<true>(a, s); }

}  // namespace ep
