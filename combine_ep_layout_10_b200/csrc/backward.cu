// backward.cu -- the backward pair.
//
// The pages state that dispatch's backward pass is carried out by a combine
// and combine's backward pass by a dispatch ("DeepSeek publica DeepEP ...",
// news.hada.io, "Patrones de uso en entrenamiento, prefill y decoding";
// "DeepEP (DeepEveryParallel) Documentation", item 10).  For this library's
// forward definitions:
//   * dispatch backward: grad_x[t] = sum over valid slots j of
//     grad_recv[pos[t][j]] -- the combine kernel with every weight 1 (see
//     combine.cu; launched by ep_dispatch_backward);
//   * combine backward (this file), with g = grad_out[t]:
//       grad_y[pos[t][j]][i] = bf16_rn(fp32_rn(w[t][j] * g[i]))   -- a weighted dispatch
//       grad_w[t][j]         = sum_i g[i] * y[pos[t][j]][i]       -- fp32 dot product
// One block per token of up to 128 threads, each owning groups of 16
// channels c = tid, tid + 128, ...: g is read once, each slot's y row once, each grad_y row written
// once.  Products of two bf16 values are exact in fp32, so the only roundings
// in grad_w are additions: a chain of 16 per channel group over the thread's
// groups, a fixed xor-shuffle tree in the warp and a fixed-order sum over the
// block's warps.  The y rows of up to 8 slots are loaded before any is used
// (16 loads in flight per thread; 128 threads x 4 blocks per SM measured best).
// The result is deterministic run to run; its distance from the exact dot
// product is bounded by (#additions on the longest path) x 2^-24 x sum|g*y|.
// Threads j < k first resolve each slot's y row and grad_y row to pointers:
// row pos[t][j] of the local buffers, or, when the ranks are real GPUs
// (PEER), row d.y of rank d.x's buffers (d = dst[t][j] of the plan) through
// the peer table: the weighted scatter then stores straight into the owner's
// gradient buffer and the dot products read the owner's y.
#include <cuda_bf16.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

constexpr int kBwdBatch = EP_BWD_BATCH;  // slots whose y rows are loaded before any is used
constexpr int kBwdMaxThreads = EP_BWD_MAX_THREADS;

template <int KMAX, bool NEED_W, bool PEER>
__global__ void __launch_bounds__(kBwdMaxThreads, EP_BWD_MIN_BLOCKS) combine_bwd_kernel(CombineBwdArgs a) {
    __shared__ const uint8_t *y_s[KMAX];
    __shared__ uint8_t *gy_s[KMAX];
    __shared__ float w_s[KMAX];
    __shared__ float red_s[kBwdMaxThreads / 32][KMAX];
    pdl_wait_then_trigger();
    const int t = blockIdx.x;
    const int tid = threadIdx.x;
    const size_t row_bytes = (size_t)a.H * 2;
    if (tid < a.k) {
        const int64_t s = (int64_t)t * a.k + tid;
        const uint8_t *yr = nullptr;
        uint8_t *gr = nullptr;
        if (PEER) {
            const int2 d = __ldg(a.dst + s);
            if (d.x >= 0) {
                gr = a.peer_grad_y[d.x] + (size_t)d.y * row_bytes;
                if (NEED_W) yr = a.peer_y[d.x] + (size_t)d.y * row_bytes;
            }
        } else {
            const int p = __ldg(a.pos + s);
            if (p >= 0) {
                gr = a.grad_y + (size_t)p * row_bytes;
                if (NEED_W) yr = a.y + (size_t)p * row_bytes;
            }
        }
        y_s[tid] = yr;
        gy_s[tid] = gr;
        w_s[tid] = __ldg(a.w + s);
    }
    __syncthreads();

    float part[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) part[j] = 0.0f;

    const uint8_t *__restrict__ g_row = a.grad_out + (size_t)t * row_bytes;
    for (int c = tid; c * 16 < a.H; c += blockDim.x) {
        const size_t off = (size_t)c * 32;      // 16 channels = 32 bytes
        const bool full = c * 16 + 16 <= a.H;  // H % 16 == 8: the last group has 8 channels
        float g[16];
        unpack8(ld_nc_v4(g_row + off), g);
        if (full) {
            unpack8(ld_nc_v4(g_row + off + 16), g + 8);
        } else {
#pragma unroll
            for (int q = 8; q < 16; ++q) g[q] = 0.0f;
        }
#pragma unroll
        for (int j0 = 0; j0 < KMAX; j0 += kBwdBatch) {
            if (j0 >= a.k) break;
            // All y loads of the batch first, so up to 16 are in flight.
            uint4 yv[kBwdBatch][2];
            if (NEED_W) {
#pragma unroll
                for (int jj = 0; jj < kBwdBatch; ++jj) {
                    const int j = j0 + jj;
                    const uint8_t *yr = (j < a.k) ? y_s[j] : nullptr;
                    yv[jj][0] = make_uint4(0u, 0u, 0u, 0u);
                    yv[jj][1] = yv[jj][0];
                    if (yr != nullptr) {
                        yv[jj][0] = ld_nc_v4(yr + off);
                        if (full) yv[jj][1] = ld_nc_v4(yr + off + 16);
                    }
                }
            }
#pragma unroll
            for (int jj = 0; jj < kBwdBatch; ++jj) {
                const int j = j0 + jj;
                uint8_t *gr = (j < a.k) ? gy_s[j] : nullptr;
                if (gr == nullptr) continue;
                if (NEED_W) {
                    float y[16];
                    unpack8(yv[jj][0], y);
                    unpack8(yv[jj][1], y + 8);  // zero past the row end: g is 0 there too
                    float acc = part[j];
#pragma unroll
                    for (int q = 0; q < 16; ++q) acc = __fmaf_rn(g[q], y[q], acc);
                    part[j] = acc;
                }
                const float wj = w_s[j];
                uint4 o0, o1;
                o0.x = pack_bf16x2(__fmul_rn(wj, g[0]), __fmul_rn(wj, g[1]));
                o0.y = pack_bf16x2(__fmul_rn(wj, g[2]), __fmul_rn(wj, g[3]));
                o0.z = pack_bf16x2(__fmul_rn(wj, g[4]), __fmul_rn(wj, g[5]));
                o0.w = pack_bf16x2(__fmul_rn(wj, g[6]), __fmul_rn(wj, g[7]));
                o1.x = pack_bf16x2(__fmul_rn(wj, g[8]), __fmul_rn(wj, g[9]));
                o1.y = pack_bf16x2(__fmul_rn(wj, g[10]), __fmul_rn(wj, g[11]));
                o1.z = pack_bf16x2(__fmul_rn(wj, g[12]), __fmul_rn(wj, g[13]));
                o1.w = pack_bf16x2(__fmul_rn(wj, g[14]), __fmul_rn(wj, g[15]));
                uint8_t *dst = gr + off;
                *reinterpret_cast<uint4 *>(dst) = o0;
                if (full) *reinterpret_cast<uint4 *>(dst + 16) = o1;
            }
        }
    }
    if (!NEED_W) return;

    // Fixed-order block reduction of the k partial dot products.
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        float v = part[j];
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if (lane == 0) red_s[warp][j] = v;
    }
    __syncthreads();
    if (tid < a.k) {
        float s = 0.0f;
        for (int w = 0; w < nwarps; ++w) s += red_s[w][tid];
        a.grad_w[(int64_t)t * a.k + tid] = (gy_s[tid] != nullptr) ? s : 0.0f;
    }
}

template <bool PEER>
cudaError_t launch_combine_backward_impl(const CombineBwdArgs &a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    // One thread per 16 channels, at most kBwdMaxThreads; threads loop over the rest.
    const int groups = (a.H + 15) / 16;
    const int threads = groups >= kBwdMaxThreads ? kBwdMaxThreads : ((groups + 31) / 32) * 32;
    const bool need_w = a.grad_w != nullptr;
    if (a.k <= 8)
        return need_w ? launch_kernel(combine_bwd_kernel<8, true, PEER>, a.T, threads, 0, s, a)
                      : launch_kernel(combine_bwd_kernel<8, false, PEER>, a.T, threads, 0, s, a);
    return need_w ? launch_kernel(combine_bwd_kernel<kMaxTopk, true, PEER>, a.T, threads, 0, s, a)
                  : launch_kernel(combine_bwd_kernel<kMaxTopk, false, PEER>, a.T, threads, 0, s, a);
}

}  // namespace

cudaError_t launch_combine_backward(const CombineBwdArgs &a, cudaStream_t s) {
    return launch_combine_backward_impl<false>(a, s);
}

cudaError_t launch_combine_backward_peer(const CombineBwdArgs &a, cudaStream_t s) {
    return launch_combine_backward_impl<true>(a, s);
}

}  // namespace ep
