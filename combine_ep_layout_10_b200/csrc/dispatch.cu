// dispatch.cu -- scatter every token's hidden row to the receive rows of its
// slots, as BF16 bit copies or fused-quantised to FP8 e4m3 with one fp32
// scale per 128 channels.
//
// Dispatch as the pages describe it ("DeepEP (DeepEveryParallel)
// Documentation", item 10; FP8 dispatch in "deepseek-ai/DeepEP", repolode,
// "Funciones clave"): each token is read once and written once per routed
// expert.  On one B200 that is an HBM-bound scatter whose write side is k
// times its read side (81% writes for FP8 at top-8, 89% for BF16).
//
// One block per (token, chunk of at most EP_DISPATCH_MAX_CHUNK channels); the
// k receive rows of the token are read from the handle once per block.  The
// data never touches shared memory: every thread loads its channels with
// 16-byte non-allocating loads and writes them to the k rows with 16-byte
// stores, so each warp-wide store covers 512 contiguous bytes of a row.
//   * FP8: a thread owns 16 consecutive channels, so a 128-channel group is
//     8 consecutive lanes; the group amax takes three xor shuffles, then one
//     correctly rounded 448/amax, 16 multiplies and the hardware
//     round-to-nearest-even satfinite e4m3 conversion give 16 code bytes; the
//     group's first lane writes the scale.
//   * BF16: a thread owns two 16-byte vectors a block apart and copies them.
//   * FP8 input already quantised (codes + scales): a thread copies 16 codes,
//     the group's first lane copies the scale.
// FP8 scales are written at p * s_row + g * s_grp (row-major [rows, H/128],
// or column-major with a caller-chosen leading dimension for FP8 GEMMs).
// Column-major scales written this way are one scattered 4-byte store per
// (row, group): rows p and p + 1 of an expert come from different tokens and
// so from different blocks, and nothing coalesces.  The faster form writes
// each token's H/128 scales once to a per-token table (contiguous, small
// enough to stay in L2) and leaves the receive rows' scales to
// scale_fill_kernel, which walks the receive rows in order, gathers their
// tokens' table rows into shared memory and stores every column as a
// contiguous run.
// Threads j < k resolve the block's k destination rows to pointers first:
// row pos[t][j] of the local receive buffer, or, when the ranks are real GPUs
// (PEER), row d.y of rank d.x's receive buffer, d = dst[t][j] of the plan,
// reached through that rank's mapping in this process (NVLink peer stores).
// A TMA variant (bulk load into a shared ring, k bulk stores from shared
// memory) was measured slower on this path: bulk stores of scattered 7-14 KB
// rows sustain less write bandwidth on B200 than plain 16-byte stores.
#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

// Store of one 16-byte vector of a receive row.
__device__ __forceinline__ void st_row_v4(void *p, const uint4 &v) {
#if EP_DISPATCH_STORE_CS
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
#else
    *reinterpret_cast<uint4 *>(p) = v;
#endif
}

// Store of a per-token table entry with an evict-last L2 policy, so that the
// table survives the receive rows streaming through L2 until the fill pass
// reads it.
__device__ __forceinline__ void st_table_keep(float *p, float v) {
#if EP_DISPATCH_TABLE_KEEP_L2
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
#else
    *p = v;
#endif
}

__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    f[0] = bf16_bits_to_f32(v.x & 0xffffu);
    f[1] = bf16_bits_to_f32(v.x >> 16);
    f[2] = bf16_bits_to_f32(v.y & 0xffffu);
    f[3] = bf16_bits_to_f32(v.y >> 16);
    f[4] = bf16_bits_to_f32(v.z & 0xffffu);
    f[5] = bf16_bits_to_f32(v.z >> 16);
    f[6] = bf16_bits_to_f32(v.w & 0xffffu);
    f[7] = bf16_bits_to_f32(v.w >> 16);
}

// Receive-row pointers of token t's k slots (nullptr for a slot without a
// row), written to shared memory by threads j < k.
template <bool PEER>
__device__ __forceinline__ void slot_rows(const DispatchArgs &a, int t, size_t row_bytes, uint8_t **row_s,
                                          float **srow_s) {
    const int j = threadIdx.x;
    if (j >= a.k) return;
    const int64_t s = (int64_t)t * a.k + j;
    uint8_t *row = nullptr;
    float *srow = nullptr;
    if (PEER) {
        const int2 d = __ldg(a.dst + s);
        if (d.x >= 0) {
            row = a.peer_recv[d.x] + (size_t)d.y * row_bytes;
            if (a.peer_scales != nullptr) srow = a.peer_scales[d.x] + (int64_t)d.y * a.s_row;
        }
    } else {
        const int p = __ldg(a.pos + s);
        if (p >= 0) {
            row = a.recv + (size_t)p * row_bytes;
            if (a.scales != nullptr) srow = a.scales + (int64_t)p * a.s_row;
        }
    }
    row_s[j] = row;
    srow_s[j] = srow;
}

// The FP8 kernels below take one (token, chunk) unit per block (the grid is
// the unit count); a grid capped by the caller (num_sms) runs the pipelined
// grid-stride kernels further down instead.  The BF16 kernel keeps a plain
// grid stride (LOOP) for a capped grid.

template <bool PEER>
__global__ void __launch_bounds__(512) dispatch_fp8_kernel(DispatchArgs a) {
    __shared__ uint8_t *row_s[kMaxTopk];
    __shared__ float *srow_s[kMaxTopk];
    __shared__ float *tok_s;  // the token's row of the per-token scale table, or nullptr
#if EP_DISPATCH_EARLY_TRIGGER
    pdl_wait_then_trigger();
#else
    pdl_wait();
#endif
    const int tid = threadIdx.x;
    const bool leader = (tid & 7) == 0;
    {
        const int u = blockIdx.x;
        const int t = u / a.nchunks;
        const int ch0 = (u - t * a.nchunks) * a.chunk;
        const int chn = min(a.chunk, a.H - ch0);
        const int ch = ch0 + tid * 16;
        const bool act = tid * 16 < chn;
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (act) {
            const uint8_t *src = a.x + ((int64_t)t * a.H + ch) * 2;
            v0 = ld_nc_v4(src);
            v1 = ld_nc_v4(src + 16);
        }
        slot_rows<PEER>(a, t, (size_t)a.H, row_s, srow_s);  // after the x loads are in flight
        if (tid == 0) tok_s = a.tok_scales != nullptr ? a.tok_scales + (int64_t)t * (a.H / 128) : nullptr;
        __syncthreads();
        float f[16];
        unpack8(v0, f);
        unpack8(v1, f + 8);
        float amax = 0.0f;
#pragma unroll
        for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(f[q]));
        // A 128-channel group is 8 consecutive lanes: xor distances < 8 stay inside it.
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        if (act) {
            uint4 q16 = make_uint4(0u, 0u, 0u, 0u);
            float scale = 0.0f;
            if (amax != 0.0f) {
                scale = __fdiv_rn(amax, 448.0f);
                const float inv = __fdiv_rn(448.0f, amax);
                uint32_t b[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float2 pr = make_float2(__fmul_rn(f[2 * q], inv), __fmul_rn(f[2 * q + 1], inv));
                    b[q] = (uint32_t)__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
                }
                q16.x = b[0] | (b[1] << 16);
                q16.y = b[2] | (b[3] << 16);
                q16.z = b[4] | (b[5] << 16);
                q16.w = b[6] | (b[7] << 16);
            }
            const int g = ch / 128;
            if (leader && tok_s != nullptr) st_table_keep(tok_s + g, scale);
            for (int j = 0; j < a.k; ++j) {
                uint8_t *row = row_s[j];
                if (row == nullptr) continue;
                st_row_v4(row + ch, q16);
                if (leader && srow_s[j] != nullptr) srow_s[j][(int64_t)g * a.s_grp] = scale;
            }
        }
    }
}

// The 16 e4m3 codes of a thread's channels given its group's 448 / amax
// (RNE-satfinite e4m3 of the correctly rounded product), as in
// dispatch_fp8_kernel.
__device__ __forceinline__ uint4 e4m3_codes16(const float *f, float inv) {
    uint32_t b[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float2 pr = make_float2(__fmul_rn(f[2 * q], inv), __fmul_rn(f[2 * q + 1], inv));
        b[q] = (uint32_t)__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
    }
    return make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16), b[6] | (b[7] << 16));
}

// The grid-capped form (an SM budget) of dispatch_fp8_kernel: a block walks
// the units with a grid stride, and as soon as a unit's codes are made the
// next unit's x vectors and row positions are loaded, so that their round
// trip overlaps this unit's stores; the next unit's row pointers go to the
// other half of a double buffer.  Same arithmetic as dispatch_fp8_kernel.
template <bool PEER>
__global__ void __launch_bounds__(512) dispatch_fp8_loop_kernel(DispatchArgs a) {
    __shared__ uint8_t *row_s[2][kMaxTopk];
    __shared__ float *srow_s[2][kMaxTopk];
    __shared__ float *tok_s[2];  // the unit's token row of the per-token scale table, or nullptr
#if EP_DISPATCH_EARLY_TRIGGER
    pdl_wait_then_trigger();
#else
    pdl_wait();
#endif
    const int tid = threadIdx.x;
    const bool leader = (tid & 7) == 0;
    const int G = a.H / 128;
    int u = blockIdx.x;
    if (u >= a.nunits) return;
    uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
    {
        const int t = u / a.nchunks;
        const int ch0 = (u - t * a.nchunks) * a.chunk;
        if (tid * 16 < min(a.chunk, a.H - ch0)) {
            const uint8_t *src = a.x + ((int64_t)t * a.H + ch0 + tid * 16) * 2;
            v0 = ld_nc_v4(src);
            v1 = ld_nc_v4(src + 16);
        }
        slot_rows<PEER>(a, t, (size_t)a.H, row_s[0], srow_s[0]);
        if (tid == 0) tok_s[0] = a.tok_scales != nullptr ? a.tok_scales + (int64_t)t * G : nullptr;
    }
    int cur = 0;
#pragma unroll 1
    for (; u < a.nunits; u += gridDim.x) {
        __syncthreads();  // buffer cur is published; nobody reads buffer cur ^ 1 any more
        const int t = u / a.nchunks;
        const int ch0 = (u - t * a.nchunks) * a.chunk;
        const int chn = min(a.chunk, a.H - ch0);
        const int ch = ch0 + tid * 16;
        const bool act = tid * 16 < chn;
        float f[16];
        unpack8(v0, f);
        unpack8(v1, f + 8);
        float amax = 0.0f;
#pragma unroll
        for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(f[q]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        uint4 q16 = make_uint4(0u, 0u, 0u, 0u);
        float scale = 0.0f;
        if (act && amax != 0.0f) {
            scale = __fdiv_rn(amax, 448.0f);
            q16 = e4m3_codes16(f, __fdiv_rn(448.0f, amax));
        }
        // The next unit's loads, issued before this unit's stores.
        const int un = u + gridDim.x;
        const bool more = un < a.nunits;
        const int tn = more ? un / a.nchunks : 0;
        v0 = make_uint4(0u, 0u, 0u, 0u);
        v1 = v0;
        int np = -1;
        int2 nd = make_int2(-1, -1);
        if (more) {
            const int nch0 = (un - tn * a.nchunks) * a.chunk;
            if (tid * 16 < min(a.chunk, a.H - nch0)) {
                const uint8_t *src = a.x + ((int64_t)tn * a.H + nch0 + tid * 16) * 2;
                v0 = ld_nc_v4(src);
                v1 = ld_nc_v4(src + 16);
            }
            if (tid < a.k) {
                if (PEER)
                    nd = __ldg(a.dst + (int64_t)tn * a.k + tid);
                else
                    np = __ldg(a.pos + (int64_t)tn * a.k + tid);
            }
        }
        if (act) {
            const int g = ch / 128;
            if (leader && tok_s[cur] != nullptr) st_table_keep(tok_s[cur] + g, scale);
            for (int j = 0; j < a.k; ++j) {
                uint8_t *row = row_s[cur][j];
                if (row == nullptr) continue;
                st_row_v4(row + ch, q16);
                if (leader && srow_s[cur][j] != nullptr) srow_s[cur][j][(int64_t)g * a.s_grp] = scale;
            }
        }
        if (more) {
            if (tid < a.k) {
                uint8_t *row = nullptr;
                float *srow = nullptr;
                if (PEER) {
                    if (nd.x >= 0) {
                        row = a.peer_recv[nd.x] + (size_t)nd.y * a.H;
                        if (a.peer_scales != nullptr) srow = a.peer_scales[nd.x] + (int64_t)nd.y * a.s_row;
                    }
                } else if (np >= 0) {
                    row = a.recv + (size_t)np * a.H;
                    if (a.scales != nullptr) srow = a.scales + (int64_t)np * a.s_row;
                }
                row_s[cur ^ 1][tid] = row;
                srow_s[cur ^ 1][tid] = srow;
            }
            if (tid == 0) tok_s[cur ^ 1] = a.tok_scales != nullptr ? a.tok_scales + (int64_t)tn * G : nullptr;
        }
        cur ^= 1;
    }
}

// The same pipelining for pre-quantised FP8 input (codes and scales copied):
// the next unit's codes, scales and row positions are loaded before this
// unit's stores; same store pattern as dispatch_fp8_copy_kernel.  (BF16
// copies keep the plain grid stride: pipelined, the kernel needs more than
// 32 registers and loses a resident block per SM, which measured slower.)
template <bool PEER>
__global__ void __launch_bounds__(512) dispatch_fp8_copy_loop_kernel(DispatchArgs a) {
    __shared__ uint8_t *row_s[2][kMaxTopk];
    __shared__ float *srow_s[2][kMaxTopk];
#if EP_DISPATCH_EARLY_TRIGGER
    pdl_wait_then_trigger();
#else
    pdl_wait();
#endif
    const int tid = threadIdx.x;
    const bool leader = (tid & 7) == 0;
    const int G = a.H / 128;
    // Codes and scale of unit u for this thread (zero past the chunk).
    auto load_unit = [&](int u, uint4 &v, float &sc) {
        v = make_uint4(0u, 0u, 0u, 0u);
        sc = 0.0f;
        const int t = u / a.nchunks;
        const int ch = (u - t * a.nchunks) * a.chunk + tid * 16;
        if (tid * 16 < min(a.chunk, a.H - (ch - tid * 16))) {
            v = ld_nc_v4(a.x + (int64_t)t * a.H + ch);
            if (leader) sc = __ldg(a.x_scales + (int64_t)t * G + ch / 128);
        }
    };
    int u = blockIdx.x;
    if (u >= a.nunits) return;
    uint4 v;
    float sc;
    load_unit(u, v, sc);
    slot_rows<PEER>(a, u / a.nchunks, (size_t)a.H, row_s[0], srow_s[0]);
    int cur = 0;
#pragma unroll 1
    for (; u < a.nunits; u += gridDim.x) {
        __syncthreads();  // buffer cur is published; nobody reads buffer cur ^ 1 any more
        const int t = u / a.nchunks;
        const int ch0 = (u - t * a.nchunks) * a.chunk;
        const int ch = ch0 + tid * 16;
        const bool act = tid * 16 < min(a.chunk, a.H - ch0);
        const uint4 q = v;  // this unit's codes and scale
        const float scale = sc;
        // The next unit's loads, issued before this unit's stores.
        const int un = u + gridDim.x;
        const bool more = un < a.nunits;
        const int tn = more ? un / a.nchunks : 0;
        int np = -1;
        int2 nd = make_int2(-1, -1);
        if (more) {
            load_unit(un, v, sc);
            if (tid < a.k) {
                if (PEER)
                    nd = __ldg(a.dst + (int64_t)tn * a.k + tid);
                else
                    np = __ldg(a.pos + (int64_t)tn * a.k + tid);
            }
        }
        if (act) {
            const int g = ch / 128;
            for (int j = 0; j < a.k; ++j) {
                uint8_t *row = row_s[cur][j];
                if (row == nullptr) continue;
                st_row_v4(row + ch, q);
                if (leader && srow_s[cur][j] != nullptr) srow_s[cur][j][(int64_t)g * a.s_grp] = scale;
            }
        }
        // The next unit's row pointers, into the other buffer.
        if (more && tid < a.k) {
            uint8_t *row = nullptr;
            float *srow = nullptr;
            if (PEER) {
                if (nd.x >= 0) {
                    row = a.peer_recv[nd.x] + (size_t)nd.y * a.H;
                    if (a.peer_scales != nullptr) srow = a.peer_scales[nd.x] + (int64_t)nd.y * a.s_row;
                }
            } else if (np >= 0) {
                row = a.recv + (size_t)np * a.H;
                if (a.scales != nullptr) srow = a.scales + (int64_t)np * a.s_row;
            }
            row_s[cur ^ 1][tid] = row;
            srow_s[cur ^ 1][tid] = srow;
        }
        cur ^= 1;
    }
}

// Pre-quantised FP8 input: codes and scales are copied, not recomputed.
template <bool PEER>
__global__ void __launch_bounds__(512) dispatch_fp8_copy_kernel(DispatchArgs a) {
    __shared__ uint8_t *row_s[kMaxTopk];
    __shared__ float *srow_s[kMaxTopk];
#if EP_DISPATCH_EARLY_TRIGGER
    pdl_wait_then_trigger();
#else
    pdl_wait();
#endif
    const int tid = threadIdx.x;
    const bool leader = (tid & 7) == 0;
    const int G_row = a.H / 128;
    {
        const int u = blockIdx.x;
        const int t = u / a.nchunks;
        const int ch0 = (u - t * a.nchunks) * a.chunk;
        const int chn = min(a.chunk, a.H - ch0);
        const int ch = ch0 + tid * 16;
        const bool act = tid * 16 < chn;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        float scale = 0.0f;
        if (act) {
            v = ld_nc_v4(a.x + (int64_t)t * a.H + ch);
            if (leader) scale = __ldg(a.x_scales + (int64_t)t * G_row + ch / 128);
        }
        slot_rows<PEER>(a, t, (size_t)a.H, row_s, srow_s);  // after the x loads are in flight
        __syncthreads();
        if (act) {
            const int g = ch / 128;
            for (int j = 0; j < a.k; ++j) {
                uint8_t *row = row_s[j];
                if (row == nullptr) continue;
                st_row_v4(row + ch, v);
                if (leader && srow_s[j] != nullptr) srow_s[j][(int64_t)g * a.s_grp] = scale;
            }
        }
    }
}

template <bool LOOP, bool PEER>
__global__ void __launch_bounds__(512) dispatch_bf16_kernel(DispatchArgs a) {
    __shared__ uint8_t *row_s[kMaxTopk];
    __shared__ float *srow_s[kMaxTopk];
#if EP_DISPATCH_EARLY_TRIGGER
    pdl_wait_then_trigger();
#else
    pdl_wait();
#endif
    const int tid = threadIdx.x;
    // One unit per block unless the grid is capped (LOOP): then a grid stride.
    for (int u = blockIdx.x; u < a.nunits; u += gridDim.x) {
        const int t = u / a.nchunks;
        const int ch0 = (u - t * a.nchunks) * a.chunk;
        const int chn = min(a.chunk, a.H - ch0);
        // Two 16-byte vectors per thread, a block apart, so that every warp-wide
        // load and store covers 512 contiguous bytes.
        const int nv = chn / 8;
        const int u0 = tid, u1 = tid + blockDim.x;
        const bool act0 = u0 < nv, act1 = u1 < nv;
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        const uint8_t *src = a.x + ((int64_t)t * a.H + ch0) * 2;
        if (act0) v0 = ld_nc_v4(src + (size_t)u0 * 16);
        if (act1) v1 = ld_nc_v4(src + (size_t)u1 * 16);
        slot_rows<PEER>(a, t, (size_t)a.H * 2, row_s, srow_s);  // after the x loads are in flight
        __syncthreads();
        if (act0) {
            for (int j = 0; j < a.k; ++j) {
                uint8_t *row = row_s[j];
                if (row == nullptr) continue;
                uint8_t *dst = row + (size_t)ch0 * 2;
                st_row_v4(dst + (size_t)u0 * 16, v0);
                if (act1) st_row_v4(dst + (size_t)u1 * 16, v1);
            }
        }
        if (!LOOP) break;
        __syncthreads();  // row_s is rewritten by the next unit
    }
}

template <bool PEER>
cudaError_t launch_dispatch_impl(const DispatchArgs &a, cudaStream_t st) {
    if (a.nunits == 0) return cudaSuccess;
    // One block per unit, one thread per 16 channels (chunk <= 8192 -> <= 512 threads).
    const int threads = (((a.chunk + 15) / 16 + 31) / 32) * 32;
    const bool loop = a.num_sms > 0;
    void (*kernel)(DispatchArgs) =
        a.mode == kDispatchQuantFp8
            ? (loop ? dispatch_fp8_loop_kernel<PEER> : dispatch_fp8_kernel<PEER>)
        : a.mode == kDispatchCopyFp8
            ? (loop ? dispatch_fp8_copy_loop_kernel<PEER> : dispatch_fp8_copy_kernel<PEER>)
            : (loop ? dispatch_bf16_kernel<true, PEER> : dispatch_bf16_kernel<false, PEER>);
    int grid = a.nunits;
    if (loop) {
        int per_sm = 0;
        cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
        if (err != cudaSuccess) return err;
        const long long cap = (long long)a.num_sms * (per_sm > 0 ? per_sm : 1);
        if (cap < grid) grid = (int)cap;
    }
    return launch_kernel(kernel, (unsigned)grid, threads, 0, st, a);
}

// Column-major scales from the per-token table.  A block takes tiles of
// kFillRows consecutive receive rows and up to kFillGroups groups: it reads
// the tiles' source tokens, gathers each token's table row (contiguous
// floats; 16-byte loads when rows allow, all of a thread's loads issued
// before any is used, so a tile costs about one memory round trip) into
// shared memory and then stores every group's column of the tile as one
// contiguous run of up to kFillRows floats.
// Behind the quantising dispatch the pass is bound by what that kernel
// leaves behind, not by its own work (measured, metric workload, with
// per-block timestamps): its blocks are released about 0.9 us after the
// dispatch's last block has issued its stores, the one gather round trip
// then takes 1.6-4.1 us (median 2.4) and issuing the column stores 2.0-3.2 us
// (median 2.8), because L2 is full of the dispatch's dirty code lines and
// every new line waits for one to be written back; neither an all-hit table
// (every row reading one of 64 tokens) nor dropping the stores' DRAM
// traffic changed the call's time.
constexpr int kFillRows = 128;
constexpr int kFillGroups = 64;
constexpr int kFillThreads = 256;
constexpr int kFillVecPerThread = kFillRows / (2 * (kFillThreads / 32));  // rows of a thread in the 16-byte gather
static_assert(kFillGroups / 4 <= 16, "a half-warp holds one row's 16-byte pieces");

// Table loads use the default L2 policy: every entry is read once per
// receive row of its token (k times), so it should stay (measured: an
// evict-first policy here cost the pre-quantised column-major call about
// 0.5 us; evict-last and evict-unchanged were no better than the default).
__device__ __forceinline__ float4 ld_table_v4(const float *p) {
    float4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float ld_table(const float *p) {
    float r;
    asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(r) : "l"(p));
    return r;
}

__global__ void __launch_bounds__(kFillThreads) scale_fill_kernel(ScaleFillArgs a) {
    __shared__ float tile_s[kFillRows * (kFillGroups + 1)];
    __shared__ int32_t src_s[kFillRows];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    constexpr int kWarps = kFillThreads / 32;
    const int64_t ntiles = (a.n_rows + kFillRows - 1) / kFillRows;
    // The source tokens of the first tile are read before the wait for the
    // dispatch: the layout wrote them, and it completed before the dispatch
    // (this kernel's predecessor) began.  The table is read only after it,
    // unless it is the caller's input (then there is no wait here at all).
    if (blockIdx.x < ntiles) {
        const int64_t p0 = (int64_t)blockIdx.x * kFillRows;
        const int n = (int)min((int64_t)kFillRows, a.n_rows - p0);
        for (int i = tid; i < n; i += kFillThreads) src_s[i] = __ldg(a.src_idx + p0 + i);
    }
    if (a.table_is_input)
        pdl_trigger();  // nothing this pass reads or writes is touched by the copy kernel
    else
        pdl_wait_then_trigger();
    const int g0 = blockIdx.y * kFillGroups;
    const int gn = min(kFillGroups, a.G - g0);
    const int ldt = gn | 1;  // odd row stride: the column reads below hit distinct banks
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t p0 = tile * kFillRows;
        const int n = (int)min((int64_t)kFillRows, a.n_rows - p0);
        if (tile != blockIdx.x)
            for (int i = tid; i < n; i += kFillThreads) src_s[i] = __ldg(a.src_idx + p0 + i);
        __syncthreads();
        if (a.vec_in) {
            // 16-byte pieces (G % 4 == 0, so gn % 4 == 0 and every table row is
            // 16-byte aligned): a warp takes two rows at a time, a half-warp per
            // row, a lane per piece (gn / 4 <= 16); no integer division.
            const int gv = gn >> 2;
            const int c = lane & 15;
            float4 v[kFillVecPerThread];
#pragma unroll
            for (int q = 0; q < kFillVecPerThread; ++q) {
                const int i = (q * kWarps + warp) * 2 + (lane >> 4);
                v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < n && c < gv) {
                    const int32_t t = src_s[i];
                    if (t >= 0) v[q] = ld_table_v4(a.table + (int64_t)t * a.G + g0 + 4 * c);
                }
            }
#pragma unroll
            for (int q = 0; q < kFillVecPerThread; ++q) {
                const int i = (q * kWarps + warp) * 2 + (lane >> 4);
                if (i < n && c < gv) {
                    float *d = tile_s + i * ldt + 4 * c;
                    d[0] = v[q].x;
                    d[1] = v[q].y;
                    d[2] = v[q].z;
                    d[3] = v[q].w;
                }
            }
        } else {
            // A warp per row, a lane per group (two passes of 32 groups).
            for (int i = warp; i < n; i += kWarps) {
                const int32_t t = src_s[i];
#pragma unroll
                for (int h = 0; h < kFillGroups; h += 32) {
                    const int g = h + lane;
                    if (g < gn) tile_s[i * ldt + g] = t >= 0 ? ld_table(a.table + (int64_t)t * a.G + g0 + g) : 0.0f;
                }
            }
        }
        __syncthreads();
        // Store: a warp per column of the tile, consecutive lanes on consecutive rows.
        for (int g = warp; g < gn; g += kWarps) {
            float *col = a.scales + (int64_t)(g0 + g) * a.ld + p0;
#pragma unroll
            for (int i0 = 0; i0 < kFillRows; i0 += 32) {
                const int i = i0 + lane;
                if (i < n && src_s[i] >= 0) col[i] = tile_s[i * ldt + g];
            }
        }
        __syncthreads();  // src_s / tile_s are rewritten by the next tile
    }
    // Started early: complete only after the copy kernel has, so that what
    // follows in the stream sees both.
    if (a.table_is_input) pdl_wait();
}

}  // namespace

cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t st) { return launch_dispatch_impl<false>(a, st); }

cudaError_t launch_scale_fill(const ScaleFillArgs &a, cudaStream_t st) {
    if (a.n_rows == 0 || a.G == 0) return cudaSuccess;
    if (a.vec_in && (a.G % 4 != 0 || (reinterpret_cast<uintptr_t>(a.table) & 15u) != 0))
        return cudaErrorInvalidValue;
    if (a.table_is_input && a.num_sms > 0) return cudaErrorInvalidValue;
    const int64_t ntiles = (a.n_rows + kFillRows - 1) / kFillRows;
    const int gchunks = (a.G + kFillGroups - 1) / kFillGroups;
    int64_t grid = ntiles;
    if (a.num_sms > 0) {
        int per_sm = 0;
        cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, scale_fill_kernel, kFillThreads, 0);
        if (err != cudaSuccess) return err;
        const int64_t cap = (int64_t)a.num_sms * (per_sm > 0 ? per_sm : 1);
        const int64_t per_chunk = (cap + gchunks - 1) / gchunks;  // blocks of the grid's x dimension
        if (per_chunk < grid) grid = per_chunk;
    }
    if (grid > 0x7fffffff) grid = 0x7fffffff;
    return launch_kernel(scale_fill_kernel, dim3((unsigned)grid, (unsigned)gchunks), kFillThreads, 0, st, a);
}

cudaError_t launch_dispatch_peer(const DispatchArgs &a, cudaStream_t st) { return launch_dispatch_impl<true>(a, st); }

}  // namespace ep
