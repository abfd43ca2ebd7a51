// dispatch.cu -- scatter every token's hidden row to the receive rows of its
// slots, as BF16 bit copies or fused-quantised to FP8 e4m3 with one fp32
// scale per 128 channels.
//
// Dispatch as the pages describe it ("DeepEP (DeepEveryParallel)
// Documentation", item 10; FP8 dispatch in "deepseek-ai/DeepEP", repolode,
// "Funciones clave"): each token is read once and written once per routed
// expert.  On one B200 that is an HBM-bound copy whose write side is k times
// its read side, so the design keeps the SM out of the data path as far as
// possible:
//   * persistent grid (SM count x resident CTAs), work units = (token, row
//     chunk) strided statically over CTAs -- per-token work is the same for
//     every token, so skewed routing creates no stragglers;
//   * the chunk of x is fetched with one TMA bulk copy (cp.async.bulk) into a
//     shared-memory ring completed on an mbarrier;
//   * BF16: the staged chunk is written to the k receive rows by k TMA bulk
//     stores straight from shared memory -- no register traffic at all;
//   * FP8: 4 warps read the chunk from shared memory, take each 128-channel
//     group's amax with half-warp shuffles, scale by one rounded 448/amax and
//     convert with the hardware round-to-nearest-even satfinite e4m3
//     conversion into a second shared-memory buffer, which k TMA bulk stores
//     write out; the group scales go out with plain coalesced stores.
// Every mbarrier wait is bounded; on timeout the kernel flags the handle's
// error word, drains its own bulk stores and returns.
#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kFp8Threads = 128;
constexpr int kBf16Threads = 32;
constexpr int kOutBufs = 3;       // FP8 output staging ring
constexpr int kHeaderBytes = 512; // mbarriers + pos staging

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) return false;
    }
    return true;
}

__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_store(void *dst, const void *src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_addr(src_smem)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// After an abort, wait (bounded) for the loads this CTA issued for units
// [first, last) so that none lands in shared memory after the CTA retires.
__device__ __forceinline__ void drain_loads(uint64_t *bar, int S, int first, int last) {
    const long long t0 = clock64();
    for (int u = first; u < last; ++u) {
        while (!mbar_try_wait(&bar[u % S], (uint32_t)((u / S) & 1))) {
            if (clock64() - t0 > kWaitLimitCycles) return;
        }
    }
}

struct Unit {
    int t;        // token
    int ch0;      // first channel of the chunk
    int chn;      // channels in the chunk
};

__device__ __forceinline__ Unit unit_of(const DispatchArgs &a, long long u) {
    Unit r;
    r.t = (int)(u / a.nchunks);
    const int c = (int)(u - (long long)r.t * a.nchunks);
    r.ch0 = c * a.chunk;
    r.chn = min(a.chunk, a.H - r.ch0);
    return r;
}

__device__ __forceinline__ int units_of_cta(const DispatchArgs &a) {
    if ((long long)blockIdx.x >= a.nunits) return 0;
    return (int)((a.nunits - blockIdx.x + gridDim.x - 1) / gridDim.x);
}

// ---------------------------------------------------------------------------
// BF16: TMA in, k TMA stores out, one warp per CTA (lane 0 drives the copies).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBf16Threads) dispatch_bf16_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
    unsigned char *ring = smem + kHeaderBytes;
    const int stage_bytes = a.chunk * 2;
    const int S = a.stages;
    const int lane = threadIdx.x;
    const int n = units_of_cta(a);

    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    int issued = 0;  // lane 0: loads issued so far (units [0, issued))
    auto issue_load = [&](int i) {
        const Unit w = unit_of(a, blockIdx.x + (long long)i * gridDim.x);
        const int s = i % S;
        const uint32_t bytes = (uint32_t)w.chn * 2u;
        mbar_expect_tx(&bar[s], bytes);
        bulk_load(ring + (size_t)s * stage_bytes, a.x + ((int64_t)w.t * a.H + w.ch0) * 2, bytes,
                  &bar[s]);
        issued = i + 1;
    };

    if (lane == 0) {
        for (int i = 0; i < min(S - 1, n); ++i) issue_load(i);
    }
    bool ok = true;
    int failed_at = n;
    for (int i = 0; i < n; ++i) {
        const Unit w = unit_of(a, blockIdx.x + (long long)i * gridDim.x);
        const int pj = (lane < a.k) ? __ldg(a.pos + (int64_t)w.t * a.k + lane) : -1;
        const int s = i % S;
        if (lane == 0) {
            ok = mbar_wait(&bar[s], (uint32_t)((i / S) & 1));
            if (!ok) atomicOr(a.err, kErrTimeout);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) {
            failed_at = i;
            break;
        }
        const unsigned char *src = ring + (size_t)s * stage_bytes;
        for (int j = 0; j < a.k; ++j) {
            const int p = __shfl_sync(0xffffffffu, pj, j);
            if (lane == 0 && p >= 0)
                bulk_store(a.recv + ((int64_t)p * a.H + w.ch0) * 2, src, (uint32_t)w.chn * 2u);
        }
        if (lane == 0) {
            bulk_commit();
            // Refill the slot the previous unit's stores read from once they are done.
            if (i + S - 1 < n) {
                if (i >= 1) bulk_wait_read<1>();
                issue_load(i + S - 1);
            }
        }
    }
    if (lane == 0) {
        bulk_wait_all();
        if (!ok) drain_loads(bar, S, failed_at, issued);
    }
}

// ---------------------------------------------------------------------------
// FP8: TMA in, quantise in shared memory, k TMA stores + scale stores out.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}

__global__ void __launch_bounds__(kFp8Threads) dispatch_fp8_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);                 // [S]
    int32_t *pos_s = reinterpret_cast<int32_t *>(smem + 128);           // [2][32]
    const int S = a.stages;
    const int in_bytes = a.chunk * 2;
    const int out_bytes = a.chunk;
    const int sc_bytes = ((a.chunk / 128) * 4 + 15) & ~15;
    unsigned char *in_ring = smem + kHeaderBytes;
    unsigned char *out_ring = in_ring + (size_t)S * in_bytes;
    float *sc_ring = reinterpret_cast<float *>(out_ring + (size_t)kOutBufs * out_bytes);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int n = units_of_cta(a);
    const int G_row = a.H / 128;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    int issued = 0;  // thread 0: loads issued so far (units [0, issued))
    auto issue_load = [&](int i) {
        const Unit w = unit_of(a, blockIdx.x + (long long)i * gridDim.x);
        const int s = i % S;
        const uint32_t bytes = (uint32_t)w.chn * 2u;
        mbar_expect_tx(&bar[s], bytes);
        bulk_load(in_ring + (size_t)s * in_bytes, a.x + ((int64_t)w.t * a.H + w.ch0) * 2, bytes,
                  &bar[s]);
        issued = i + 1;
    };

    if (tid == 0) {
        for (int i = 0; i < min(S, n); ++i) issue_load(i);
    }
    int failed_at = n;

    for (int i = 0; i < n; ++i) {
        const Unit w = unit_of(a, blockIdx.x + (long long)i * gridDim.x);
        const int s = i % S;
        const int ob = i % kOutBufs;
        int32_t *pbuf = pos_s + (i & 1) * 32;
        int pj = -1;
        if (warp == 0 && lane < a.k) pj = __ldg(a.pos + (int64_t)w.t * a.k + lane);

        const bool ok = mbar_wait(&bar[s], (uint32_t)((i / S) & 1));

        const unsigned char *in = in_ring + (size_t)s * in_bytes;
        unsigned char *out = out_ring + (size_t)ob * out_bytes;
        float *sc = sc_ring + (size_t)ob * (sc_bytes / 4);
        const int G = w.chn / 128;
        const int half = lane >> 4;
        const int hl = lane & 15;
        for (int pp = warp; pp < (G + 1) / 2; pp += nwarps) {
            const int g = pp * 2 + half;
            const bool act = g < G;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (act) v = *reinterpret_cast<const uint4 *>(in + ((size_t)g * 128 + hl * 8) * 2);
            float f[8];
            f[0] = bf16_bits_to_f32(v.x & 0xffffu);
            f[1] = bf16_bits_to_f32(v.x >> 16);
            f[2] = bf16_bits_to_f32(v.y & 0xffffu);
            f[3] = bf16_bits_to_f32(v.y >> 16);
            f[4] = bf16_bits_to_f32(v.z & 0xffffu);
            f[5] = bf16_bits_to_f32(v.z >> 16);
            f[6] = bf16_bits_to_f32(v.w & 0xffffu);
            f[7] = bf16_bits_to_f32(v.w >> 16);
            float amax = 0.0f;
#pragma unroll
            for (int q = 0; q < 8; ++q) amax = fmaxf(amax, fabsf(f[q]));
            // 128-channel group = 16 lanes: xor distances < 16 stay in the half-warp.
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 8));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            uint2 q8 = make_uint2(0u, 0u);
            float scale = 0.0f;
            if (amax != 0.0f) {
                scale = __fdiv_rn(amax, 448.0f);
                const float inv = __fdiv_rn(448.0f, amax);
                uint32_t b[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 pr = make_float2(__fmul_rn(f[2 * q], inv), __fmul_rn(f[2 * q + 1], inv));
                    b[q] = (uint32_t)__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
                }
                q8.x = b[0] | (b[1] << 16);
                q8.y = b[2] | (b[3] << 16);
            }
            if (act) {
                *reinterpret_cast<uint2 *>(out + (size_t)g * 128 + hl * 8) = q8;
                if (hl == 0) sc[g] = scale;
            }
        }
        if (warp == 0 && lane < a.k) pbuf[lane] = pj;
        fence_proxy_async_smem();
        // The stores of unit i-2 read out[(i+1) % 3]; unit i+1 writes it next.
        if (tid == 0) bulk_wait_read<kOutBufs - 2>();
        const bool all_ok = __syncthreads_and(ok) != 0;
        if (!all_ok) {
            if (tid == 0) atomicOr(a.err, kErrTimeout);
            failed_at = i;
            break;
        }
        if (tid == 0) {
            for (int j = 0; j < a.k; ++j) {
                const int p = pbuf[j];
                if (p >= 0) bulk_store(a.recv + (int64_t)p * a.H + w.ch0, out, (uint32_t)w.chn);
            }
            bulk_commit();
            if (i + S < n) issue_load(i + S);  // every thread is past its reads of in[s]
        }
        const int gbase = w.ch0 / 128;
        for (int idx = tid; idx < a.k * G; idx += blockDim.x) {
            const int j = idx / G;
            const int g = idx - j * G;
            const int p = pbuf[j];
            if (p >= 0) a.scales[(int64_t)p * G_row + gbase + g] = sc[g];
        }
    }
    if (tid == 0) {
        bulk_wait_all();
        if (failed_at < n) drain_loads(bar, S, failed_at, issued);
    }
}

}  // namespace

cudaError_t launch_dispatch(const DispatchArgs &a0, bool fp8, int num_sms, cudaStream_t st) {
    DispatchArgs a = a0;
    if (a.nunits == 0) return cudaSuccess;
    cudaError_t err;
    int threads, per_sm = 0;
    size_t smem;
    if (fp8) {
        const int sc_bytes = ((a.chunk / 128) * 4 + 15) & ~15;
        smem = kHeaderBytes + (size_t)a.stages * a.chunk * 2 + (size_t)kOutBufs * (a.chunk + sc_bytes);
        threads = kFp8Threads;
        if ((err = cudaFuncSetAttribute(dispatch_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem)) != cudaSuccess)
            return err;
        if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_fp8_kernel, threads,
                                                                 smem)) != cudaSuccess)
            return err;
    } else {
        smem = kHeaderBytes + (size_t)a.stages * a.chunk * 2;
        threads = kBf16Threads;
        if ((err = cudaFuncSetAttribute(dispatch_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem)) != cudaSuccess)
            return err;
        if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_bf16_kernel, threads,
                                                                 smem)) != cudaSuccess)
            return err;
    }
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = (long long)per_sm * num_sms;
    if (grid > a.nunits) grid = a.nunits;
    if (fp8)
        dispatch_fp8_kernel<<<(unsigned)grid, threads, smem, st>>>(a);
    else
        dispatch_bf16_kernel<<<(unsigned)grid, threads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ep
