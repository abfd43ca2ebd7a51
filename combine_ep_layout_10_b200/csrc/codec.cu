// codec.cu -- fp32 -> FP8 e4m3 encoding exactly as the dispatch kernels do it.
//
// FP8 dispatch ("deepseek-ai/DeepEP", repolode, "Funciones clave") encodes
// every scaled value with the hardware's round-to-nearest-even, saturating
// e4m3 conversion (OCP FP8 E4M3: no infinities, finite overflow saturates to
// +-448, NaN stays NaN).  This kernel applies the same conversion, two values
// per instruction, to a caller's array, so callers can pre-quantise with the
// dispatch's rounding (ep_dispatch_ex accepts pre-quantised input) and the
// conversion itself can be checked value by value against a software encoder.
// One thread per 8 values: two 16-byte loads, four conversions, one 8-byte
// store; a scalar tail for the last n % 8 values.
#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kCodecThreads = 256;

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

__global__ void __launch_bounds__(kCodecThreads) e4m3_encode_kernel(const float *__restrict__ x,
                                                                    uint8_t *__restrict__ out, int64_t n) {
    pdl_wait_then_trigger();
    const int64_t i = ((int64_t)blockIdx.x * kCodecThreads + threadIdx.x) * 8;
    if (i + 8 <= n) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(x + i));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(x + i + 4));
        uint2 q;
        q.x = e4m3x2(a.x, a.y) | (e4m3x2(a.z, a.w) << 16);
        q.y = e4m3x2(b.x, b.y) | (e4m3x2(b.z, b.w) << 16);
        *reinterpret_cast<uint2 *>(out + i) = q;
    } else {
        for (int64_t j = i; j < n; ++j) out[j] = (uint8_t)(e4m3x2(__ldg(x + j), 0.0f) & 0xffu);
    }
}

}  // namespace

cudaError_t launch_e4m3_encode(const float *x, uint8_t *out, int64_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int64_t threads_needed = (n + 7) / 8;
    const int64_t blocks = (threads_needed + kCodecThreads - 1) / kCodecThreads;
    return launch_kernel(e4m3_encode_kernel, dim3((unsigned)blocks), dim3(kCodecThreads), 0, s, x, out, n);
}

}  // namespace ep
