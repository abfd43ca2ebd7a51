// api_common.cuh -- host-side helpers shared by the C ABI's translation
// units (ep_api.cu, peer_api.cu): argument checks, CUDA error mapping, the
// current device, and the stream-ordered memory pool of handles and plans.
#pragma once

#include <cstdio>
#include <cstdlib>

#include "ep_internal.cuh"

namespace ep {

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline ep_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return EP_OK;
    if (e == cudaErrorMemoryAllocation) return EP_ERR_OOM;
    if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver || e == cudaErrorNoKernelImageForDevice)
        return EP_ERR_NO_DEVICE;
    return EP_ERR_CUDA;
}

// The current device, checked to be a Blackwell sm_100 part.
inline ep_status current_device(int *dev, DeviceInfo *info) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_status(e);
    if ((e = device_info(*dev, info)) != cudaSuccess) return cuda_status(e);
    if (info->cc_major != 10) return EP_ERR_NO_DEVICE;
    return EP_OK;
}

// Host logging of each call's launch shape to stderr when the environment
// sets EP_DEBUG (to anything but "0"); read once per process.
inline bool debug_enabled() {
    static const bool on = [] {
        const char *v = std::getenv("EP_DEBUG");
        return v != nullptr && v[0] != '\0' && !(v[0] == '0' && v[1] == '\0');
    }();
    return on;
}

// Stream-ordered pool (one per device, kept for the life of the process)
// from which handles and plans take their device memory.
cudaError_t handle_pool(int device, cudaMemPool_t *out);

}  // namespace ep
