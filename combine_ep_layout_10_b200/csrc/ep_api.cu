// ep_api.cu -- the C ABI declared in include/ep.h: argument validation,
// ownership of handles, plans and peer tables, CUDA IPC, and kernel launches.
// Every step of the data path runs in the kernels of layout.cu, dispatch.cu,
// combine.cu, backward.cu, recv_topk.cu and plan.cu; nothing here touches
// tensor data on the host.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceInfo g_info[kMaxDevices];
bool g_have[kMaxDevices];
cudaMemPool_t g_pool[kMaxDevices];

// Stream-ordered pool for handle metadata, one per device, created on first
// use and kept for the life of the process.  Its release threshold is
// unbounded, so memory freed by ep_handle_free stays in the pool and the next
// layout's allocation is pure bookkeeping (the default pool would return it
// to the driver at every synchronisation and map it again).
cudaError_t handle_pool(int device, cudaMemPool_t *out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_pool[device] == nullptr) {
        cudaMemPoolProps props{};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = device;
        cudaMemPool_t pool = nullptr;
        cudaError_t e = cudaMemPoolCreate(&pool, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = ~0ull;
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return e;
        }
        g_pool[device] = pool;
    }
    *out = g_pool[device];
    return cudaSuccess;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

ep_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return EP_OK;
    if (e == cudaErrorMemoryAllocation) return EP_ERR_OOM;
    if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver || e == cudaErrorNoKernelImageForDevice)
        return EP_ERR_NO_DEVICE;
    return EP_ERR_CUDA;
}

// The current device, checked to be a Blackwell sm_100 part.
ep_status current_device(int *dev, DeviceInfo *info) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_status(e);
    if ((e = device_info(*dev, info)) != cudaSuccess) return cuda_status(e);
    if (info->cc_major != 10) return EP_ERR_NO_DEVICE;
    return EP_OK;
}

}  // namespace

cudaError_t device_info(int device, DeviceInfo *out) {
    if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_have[device]) {
        DeviceInfo d{};
        cudaError_t e;
        if ((e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, device)) != cudaSuccess)
            return e;
        if ((e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, device)) != cudaSuccess)
            return e;
        if ((e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, device)) != cudaSuccess)
            return e;
        if ((e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                        device)) != cudaSuccess)
            return e;
        g_info[device] = d;
        g_have[device] = true;
    }
    *out = g_info[device];
    return cudaSuccess;
}

}  // namespace ep

using namespace ep;

extern "C" {

const char *ep_status_str(ep_status s) {
    switch (s) {
        case EP_OK: return "EP_OK";
        case EP_ERR_INVALID_ARG: return "EP_ERR_INVALID_ARG";
        case EP_ERR_BAD_EXPERT_ID: return "EP_ERR_BAD_EXPERT_ID";
        case EP_ERR_CAPACITY: return "EP_ERR_CAPACITY";
        case EP_ERR_CUDA: return "EP_ERR_CUDA";
        case EP_ERR_OOM: return "EP_ERR_OOM";
        case EP_ERR_TIMEOUT: return "EP_ERR_TIMEOUT";
        case EP_ERR_NO_DEVICE: return "EP_ERR_NO_DEVICE";
        case EP_ERR_SCRATCH_LIMIT: return "EP_ERR_SCRATCH_LIMIT";
    }
    return "EP_ERR_UNKNOWN";
}

size_t ep_max_recv_rows(int T, int k, int E, int A, int C) {
    if (T < 0 || k < 1 || k > kMaxTopk || E < 1 || E > kMaxExperts || A < 1 || C < 0) return 0;
    if (C > 0) return (size_t)E * (size_t)C;
    return (size_t)T * (size_t)k + (size_t)E * (size_t)(A - 1);
}

ep_status ep_layout(const int32_t *topk_idx, int T, int k, int E, int R, int A, int C,
                    int32_t *out_cnt, int32_t *out_rank_tok, uint8_t *out_in_rank,
                    ep_handle **out_handle, ep_stream_t stream) {
    if (out_handle == nullptr) return EP_ERR_INVALID_ARG;
    *out_handle = nullptr;
    if (T < 0 || k < 1 || k > kMaxTopk || E < 1 || E > kMaxExperts || R < 1 || R > E || E % R != 0 ||
        A < 1 || C < 0 || (C > 0 && C % A != 0))
        return EP_ERR_INVALID_ARG;
    if ((int64_t)T * k >= (int64_t)1 << 31) return EP_ERR_INVALID_ARG;
    const size_t n_rows = ep_max_recv_rows(T, k, E, A, C);
    if (n_rows >= ((size_t)1 << 31)) return EP_ERR_INVALID_ARG;
    if (T > 0 && (topk_idx == nullptr || !aligned(topk_idx, 4))) return EP_ERR_INVALID_ARG;
    if ((out_cnt && !aligned(out_cnt, 4)) || (out_rank_tok && !aligned(out_rank_tok, 4)))
        return EP_ERR_INVALID_ARG;

    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;

    const LayoutGeometry geo = layout_geometry(T, k, E, R);
    const int ntiles = geo.ntiles;

    // One stream-ordered allocation, every array 256-byte aligned.
    size_t off = 0;
    auto carve = [&](size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    };
    const size_t o_err = carve(4);
    const size_t o_pos = carve((size_t)T * k * 4);
    const size_t o_src = carve(n_rows * 4);
    const size_t o_seg = carve((size_t)(E + 1) * 4);
    const size_t o_roff = carve((size_t)(R + 1) * 4);
    const size_t o_cnt = carve((size_t)E * 4);
    const size_t o_tcnt = carve((size_t)ntiles * E * 4);
    const size_t o_trank = carve((size_t)ntiles * R * 4);
    const size_t o_terr = carve((size_t)ntiles * 4);
    void *block = nullptr;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = handle_pool(dev, &pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&block, off, pool, stream);
    if (e != cudaSuccess) return cuda_status(e);

    ep_handle *h = new (std::nothrow) ep_handle;
    if (h == nullptr) {
        cudaFreeAsync(block, stream);
        return EP_ERR_OOM;
    }
    unsigned char *b = static_cast<unsigned char *>(block);
    h->T = T; h->k = k; h->E = E; h->R = R; h->align = A; h->capacity = C;
    h->experts_per_rank = E / R;
    h->tile_tokens = geo.tile_tokens;
    h->ntiles = ntiles;
    h->n_rows = (int64_t)n_rows;
    h->device = dev;
    h->stream = stream;
    h->block = block;
    h->err = reinterpret_cast<uint32_t *>(b + o_err);
    h->pos = reinterpret_cast<int32_t *>(b + o_pos);
    h->src_idx = reinterpret_cast<int32_t *>(b + o_src);
    h->seg = reinterpret_cast<int32_t *>(b + o_seg);
    h->rank_off = reinterpret_cast<int32_t *>(b + o_roff);
    h->cnt = reinterpret_cast<int32_t *>(b + o_cnt);
    h->tile_cnt = reinterpret_cast<int32_t *>(b + o_tcnt);
    h->tile_rank = reinterpret_cast<int32_t *>(b + o_trank);
    h->tile_err = reinterpret_cast<uint32_t *>(b + o_terr);

    LayoutArgs a{};
    a.topk_idx = topk_idx;
    a.T = T; a.k = k; a.E = E; a.R = R; a.epr = E / R; a.align = A; a.capacity = C;
    a.tile_tokens = geo.tile_tokens;
    a.ntiles = ntiles;
    a.sub_tokens = geo.sub_tokens;
    a.pos_warps = geo.pos_warps;
    a.ids_in_smem = geo.ids_in_smem;
    a.small = geo.small;
    a.n_rows = (int64_t)n_rows;
    a.pos = h->pos; a.src_idx = h->src_idx; a.seg = h->seg; a.rank_off = h->rank_off;
    a.cnt = h->cnt; a.tile_cnt = h->tile_cnt; a.tile_rank = h->tile_rank;
    a.tile_err = h->tile_err; a.err = h->err;
    a.out_cnt = out_cnt;
    a.out_rank_tok = out_rank_tok;
    a.out_in_rank = out_in_rank;

    e = launch_layout(a, stream);  // also (re)initialises the error word
    if (e != cudaSuccess) {
        cudaFreeAsync(block, stream);
        delete h;
        return cuda_status(e);
    }
    *out_handle = h;
    return EP_OK;
}

ep_status ep_dispatch_ex(const ep_handle *h, const void *x, const float *x_scales, int H, int in_format,
                         int out_format, void *recv_x, float *recv_scales, int64_t scale_row_stride,
                         int64_t scale_group_stride, int32_t *recv_src_idx, size_t recv_rows, int num_sms,
                         ep_stream_t stream) {
    if (h == nullptr || H < 8 || H % 8 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
    const bool in_fp8 = in_format == EP_FORMAT_E4M3;
    const bool out_fp8 = out_format == EP_FORMAT_E4M3;
    if ((in_format != EP_FORMAT_BF16 && !in_fp8) || (out_format != EP_FORMAT_BF16 && !out_fp8))
        return EP_ERR_INVALID_ARG;
    if (in_fp8 && !out_fp8) return EP_ERR_INVALID_ARG;  // no dequantising dispatch
    if (out_fp8 && H % 128 != 0) return EP_ERR_INVALID_ARG;
    if (recv_rows < (size_t)h->n_rows) return EP_ERR_INVALID_ARG;
    const int64_t G = H / 128;
    if (out_fp8) {
        // Non-overlapping scale layouts only: row-major-like or column-major-like.
        const bool row_like = scale_group_stride == 1 && scale_row_stride >= G;
        const bool col_like = scale_row_stride == 1 && scale_group_stride >= (int64_t)recv_rows;
        if (!(row_like || col_like)) return EP_ERR_INVALID_ARG;
    }
    if (h->T > 0) {
        if (x == nullptr || recv_x == nullptr || !aligned(x, 16) || !aligned(recv_x, 16))
            return EP_ERR_INVALID_ARG;
        if (out_fp8 && (recv_scales == nullptr || !aligned(recv_scales, 4))) return EP_ERR_INVALID_ARG;
        if (in_fp8 && (x_scales == nullptr || !aligned(x_scales, 4))) return EP_ERR_INVALID_ARG;
    }
    if (recv_src_idx != nullptr && !aligned(recv_src_idx, 4)) return EP_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != h->device) return EP_ERR_INVALID_ARG;

    int chunk, nchunks;
    dispatch_chunking(h->T, H, out_fp8 ? 128 : 8, info.num_sms, &chunk, &nchunks);

    DispatchArgs a{};
    a.x = static_cast<const uint8_t *>(x);
    a.x_scales = x_scales;
    a.pos = h->pos;
    a.recv = static_cast<uint8_t *>(recv_x);
    a.scales = recv_scales;
    a.s_row = scale_row_stride;
    a.s_grp = scale_group_stride;
    a.mode = !out_fp8 ? kDispatchCopyBf16 : in_fp8 ? kDispatchCopyFp8 : kDispatchQuantFp8;
    a.num_sms = num_sms;
    a.T = h->T; a.k = h->k; a.H = H;
    a.chunk = chunk;
    a.nchunks = nchunks;
    if ((int64_t)h->T * a.nchunks >= ((int64_t)1 << 31)) return EP_ERR_INVALID_ARG;
    a.nunits = h->T * a.nchunks;
    cudaError_t e = launch_dispatch(a, stream);
    if (e == cudaSuccess && recv_src_idx != nullptr && h->n_rows > 0)
        e = cudaMemcpyAsync(recv_src_idx, h->src_idx, (size_t)h->n_rows * 4, cudaMemcpyDeviceToDevice, stream);
    return cuda_status(e);
}

ep_status ep_dispatch(const ep_handle *h, const void *x, int H, int use_fp8, void *recv_x,
                      float *recv_scales, int32_t *recv_src_idx, size_t recv_rows, ep_stream_t stream) {
    return ep_dispatch_ex(h, x, nullptr, H, EP_FORMAT_BF16, use_fp8 ? EP_FORMAT_E4M3 : EP_FORMAT_BF16, recv_x,
                          recv_scales, H / 128, 1, recv_src_idx, recv_rows, 0, stream);
}

ep_status ep_combine_ex(const ep_handle *h, const void *y, const float *topk_w, int H, size_t recv_rows,
                        void *out, int num_sms, ep_stream_t stream) {
    if (h == nullptr || H < 8 || H % 8 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
    if (recv_rows < (size_t)h->n_rows) return EP_ERR_INVALID_ARG;
    if (h->T > 0) {
        if (y == nullptr || out == nullptr || topk_w == nullptr) return EP_ERR_INVALID_ARG;
        if (!aligned(y, 16) || !aligned(out, 16) || !aligned(topk_w, 4)) return EP_ERR_INVALID_ARG;
    }
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != h->device) return EP_ERR_INVALID_ARG;

    CombineArgs a{};
    a.y = static_cast<const uint8_t *>(y);
    a.w = topk_w;
    a.pos = h->pos;
    a.out = static_cast<uint8_t *>(out);
    a.T = h->T; a.k = h->k; a.H = H;
    a.nvec = H / 8;
    a.vpt = EP_COMBINE_VPT;
    a.blocks_per_token = (a.nvec + EP_COMBINE_THREADS * a.vpt - 1) / (EP_COMBINE_THREADS * a.vpt);
    if ((int64_t)h->T * a.blocks_per_token >= ((int64_t)1 << 31)) return EP_ERR_INVALID_ARG;
    a.num_sms = num_sms;
    return cuda_status(launch_combine(a, stream));
}

ep_status ep_combine(const ep_handle *h, const void *y, const float *topk_w, int H, size_t recv_rows,
                     void *out, ep_stream_t stream) {
    return ep_combine_ex(h, y, topk_w, H, recv_rows, out, 0, stream);
}

ep_status ep_dispatch_backward(const ep_handle *h, const void *grad_recv, int H, size_t recv_rows,
                               void *grad_x, ep_stream_t stream) {
    if (h == nullptr || H < 8 || H % 8 != 0) return EP_ERR_INVALID_ARG;
    if (recv_rows < (size_t)h->n_rows) return EP_ERR_INVALID_ARG;
    if (h->T > 0 && (grad_recv == nullptr || grad_x == nullptr || !aligned(grad_recv, 16) || !aligned(grad_x, 16)))
        return EP_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != h->device) return EP_ERR_INVALID_ARG;
    CombineArgs a{};
    a.y = static_cast<const uint8_t *>(grad_recv);
    a.w = nullptr;  // unit weights
    a.pos = h->pos;
    a.out = static_cast<uint8_t *>(grad_x);
    a.T = h->T; a.k = h->k; a.H = H;
    a.nvec = H / 8;
    a.vpt = EP_COMBINE_VPT;
    a.blocks_per_token = (a.nvec + EP_COMBINE_THREADS * a.vpt - 1) / (EP_COMBINE_THREADS * a.vpt);
    if ((int64_t)h->T * a.blocks_per_token >= ((int64_t)1 << 31)) return EP_ERR_INVALID_ARG;
    a.num_sms = 0;
    return cuda_status(launch_combine(a, stream));
}

ep_status ep_combine_backward(const ep_handle *h, const void *grad_out, const void *y, const float *topk_w,
                              int H, size_t recv_rows, void *grad_y, float *grad_w, ep_stream_t stream) {
    if (h == nullptr || H < 8 || H % 8 != 0) return EP_ERR_INVALID_ARG;
    if (recv_rows < (size_t)h->n_rows) return EP_ERR_INVALID_ARG;
    if (h->T > 0) {
        if (grad_out == nullptr || topk_w == nullptr || grad_y == nullptr) return EP_ERR_INVALID_ARG;
        if (!aligned(grad_out, 16) || !aligned(grad_y, 16) || !aligned(topk_w, 4)) return EP_ERR_INVALID_ARG;
        if (grad_w != nullptr && (y == nullptr || !aligned(y, 16) || !aligned(grad_w, 4))) return EP_ERR_INVALID_ARG;
    }
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != h->device) return EP_ERR_INVALID_ARG;
    CombineBwdArgs a{};
    a.grad_out = static_cast<const uint8_t *>(grad_out);
    a.y = static_cast<const uint8_t *>(y);
    a.w = topk_w;
    a.pos = h->pos;
    a.grad_y = static_cast<uint8_t *>(grad_y);
    a.grad_w = grad_w;
    a.T = h->T; a.k = h->k; a.H = H;
    return cuda_status(launch_combine_backward(a, stream));
}

ep_status ep_dispatch_topk(const ep_handle *h, const float *topk_w, int32_t *recv_topk_idx,
                           float *recv_topk_weights, int32_t *recv_slot, size_t recv_rows,
                           ep_stream_t stream) {
    if (h == nullptr) return EP_ERR_INVALID_ARG;
    if (recv_rows < (size_t)h->n_rows) return EP_ERR_INVALID_ARG;
    if (recv_topk_weights != nullptr && h->T > 0 && (topk_w == nullptr || !aligned(topk_w, 4)))
        return EP_ERR_INVALID_ARG;
    if ((recv_topk_idx && !aligned(recv_topk_idx, 4)) || (recv_topk_weights && !aligned(recv_topk_weights, 4)) ||
        (recv_slot && !aligned(recv_slot, 4)))
        return EP_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != h->device) return EP_ERR_INVALID_ARG;
    if (recv_topk_idx == nullptr && recv_topk_weights == nullptr && recv_slot == nullptr) return EP_OK;
    RecvTopkArgs a{};
    a.src_idx = h->src_idx;
    a.pos = h->pos;
    a.seg = h->seg;
    a.w = recv_topk_weights != nullptr ? topk_w : nullptr;
    a.out_idx = recv_topk_idx;
    a.out_w = recv_topk_weights;
    a.out_slot = recv_slot;
    a.T = h->T; a.k = h->k; a.E = h->E;
    a.n_rows = h->n_rows;
    return cuda_status(launch_recv_topk(a, stream));
}

void ep_handle_free(ep_handle *h) {
    if (h == nullptr) return;
    if (h->block != nullptr) {
        if (cudaFreeAsync(h->block, h->stream) != cudaSuccess) {
            (void)cudaGetLastError();
            cudaFree(h->block);
        }
    }
    delete h;
}

ep_status ep_handle_get_info(const ep_handle *h, ep_handle_info *info) {
    if (h == nullptr || info == nullptr) return EP_ERR_INVALID_ARG;
    info->num_tokens = h->T;
    info->num_topk = h->k;
    info->num_experts = h->E;
    info->num_ranks = h->R;
    info->expert_alignment = h->align;
    info->capacity = h->capacity;
    info->num_recv_rows = (size_t)h->n_rows;
    return EP_OK;
}

ep_status ep_handle_export(const ep_handle *h, int32_t *pos, int32_t *src_idx, int32_t *seg,
                           int32_t *rank_off, ep_stream_t stream) {
    if (h == nullptr) return EP_ERR_INVALID_ARG;
    cudaError_t e = cudaSuccess;
    if (pos && h->T > 0)
        e = cudaMemcpyAsync(pos, h->pos, (size_t)h->T * h->k * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess && src_idx && h->n_rows > 0)
        e = cudaMemcpyAsync(src_idx, h->src_idx, (size_t)h->n_rows * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess && seg)
        e = cudaMemcpyAsync(seg, h->seg, (size_t)(h->E + 1) * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess && rank_off)
        e = cudaMemcpyAsync(rank_off, h->rank_off, (size_t)(h->R + 1) * 4, cudaMemcpyDeviceToDevice, stream);
    return cuda_status(e);
}

ep_status ep_handle_counts_host(const ep_handle *h, int32_t *host_counts, ep_stream_t stream) {
    if (h == nullptr || host_counts == nullptr) return EP_ERR_INVALID_ARG;
    cudaError_t e = cudaMemcpyAsync(host_counts, h->cnt, (size_t)h->E * 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    return cuda_status(e);
}

ep_status ep_handle_check(const ep_handle *h, ep_stream_t stream) {
    if (h == nullptr) return EP_ERR_INVALID_ARG;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, h->err, 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_status(e);
    if (word & kErrBadExpertId) return EP_ERR_BAD_EXPERT_ID;
    if (word & kErrCapacity) return EP_ERR_CAPACITY;
    if (word & kErrTimeout) return EP_ERR_TIMEOUT;
    return EP_OK;
}

}  // extern "C"

/* ------------------------------------------------------------------------- */
/* Expert parallelism across GPUs                                             */
/* ------------------------------------------------------------------------- */

extern "C" {

size_t ep_peer_max_recv_rows(int64_t total_tokens, int k, int E, int world, int A, int C) {
    if (total_tokens < 0 || k < 1 || E < 1 || world < 1 || E % world != 0 || A < 1 || C < 0) return 0;
    const int64_t epr = E / world;
    if (C > 0) return (size_t)(epr * C);
    return (size_t)(total_tokens * k + epr * (A - 1));
}

ep_status ep_plan_create(const ep_handle *h, const int32_t *topk_idx, const int32_t *all_counts, int rank,
                         int world, int A, int C, size_t recv_rows, ep_plan **out, ep_stream_t stream) {
    if (out == nullptr) return EP_ERR_INVALID_ARG;
    *out = nullptr;
    if (h == nullptr || world < 1 || rank < 0 || rank >= world || A < 1 || C < 0) return EP_ERR_INVALID_ARG;
    if (C > 0 && C % A != 0) return EP_ERR_INVALID_ARG;
    // The local layout must be the packed, unaligned one over `world` ranks:
    // its positions then count each expert's local slots from 0.
    if (h->R != world || h->align != 1 || h->capacity != 0) return EP_ERR_INVALID_ARG;
    if (recv_rows >= ((size_t)1 << 31)) return EP_ERR_INVALID_ARG;
    if (all_counts == nullptr || !aligned(all_counts, 4)) return EP_ERR_INVALID_ARG;
    if (h->T > 0 && (topk_idx == nullptr || !aligned(topk_idx, 4))) return EP_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != h->device) return EP_ERR_INVALID_ARG;

    ep_plan *p = new (std::nothrow) ep_plan{};
    if (p == nullptr) return EP_ERR_OOM;
    p->T = h->T; p->k = h->k; p->E = h->E; p->world = world; p->rank = rank;
    p->epr = h->E / world; p->align = A; p->capacity = C;
    p->recv_rows = (int64_t)recv_rows;
    p->device = dev;
    p->stream = stream;
    size_t off = 0;
    auto carve = [&](size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    };
    const size_t o_err = carve(4);
    const size_t o_dst = carve((size_t)h->T * h->k * sizeof(int2));
    const size_t o_pre = carve((size_t)h->E * 4);
    const size_t o_offs = carve((size_t)h->E * 4);
    const size_t o_seg = carve((size_t)(p->epr + 1) * 4);
    const size_t o_cnt = carve((size_t)p->epr * 4);
    cudaMemPool_t pool;
    cudaError_t e = handle_pool(dev, &pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&p->block, off, pool, stream);
    if (e != cudaSuccess) {
        delete p;
        return cuda_status(e);
    }
    uint8_t *b = static_cast<uint8_t *>(p->block);
    p->err = reinterpret_cast<uint32_t *>(b + o_err);
    p->dst = reinterpret_cast<int2 *>(b + o_dst);
    p->pre = reinterpret_cast<int32_t *>(b + o_pre);
    p->offs = reinterpret_cast<int32_t *>(b + o_offs);
    p->recv_seg = reinterpret_cast<int32_t *>(b + o_seg);
    p->recv_cnt = reinterpret_cast<int32_t *>(b + o_cnt);
    e = cudaMemsetAsync(p->err, 0, 4, stream);
    if (e == cudaSuccess) {
        PlanArgs a{};
        a.topk_idx = topk_idx;
        a.pos = h->pos;
        a.seg = h->seg;
        a.counts = all_counts;
        a.T = p->T; a.k = p->k; a.E = p->E; a.world = world; a.rank = rank; a.epr = p->epr;
        a.align = A; a.capacity = C;
        a.recv_rows = p->recv_rows;
        a.dst = p->dst; a.pre = p->pre; a.offs = p->offs; a.recv_seg = p->recv_seg; a.recv_cnt = p->recv_cnt;
        a.err = p->err;
        e = launch_plan(a, stream);
    }
    if (e != cudaSuccess) {
        ep_plan_free(p);
        return cuda_status(e);
    }
    *out = p;
    return EP_OK;
}

void ep_plan_free(ep_plan *p) {
    if (p == nullptr) return;
    if (p->block != nullptr) {
        if (cudaFreeAsync(p->block, p->stream) != cudaSuccess) {
            (void)cudaGetLastError();
            cudaFree(p->block);
        }
    }
    delete p;
}

ep_status ep_plan_export(const ep_plan *p, int32_t *dst, int32_t *recv_seg, int32_t *recv_counts,
                         ep_stream_t stream) {
    if (p == nullptr) return EP_ERR_INVALID_ARG;
    cudaError_t e = cudaSuccess;
    if (dst && p->T > 0)
        e = cudaMemcpyAsync(dst, p->dst, (size_t)p->T * p->k * sizeof(int2), cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess && recv_seg)
        e = cudaMemcpyAsync(recv_seg, p->recv_seg, (size_t)(p->epr + 1) * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess && recv_counts)
        e = cudaMemcpyAsync(recv_counts, p->recv_cnt, (size_t)p->epr * 4, cudaMemcpyDeviceToDevice, stream);
    return cuda_status(e);
}

ep_status ep_plan_recv_rows_host(const ep_plan *p, int64_t *rows, ep_stream_t stream) {
    if (p == nullptr || rows == nullptr) return EP_ERR_INVALID_ARG;
    int32_t n = 0;
    cudaError_t e = cudaMemcpyAsync(&n, p->recv_seg + p->epr, 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_status(e);
    *rows = n;
    return EP_OK;
}

ep_status ep_plan_check(const ep_plan *p, ep_stream_t stream) {
    if (p == nullptr) return EP_ERR_INVALID_ARG;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, p->err, 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_status(e);
    if (word & kErrCapacity) return EP_ERR_CAPACITY;
    return EP_OK;
}

}  // extern "C"

// The peer table of the ABI: every rank's buffers as mapped in this process.
struct ep_peers {
    int world;
    int device;
    size_t recv_rows;
    void *block;                 // device copy of the three pointer tables
    uint8_t *const *recv_x;      // [world]
    float *const *recv_scales;   // [world] or nullptr
    const uint8_t *const *y;     // [world] or nullptr
    uint8_t *const *grad_y;      // [world] or nullptr
};

extern "C" {

ep_status ep_peers_create(int world, void *const *recv_x, float *const *recv_scales, void *const *y,
                          void *const *grad_y, size_t recv_rows, ep_peers **out) {
    if (out == nullptr) return EP_ERR_INVALID_ARG;
    *out = nullptr;
    if (world < 1 || recv_x == nullptr) return EP_ERR_INVALID_ARG;
    for (int r = 0; r < world; ++r) {
        if (recv_x[r] == nullptr || !aligned(recv_x[r], 16)) return EP_ERR_INVALID_ARG;
        if (recv_scales && (recv_scales[r] == nullptr || !aligned(recv_scales[r], 16))) return EP_ERR_INVALID_ARG;
        if (y && (y[r] == nullptr || !aligned(y[r], 16))) return EP_ERR_INVALID_ARG;
        if (grad_y && (grad_y[r] == nullptr || !aligned(grad_y[r], 16))) return EP_ERR_INVALID_ARG;
    }
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    ep_peers *p = new (std::nothrow) ep_peers{};
    if (p == nullptr) return EP_ERR_OOM;
    p->world = world;
    p->device = dev;
    p->recv_rows = recv_rows;
    const size_t n = (size_t)world;
    uintptr_t *host = static_cast<uintptr_t *>(std::malloc(4 * n * sizeof(uintptr_t)));
    if (host == nullptr) {
        delete p;
        return EP_ERR_OOM;
    }
    for (size_t r = 0; r < n; ++r) {
        host[r] = reinterpret_cast<uintptr_t>(recv_x[r]);
        host[n + r] = recv_scales ? reinterpret_cast<uintptr_t>(recv_scales[r]) : 0;
        host[2 * n + r] = y ? reinterpret_cast<uintptr_t>(y[r]) : 0;
        host[3 * n + r] = grad_y ? reinterpret_cast<uintptr_t>(grad_y[r]) : 0;
    }
    cudaError_t e = cudaMalloc(&p->block, 4 * n * sizeof(uintptr_t));
    if (e == cudaSuccess) e = cudaMemcpy(p->block, host, 4 * n * sizeof(uintptr_t), cudaMemcpyHostToDevice);
    std::free(host);
    if (e != cudaSuccess) {
        if (p->block) cudaFree(p->block);
        delete p;
        return cuda_status(e);
    }
    uintptr_t *tab = static_cast<uintptr_t *>(p->block);
    p->recv_x = reinterpret_cast<uint8_t *const *>(tab);
    p->recv_scales = recv_scales ? reinterpret_cast<float *const *>(tab + n) : nullptr;
    p->y = y ? reinterpret_cast<const uint8_t *const *>(tab + 2 * n) : nullptr;
    p->grad_y = grad_y ? reinterpret_cast<uint8_t *const *>(tab + 3 * n) : nullptr;
    *out = p;
    return EP_OK;
}

void ep_peers_free(ep_peers *p) {
    if (p == nullptr) return;
    if (p->block) cudaFree(p->block);
    delete p;
}

ep_status ep_dispatch_peer(const ep_plan *plan, const ep_peers *peers, const void *x, const float *x_scales,
                           int H, int in_format, int out_format, int num_sms, ep_stream_t stream) {
    if (plan == nullptr || peers == nullptr || H < 8 || H % 8 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
    if (peers->world != plan->world || peers->recv_rows < (size_t)plan->recv_rows) return EP_ERR_INVALID_ARG;
    const bool in_fp8 = in_format == EP_FORMAT_E4M3;
    const bool out_fp8 = out_format == EP_FORMAT_E4M3;
    if ((in_format != EP_FORMAT_BF16 && !in_fp8) || (out_format != EP_FORMAT_BF16 && !out_fp8))
        return EP_ERR_INVALID_ARG;
    if (in_fp8 && !out_fp8) return EP_ERR_INVALID_ARG;
    if (out_fp8 && (H % 128 != 0 || peers->recv_scales == nullptr)) return EP_ERR_INVALID_ARG;
    if (plan->T > 0) {
        if (x == nullptr || !aligned(x, 16)) return EP_ERR_INVALID_ARG;
        if (in_fp8 && (x_scales == nullptr || !aligned(x_scales, 4))) return EP_ERR_INVALID_ARG;
    }
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != plan->device || dev != peers->device) return EP_ERR_INVALID_ARG;

    int chunk, nchunks;
    dispatch_chunking(plan->T, H, out_fp8 ? 128 : 8, info.num_sms, &chunk, &nchunks);
    DispatchArgs a{};
    a.x = static_cast<const uint8_t *>(x);
    a.x_scales = x_scales;
    a.dst = plan->dst;
    a.peer_recv = peers->recv_x;
    a.peer_scales = out_fp8 ? peers->recv_scales : nullptr;
    a.s_row = H / 128;
    a.s_grp = 1;
    a.mode = !out_fp8 ? kDispatchCopyBf16 : in_fp8 ? kDispatchCopyFp8 : kDispatchQuantFp8;
    a.num_sms = num_sms;
    a.T = plan->T; a.k = plan->k; a.H = H;
    a.chunk = chunk;
    a.nchunks = nchunks;
    if ((int64_t)plan->T * a.nchunks >= ((int64_t)1 << 31)) return EP_ERR_INVALID_ARG;
    a.nunits = plan->T * a.nchunks;
    return cuda_status(launch_dispatch_peer(a, stream));
}

ep_status ep_combine_peer(const ep_plan *plan, const ep_peers *peers, const float *topk_w, int H, void *out,
                          int num_sms, ep_stream_t stream) {
    if (plan == nullptr || peers == nullptr || H < 8 || H % 8 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
    if (peers->world != plan->world || peers->y == nullptr || peers->recv_rows < (size_t)plan->recv_rows)
        return EP_ERR_INVALID_ARG;
    if (plan->T > 0) {
        if (out == nullptr || !aligned(out, 16)) return EP_ERR_INVALID_ARG;
        if (topk_w != nullptr && !aligned(topk_w, 4)) return EP_ERR_INVALID_ARG;
    }
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != plan->device || dev != peers->device) return EP_ERR_INVALID_ARG;
    CombineArgs a{};
    a.w = topk_w;  // nullptr: unit weights (the backward of ep_dispatch_peer)
    a.src = plan->dst;
    a.peer_y = peers->y;
    a.out = static_cast<uint8_t *>(out);
    a.T = plan->T; a.k = plan->k; a.H = H;
    a.nvec = H / 8;
    a.vpt = 1;
    a.blocks_per_token = (a.nvec + EP_COMBINE_THREADS - 1) / EP_COMBINE_THREADS;
    if ((int64_t)plan->T * a.blocks_per_token >= ((int64_t)1 << 31)) return EP_ERR_INVALID_ARG;
    a.num_sms = num_sms;
    return cuda_status(launch_combine_peer(a, stream));
}

ep_status ep_combine_backward_peer(const ep_plan *plan, const ep_peers *peers, const void *grad_out,
                                   const float *topk_w, int H, float *grad_w, ep_stream_t stream) {
    if (plan == nullptr || peers == nullptr || H < 8 || H % 8 != 0) return EP_ERR_INVALID_ARG;
    if (peers->world != plan->world || peers->grad_y == nullptr || peers->recv_rows < (size_t)plan->recv_rows)
        return EP_ERR_INVALID_ARG;
    if (grad_w != nullptr && peers->y == nullptr) return EP_ERR_INVALID_ARG;
    if (plan->T > 0) {
        if (grad_out == nullptr || topk_w == nullptr) return EP_ERR_INVALID_ARG;
        if (!aligned(grad_out, 16) || !aligned(topk_w, 4)) return EP_ERR_INVALID_ARG;
        if (grad_w != nullptr && !aligned(grad_w, 4)) return EP_ERR_INVALID_ARG;
    }
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != plan->device || dev != peers->device) return EP_ERR_INVALID_ARG;
    CombineBwdArgs a{};
    a.grad_out = static_cast<const uint8_t *>(grad_out);
    a.w = topk_w;
    a.grad_w = grad_w;
    a.dst = plan->dst;
    a.peer_y = peers->y;
    a.peer_grad_y = peers->grad_y;
    a.T = plan->T; a.k = plan->k; a.H = H;
    return cuda_status(launch_combine_backward_peer(a, stream));
}

ep_status ep_ipc_export(const void *ptr, void *handle, uint64_t *offset) {
    if (ptr == nullptr || handle == nullptr || offset == nullptr) return EP_ERR_INVALID_ARG;
    static_assert(sizeof(cudaIpcMemHandle_t) == EP_IPC_HANDLE_BYTES, "IPC handle size");
    // The handle names the whole allocation that holds ptr; the offset of ptr
    // inside it comes from the driver's address-range query.
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || fn == nullptr || q != cudaDriverEntryPointSuccess) return EP_ERR_CUDA;
    using range_fn = int (*)(unsigned long long *, size_t *, unsigned long long);
    unsigned long long base = 0;
    size_t size = 0;
    if (reinterpret_cast<range_fn>(fn)(&base, &size, reinterpret_cast<unsigned long long>(ptr)) != 0)
        return EP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    e = cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base));
    if (e != cudaSuccess) return cuda_status(e);
    std::memcpy(handle, &h, sizeof(h));
    *offset = reinterpret_cast<unsigned long long>(ptr) - base;
    return EP_OK;
}

ep_status ep_ipc_import(const void *handle, uint64_t offset, void **ptr) {
    if (handle == nullptr || ptr == nullptr) return EP_ERR_INVALID_ARG;
    *ptr = nullptr;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void *base = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_status(e);
    *ptr = static_cast<uint8_t *>(base) + offset;
    return EP_OK;
}

ep_status ep_ipc_release(void *ptr, uint64_t offset) {
    if (ptr == nullptr) return EP_ERR_INVALID_ARG;
    return cuda_status(cudaIpcCloseMemHandle(static_cast<uint8_t *>(ptr) - offset));
}

}  // extern "C"
