// peer_api.cu -- the multi-GPU part of the C ABI declared in include/ep.h:
// plans (where every local slot goes on which rank), peer tables, the
// peer-addressed dispatch, combine and combine backward, and CUDA IPC.  The
// data path runs in the kernels of plan.cu, dispatch.cu, combine.cu and
// backward.cu; nothing here touches tensor data on the host.
#include <cstdlib>
#include <cstring>
#include <new>

#include "api_common.cuh"

using namespace ep;

/* ------------------------------------------------------------------------- */
/* Expert parallelism across GPUs                                             */
/* ------------------------------------------------------------------------- */

extern "C" {

size_t ep_peer_max_recv_rows(int64_t total_tokens, int k, int E, int world, int A, int C) {
    if (total_tokens < 0 || k < 1 || k > kMaxTopk || E < 1 || E > kMaxExperts || world < 1 || E % world != 0 ||
        A < 1 || C < 0)
        return 0;
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
        if (debug_enabled())
            std::fprintf(stderr, "ep: plan rank=%d world=%d T=%d k=%d E=%d align=%d capacity=%d recv_rows=%lld\n",
                         rank, world, p->T, p->k, p->E, A, C, (long long)recv_rows);
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
    void *topk_block;            // device copy of the per-row output tables (ep_peers_set_topk)
    int32_t *const *topk_idx;    // [world] or nullptr
    float *const *topk_w;        // [world] or nullptr
    int32_t *const *topk_src;    // [world] or nullptr
    int32_t *const *topk_slot;   // [world] or nullptr
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
    if (p->topk_block) cudaFree(p->topk_block);
    delete p;
}

ep_status ep_peers_set_topk(ep_peers *p, int32_t *const *recv_topk_idx, float *const *recv_topk_weights,
                            int32_t *const *recv_src_rank, int32_t *const *recv_slot) {
    if (p == nullptr) return EP_ERR_INVALID_ARG;
    const void *const *tabs[4] = {reinterpret_cast<const void *const *>(recv_topk_idx),
                                  reinterpret_cast<const void *const *>(recv_topk_weights),
                                  reinterpret_cast<const void *const *>(recv_src_rank),
                                  reinterpret_cast<const void *const *>(recv_slot)};
    for (const void *const *t : tabs)
        if (t != nullptr)
            for (int r = 0; r < p->world; ++r)
                if (t[r] == nullptr || !aligned(t[r], 4)) return EP_ERR_INVALID_ARG;
    const size_t n = (size_t)p->world;
    uintptr_t *host = static_cast<uintptr_t *>(std::malloc(4 * n * sizeof(uintptr_t)));
    if (host == nullptr) return EP_ERR_OOM;
    for (int i = 0; i < 4; ++i)
        for (size_t r = 0; r < n; ++r) host[i * n + r] = tabs[i] ? reinterpret_cast<uintptr_t>(tabs[i][r]) : 0;
    void *block = nullptr;
    cudaError_t e = cudaMalloc(&block, 4 * n * sizeof(uintptr_t));
    if (e == cudaSuccess) e = cudaMemcpy(block, host, 4 * n * sizeof(uintptr_t), cudaMemcpyHostToDevice);
    std::free(host);
    if (e != cudaSuccess) {
        if (block) cudaFree(block);
        return cuda_status(e);
    }
    if (p->topk_block) cudaFree(p->topk_block);
    p->topk_block = block;
    uintptr_t *tab = static_cast<uintptr_t *>(block);
    p->topk_idx = recv_topk_idx ? reinterpret_cast<int32_t *const *>(tab) : nullptr;
    p->topk_w = recv_topk_weights ? reinterpret_cast<float *const *>(tab + n) : nullptr;
    p->topk_src = recv_src_rank ? reinterpret_cast<int32_t *const *>(tab + 2 * n) : nullptr;
    p->topk_slot = recv_slot ? reinterpret_cast<int32_t *const *>(tab + 3 * n) : nullptr;
    return EP_OK;
}

ep_status ep_dispatch_topk_peer(const ep_plan *plan, const ep_peers *peers, const int32_t *topk_idx,
                                const float *topk_w, ep_stream_t stream) {
    if (plan == nullptr || peers == nullptr || peers->world != plan->world) return EP_ERR_INVALID_ARG;
    if (peers->recv_rows < (size_t)plan->recv_rows) return EP_ERR_INVALID_ARG;
    if (peers->topk_idx == nullptr && peers->topk_w == nullptr && peers->topk_src == nullptr &&
        peers->topk_slot == nullptr)
        return EP_ERR_INVALID_ARG;  // no tables registered (ep_peers_set_topk)
    if (plan->T > 0) {
        if (topk_idx == nullptr || !aligned(topk_idx, 4)) return EP_ERR_INVALID_ARG;
        if (peers->topk_w != nullptr && (topk_w == nullptr || !aligned(topk_w, 4))) return EP_ERR_INVALID_ARG;
    }
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != plan->device || dev != peers->device) return EP_ERR_INVALID_ARG;
    RecvTopkPeerArgs a{};
    a.dst = plan->dst;
    a.topk_idx = topk_idx;
    a.w = topk_w;
    a.T = plan->T; a.k = plan->k; a.rank = plan->rank; a.epr = plan->epr; a.capacity = plan->capacity;
    a.p_idx = peers->topk_idx;
    a.p_w = peers->topk_w;
    a.p_src = peers->topk_src;
    a.p_slot = peers->topk_slot;
    a.recv_seg = plan->recv_seg;
    a.recv_cnt = plan->recv_cnt;
    return cuda_status(launch_recv_topk_peer(a, stream));
}

ep_status ep_dispatch_peer(const ep_plan *plan, const ep_peers *peers, const void *x, const float *x_scales,
                           int H, int in_format, int out_format, int64_t scale_row_stride,
                           int64_t scale_group_stride, int num_sms, ep_stream_t stream) {
    if (plan == nullptr || peers == nullptr || H < 8 || H > kMaxHidden || H % 8 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
    if (peers->world != plan->world || peers->recv_rows < (size_t)plan->recv_rows) return EP_ERR_INVALID_ARG;
    const bool in_fp8 = in_format == EP_FORMAT_E4M3;
    const bool out_fp8 = out_format == EP_FORMAT_E4M3;
    if ((in_format != EP_FORMAT_BF16 && !in_fp8) || (out_format != EP_FORMAT_BF16 && !out_fp8))
        return EP_ERR_INVALID_ARG;
    if (in_fp8 && !out_fp8) return EP_ERR_INVALID_ARG;
    if (out_fp8 && (H % 128 != 0 || peers->recv_scales == nullptr)) return EP_ERR_INVALID_ARG;
    if (out_fp8) {
        // Non-overlapping scale layouts only, as ep_dispatch_ex: row-major-like or column-major-like.
        const int64_t G = H / 128;
        const bool row_like = scale_group_stride == 1 && scale_row_stride >= G;
        const bool col_like = scale_row_stride == 1 && scale_group_stride >= (int64_t)peers->recv_rows;
        if (!(row_like || col_like)) return EP_ERR_INVALID_ARG;
    }
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
    a.s_row = scale_row_stride;
    a.s_grp = scale_group_stride;
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
    if (plan == nullptr || peers == nullptr || H < 8 || H > kMaxHidden || H % 8 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
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
    if (plan == nullptr || peers == nullptr || H < 8 || H > kMaxHidden || H % 8 != 0) return EP_ERR_INVALID_ARG;
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
