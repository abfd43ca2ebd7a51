// ep_api.cu -- the single-GPU part of the C ABI declared in include/ep.h:
// argument validation, handle ownership and kernel launches (the multi-GPU
// calls are in peer_api.cu).  Every step of the data path runs in the kernels
// of layout.cu, dispatch.cu, combine.cu, backward.cu and recv_topk.cu;
// nothing here touches tensor data on the host.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "api_common.cuh"

namespace ep {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceInfo g_info[kMaxDevices];
bool g_have[kMaxDevices];
cudaMemPool_t g_pool[kMaxDevices];

}  // namespace

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

    const LayoutGeometry geo = layout_geometry(T, k, E, R, C);
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
    a.tile_threads = geo.tile_threads;
    a.ids_in_smem = geo.ids_in_smem;
    a.small = geo.small;
    a.rank_early = 2LL * ntiles <= info.num_sms;
    a.n_rows = (int64_t)n_rows;
    a.pos = h->pos; a.src_idx = h->src_idx; a.seg = h->seg; a.rank_off = h->rank_off;
    a.cnt = h->cnt; a.tile_cnt = h->tile_cnt; a.tile_rank = h->tile_rank;
    a.tile_err = h->tile_err; a.err = h->err;
    a.out_cnt = out_cnt;
    a.out_rank_tok = out_rank_tok;
    a.out_in_rank = out_in_rank;
    h->layout_path = ntiles == 0 ? kLayoutPathEmpty : geo.small ? kLayoutPathOneCta : kLayoutPathTiled;
    h->layout_kernels = h->layout_path == kLayoutPathTiled ? 2 : 1;

    if (debug_enabled())
        std::fprintf(stderr,
                     "ep: layout T=%d k=%d E=%d R=%d align=%d capacity=%d rows=%lld path=%s tiles=%d "
                     "tile_tokens=%d threads=%d\n",
                     T, k, E, R, A, C, (long long)n_rows, geo.small ? "one-cta" : "tiled", geo.ntiles,
                     geo.tile_tokens, geo.small ? 1024 : geo.tile_threads);
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
    if (h == nullptr || H < 8 || H > kMaxHidden || H % 8 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
    const bool in_fp8 = in_format == EP_FORMAT_E4M3;
    const bool out_fp8 = out_format == EP_FORMAT_E4M3;
    if ((in_format != EP_FORMAT_BF16 && !in_fp8) || (out_format != EP_FORMAT_BF16 && !out_fp8))
        return EP_ERR_INVALID_ARG;
    if (in_fp8 && !out_fp8) return EP_ERR_INVALID_ARG;  // no dequantising dispatch
    if (out_fp8 && H % 128 != 0) return EP_ERR_INVALID_ARG;
    if (recv_rows < (size_t)h->n_rows) return EP_ERR_INVALID_ARG;
    const int64_t G = H / 128;
    bool col_fill = false;  // pre-quantised input, column-major scales: codes copied, then the fill pass
    if (out_fp8) {
        // Non-overlapping scale layouts only: row-major-like or column-major-like.
        const bool row_like = scale_group_stride == 1 && scale_row_stride >= G;
        const bool col_like = scale_row_stride == 1 && scale_group_stride >= (int64_t)recv_rows;
        if (!(row_like || col_like)) return EP_ERR_INVALID_ARG;
        col_fill = in_fp8 && col_like && !row_like;
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
    a.scales = col_fill ? nullptr : recv_scales;
    a.s_row = scale_row_stride;
    a.s_grp = scale_group_stride;
    a.mode = !out_fp8 ? kDispatchCopyBf16 : in_fp8 ? kDispatchCopyFp8 : kDispatchQuantFp8;
    a.num_sms = num_sms;
    a.T = h->T; a.k = h->k; a.H = H;
    a.chunk = chunk;
    a.nchunks = nchunks;
    if ((int64_t)h->T * a.nchunks >= ((int64_t)1 << 31)) return EP_ERR_INVALID_ARG;
    a.nunits = h->T * a.nchunks;
    if (debug_enabled())
        std::fprintf(stderr, "ep: dispatch T=%d H=%d mode=%s chunk=%d units=%d num_sms=%d\n", h->T, H,
                     a.mode == kDispatchQuantFp8 ? "bf16->e4m3" : a.mode == kDispatchCopyFp8 ? "e4m3" : "bf16",
                     a.chunk, a.nunits, num_sms);
    cudaError_t e = launch_dispatch(a, stream);
    if (e == cudaSuccess && col_fill && h->T > 0) {
        // The input's own scale table [T, H/128] is the fill pass's source.
        ScaleFillArgs f{};
        f.src_idx = h->src_idx;
        f.table = x_scales;
        f.scales = recv_scales;
        f.ld = scale_group_stride;
        f.n_rows = h->n_rows;
        f.G = (int)G;
        f.num_sms = num_sms;
        f.vec_in = G % 4 == 0 && aligned(x_scales, 16);
        // Without an SM budget the pass starts in the copy kernel's last wave:
        // the input table predates it (with a budget its blocks would wait on
        // SMs the caller left to other work).
        f.table_is_input = EP_FILL_EARLY_START && num_sms == 0;
        e = launch_scale_fill(f, stream);
    }
    if (e == cudaSuccess && recv_src_idx != nullptr && h->n_rows > 0)
        e = cudaMemcpyAsync(recv_src_idx, h->src_idx, (size_t)h->n_rows * 4, cudaMemcpyDeviceToDevice, stream);
    return cuda_status(e);
}

ep_status ep_dispatch_fp8_colmajor(const ep_handle *h, const void *x, int H, void *recv_x, float *recv_scales,
                                   int64_t scale_ld, float *token_scales, int32_t *recv_src_idx,
                                   size_t recv_rows, int num_sms, ep_stream_t stream) {
    if (h == nullptr || H < 128 || H > kMaxHidden || H % 128 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
    if (scale_ld < 1 || recv_rows > ((size_t)1 << 62) || scale_ld < (int64_t)recv_rows) return EP_ERR_INVALID_ARG;
    if (recv_rows < (size_t)h->n_rows) return EP_ERR_INVALID_ARG;
    if (h->T > 0) {
        if (x == nullptr || recv_x == nullptr || recv_scales == nullptr || token_scales == nullptr)
            return EP_ERR_INVALID_ARG;
        if (!aligned(x, 16) || !aligned(recv_x, 16) || !aligned(recv_scales, 4) || !aligned(token_scales, 4))
            return EP_ERR_INVALID_ARG;
    }
    if (recv_src_idx != nullptr && !aligned(recv_src_idx, 4)) return EP_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    if (dev != h->device) return EP_ERR_INVALID_ARG;

    int chunk, nchunks;
    dispatch_chunking(h->T, H, 128, info.num_sms, &chunk, &nchunks);
    if ((int64_t)h->T * nchunks >= ((int64_t)1 << 31)) return EP_ERR_INVALID_ARG;
    DispatchArgs a{};
    a.x = static_cast<const uint8_t *>(x);
    a.pos = h->pos;
    a.recv = static_cast<uint8_t *>(recv_x);
    a.scales = nullptr;         // the receive rows' scales come from the fill pass
    a.tok_scales = token_scales;
    a.s_row = 1;
    a.s_grp = scale_ld;
    a.mode = kDispatchQuantFp8;
    a.num_sms = num_sms;
    a.T = h->T; a.k = h->k; a.H = H;
    a.chunk = chunk;
    a.nchunks = nchunks;
    a.nunits = h->T * nchunks;
    if (debug_enabled())
        std::fprintf(stderr, "ep: dispatch_fp8_colmajor T=%d H=%d chunk=%d units=%d ld=%lld num_sms=%d\n", h->T,
                     H, a.chunk, a.nunits, (long long)scale_ld, num_sms);
    cudaError_t e = launch_dispatch(a, stream);
    if (e == cudaSuccess && h->T > 0) {
        ScaleFillArgs f{};
        f.src_idx = h->src_idx;
        f.table = token_scales;
        f.scales = recv_scales;
        f.ld = scale_ld;
        f.n_rows = h->n_rows;
        f.G = H / 128;
        f.num_sms = num_sms;
        f.vec_in = f.G % 4 == 0 && aligned(token_scales, 16);
        e = launch_scale_fill(f, stream);
    }
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
    if (h == nullptr || H < 8 || H > kMaxHidden || H % 8 != 0 || num_sms < 0) return EP_ERR_INVALID_ARG;
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
    a.pos_early = (int64_t)h->T * a.blocks_per_token <= (int64_t)EP_COMBINE_EARLY_MAX_BLOCKS_PER_SM * info.num_sms;
    if (debug_enabled())
        std::fprintf(stderr, "ep: combine T=%d H=%d blocks=%lld num_sms=%d\n", h->T, H,
                     (long long)h->T * a.blocks_per_token, num_sms);
    return cuda_status(launch_combine(a, stream));
}

ep_status ep_combine(const ep_handle *h, const void *y, const float *topk_w, int H, size_t recv_rows,
                     void *out, ep_stream_t stream) {
    return ep_combine_ex(h, y, topk_w, H, recv_rows, out, 0, stream);
}

ep_status ep_dispatch_backward(const ep_handle *h, const void *grad_recv, int H, size_t recv_rows,
                               void *grad_x, ep_stream_t stream) {
    if (h == nullptr || H < 8 || H > kMaxHidden || H % 8 != 0) return EP_ERR_INVALID_ARG;
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
    a.pos_early = (int64_t)h->T * a.blocks_per_token <= (int64_t)EP_COMBINE_EARLY_MAX_BLOCKS_PER_SM * info.num_sms;
    return cuda_status(launch_combine(a, stream));
}

ep_status ep_combine_backward(const ep_handle *h, const void *grad_out, const void *y, const float *topk_w,
                              int H, size_t recv_rows, void *grad_y, float *grad_w, ep_stream_t stream) {
    if (h == nullptr || H < 8 || H > kMaxHidden || H % 8 != 0) return EP_ERR_INVALID_ARG;
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

ep_status ep_e4m3_encode(const float *x, uint8_t *codes, size_t n, ep_stream_t stream) {
    if (n == 0) return EP_OK;
    if (x == nullptr || codes == nullptr || !aligned(x, 16) || !aligned(codes, 16)) return EP_ERR_INVALID_ARG;
    if (n >= ((size_t)1 << 40)) return EP_ERR_INVALID_ARG;
    int dev;
    DeviceInfo info;
    ep_status st = current_device(&dev, &info);
    if (st != EP_OK) return st;
    return cuda_status(launch_e4m3_encode(x, codes, (int64_t)n, stream));
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
    info->layout_kernels = h->layout_kernels;
    info->layout_path = h->layout_path;
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
