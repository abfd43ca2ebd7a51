// noalloc.cu -- ep_layout_noalloc: the routing layout without any device
// allocation, for callers that cannot allocate.
//
// Who needs it: a serving loop whose device memory is planned once at start-up
// by a static memory planner (every byte pre-carved, no allocator on the hot
// path); code that runs under another framework's allocator and may not touch
// the CUDA allocator behind its back; and latency-critical loops that must not
// risk cudaMalloc's implicit device synchronisation.  Those callers pass every
// input and output buffer themselves; the only other device memory this call
// uses is the fixed scratch array below.
//
// The scratch (the layout's per-tile count matrices, a per-expert count
// buffer and a fallback error word) is a file-scope __device__ array of
// EP_NOALLOC_SCRATCH_WORDS 32-bit words: it is created when the library's
// device code is loaded and every GPU that loads the library holds it until
// the process exits.  Its device address is looked up with
// cudaGetSymbolAddress (host code cannot use the array's name as a device
// pointer) by the first call on a device, with that device current, and kept
// together with the unique id of the CUDA context it belongs to.  A later call
// that finds another context current on that device (the device was reset
// and the library's module loaded again, possibly at another address) looks
// the address up again, so no call launches on a stale pointer.  All
// calls on a device share the array, so two calls whose work overlaps on the
// GPU (different streams, no ordering between them) race on it; calls on one
// stream are ordered and safe.  Nothing in it needs to start at zero: the
// count kernel overwrites every tile entry the position kernel reads, and the
// position kernel (or, for T == 0, the empty-layout kernel) overwrites the
// error word.
#include <cuda.h>

#include <mutex>

#include "api_common.cuh"

namespace ep {
namespace {

static __device__ __align__(256) int32_t g_layout_scratch[EP_NOALLOC_SCRATCH_WORDS];

constexpr int kMaxDevicesNoAlloc = 64;
std::mutex g_scratch_mu;
int32_t *g_scratch_ptr[kMaxDevicesNoAlloc];
unsigned long long g_scratch_ctx[kMaxDevicesNoAlloc];  // context id the address belongs to

// Unique id of the current CUDA context (cuCtxGetId, reached through the
// runtime's driver entry point so that the library needs no -lcuda); false
// when there is no current context yet or the driver lacks the call.
bool current_context_id(unsigned long long *id) {
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    static GetId fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<GetId>(p);
    }();
    return fn != nullptr && fn(nullptr, id) == CUDA_SUCCESS;
}

bool is_aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

ep_status status_of(cudaError_t e) {
    if (e == cudaSuccess) return EP_OK;
    if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver || e == cudaErrorNoKernelImageForDevice)
        return EP_ERR_NO_DEVICE;
    return EP_ERR_CUDA;
}

// Device address of the scratch array on `dev` (which is current): looked up
// on the first call on the device and again whenever the current context is
// not the one the kept address belongs to.
ep_status scratch_for_device(int dev, int32_t **out) {
    if (dev < 0 || dev >= kMaxDevicesNoAlloc) return EP_ERR_INVALID_ARG;
    unsigned long long ctx = 0;
    const bool have_ctx = current_context_id(&ctx);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr || !have_ctx || g_scratch_ctx[dev] != ctx) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_layout_scratch);  // creates the context if needed
        if (e != cudaSuccess || p == nullptr) return e != cudaSuccess ? status_of(e) : EP_ERR_CUDA;
        unsigned long long now = 0;
        // Without a context id the address is not kept: every call looks it up.
        g_scratch_ptr[dev] = current_context_id(&now) ? static_cast<int32_t *>(p) : nullptr;
        g_scratch_ctx[dev] = now;
        *out = static_cast<int32_t *>(p);
        return EP_OK;
    }
    *out = g_scratch_ptr[dev];
    return EP_OK;
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" ep_status ep_layout_noalloc(const int32_t *topk_idx, int T, int k, int E, int R, int A, int C,
                                       int32_t *out_cnt, int32_t *out_rank_tok, uint8_t *out_in_rank,
                                       int32_t *pos, int32_t *src_idx, int32_t *seg, int32_t *rank_off,
                                       uint32_t *error_word, ep_stream_t stream) {
    if (T < 0 || k < 1 || k > kMaxTopk || E < 1 || E > kMaxExperts || R < 1 || R > E || E % R != 0 ||
        A < 1 || C < 0 || (C > 0 && C % A != 0))
        return EP_ERR_INVALID_ARG;
    if ((int64_t)T * k >= (int64_t)1 << 31) return EP_ERR_INVALID_ARG;
    const size_t n_rows = ep_max_recv_rows(T, k, E, A, C);
    if (n_rows >= ((size_t)1 << 31)) return EP_ERR_INVALID_ARG;
    if (T > 0 && (topk_idx == nullptr || !is_aligned(topk_idx, 4) || pos == nullptr || !is_aligned(pos, 4)))
        return EP_ERR_INVALID_ARG;
    if (seg == nullptr || rank_off == nullptr || !is_aligned(seg, 4) || !is_aligned(rank_off, 4))
        return EP_ERR_INVALID_ARG;
    if (n_rows > 0 && (src_idx == nullptr || !is_aligned(src_idx, 4))) return EP_ERR_INVALID_ARG;
    if ((out_cnt && !is_aligned(out_cnt, 4)) || (out_rank_tok && !is_aligned(out_rank_tok, 4)) ||
        (error_word && !is_aligned(error_word, 4)))
        return EP_ERR_INVALID_ARG;

    // Same tile geometry as ep_layout.
    const LayoutGeometry geo = layout_geometry(T, k, E, R, C);
    const int ntiles = geo.ntiles;

    // Scratch words (16-byte aligned blocks): tile_cnt, tile_rank, per-expert
    // counts, per-tile bad-id flags, error word.
    const size_t w_tcnt = (size_t)align4(ntiles * E);
    const size_t w_trank = (size_t)align4(ntiles * R);
    const size_t w_cnt = (size_t)align4(E);
    const size_t w_terr = (size_t)align4(ntiles);
    const size_t need = w_tcnt + w_trank + w_cnt + w_terr + 1;
    if (need > (size_t)EP_NOALLOC_SCRATCH_WORDS) return EP_ERR_SCRATCH_LIMIT;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return status_of(e);
    DeviceInfo info;
    if ((e = device_info(dev, &info)) != cudaSuccess) return status_of(e);
    if (info.cc_major != 10) return EP_ERR_NO_DEVICE;
    int32_t *scratch = nullptr;
    const ep_status st = scratch_for_device(dev, &scratch);
    if (st != EP_OK) return st;

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
    a.pos = pos;
    a.src_idx = src_idx;
    a.seg = seg;
    a.rank_off = rank_off;
    a.tile_cnt = scratch;
    a.tile_rank = scratch + w_tcnt;
    a.cnt = scratch + w_tcnt + w_trank;
    a.tile_err = reinterpret_cast<uint32_t *>(scratch + w_tcnt + w_trank + w_cnt);
    a.err = error_word != nullptr ? error_word
                                  : reinterpret_cast<uint32_t *>(scratch + w_tcnt + w_trank + w_cnt + w_terr);
    a.out_cnt = out_cnt;
    a.out_rank_tok = out_rank_tok;
    a.out_in_rank = out_in_rank;

    if (debug_enabled())
        std::fprintf(stderr,
                     "ep: layout_noalloc T=%d k=%d E=%d R=%d align=%d capacity=%d rows=%lld path=%s tiles=%d "
                     "tile_tokens=%d threads=%d scratch_words=%zu of %d\n",
                     T, k, E, R, A, C, (long long)n_rows, geo.small ? "one-cta" : "tiled", geo.ntiles,
                     geo.tile_tokens, geo.small ? 1024 : geo.tile_threads, need, EP_NOALLOC_SCRATCH_WORDS);
    // The layout kernels overwrite the error word; nothing else needs clearing.
    return status_of(launch_layout(a, stream));
}
