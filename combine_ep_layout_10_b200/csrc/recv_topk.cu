// recv_topk.cu -- per-row routing outputs of dispatch.
//
// Besides the received rows, the pages' dispatch returns recv_topk_idx and
// recv_topk_weights ("DeepEP (DeepEveryParallel) Documentation", item 10
// "Perform MoE Dispatch and Combine for Training or Prefilling").  Every
// receive row of the expert-major layout holds exactly one slot (t, j), so
// the per-row outputs are that slot's expert id, its routing weight and its
// flat index t*k + j; a row that no slot fills gets -1, 0.0f, -1.
//
// One thread per receive row, 256 rows per block (coalesced reads of
// src_idx and coalesced writes): a row's source token is src_idx[r]; its slot
// j is the one of the token's k positions equal to r; its expert is the
// segment [seg[e], seg[e+1]) that holds r, found by binary search over a copy
// of seg in shared memory (the handle keeps no copy of topk_idx).  The k
// positions and k weights of the token are loaded by one fully unrolled,
// predicated loop, so they are all in flight together and the seg copy loads
// meanwhile: the critical path is two dependent global loads (src_idx, then
// pos/w), not one per slot or per search step.
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kTopkThreads = 256;

template <int KMAX>
__global__ void __launch_bounds__(kTopkThreads) recv_topk_kernel(RecvTopkArgs a) {
    extern __shared__ int32_t seg_s[];  // [E + 1]
    pdl_wait_then_trigger();
    const int64_t r = (int64_t)blockIdx.x * kTopkThreads + threadIdx.x;
    const int t = r < a.n_rows ? __ldg(a.src_idx + r) : -1;
    for (int e = threadIdx.x; e <= a.E; e += kTopkThreads) seg_s[e] = __ldg(a.seg + e);
    int j = -1;
    float wsel = 0.0f;
    if (t >= 0 && t < a.T) {
        const int64_t s0 = (int64_t)t * a.k;
        int32_t p[KMAX];
        float wv[KMAX];
        if ((a.k & 3) == 0) {
            // k a multiple of 4: the token's run of pos starts on a 16-byte
            // boundary (the handle's arrays are 256-byte aligned), and so does
            // its run of weights when the caller's array is 16-byte aligned;
            // such runs are read with 16-byte loads.
            const int4 *p4 = reinterpret_cast<const int4 *>(a.pos + s0);
            const bool w_vec = a.w != nullptr && (reinterpret_cast<uintptr_t>(a.w) & 15) == 0;
#pragma unroll
            for (int q = 0; q < KMAX / 4; ++q) {
                int4 pv = make_int4(-1, -1, -1, -1);
                float4 ww = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (4 * q < a.k) {
                    pv = __ldg(p4 + q);
                    if (w_vec) {
                        ww = __ldg(reinterpret_cast<const float4 *>(a.w + s0) + q);
                    } else if (a.w != nullptr) {
                        ww = make_float4(__ldg(a.w + s0 + 4 * q), __ldg(a.w + s0 + 4 * q + 1),
                                         __ldg(a.w + s0 + 4 * q + 2), __ldg(a.w + s0 + 4 * q + 3));
                    }
                }
                p[4 * q] = pv.x; p[4 * q + 1] = pv.y; p[4 * q + 2] = pv.z; p[4 * q + 3] = pv.w;
                wv[4 * q] = ww.x; wv[4 * q + 1] = ww.y; wv[4 * q + 2] = ww.z; wv[4 * q + 3] = ww.w;
            }
        } else {
#pragma unroll
            for (int jj = 0; jj < KMAX; ++jj) {
                p[jj] = jj < a.k ? __ldg(a.pos + s0 + jj) : -1;
                wv[jj] = (jj < a.k && a.w != nullptr) ? __ldg(a.w + s0 + jj) : 0.0f;
            }
        }
#pragma unroll
        for (int jj = KMAX - 1; jj >= 0; --jj) {  // the first slot with position r wins
            if (p[jj] == (int32_t)r) {
                j = jj;
                wsel = wv[jj];
            }
        }
    }
    __syncthreads();
    if (r >= a.n_rows) return;
    int32_t e_out = -1, s_out = -1;
    float w_out = 0.0f;
    if (j >= 0) {
        // Largest e < E with seg[e] <= r; seg is non-decreasing, seg[0] = 0.
        int lo = 0, hi = a.E;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (seg_s[mid] <= r) lo = mid;
            else hi = mid;
        }
        if (seg_s[lo] <= r && r < seg_s[lo + 1]) {
            e_out = lo;
            s_out = (int32_t)((int64_t)t * a.k + j);
            w_out = wsel;
        }
    }
    if (a.out_idx != nullptr) a.out_idx[r] = e_out;
    if (a.out_w != nullptr) a.out_w[r] = w_out;
    if (a.out_slot != nullptr) a.out_slot[r] = s_out;
}

// Across GPUs (ep_dispatch_topk_peer): every source rank writes, for each of
// its slots, the expert id, the weight, its rank and the slot's flat index
// into the owner's per-row tables at the plan's (rank, row); and every rank
// fills its own padding rows (which no source writes) with -1, 0, -1, -1,
// so the two parts need no ordering between them.
constexpr int kTopkPeerThreads = 256;

__global__ void __launch_bounds__(kTopkPeerThreads) recv_topk_peer_scatter_kernel(RecvTopkPeerArgs a) {
    pdl_wait_then_trigger();
    const int64_t s = (int64_t)blockIdx.x * kTopkPeerThreads + threadIdx.x;
    if (s >= (int64_t)a.T * a.k) return;
    const int2 d = __ldg(a.dst + s);
    if (d.x < 0) return;
    if (a.p_idx != nullptr) a.p_idx[d.x][d.y] = __ldg(a.topk_idx + s);
    if (a.p_w != nullptr) a.p_w[d.x][d.y] = a.w != nullptr ? __ldg(a.w + s) : 0.0f;
    if (a.p_src != nullptr) a.p_src[d.x][d.y] = a.rank;
    if (a.p_slot != nullptr) a.p_slot[d.x][d.y] = (int32_t)s;
}

__global__ void __launch_bounds__(kTopkPeerThreads) recv_topk_peer_pad_kernel(RecvTopkPeerArgs a) {
    pdl_wait_then_trigger();
    const int lane = threadIdx.x & 31;
    const int le = blockIdx.x * (kTopkPeerThreads / 32) + (threadIdx.x >> 5);  // this rank's expert
    if (le >= a.epr) return;
    int32_t used = __ldg(a.recv_cnt + le);
    if (a.capacity > 0 && used > a.capacity) used = a.capacity;
    const int64_t start = (int64_t)__ldg(a.recv_seg + le) + used;
    const int64_t end = __ldg(a.recv_seg + le + 1);
    int32_t *idx = a.p_idx != nullptr ? a.p_idx[a.rank] : nullptr;
    float *w = a.p_w != nullptr ? a.p_w[a.rank] : nullptr;
    int32_t *src = a.p_src != nullptr ? a.p_src[a.rank] : nullptr;
    int32_t *slot = a.p_slot != nullptr ? a.p_slot[a.rank] : nullptr;
    for (int64_t row = start + lane; row < end; row += 32) {
        if (idx != nullptr) idx[row] = -1;
        if (w != nullptr) w[row] = 0.0f;
        if (src != nullptr) src[row] = -1;
        if (slot != nullptr) slot[row] = -1;
    }
}

}  // namespace

cudaError_t launch_recv_topk_peer(const RecvTopkPeerArgs &a, cudaStream_t s) {
    const int64_t slots = (int64_t)a.T * a.k;
    cudaError_t e = cudaSuccess;
    if (slots > 0)
        e = launch_kernel(recv_topk_peer_scatter_kernel, (unsigned)((slots + kTopkPeerThreads - 1) / kTopkPeerThreads),
                          kTopkPeerThreads, 0, s, a);
    if (e != cudaSuccess || a.epr == 0) return e;
    const int per_block = kTopkPeerThreads / 32;
    return launch_kernel(recv_topk_peer_pad_kernel, (a.epr + per_block - 1) / per_block, kTopkPeerThreads, 0, s, a);
}

cudaError_t launch_recv_topk(const RecvTopkArgs &a, cudaStream_t s) {
    if (a.n_rows == 0) return cudaSuccess;
    const int64_t blocks = (a.n_rows + kTopkThreads - 1) / kTopkThreads;
    const size_t smem = (size_t)(a.E + 1) * sizeof(int32_t);  // <= 16 KB for E <= 4096
    if (a.k <= 8) return launch_kernel(recv_topk_kernel<8>, dim3((unsigned)blocks), dim3(kTopkThreads), smem, s, a);
    return launch_kernel(recv_topk_kernel<kMaxTopk>, dim3((unsigned)blocks), dim3(kTopkThreads), smem, s, a);
}

}  // namespace ep
