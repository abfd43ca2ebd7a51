// plan.cu -- where every local slot goes when the expert-parallel ranks are
// real GPUs.
//
// The pages' dispatch sends every token to its experts on all ranks and
// combine brings the outputs back to the rank the token came from ("DeepSeek
// publica DeepEP ...", news.hada.io, "Patrones de uso en entrenamiento,
// prefill y decoding"; "DeepEP (DeepEveryParallel) Documentation", item 10).
// This library orders the rows a rank receives exactly as the single-GPU
// layout of all ranks' tokens concatenated in rank order would: rank r owns
// experts [r*E/W, (r+1)*E/W); inside its receive buffer expert e's segment
// starts after the (aligned, or capacity-sized) segments of r's lower
// experts, and holds the slots of e from source rank 0, then 1, ..., each in
// (token, slot) order.  So the row of source rank s's i-th slot of expert e
// (i counted in s's own (token, slot) order, which is what s's local layout
// gives: i = pos_local - seg_local[e]) is
//     segdest(e) + sum_{s' < s} counts[s'][e] + i,
// where counts[s'][e] are the per-expert slot counts every rank computed
// locally and the caller all-gathered.
//
// Two kernels: one block computes segdest and the per-expert offsets from
// the [W, E] count matrix (a block scan over the experts, restarted at each
// owner rank's first expert); then one thread per local slot writes its
// (owner, row).  A row outside the receive buffer (recv_rows) or past a
// padded expert's capacity is not assigned (-1) and sets the plan's error
// word, so the peer kernels never write outside any rank's buffer.
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kPlanThreads = 1024;
constexpr int kSlotThreads = 256;

__global__ void __launch_bounds__(kPlanThreads) plan_offsets_kernel(PlanArgs a) {
    extern __shared__ int32_t S[];  // [E + 1] exclusive prefix of the segment sizes
    __shared__ int32_t warp_s[33];
    pdl_wait_then_trigger();
    const int E = a.E;
    uint32_t bad = 0;
    int32_t carry = 0;
    for (int base = 0; base < E; base += kPlanThreads) {
        const int e = base + threadIdx.x;
        int32_t sz = 0;
        if (e < E) {
            int32_t tot = 0, pre = 0;
            for (int s = 0; s < a.world; ++s) {
                const int32_t c = __ldg(a.counts + (int64_t)s * E + e);
                tot += c;
                if (s < a.rank) pre += c;
            }
            if (a.capacity > 0) {
                sz = a.capacity;
                if (tot > a.capacity) bad |= kErrCapacity;
            } else {
                sz = (tot + a.align - 1) / a.align * a.align;
            }
            a.pre[e] = pre;
            if (e / a.epr == a.rank) a.recv_cnt[e - a.rank * a.epr] = tot;
        }
        int32_t total;
        const int32_t excl = block_exclusive_scan(sz, &total, warp_s);
        if (e < E) S[e] = carry + excl;
        carry += total;
    }
    if (threadIdx.x == 0) S[E] = carry;
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kPlanThreads) {
        const int g0 = e / a.epr * a.epr;        // owner's first expert
        const int32_t segdest = S[e] - S[g0];
        const int32_t owner_rows = S[g0 + a.epr] - S[g0];
        if (owner_rows > a.recv_rows) bad |= kErrCapacity;  // the owner's buffer is too small
        a.offs[e] = segdest + a.pre[e];
    }
    const int r0 = a.rank * a.epr;
    for (int le = threadIdx.x; le <= a.epr; le += kPlanThreads) a.recv_seg[le] = S[r0 + le] - S[r0];
    if (bad) atomicOr(a.err, bad);
}

__global__ void __launch_bounds__(kSlotThreads) plan_slots_kernel(PlanArgs a) {
    pdl_wait_then_trigger();
    const int64_t s = (int64_t)blockIdx.x * kSlotThreads + threadIdx.x;
    if (s >= (int64_t)a.T * a.k) return;
    int2 d = make_int2(-1, -1);
    const int e = __ldg(a.topk_idx + s);
    const int p = __ldg(a.pos + s);
    if (e >= 0 && e < a.E && p >= 0) {
        const int32_t i = p - __ldg(a.seg + e);               // index among this rank's slots of e
        const int32_t within = __ldg(a.pre + e) + i;           // ... among all ranks' slots of e
        const int64_t row = (int64_t)__ldg(a.offs + e) + i;
        if (a.capacity > 0 && within >= a.capacity) {
            atomicOr(a.err, kErrCapacity);
        } else if (row >= a.recv_rows) {
            atomicOr(a.err, kErrCapacity);
        } else {
            d = make_int2(e / a.epr, (int)row);
        }
    }
    a.dst[s] = d;
}

}  // namespace

cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)(a.E + 1) * sizeof(int32_t);  // <= 16 KB for E <= 4096
    cudaError_t e = launch_kernel(plan_offsets_kernel, 1, kPlanThreads, smem, s, a);
    if (e != cudaSuccess || a.T == 0) return e;
    const int64_t slots = (int64_t)a.T * a.k;
    const int64_t blocks = (slots + kSlotThreads - 1) / kSlotThreads;
    return launch_kernel(plan_slots_kernel, (unsigned)blocks, kSlotThreads, 0, s, a);
}

}  // namespace ep
