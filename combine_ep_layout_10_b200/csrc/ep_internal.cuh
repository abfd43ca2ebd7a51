// ep_internal.cuh -- shared definitions of the CUDA library (not part of the ABI).
//
// Kernels live in layout.cu, dispatch.cu and combine.cu; the C ABI in
// ep_api.cu validates arguments, owns the handle and launches them.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

namespace ep {

// Bits of the handle's device error word.
constexpr uint32_t kErrBadExpertId = 1u;
constexpr uint32_t kErrCapacity = 2u;
constexpr uint32_t kErrTimeout = 4u;

constexpr int kMaxTopk = 32;
constexpr int kMaxExperts = 4096;

// Bounded device waits give up after about a second at B200 clocks.
constexpr long long kWaitLimitCycles = 2000000000LL;

}  // namespace ep

// The opaque handle of the ABI.  Host struct; the arrays are device memory
// carved out of one stream-ordered allocation.
struct ep_handle {
    int T, k, E, R, align, capacity, experts_per_rank;
    int tile_tokens, ntiles;
    int64_t n_rows;          // receive rows the layout may use (ep_max_recv_rows)
    int device;
    cudaStream_t stream;     // the stream the handle was created (and is freed) on
    void *block;             // the allocation
    int32_t *pos;            // [T*k]
    int32_t *src_idx;        // [n_rows]
    int32_t *seg;            // [E+1]
    int32_t *rank_off;       // [R+1]
    int32_t *cnt;            // [E]
    int32_t *tile_cnt;       // [ntiles*E]  per-tile expert counts, then exclusive bases
    int32_t *tile_rank;      // [ntiles*R]  per-tile token-in-rank counts
    uint32_t *err;           // [1] device error word
};

namespace ep {

struct LayoutArgs {
    const int32_t *topk_idx;
    int T, k, E, R, epr, align, capacity;
    int tile_tokens, ntiles, sub_tokens;
    int scan_parts_e, scan_parts_r, pos_warps;
    int64_t n_rows;
    int32_t *pos, *src_idx, *seg, *rank_off, *cnt, *tile_cnt, *tile_rank;
    uint32_t *err;
    int32_t *out_cnt, *out_rank_tok;
    uint8_t *out_in_rank;
};

struct DispatchArgs {
    const uint8_t *x;        // bf16 [T, H]
    const int32_t *pos;      // [T, k]
    uint8_t *recv;           // [rows, H] bf16 or e4m3
    float *scales;           // [rows, H/128] (FP8 only)
    uint32_t *err;
    int T, k, H;
    int chunk;               // channels per work unit
    int nchunks;             // units per token
    long long nunits;        // T * nchunks
    int stages;              // input ring depth
};

struct CombineArgs {
    const uint8_t *y;        // bf16 [rows, H]
    const float *w;          // [T, k]
    const int32_t *pos;      // [T, k]
    uint8_t *out;            // bf16 [T, H]
    int T, k, H;
    int nvec;                // H / 8 (16-byte vectors per row)
    int vpt;                 // vectors per thread: 1, 2 or 4
    int blocks_per_token;    // ceil(nvec / (128 * vpt))
};

// Launchers (return the cudaGetLastError() of the launch).
cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s);
cudaError_t launch_dispatch(const DispatchArgs &a, bool fp8, int num_sms, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s);

// Per-device facts, cached.
struct DeviceInfo {
    int num_sms;
    int cc_major, cc_minor;
    int max_smem_optin;
};
cudaError_t device_info(int device, DeviceInfo *out);

}  // namespace ep
