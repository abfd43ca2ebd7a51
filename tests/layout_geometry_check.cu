// layout_geometry_check.cu -- host-only check of the layout's launch geometry.
//
// Built with nvcc together with the library's layout.cu and run on the CPU
// (no CUDA call is made): for every shape of a grid that spans the ABI's
// limits (T*k < 2^31, k <= 32, E <= 4096, R | E, packed and padded), the
// geometry the library would launch must be valid on B200 -- block sizes of
// whole warps within 1024 threads, dynamic shared memory within the 227 KB a
// block may opt into (static shared memory included), the per-tile count
// matrices within the fixed scratch of the no-allocation entry point, and
// tiles that cover the batch; and the dispatch's work units must tile every
// row for every hidden size up to 2^24.  Prints one line per violation and the number
// of shapes checked; exits non-zero on any violation.
#include <cstdint>
#include <cstdio>
#include <vector>

#include "ep_internal.cuh"

namespace ep {
size_t layout_small_smem(const LayoutArgs &a);
size_t layout_count_smem(const LayoutArgs &a);
size_t layout_pos_smem(const LayoutArgs &a);
}  // namespace ep

using namespace ep;

static const size_t kMaxSmem = 227 * 1024;  // per block, opt-in, sm_100
static const size_t kStaticSmem = 1024;     // headroom for the kernels' static shared arrays

int main() {
    const long long Ts[] = {1, 2, 31, 127, 128, 129, 383, 1000, 1536, 1537, 4095, 4096, 8192, 8193,
                            70000, 262144, 1 << 20, (1 << 22) + 7, 1 << 24, 67108863, 268435455,
                            (1LL << 31) - 129, (1LL << 31) - 1};
    const int ks[] = {1, 2, 3, 8, 17, 32};
    const int Es[] = {1, 2, 8, 16, 96, 256, 512, 513, 1024, 4096};
    const int Cs[] = {0, 1, 16, 128, 2048};
    long long checked = 0, bad = 0;
    for (long long T : Ts)
        for (int k : ks)
            for (int E : Es) {
                std::vector<int> Rs = {1, E};
                for (int r : {2, 8, 64}) if (E % r == 0 && r < E) Rs.push_back(r);
                for (int R : Rs)
                    for (int C : Cs) {
                        if (T * k >= (1LL << 31)) continue;
                        const long long rows = C > 0 ? (long long)E * C : T * k;
                        if (rows >= (1LL << 31)) continue;
                        const LayoutGeometry g = layout_geometry((int)T, k, E, R, C);
                        LayoutArgs a{};
                        a.T = (int)T; a.k = k; a.E = E; a.R = R; a.epr = E / R; a.capacity = C;
                        a.tile_tokens = g.tile_tokens; a.ntiles = g.ntiles; a.sub_tokens = g.sub_tokens;
                        a.pos_warps = g.pos_warps; a.tile_threads = g.tile_threads;
                        a.ids_in_smem = g.ids_in_smem; a.small = g.small; a.n_rows = rows;
                        ++checked;
                        auto fail = [&](const char *what, long long v) {
                            ++bad;
                            if (bad <= 40)
                                std::printf("T=%lld k=%d E=%d R=%d C=%d: %s (%lld)\n", T, k, E, R, C, what, v);
                        };
                        if (g.ntiles < 1 || (long long)g.ntiles * g.tile_tokens < T ||
                            (long long)(g.ntiles - 1) * g.tile_tokens >= T)
                            fail("tiles do not cover the batch exactly", g.ntiles);
                        if (g.small) {
                            if (layout_small_smem(a) + kStaticSmem > kMaxSmem)
                                fail("one-CTA shared memory", (long long)layout_small_smem(a));
                            continue;
                        }
                        if (g.tile_threads < 256 || g.tile_threads > 1024 || g.tile_threads % 32)
                            fail("tile threads", g.tile_threads);
                        if (g.pos_warps < 1 || g.pos_warps > g.tile_threads / 32)
                            fail("position-kernel warps", g.pos_warps);
                        if ((long long)g.ntiles * (E + R) > kLayoutMatWords &&
                            g.tile_tokens < (1 << 29))
                            fail("count matrices exceed their bound", (long long)g.ntiles * (E + R));
                        if (g.sub_tokens < 1 || g.sub_tokens > g.tile_tokens)
                            fail("sub-block tokens", g.sub_tokens);
                        if (layout_count_smem(a) + kStaticSmem > kMaxSmem)
                            fail("count-kernel shared memory", (long long)layout_count_smem(a));
                        if (layout_pos_smem(a) + kStaticSmem > kMaxSmem)
                            fail("position-kernel shared memory", (long long)layout_pos_smem(a));
                    }
            }
    // Dispatch work units: chunks of whole 8- (BF16) or 128-channel (FP8)
    // groups, at most EP_DISPATCH_MAX_CHUNK channels (so at most 512 threads
    // of 16 channels), that tile the row exactly.
    for (int H = 8; H <= kMaxHidden; H = H < 65536 ? H + 8 * 37 : H * 2 + 8)
        for (int align_ch : {8, 128})
            for (long long T : {1LL, 7LL, 148LL, 8192LL, 1LL << 20}) {
                if (align_ch == 128 && H % 128) continue;
                int chunk = 0, n = 0;
                dispatch_chunking((int)T, H, align_ch, 148, &chunk, &n);
                ++checked;
                const int threads = (((chunk + 15) / 16 + 31) / 32) * 32;
                if (chunk < align_ch || chunk % align_ch || chunk > EP_DISPATCH_MAX_CHUNK || n < 1 ||
                    (long long)n * chunk < H || (long long)(n - 1) * chunk >= H || threads > 512) {
                    ++bad;
                    std::printf("dispatch H=%d align=%d T=%lld: chunk %d x %d, %d threads\n", H, align_ch, T,
                                chunk, n, threads);
                }
            }
    std::printf("checked %lld shapes, %lld violations\n", checked, bad);
    return bad == 0 ? 0 : 1;
}
