/*
 * ep_oracle.c -- plain, slow, single-threaded CPU oracle for the MoE
 * expert-parallel layout / dispatch / combine path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library under combine_ep_layout_10_b200/) never calls it, shares
 * no code, header, table or helper with it, and fails loudly when its own
 * CUDA extension is missing.
 *
 * What is computed, and where it comes from:
 *   - The pages ("DeepSeek publica DeepEP, una biblioteca open source para
 *     entrenamiento e inferencia MoE", news.hada.io, section "Patrones de uso
 *     en entrenamiento, prefill y decoding"; and "DeepEP (DeepEveryParallel)
 *     Documentation", docsearch.algolia.com, item 10 "Perform MoE Dispatch and
 *     Combine for Training or Prefilling") say that dispatch routes every
 *     token to the experts its top-k ids name, that the handle it returns
 *     carries the routing metadata and the per-expert token counts a grouped
 *     GEMM needs, and that combine reduces the expert outputs back to the
 *     source tokens.  FP8 dispatch with scale factors is named in
 *     "deepseek-ai/DeepEP" (repolode.com, "Funciones clave").
 *   - The pages do not fix the arithmetic.  This library fixes it as:
 *       receive rows in (expert, source token, slot) order, expert-major;
 *       virtual rank r owns experts [r*E/R, (r+1)*E/R) and the contiguous row
 *       slice of those experts;
 *       FP8 e4m3 with one fp32 scale per 128 channels, scale = amax / 448;
 *       combine = fp32 fused multiply-add chain over the k slots in slot
 *       order, rounded once to bf16 (round to nearest even).
 *     Each function below writes that definition out step by step, with no
 *     blocking, fusion or reordering.
 *
 * Floating point: IEEE binary32, round to nearest even, compiled without
 * fast-math and with floating-point contraction off, so every multiply and
 * divide is rounded exactly once and the only fused operation is the
 * explicit fmaf() of the combine definition.
 *
 * Pins (all CPU tests, see tests/test_oracle_*.py): brute-force enumeration
 * of positions, torch.sort(stable=True) of the flattened expert ids,
 * layout invariants, hand-derived golden fixtures, the e4m3 codec against the
 * OCP FP8 definition and torch.float8_e4m3fn, bf16 rounding against
 * torch.bfloat16, exact small-integer combines, and the closed-form
 * dispatch->combine round trip.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status codes of this oracle (its own numbering, documented in oracle/__init__.py). */
#define OR_OK 0
#define OR_ERR_INVALID_ARG 1
#define OR_ERR_BAD_EXPERT_ID 2
#define OR_ERR_CAPACITY 3

/* ------------------------------------------------------------------------- */
/* Number formats                                                             */
/* ------------------------------------------------------------------------- */

/* bf16 -> fp32: bf16 is the upper half of a binary32 word, so widening is exact. */
float oracle_bf16_to_f32(uint16_t h) {
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even.  Drops the low 16 bits of the
 * binary32 word and rounds the kept part by comparing the dropped part with
 * one half of the kept part's last place. */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    if ((bits & 0x7fffffffu) > 0x7f800000u) {
        /* NaN: keep the sign, return a quiet NaN. */
        return (uint16_t)(((bits >> 16) & 0x8000u) | 0x7fc0u);
    }
    uint32_t upper = bits >> 16;
    uint32_t lower = bits & 0xffffu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) {
        upper += 1u; /* a carry into the exponent is the correct result (up to inf) */
    }
    return (uint16_t)upper;
}

/* OCP 8-bit floating point, E4M3 variant ("e4m3fn"): 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits, no infinities, a single NaN pattern per
 * sign (S.1111.111), largest finite magnitude 448 = 1.75 * 2^8, subnormals
 * m * 2^-9 for m = 1..7.  Returns the value of a code. */
float oracle_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int ef = (code >> 3) & 0xf;
    int m = code & 7;
    double v;
    if (ef == 15 && m == 7) {
        return nanf("");
    }
    if (ef == 0) {
        v = ldexp((double)m, -9);
    } else {
        v = ldexp(1.0 + (double)m / 8.0, ef - 7);
    }
    return (float)(sign ? -v : v);
}

/* fp32 -> e4m3: round to nearest, ties to even, then saturate finite results
 * (and infinities) to +-448.  The sign of zero is kept.  NaN maps to 0x7f. */
uint8_t oracle_e4m3_encode(float v) {
    uint32_t bits;
    memcpy(&bits, &v, sizeof bits);
    uint8_t sign = (uint8_t)((bits >> 24) & 0x80u);
    uint32_t mag = bits & 0x7fffffffu;
    if (mag > 0x7f800000u) {
        return 0x7f;
    }
    float a = fabsf(v);
    /* Every magnitude >= 448 either rounds to 448 (below the 448/480
     * midpoint 464, or exactly on it: 448 has the even mantissa) or to 480,
     * which e4m3fn cannot hold and satfinite turns back into 448. */
    if (a >= 448.0f) {
        return (uint8_t)(sign | 0x7e);
    }
    if (a < 0.015625f) { /* below 2^-6, the smallest normal: subnormal grid of step 2^-9 */
        double d = (double)a * 512.0; /* exact: power-of-two scaling of a binary32 value */
        double n = floor(d);
        double frac = d - n;
        if (frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) != 0.0)) {
            n += 1.0;
        }
        /* n == 8 is the code 0x08, i.e. 1.0 * 2^-6: the smallest normal. */
        return (uint8_t)(sign | (uint8_t)n);
    }
    /* Normal: a = 1.m23 * 2^e with e in [-6, 8]; keep 3 mantissa bits. */
    int e = (int)(mag >> 23) - 127;
    uint32_t m23 = mag & 0x7fffffu;
    uint32_t keep = m23 >> 20;
    uint32_t rest = m23 & 0xfffffu;
    if (rest > 0x80000u || (rest == 0x80000u && (keep & 1u))) {
        keep += 1u;
    }
    if (keep == 8u) { /* mantissa overflow: next binade */
        keep = 0u;
        e += 1;
    }
    uint32_t code = ((uint32_t)(e + 7) << 3) | keep;
    if (code > 0x7eu) {
        code = 0x7eu;
    }
    return (uint8_t)(sign | code);
}

/* Element-wise loops over the two scalar conversions above (used by the tests
 * to sweep whole binades; no arithmetic of their own). */
void oracle_e4m3_encode_n(const float *v, uint8_t *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) {
        out[i] = oracle_e4m3_encode(v[i]);
    }
}

void oracle_f32_to_bf16_n(const float *v, uint16_t *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) {
        out[i] = oracle_f32_to_bf16(v[i]);
    }
}

/* ------------------------------------------------------------------------- */
/* Layout                                                                     */
/* ------------------------------------------------------------------------- */

static int64_t align_up64(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

/* An expert id as the layout uses it: ids outside [-1, E) count as -1. */
static int valid_id(int32_t e, int E) { return (e < -1 || e >= E) ? -1 : e; }

/* Upper bound on the receive rows a layout can use.
 *   capacity > 0 (padded, the decoding layout): every expert owns exactly
 *     `capacity` rows, so E * capacity.
 *   capacity == 0: expert segments are packed back to back, each rounded up
 *     to a multiple of `align` (the pages' expert_alignment), so at most
 *     T*k + E*(align-1).
 * Returns -1 for invalid arguments. */
int64_t oracle_max_recv_rows(int T, int k, int E, int align, int capacity) {
    if (T < 0 || k < 1 || E < 1 || align < 1 || capacity < 0) {
        return -1;
    }
    if (capacity > 0) {
        return (int64_t)E * capacity;
    }
    return (int64_t)T * k + (int64_t)E * (align - 1);
}

/*
 * Routing layout.  Inputs: topk_idx [T, k] (row-major, int32; -1 marks an
 * unused slot).  Outputs (all caller-allocated):
 *   cnt[E]          tokens routed to each expert (slots, counted with multiplicity)
 *   rank_tok[R]     tokens with at least one expert on virtual rank r
 *   in_rank[T*R]    1 if token t has an expert on rank r, else 0
 *   seg[E+1]        first receive row of each expert's segment; seg[E] = rows used
 *   rank_off[R+1]   first receive row of each rank's slice
 *   pos[T*k]        receive row of each slot, -1 for unused slots
 *   src_idx[n_rows] source token of each receive row, -1 for padding rows
 * The handle of the pages (news.hada.io, "Patrones de uso ..."; docsearch
 * item 10) carries exactly this metadata to the combine; cnt is its
 * per-expert token count list for the expert GEMMs.
 * Two data errors still give a complete layout, and are reported in the
 * return value:
 *   an id outside [-1, E) is taken as an unused slot (OR_ERR_BAD_EXPERT_ID);
 *   in padded mode, an expert named by more than `capacity` slots keeps its
 *   first `capacity` slots in (token, slot) order and the rest get no row
 *   (pos -1) -- the bound that num_max_tokens_per_rank (docsearch item 10)
 *   puts on a padded buffer (OR_ERR_CAPACITY).
 * A bad id is reported before an overflow when both occur.
 */
int oracle_layout(const int32_t *topk_idx, int T, int k, int E, int R, int align,
                  int capacity, int32_t *cnt, int32_t *rank_tok, uint8_t *in_rank,
                  int32_t *seg, int32_t *rank_off, int32_t *pos, int32_t *src_idx,
                  int64_t n_rows) {
    /* Step 1: arguments. */
    if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0 || align < 1 || capacity < 0) {
        return OR_ERR_INVALID_ARG;
    }
    if (capacity > 0 && capacity % align != 0) {
        return OR_ERR_INVALID_ARG;
    }
    if (n_rows < oracle_max_recv_rows(T, k, E, align, capacity)) {
        return OR_ERR_INVALID_ARG;
    }
    int experts_per_rank = E / R;

    /* Step 2: every id must name an expert or be -1; any other id is
     * reported and from here on treated as -1 (see valid_id). */
    int bad_id = 0;
    for (int64_t s = 0; s < (int64_t)T * k; ++s) {
        if (topk_idx[s] < -1 || topk_idx[s] >= E) {
            bad_id = 1;
        }
    }

    /* Step 3: per-expert counts and token-in-rank flags. */
    for (int e = 0; e < E; ++e) {
        cnt[e] = 0;
    }
    memset(in_rank, 0, (size_t)T * (size_t)R);
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = valid_id(topk_idx[(int64_t)t * k + j], E);
            if (e < 0) {
                continue;
            }
            cnt[e] += 1;
            in_rank[(int64_t)t * R + e / experts_per_rank] = 1;
        }
    }
    for (int r = 0; r < R; ++r) {
        int32_t n = 0;
        for (int t = 0; t < T; ++t) {
            n += in_rank[(int64_t)t * R + r];
        }
        rank_tok[r] = n;
    }

    /* Step 4: expert segments and rank slices. */
    int over = 0;
    seg[0] = 0;
    for (int e = 0; e < E; ++e) {
        if (capacity > 0) {
            seg[e + 1] = (int32_t)((int64_t)(e + 1) * capacity);
            if (cnt[e] > capacity) {
                over = 1;
            }
        } else {
            seg[e + 1] = (int32_t)(seg[e] + align_up64(cnt[e], align));
        }
    }
    for (int r = 0; r <= R; ++r) {
        rank_off[r] = seg[r * experts_per_rank];
    }

    /* Step 5: positions.  Walking tokens in ascending order and, inside a
     * token, slots in ascending order, and handing each expert its next free
     * row, is the definition of (expert, source token, slot) order.  A padded
     * expert whose `capacity` rows are all handed out gives no row to its
     * later slots. */
    for (int64_t p = 0; p < n_rows; ++p) {
        src_idx[p] = -1;
    }
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (fill == NULL) {
        return OR_ERR_INVALID_ARG;
    }
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int64_t s = (int64_t)t * k + j;
            int e = valid_id(topk_idx[s], E);
            if (e < 0 || (capacity > 0 && fill[e] == capacity)) {
                pos[s] = -1;
                continue;
            }
            int32_t p = seg[e] + fill[e];
            fill[e] += 1;
            pos[s] = p;
            src_idx[p] = t;
        }
    }
    free(fill);
    if (bad_id) {
        return OR_ERR_BAD_EXPERT_ID;
    }
    return over ? OR_ERR_CAPACITY : OR_OK;
}

/* ------------------------------------------------------------------------- */
/* Dispatch                                                                   */
/* ------------------------------------------------------------------------- */

/* BF16 dispatch: receive row pos[t][j] becomes a bit copy of x[t]. */
int oracle_dispatch_bf16(const uint16_t *x, int T, int H, int k, const int32_t *pos,
                         uint16_t *recv, int64_t n_rows) {
    if (T < 0 || H < 1 || k < 1) {
        return OR_ERR_INVALID_ARG;
    }
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int32_t p = pos[(int64_t)t * k + j];
            if (p < 0) {
                continue;
            }
            if (p >= n_rows) {
                return OR_ERR_INVALID_ARG;
            }
            for (int i = 0; i < H; ++i) {
                recv[(int64_t)p * H + i] = x[(int64_t)t * H + i];
            }
        }
    }
    return OR_OK;
}

/* Quantise one group of 128 channels of one token:
 *   amax = max |x_i|;
 *   amax == 0: scale 0, every byte 0x00;
 *   else scale = amax / 448 and q_i = e4m3(x_i * (448 / amax)), each a single
 *   correctly rounded binary32 operation. */
void oracle_quantize_group(const uint16_t *xg, uint8_t *qg, float *scale) {
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) {
        float a = fabsf(oracle_bf16_to_f32(xg[i]));
        if (a > amax) {
            amax = a;
        }
    }
    if (amax == 0.0f) {
        *scale = 0.0f;
        for (int i = 0; i < 128; ++i) {
            qg[i] = 0x00;
        }
        return;
    }
    *scale = amax / 448.0f;
    float inv = 448.0f / amax;
    for (int i = 0; i < 128; ++i) {
        float scaled = oracle_bf16_to_f32(xg[i]) * inv;
        qg[i] = oracle_e4m3_encode(scaled);
    }
}

/* FP8 dispatch: quantise x[t] per 128-channel group once, then write the
 * codes and the H/128 scales to every receive row of token t. */
int oracle_dispatch_fp8(const uint16_t *x, int T, int H, int k, const int32_t *pos,
                        uint8_t *recv, float *scales, int64_t n_rows) {
    if (T < 0 || H < 128 || H % 128 != 0 || k < 1) {
        return OR_ERR_INVALID_ARG;
    }
    int G = H / 128;
    uint8_t *q = (uint8_t *)malloc((size_t)H);
    float *s = (float *)malloc((size_t)G * sizeof(float));
    if (q == NULL || s == NULL) {
        free(q);
        free(s);
        return OR_ERR_INVALID_ARG;
    }
    int status = OR_OK;
    for (int t = 0; t < T && status == OR_OK; ++t) {
        for (int g = 0; g < G; ++g) {
            oracle_quantize_group(x + (int64_t)t * H + (int64_t)g * 128, q + g * 128, s + g);
        }
        for (int j = 0; j < k; ++j) {
            int32_t p = pos[(int64_t)t * k + j];
            if (p < 0) {
                continue;
            }
            if (p >= n_rows) {
                status = OR_ERR_INVALID_ARG;
                break;
            }
            memcpy(recv + (int64_t)p * H, q, (size_t)H);
            memcpy(scales + (int64_t)p * G, s, (size_t)G * sizeof(float));
        }
    }
    free(q);
    free(s);
    return status;
}

/* ------------------------------------------------------------------------- */
/* Combine                                                                    */
/* ------------------------------------------------------------------------- */

/* out[t][i] = bf16_rne( fma chain over j = 0..k-1 with pos >= 0 of
 *                       w[t][j] * y[pos[t][j]][i], starting from +0.0f ). */
int oracle_combine(const uint16_t *y, int64_t n_rows, int H, const float *w,
                   const int32_t *pos, int T, int k, uint16_t *out) {
    if (T < 0 || H < 1 || k < 1) {
        return OR_ERR_INVALID_ARG;
    }
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int32_t p = pos[(int64_t)t * k + j];
            if (p >= n_rows) {
                return OR_ERR_INVALID_ARG;
            }
        }
        for (int i = 0; i < H; ++i) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int32_t p = pos[(int64_t)t * k + j];
                if (p < 0) {
                    continue;
                }
                acc = fmaf(w[(int64_t)t * k + j], oracle_bf16_to_f32(y[(int64_t)p * H + i]), acc);
            }
            out[(int64_t)t * H + i] = oracle_f32_to_bf16(acc);
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* Backward                                                                   */
/* ------------------------------------------------------------------------- */

/* The pages ("DeepSeek publica DeepEP ...", news.hada.io, "Patrones de uso
 * en entrenamiento, prefill y decoding"; "DeepEP (DeepEveryParallel)
 * Documentation", item 10) say that the backward pass of dispatch is carried
 * out by a combine and the backward pass of combine by a dispatch.  Written
 * out for this library's forward definitions:
 *
 * dispatch backward: the gradient reaching x[t] is the sum of the gradients
 *   of its k receive rows.  That is the combine definition with every weight
 *   equal to 1 (oracle_combine with w = 1): bf16_rn of the fp32 chain
 *   acc = acc + grad_recv[pos[t][j]][i] over valid slots in slot order.
 *
 * combine backward, with g = grad_out[t] (bf16):
 *   grad_y[pos[t][j]][i] = bf16_rn( fp32_rn( w[t][j] * g[i] ) )   (a weighted dispatch)
 *   grad_w[t][j]         = sum_i g[i] * y[pos[t][j]][i]          (a dot product)
 *   The dot product is returned exactly enough to grade any fp32 summation
 *   order: every product of two bf16 values is exact in binary64 and the
 *   binary64 sum of at most 2^16 of them is within ~1e-12 relative of the
 *   exact sum.  Slots with pos < 0 get grad_w = 0 and write no row. */
int oracle_combine_backward(const uint16_t *grad_out, const uint16_t *y, int64_t n_rows, int H,
                            const float *w, const int32_t *pos, int T, int k, uint16_t *grad_y,
                            double *grad_w) {
    if (T < 0 || H < 1 || k < 1) {
        return OR_ERR_INVALID_ARG;
    }
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int64_t s = (int64_t)t * k + j;
            int32_t p = pos[s];
            if (p < 0) {
                grad_w[s] = 0.0;
                continue;
            }
            if (p >= n_rows) {
                return OR_ERR_INVALID_ARG;
            }
            double dot = 0.0;
            for (int i = 0; i < H; ++i) {
                float g = oracle_bf16_to_f32(grad_out[(int64_t)t * H + i]);
                float prod = w[s] * g;
                grad_y[(int64_t)p * H + i] = oracle_f32_to_bf16(prod);
                dot += (double)g * (double)oracle_bf16_to_f32(y[(int64_t)p * H + i]);
            }
            grad_w[s] = dot;
        }
    }
    return OR_OK;
}

/* Dispatch of input that is already FP8 ("DeepEP (DeepEveryParallel)
 * Documentation", item 10: dispatch takes BF16 input, or FP8 input given as
 * data plus scale factors).  Nothing is requantised: receive row pos[t][j]
 * becomes a bit copy of the codes xq[t] and of the H/128 scales xs[t]. */
int oracle_dispatch_fp8_prequant(const uint8_t *xq, const float *xs, int T, int H, int k,
                                 const int32_t *pos, uint8_t *recv, float *scales, int64_t n_rows) {
    if (T < 0 || H < 128 || H % 128 != 0 || k < 1) {
        return OR_ERR_INVALID_ARG;
    }
    int G = H / 128;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int32_t p = pos[(int64_t)t * k + j];
            if (p < 0) {
                continue;
            }
            if (p >= n_rows) {
                return OR_ERR_INVALID_ARG;
            }
            memcpy(recv + (int64_t)p * H, xq + (int64_t)t * H, (size_t)H);
            memcpy(scales + (int64_t)p * G, xs + (int64_t)t * G, (size_t)G * sizeof(float));
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* Per-row routing outputs of dispatch                                        */
/* ------------------------------------------------------------------------- */

/* Besides the received rows, dispatch returns recv_topk_idx and
 * recv_topk_weights ("DeepEP (DeepEveryParallel) Documentation", item 10).
 * In this layout every receive row holds exactly one slot (t, j), so the
 * per-row values are that slot's expert id topk_idx[t][j], its weight
 * topk_w[t][j] and its flat index t*k + j.  A row that no slot fills
 * (padding, alignment slack, rows left by unused slots) gets -1, 0.0f, -1.
 * Any output pointer may be NULL. */
int oracle_dispatch_topk(const int32_t *topk_idx, const float *topk_w, int T, int k,
                         const int32_t *pos, int64_t n_rows, int32_t *recv_idx,
                         float *recv_w, int32_t *recv_slot) {
    if (T < 0 || k < 1 || n_rows < 0) {
        return OR_ERR_INVALID_ARG;
    }
    for (int64_t r = 0; r < n_rows; ++r) {
        if (recv_idx) recv_idx[r] = -1;
        if (recv_w) recv_w[r] = 0.0f;
        if (recv_slot) recv_slot[r] = -1;
    }
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int64_t s = (int64_t)t * k + j;
            int32_t p = pos[s];
            if (p < 0) {
                continue;
            }
            if (p >= n_rows) {
                return OR_ERR_INVALID_ARG;
            }
            if (recv_idx) recv_idx[p] = topk_idx[s];
            if (recv_w) recv_w[p] = topk_w[s];
            if (recv_slot) recv_slot[p] = (int32_t)s;
        }
    }
    return OR_OK;
}
