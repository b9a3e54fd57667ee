/* The MoE expert layer, forward and backward, in plain C99 fp64.
 *
 * TEST INFRASTRUCTURE ONLY: a second, independent statement of what the layer
 * computes, beside the numpy oracle in moe.py.  Only the tests, the smoke
 * check and the CPU-baseline leg of the bench may load it; the product path
 * never does, and nothing here is shared with the CUDA library.
 *
 * What it follows (the pages give no formula; the readings are those of the
 * numpy oracle's docstrings, restated here):
 *
 *  - "Ai2 rebuilds Olmo's training stack for trillion-parameter MoEs",
 *    introduction: a router sends each token to a small selection of experts
 *    and the output is the routing-weighted sum of their outputs.  Reading:
 *    the k largest fp32 logits (equal values to the lower expert index, slot
 *    order = selection order), weights w_i = exp(l_i - l_0) / sum_j exp(l_j - l_0)
 *    over the selected logits.
 *  - same page, "Routing work stays on the GPU": routed rows go straight into
 *    contiguous per-expert buffers.  Reading: experts back to back, offsets the
 *    exclusive prefix sum of the counts, rows of one expert in ascending token
 *    order, i.e. dest_pos(t, i) = offsets[e] + #{t' < t : e in top-k(t')}.
 *  - Each expert is a SwiGLU FFN: a = silu(x W1^T) * (x W3^T), y = a W2^T, with
 *    W13 [E, 2f, d] (rows 0..f-1 the gate W1, f..2f-1 the up projection W3) and
 *    W2 [E, d, f]; the backward is the chain rule of the forward.
 *  - Rounding: where the device stores bf16 (GU, A, Y_perm, out, dY_perm, dH,
 *    dX_perm, dx, dW13, dW2, dW_r) the value is rounded once to bf16, nearest
 *    even; every sum is fp64.  round_bf16 = 0 keeps everything in fp64.
 *  - same page, "MXFP8 reduces compute and memory costs": a grouped GEMM on
 *    MXFP8 operands runs on the decoded values of E4M3 codes with one E8M0
 *    scale per 32 consecutive values along that GEMM's reduction axis (OCP
 *    Microscaling Formats v1.0: X = floor(log2 amax) - 8, clamped to
 *    [-127, 127], 0 for an all-zero block; code = E4M3(v / 2^X), nearest even,
 *    clamped to +-448).  For the dW GEMMs the reduction runs over an expert's
 *    rows and the blocks restart at each expert's first row.
 *
 * Evaluation is per token and per selected expert with brute-force loops.  The
 * permutation is used where it is itself an output (the row a result is stored
 * in) and for the dW sums, which run over an expert's rows.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define MOE_REF_OK 0
#define MOE_REF_BAD_ARG 1
#define MOE_REF_NO_MEMORY 2

/* bit g of mx: grouped GEMM g on MXFP8 operands */
enum { MX_GEMM1 = 1, MX_GEMM2 = 2, MX_DA = 4, MX_DW2 = 8, MX_DX = 16, MX_DW13 = 32 };

typedef struct {
    int T, d, E, k, f;
    int round_bf16; /* 1: round stored values to bf16; 0: pure fp64 */
    unsigned mx;    /* MX_* bits */
} moe_ref_shape;

/* ------------------------------------------------------------------ formats */

/* Nearest bf16 (8 significant bits, fp32's exponent range), ties to even.
 * Normal range: drop the low 45 of fp64's 52 fraction bits with a
 * round-half-even carry on the bit pattern (a carry into the exponent is the
 * correct result).  Below 2^-126 bf16 is subnormal with a fixed spacing of
 * 2^-133.  Beyond the largest finite bf16 the result is an infinity. */
static double round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    if (fabs(x) < 0x1p-126) return nearbyint(x * 0x1p133) * 0x1p-133;
    uint64_t u;
    memcpy(&u, &x, sizeof u);
    const int drop = 45;
    const uint64_t keep_lsb = (u >> drop) & 1u;
    u += (((uint64_t)1 << (drop - 1)) - 1u) + keep_lsb;
    u &= ~(((uint64_t)1 << drop) - 1u);
    double r;
    memcpy(&r, &u, sizeof r);
    if (fabs(r) >= 0x1p128) return copysign(INFINITY, x);
    return r;
}

static double stored(double x, int bf16) { return bf16 ? round_bf16(x) : x; }

/* OCP FP8 E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0
 * is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities. */
static double e4m3_value(int code) {
    const int e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return (code & 0x80) ? -v : v;
}

/* Code of the E4M3 value nearest to v (ties to the even code, magnitudes
 * beyond 448 to 448), found by scanning the 127 finite non-negative codes,
 * whose values increase with the code.  The sign of v is kept, zero included. */
static int e4m3_code(double v) {
    const double a = fabs(v);
    int best = 0;
    double best_d = a;
    for (int c = 1; c <= 0x7E; ++c) {
        const double dist = fabs(e4m3_value(c) - a);
        if (dist < best_d || (dist == best_d && (c & 1) == 0)) {
            best = c;
            best_d = dist;
        }
    }
    return signbit(v) ? (best | 0x80) : best;
}

/* One MX block of n <= 32 values read at src[i * ss]; writes the decoded
 * values code * 2^X to dst[i * ds] (and, when asked, the codes and the scale
 * byte X + 127). */
static void mx_block(const double* src, size_t ss, int n, double* dst, size_t ds,
                     uint8_t* codes, size_t cs, uint8_t* scale) {
    double amax = 0.0;
    for (int i = 0; i < n; ++i) amax = fmax(amax, fabs(src[i * ss]));
    int X = 0;
    if (amax > 0.0) {
        X = ilogb(amax) - 8; /* 8 = largest exponent of E4M3 */
        if (X < -127) X = -127;
        if (X > 127) X = 127;
    }
    for (int i = 0; i < n; ++i) {
        const int c = e4m3_code(ldexp(src[i * ss], -X));
        if (dst) dst[i * ds] = ldexp(e4m3_value(c), X);
        if (codes) codes[i * cs] = (uint8_t)c;
    }
    if (scale) *scale = (uint8_t)(X + 127);
}

/* Decoded MXFP8 copy of rows x cols (row-major) with blocks of 32 along each
 * row. */
static void mx_rows(const double* a, int64_t rows, int64_t cols, double* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c0 = 0; c0 < cols; c0 += 32) {
            const int n = (int)(cols - c0 < 32 ? cols - c0 : 32);
            mx_block(a + r * cols + c0, 1, n, out + r * cols + c0, 1, NULL, 0, NULL);
        }
}

/* Decoded MXFP8 copy of rows [r0, r1) x cols with blocks of 32 down each
 * column, the first block starting at r0. */
static void mx_cols(const double* a, int64_t r0, int64_t r1, int64_t cols, double* out) {
    for (int64_t b = r0; b < r1; b += 32) {
        const int n = (int)(r1 - b < 32 ? r1 - b : 32);
        for (int64_t c = 0; c < cols; ++c)
            mx_block(a + b * cols + c, (size_t)cols, n, out + b * cols + c, (size_t)cols, NULL, 0, NULL);
    }
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* ------------------------------------------------------------------ helpers */

static int valid(const moe_ref_shape* s) {
    return s && s->T >= 0 && s->d > 0 && s->E > 0 && s->k >= 1 && s->k <= s->E && s->f > 0;
}

static double* alloc(size_t n) { return (double*)malloc((n ? n : 1) * sizeof(double)); }

/* ------------------------------------------------------------------ forward */

/* logits_in: fp32 router logits [T, E], or NULL to compute logits = x W_r
 * from wr [d, E] in fp64 (written to logits [T, E] when that is not NULL);
 * routing then compares the fp32 rounding of those logits, and the weights
 * take the fp32 logits (the fp64 ones when round_bf16 = 0).
 * Outputs: topk_idx, topk_w [T, k]; counts [E]; offsets [E + 1];
 * dest_pos [T, k]; src_token [T k]; gu [T k, 2f]; a [T k, f]; y_perm [T k, d];
 * out [T, d].  Returns 0, or 1 for a bad argument, 2 when out of memory. */
int moe_ref_forward(const moe_ref_shape* s, const double* x, const float* logits_in,
                    const double* wr, const double* w13, const double* w2, double* logits,
                    int32_t* topk_idx, double* topk_w, int32_t* counts, int32_t* offsets,
                    int32_t* dest_pos, int32_t* src_token, double* gu, double* a,
                    double* y_perm, double* out) {
    if (!valid(s) || !x || (!logits_in && !wr) || !w13 || !w2 || !topk_idx || !topk_w ||
        !counts || !offsets || !dest_pos || !src_token || !gu || !a || !y_perm || !out)
        return MOE_REF_BAD_ARG;
    const int64_t T = s->T, d = s->d, E = s->E, k = s->k, f = s->f, f2 = 2 * s->f;
    const int bf = s->round_bf16;
    int status = MOE_REF_OK;

    /* router */
    float* lg32 = (float*)malloc((size_t)(T * E > 0 ? T * E : 1) * sizeof(float));
    double* lgw = alloc((size_t)(T * E)); /* logits the weights are taken on */
    char* chosen = (char*)malloc((size_t)E);
    int64_t* cursor = (int64_t*)malloc((size_t)E * sizeof(int64_t));
    double* xq = NULL;
    double* w13q = NULL;
    double* w2q = NULL;
    double* aq = alloc((size_t)f);
    double* pre = alloc((size_t)f2);
    if (!lg32 || !lgw || !chosen || !cursor || !aq || !pre) { status = MOE_REF_NO_MEMORY; goto done; }
    for (int64_t t = 0; t < T; ++t)
        for (int64_t e = 0; e < E; ++e) {
            if (logits_in) {
                lg32[t * E + e] = logits_in[t * E + e];
                lgw[t * E + e] = (double)logits_in[t * E + e];
            } else {
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c) acc += x[t * d + c] * wr[c * E + e];
                if (logits) logits[t * E + e] = acc;
                lg32[t * E + e] = (float)acc;
                lgw[t * E + e] = bf ? (double)(float)acc : acc;
            }
        }
    for (int64_t t = 0; t < T; ++t) {
        memset(chosen, 0, (size_t)E);
        for (int64_t i = 0; i < k; ++i) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e)
                if (!chosen[e] && (best < 0 || lg32[t * E + e] > lg32[t * E + best])) best = e;
            chosen[best] = 1;
            topk_idx[t * k + i] = (int32_t)best;
        }
        const double l0 = lgw[t * E + topk_idx[t * k]];
        double z = 0.0;
        for (int64_t i = 0; i < k; ++i) z += exp(lgw[t * E + topk_idx[t * k + i]] - l0);
        for (int64_t i = 0; i < k; ++i) topk_w[t * k + i] = exp(lgw[t * E + topk_idx[t * k + i]] - l0) / z;
    }

    /* dispatch plan: a stable counting sort of the (t, i) pairs by expert */
    for (int64_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t j = 0; j < T * k; ++j) counts[topk_idx[j]] += 1;
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    for (int64_t e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t t = 0; t < T; ++t)
        for (int64_t i = 0; i < k; ++i) {
            const int64_t r = cursor[topk_idx[t * k + i]]++;
            dest_pos[t * k + i] = (int32_t)r;
            src_token[r] = (int32_t)t;
        }

    /* operands as the GEMMs see them: MXFP8 along the reduction axis (d for
     * GEMM1, f for GEMM2) or the values themselves */
    const double* xs = x;
    const double* w13s = w13;
    const double* w2s = w2;
    if (s->mx & MX_GEMM1) {
        xq = alloc((size_t)(T * d));
        w13q = alloc((size_t)(E * f2 * d));
        if (!xq || !w13q) { status = MOE_REF_NO_MEMORY; goto done; }
        mx_rows(x, T, d, xq);
        mx_rows(w13, E * f2, d, w13q);
        xs = xq;
        w13s = w13q;
    }
    if (s->mx & MX_GEMM2) {
        w2q = alloc((size_t)(E * d * f));
        if (!w2q) { status = MOE_REF_NO_MEMORY; goto done; }
        mx_rows(w2, E * d, f, w2q);
        w2s = w2q;
    }

    /* each token through each of its experts */
    for (int64_t t = 0; t < T; ++t)
        for (int64_t i = 0; i < k; ++i) {
            const int64_t e = topk_idx[t * k + i], r = dest_pos[t * k + i];
            const double* we = w13s + e * f2 * d;
            for (int64_t j = 0; j < f2; ++j) {
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c) acc += xs[t * d + c] * we[j * d + c];
                pre[j] = acc;
                gu[r * f2 + j] = stored(acc, bf);
            }
            for (int64_t j = 0; j < f; ++j) a[r * f + j] = stored(silu(pre[j]) * pre[f + j], bf);
            if (s->mx & MX_GEMM2) mx_rows(a + r * f, 1, f, aq);
            else memcpy(aq, a + r * f, (size_t)f * sizeof(double));
            const double* w2e = w2s + e * d * f;
            for (int64_t c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < f; ++j) acc += aq[j] * w2e[c * f + j];
                y_perm[r * d + c] = stored(acc, bf);
            }
        }

    /* weighted combine, slots in order */
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < k; ++i) acc += topk_w[t * k + i] * y_perm[(int64_t)dest_pos[t * k + i] * d + c];
            out[t * d + c] = stored(acc, bf);
        }

done:
    free(lg32); free(lgw); free(chosen); free(cursor);
    free(xq); free(w13q); free(w2q); free(aq); free(pre);
    return status;
}

/* ------------------------------------------------------------------ backward */

/* From the forward's record (topk_idx, topk_w, offsets, dest_pos, src_token,
 * gu, a, y_perm) and dout = dL/dout [T, d].  Outputs: dy_perm [T k, d],
 * dw [T, k], dh [T k, 2f], dx_perm [T k, d], dw2 [E, d, f], dw13 [E, 2f, d],
 * d_logits [T, E], dx [T, d]; with wr (router projection) also the router
 * term of dx and dwr [d, E] (dwr may be NULL without wr).  An expert with no
 * rows gets dW2_e = dW13_e = 0.  Returns 0, 1 for a bad argument, 2 when out
 * of memory. */
int moe_ref_backward(const moe_ref_shape* s, const double* x, const double* wr,
                     const double* w13, const double* w2, const double* dout,
                     const int32_t* topk_idx, const double* topk_w, const int32_t* offsets,
                     const int32_t* dest_pos, const int32_t* src_token, const double* gu,
                     const double* a, const double* y_perm, double* dy_perm, double* dw,
                     double* dh, double* dx_perm, double* dw2, double* dw13, double* d_logits,
                     double* dx, double* dwr) {
    if (!valid(s) || !x || !w13 || !w2 || !dout || !topk_idx || !topk_w || !offsets ||
        !dest_pos || !src_token || !gu || !a || !y_perm || !dy_perm || !dw || !dh ||
        !dx_perm || !dw2 || !dw13 || !d_logits || !dx || (wr && !dwr))
        return MOE_REF_BAD_ARG;
    const int64_t T = s->T, d = s->d, E = s->E, k = s->k, f = s->f, f2 = 2 * s->f, M = T * k;
    const int bf = s->round_bf16;
    int status = MOE_REF_OK;
    double* w2c = NULL;   /* W2 as the dA GEMM sees it (blocks along d) */
    double* w13c = NULL;  /* W13 as the dX GEMM sees it (blocks along 2f) */
    double* xperm = alloc((size_t)(M * d));
    double* dyg = NULL;   /* dW2 operands (blocks down each expert's rows) */
    double* ag = NULL;
    double* dhg = NULL;   /* dW13 operands */
    double* xg = NULL;
    double* dyq = alloc((size_t)d);
    double* dhq = alloc((size_t)f2);
    if (!xperm || !dyq || !dhq) { status = MOE_REF_NO_MEMORY; goto done; }
    for (int64_t r = 0; r < M; ++r) memcpy(xperm + r * d, x + (int64_t)src_token[r] * d, (size_t)d * sizeof(double));

    /* combine backward */
    for (int64_t t = 0; t < T; ++t)
        for (int64_t i = 0; i < k; ++i) {
            const int64_t r = dest_pos[t * k + i];
            double acc = 0.0;
            for (int64_t c = 0; c < d; ++c) {
                dy_perm[r * d + c] = stored(topk_w[t * k + i] * dout[t * d + c], bf);
                acc += dout[t * d + c] * y_perm[r * d + c];
            }
            dw[t * k + i] = acc;
        }

    const double* w2s = w2;
    const double* w13s = w13;
    if (s->mx & MX_DA) {
        w2c = alloc((size_t)(E * d * f));
        if (!w2c) { status = MOE_REF_NO_MEMORY; goto done; }
        for (int64_t e = 0; e < E; ++e) mx_cols(w2 + e * d * f, 0, d, f, w2c + e * d * f);
        w2s = w2c;
    }
    if (s->mx & MX_DX) {
        w13c = alloc((size_t)(E * f2 * d));
        if (!w13c) { status = MOE_REF_NO_MEMORY; goto done; }
        for (int64_t e = 0; e < E; ++e) mx_cols(w13 + e * f2 * d, 0, f2, d, w13c + e * f2 * d);
        w13s = w13c;
    }

    /* per routed row: dA = dY W2_e, SwiGLU backward, dX = dH W13_e */
    for (int64_t t = 0; t < T; ++t)
        for (int64_t i = 0; i < k; ++i) {
            const int64_t e = topk_idx[t * k + i], r = dest_pos[t * k + i];
            if (s->mx & MX_DA) mx_rows(dy_perm + r * d, 1, d, dyq);
            else memcpy(dyq, dy_perm + r * d, (size_t)d * sizeof(double));
            const double* w2e = w2s + e * d * f;
            for (int64_t j = 0; j < f; ++j) {
                double da = 0.0;
                for (int64_t c = 0; c < d; ++c) da += dyq[c] * w2e[c * f + j];
                const double g = gu[r * f2 + j], u = gu[r * f2 + f + j];
                const double sg = 1.0 / (1.0 + exp(-g));
                dh[r * f2 + j] = stored(da * u * sg * (1.0 + g * (1.0 - sg)), bf);
                dh[r * f2 + f + j] = stored(da * g * sg, bf);
            }
            if (s->mx & MX_DX) mx_rows(dh + r * f2, 1, f2, dhq);
            else memcpy(dhq, dh + r * f2, (size_t)f2 * sizeof(double));
            const double* w13e = w13s + e * f2 * d;
            for (int64_t c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < f2; ++j) acc += dhq[j] * w13e[j * d + c];
                dx_perm[r * d + c] = stored(acc, bf);
            }
        }

    /* weight gradients: sums over each expert's rows */
    const double* dys = dy_perm;
    const double* as = a;
    const double* dhs = dh;
    const double* xs = xperm;
    if (s->mx & MX_DW2) {
        dyg = alloc((size_t)(M * d));
        ag = alloc((size_t)(M * f));
        if (!dyg || !ag) { status = MOE_REF_NO_MEMORY; goto done; }
        for (int64_t e = 0; e < E; ++e) {
            mx_cols(dy_perm, offsets[e], offsets[e + 1], d, dyg);
            mx_cols(a, offsets[e], offsets[e + 1], f, ag);
        }
        dys = dyg;
        as = ag;
    }
    if (s->mx & MX_DW13) {
        dhg = alloc((size_t)(M * f2));
        xg = alloc((size_t)(M * d));
        if (!dhg || !xg) { status = MOE_REF_NO_MEMORY; goto done; }
        for (int64_t e = 0; e < E; ++e) {
            mx_cols(dh, offsets[e], offsets[e + 1], f2, dhg);
            mx_cols(xperm, offsets[e], offsets[e + 1], d, xg);
        }
        dhs = dhg;
        xs = xg;
    }
    for (int64_t e = 0; e < E; ++e) {
        const int64_t r0 = offsets[e], r1 = offsets[e + 1];
        for (int64_t c = 0; c < d; ++c)
            for (int64_t j = 0; j < f; ++j) {
                double acc = 0.0;
                for (int64_t r = r0; r < r1; ++r) acc += dys[r * d + c] * as[r * f + j];
                dw2[(e * d + c) * f + j] = stored(acc, bf);
            }
        for (int64_t j = 0; j < f2; ++j)
            for (int64_t c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int64_t r = r0; r < r1; ++r) acc += dhs[r * f2 + j] * xs[r * d + c];
                dw13[(e * f2 + j) * d + c] = stored(acc, bf);
            }
    }

    /* router: softmax over the selected logits, differentiated; 0 off the
     * selection (the selection itself is piecewise constant) */
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) d_logits[t * E + e] = 0.0;
        double inner = 0.0;
        for (int64_t i = 0; i < k; ++i) inner += topk_w[t * k + i] * dw[t * k + i];
        for (int64_t i = 0; i < k; ++i)
            d_logits[t * E + topk_idx[t * k + i]] = topk_w[t * k + i] * (dw[t * k + i] - inner);
    }

    /* dx: the token's routed rows summed, plus the router projection's term */
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < k; ++i) acc += dx_perm[(int64_t)dest_pos[t * k + i] * d + c];
            if (wr) {
                double rt = 0.0;
                for (int64_t e = 0; e < E; ++e) rt += d_logits[t * E + e] * wr[c * E + e];
                acc += rt;
            }
            dx[t * d + c] = stored(acc, bf);
        }
    if (wr)
        for (int64_t c = 0; c < d; ++c)
            for (int64_t e = 0; e < E; ++e) {
                double acc = 0.0;
                for (int64_t t = 0; t < T; ++t) acc += x[t * d + c] * d_logits[t * E + e];
                dwr[c * E + e] = stored(acc, bf);
            }

done:
    free(w2c); free(w13c); free(xperm); free(dyg); free(ag); free(dhg); free(xg);
    free(dyq); free(dhq);
    return status;
}

/* ------------------------------------------------------------------ formats, exported for pins */

void moe_ref_round_bf16(const double* x, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(x[i]);
}

void moe_ref_e4m3_decode(const uint8_t* codes, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
}

void moe_ref_e4m3_encode(const double* v, int64_t n, uint8_t* codes) {
    for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)e4m3_code(v[i]);
}

/* MXFP8 of rows x cols with blocks of 32 along each row: codes [rows, cols],
 * scale bytes [rows, ceil(cols / 32)]. */
void moe_ref_mx_rowwise(const double* x, int64_t rows, int64_t cols, uint8_t* codes,
                        uint8_t* scales) {
    const int64_t nb = (cols + 31) / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            const int n = (int)(cols - 32 * b < 32 ? cols - 32 * b : 32);
            mx_block(x + r * cols + 32 * b, 1, n, NULL, 0, codes + r * cols + 32 * b, 1,
                     scales + r * nb + b);
        }
}
