/*
 * Oracle for the one-GPU Mixture-of-Experts layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, obviously-correct CPU
 * restatement of what the layer computes, used by the tests, the smoke check
 * and the CPU baseline of the benchmark to judge the CUDA path.  It shares no
 * code with the CUDA library and the product path never calls it.
 *
 * Arithmetic: every input is converted exactly to double (bf16 and e4m3 by
 * this file's own decoders, written from the formats' definitions) and all
 * sums are taken in double, in ascending index order, with naive loops.
 * Nothing is blocked, fused or reordered; OpenMP only spreads independent
 * output rows over threads, so results do not depend on the thread count.
 *
 * Sources (web pages on MoE routing and grouped matmuls):
 *  - "Advanced GPU Optimization: How to tech an LLM with CUDA and ROCm? -
 *    Part 5", section 1.1 The Router Kernel (Top-k Gating): per-token expert
 *    scores from the router weights, the top-2 kept, softmax applied only to
 *    the kept scores.  Section 1.2: tokens are grouped by destination expert
 *    and each expert's FFN runs on the tokens it received.
 *  - "aclnnQuantGroupedMatMulAlltoAllv" (Ascend CANN), function and formula
 *    sections: gmmY = (gmmX @ gmmWeight) * gmmXScale * gmmWeightScale,
 *    unpermuteOut = Unpermute(gmmY); shared expert
 *    mmY = (mmX @ mmWeight) * mmXScale * mmWeightScale; quant mode 1 =
 *    per-tensor; constraints: K in [2, 8], deterministic by default.
 *    Quant modes 4 (pergroup) and 5 (perblock): read as fp32 scales per
 *    group of 128 elements of K (per output channel, or per 128 x 128 weight
 *    block, with per-token-per-group activation scales).
 *    Quant mode 6 ("mx"): read as OCP MXFP8, e4m3 elements in blocks of 32
 *    along the reduction dimension, each block with an E8M0 power-of-two scale.
 *  - zyxy.net "SpMM ... MoE inference", MoE structure: y = sum_i g_i(x)*E_i(x);
 *    expert selection: gating matrix (N, E), top-K index matrix (N, K),
 *    binary expert-activation matrix (N, E); SpMM section: C = A @ B.
 *
 * Readings where the pages are silent: ties in the top-K go to the lower
 * expert index; the K kept slots are ordered by descending logit; the
 * softmax subtracts the largest kept logit; within one expert the permuted
 * rows are ordered by (token, slot) ascending; expert FFNs have no biases;
 * SwiGLU h = silu(x Wg) * (x Wu), silu(z) = z / (1 + exp(-z)).
 *
 * Weight layout: each expert matrix is stored output-major,
 * W[e][n][k] = (E, d_out, d_in) row-major, the transpose of the page's
 * logical (e, H1, N1).  Router weight W_r is (d, E) row-major fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2

#define ORC_ACT_NONE 0
#define ORC_ACT_RELU 1
#define ORC_ACT_SWIGLU 2

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_INDEX 2

/* ------------------------------------------------------------------------ */
/* number formats                                                           */
/* ------------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
double orc_bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* OCP FP8 E4M3 ("FN"): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; exponent field 0 is subnormal. */
double orc_e4m3_to_f64(uint8_t c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);              /* m/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* double -> e4m3, round to nearest even, saturating to +-448 (NaN -> 0x7F). */
uint8_t orc_f64_to_e4m3(double v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs(v);
    if (a > 448.0) a = 448.0;
    if (a < ldexp(1.0, -6)) {
        int q = (int)nearbyint(ldexp(a, 9));   /* q == 8 is the smallest normal */
        return sign | (uint8_t)q;
    }
    int ex;
    frexp(a, &ex);
    int e = ex - 1;                            /* a = s * 2^e, s in [1,2) */
    double s = ldexp(a, -e);
    int q = (int)nearbyint((s - 1.0) * 8.0);
    if (q == 8) { q = 0; e += 1; }
    return sign | (uint8_t)(((e + 7) << 3) | q);
}

/* double -> bf16, round to nearest even (inf on overflow). */
uint16_t orc_f64_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);
    int e = ex - 1;
    if (e < -126) {                            /* subnormal: step 2^-133 */
        long q = lrint(ldexp(a, 133));
        return sign | (uint16_t)q;             /* q == 128 is the smallest normal */
    }
    double s = ldexp(a, -e);
    long q = lrint(s * 128.0);                 /* 8 significant bits */
    if (q == 256) { q = 128; e += 1; }
    if (e > 127) return sign | 0x7F80;
    return sign | (uint16_t)(((e + 127) << 7) | (q - 128));
}

static double load_elem(const void* base, int dtype, int64_t i) {
    switch (dtype) {
    case ORC_F32: return (double)((const float*)base)[i];
    case ORC_BF16: return orc_bf16_to_f64(((const uint16_t*)base)[i]);
    default: return orc_e4m3_to_f64(((const uint8_t*)base)[i]);
    }
}


/* Convert n elements starting at element `first` to double. */
void orc_to_f64(const void* base, int dtype, int64_t first, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = load_elem(base, dtype, first + i);
}

/* ------------------------------------------------------------------------ */
/* router: logits, top-K, softmax over the kept K                           */
/* ------------------------------------------------------------------------ */

/* One token: L[e] = sum_k x[k] * W_r[k][e] (+ b[e]), summed over k ascending. */
static void token_logits(int d, int E, const double* x, const float* w_r, const float* bias,
                         double* L) {
    for (int e = 0; e < E; ++e) L[e] = 0.0;
    for (int k = 0; k < d; ++k) {
        double xk = x[k];
        const float* wrow = w_r + (int64_t)k * E;
        for (int e = 0; e < E; ++e) L[e] += xk * (double)wrow[e];
    }
    if (bias)
        for (int e = 0; e < E; ++e) L[e] += (double)bias[e];
}

/* Keep the K largest logits: K passes, each taking the largest not yet
 * taken; equal values go to the lower expert index (strict '>' while
 * scanning e upward).  margin = (K-th largest) - ((K+1)-th largest), +inf
 * when K == E.  Gates: softmax over the kept logits only. */
static void token_topk(int E, int K, const double* L, int32_t* ids, double* gates,
                       double* margin, unsigned char* taken) {
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < K; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || L[e] > L[best])) best = e;
        taken[best] = 1;
        ids[j] = best;
    }
    if (margin) {
        if (K == E) {
            *margin = INFINITY;
        } else {
            int next = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (next < 0 || L[e] > L[next])) next = e;
            *margin = L[ids[K - 1]] - L[next];
        }
    }
    if (gates) {
        double lmax = L[ids[0]], z = 0.0;
        for (int j = 0; j < K; ++j) z += exp(L[ids[j]] - lmax);
        for (int j = 0; j < K; ++j) gates[j] = exp(L[ids[j]] - lmax) / z;
    }
}

/* Router over N tokens.  x: (N, d) in x_dtype; w_r: (d, E) fp32; bias: (E)
 * or NULL.  Outputs ids (N, K), gates (N, K), margin (N) (may be NULL),
 * logits (N, E) (may be NULL). */
int orc_router(int N, int d, int E, int K, int x_dtype, const void* x, const float* w_r,
               const float* bias, int32_t* ids, double* gates, double* margin, double* logits) {
    if (N < 0 || d <= 0 || E <= 0 || K <= 0 || K > E || !x || !w_r || !ids) return ORC_ERR_ARG;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)d);
        double* L = (double*)malloc(sizeof(double) * (size_t)E);
        unsigned char* taken = (unsigned char*)malloc((size_t)E);
#pragma omp for schedule(static)
        for (int t = 0; t < N; ++t) {
            orc_to_f64(x, x_dtype, (int64_t)t * d, d, xr);
            token_logits(d, E, xr, w_r, bias, L);
            if (logits) memcpy(logits + (int64_t)t * E, L, sizeof(double) * (size_t)E);
            token_topk(E, K, L, ids + (int64_t)t * K, gates ? gates + (int64_t)t * K : NULL,
                       margin ? margin + t : NULL, taken);
        }
        free(xr); free(L); free(taken);
    }
    return ORC_OK;
}

/* Top-K + sparse softmax on given logits (N, E) (used by the pins). */
int orc_topk_from_logits(int N, int E, int K, const double* logits, int32_t* ids, double* gates,
                         double* margin) {
    if (N < 0 || E <= 0 || K <= 0 || K > E) return ORC_ERR_ARG;
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    for (int t = 0; t < N; ++t)
        token_topk(E, K, logits + (int64_t)t * E, ids + (int64_t)t * K,
                   gates ? gates + (int64_t)t * K : NULL, margin ? margin + t : NULL, taken);
    free(taken);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* permute: histogram, exclusive scan, stable expert-major placement        */
/* ------------------------------------------------------------------------ */

/* counts[e] = #{(t,j) : ids[t][j] = e}; offsets = exclusive prefix sum of
 * counts (E+1 entries, offsets[E] = N*K); pos[t*K+j] = offsets[e] + number
 * of earlier (t',j') in (token, slot) order with the same expert; src[pos] =
 * t; x_perm[pos] = x[t] (byte copy of row_bytes; skipped when x or x_perm is
 * NULL).  One sequential pass with a cursor per expert. */
int orc_permute(int N, int K, int E, const int32_t* ids, const void* x, int64_t row_bytes,
                int32_t* counts, int32_t* offsets, int32_t* pos, int32_t* src, void* x_perm) {
    if (N < 0 || K <= 0 || E <= 0 || !ids || !counts || !offsets) return ORC_ERR_ARG;
    for (int64_t i = 0; i < (int64_t)N * K; ++i)
        if (ids[i] < 0 || ids[i] >= E) return ORC_ERR_INDEX;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < (int64_t)N * K; ++i) counts[ids[i]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int t = 0; t < N; ++t)
        for (int j = 0; j < K; ++j) {
            int e = ids[(int64_t)t * K + j];
            int p = cursor[e]++;
            if (pos) pos[(int64_t)t * K + j] = p;
            if (src) src[p] = t;
            if (x && x_perm)
                memcpy((char*)x_perm + (int64_t)p * row_bytes, (const char*)x + (int64_t)t * row_bytes,
                       (size_t)row_bytes);
        }
    free(cursor);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* expert FFN                                                               */
/* ------------------------------------------------------------------------ */

/* sum_k a[k] * W[row][k] over k ascending, W in w_dtype, row-major (.., din). */
static double dot_row(int din, const double* a, const void* w, int w_dtype, int64_t row) {
    double acc = 0.0;
    int64_t base = row * din;
    switch (w_dtype) {
    case ORC_F32: {
        const float* p = (const float*)w + base;
        for (int k = 0; k < din; ++k) acc += a[k] * (double)p[k];
        break;
    }
    case ORC_BF16: {
        const uint16_t* p = (const uint16_t*)w + base;
        for (int k = 0; k < din; ++k) acc += a[k] * orc_bf16_to_f64(p[k]);
        break;
    }
    default: {
        const uint8_t* p = (const uint8_t*)w + base;
        for (int k = 0; k < din; ++k) acc += a[k] * orc_e4m3_to_f64(p[k]);
        break;
    }
    }
    return acc;
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* One expert on one input row (already in double).
 *  act NONE:   y[n] = (sum_k x[k] W1[e][n][k]) * x_scale * w_scale,  n < F
 *  act RELU:   h = relu(x W1[e]^T) (F),  y = h W2[e]^T (din)
 *  act SWIGLU: h = silu(x W1[e]^T) * (x W3[e]^T),  y = h W2[e]^T (din)
 * h is kept in double (not rounded). */
static void expert_row(int e, int din, int F, int act, int w_dtype, const void* w1, const void* w3,
                       const void* w2, double x_scale, double w_scale, const double* x, double* h,
                       double* y) {
    if (act == ORC_ACT_NONE) {
        for (int n = 0; n < F; ++n)
            y[n] = dot_row(din, x, w1, w_dtype, (int64_t)e * F + n) * x_scale * w_scale;
        return;
    }
    for (int n = 0; n < F; ++n) {
        double g = dot_row(din, x, w1, w_dtype, (int64_t)e * F + n);
        if (act == ORC_ACT_RELU) {
            h[n] = g > 0.0 ? g : 0.0;
        } else {
            double u = dot_row(din, x, w3, w_dtype, (int64_t)e * F + n);
            h[n] = silu(g) * u;
        }
    }
    for (int n = 0; n < din; ++n) y[n] = dot_row(F, h, w2, w_dtype, (int64_t)e * din + n);
}

static int ffn_args_ok(int din, int F, int act, const void* w1, const void* w3, const void* w2) {
    if (din <= 0 || F <= 0 || !w1) return 0;
    if (act == ORC_ACT_SWIGLU && (!w3 || !w2)) return 0;
    if (act == ORC_ACT_RELU && !w2) return 0;
    return act >= ORC_ACT_NONE && act <= ORC_ACT_SWIGLU;
}

/* Run expert row_expert[r] on input row r of xrows (nrows, din) in x_dtype.
 * y: (nrows, d_out), d_out = F for act NONE else din.  A row whose expert is
 * negative is skipped (left untouched). */
int orc_expert_rows(int nrows, const int32_t* row_expert, int E, int din, int x_dtype,
                    const void* xrows, int act, int F, int w_dtype, const void* w1, const void* w3,
                    const void* w2, double x_scale, double w_scale, double* y) {
    if (nrows < 0 || !row_expert || !xrows || !y || !ffn_args_ok(din, F, act, w1, w3, w2))
        return ORC_ERR_ARG;
    for (int r = 0; r < nrows; ++r)
        if (row_expert[r] >= E) return ORC_ERR_INDEX;
    int dout = act == ORC_ACT_NONE ? F : din;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)din);
        double* h = (double*)malloc(sizeof(double) * (size_t)F);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            if (row_expert[r] < 0) continue;
            orc_to_f64(xrows, x_dtype, (int64_t)r * din, din, xr);
            expert_row(row_expert[r], din, F, act, w_dtype, w1, w3, w2, x_scale, w_scale, xr, h,
                       y + (int64_t)r * dout);
        }
        free(xr); free(h);
    }
    return ORC_OK;
}

/* Single-matrix experts with finer scales (Ascend quant modes 2 = per-channel
 * for the weights, 3 = per-token for the activations):
 *   y[r][n] = (sum_k x[r][k] W[e][n][k]) * xs[r] * ws[e][n]
 * xs: one scale per input row (NULL: x_scale for all); ws: (E, F) per output
 * channel of each expert (NULL: w_scale for all). */
int orc_expert_rows_scaled(int nrows, const int32_t* row_expert, int E, int din, int x_dtype,
                           const void* xrows, int F, int w_dtype, const void* w1, double x_scale,
                           const double* xs, double w_scale, const double* ws, double* y) {
    if (nrows < 0 || !row_expert || !xrows || !y || !w1 || din <= 0 || F <= 0) return ORC_ERR_ARG;
    for (int r = 0; r < nrows; ++r)
        if (row_expert[r] >= E) return ORC_ERR_INDEX;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)din);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            int e = row_expert[r];
            if (e < 0) continue;
            orc_to_f64(xrows, x_dtype, (int64_t)r * din, din, xr);
            double sx = xs ? xs[r] : x_scale;
            for (int n = 0; n < F; ++n) {
                double sw = ws ? ws[(int64_t)e * F + n] : w_scale;
                y[(int64_t)r * F + n] = dot_row(din, xr, w1, w_dtype, (int64_t)e * F + n) * sx * sw;
            }
        }
        free(xr);
    }
    return ORC_OK;
}

/* E8M0 (OCP Microscaling Formats v1.0, the shared block scale): eight
 * exponent bits with bias 127, no sign and no mantissa; 0xFF encodes NaN. */
double orc_e8m0_to_f64(uint8_t s) {
    if (s == 0xFF) return NAN;
    return ldexp(1.0, (int)s - 127);
}

/* Single-matrix experts with MX block scales (Ascend quant mode 6, "mx"; the
 * block format is OCP MXFP8: 32 consecutive e4m3 elements along the
 * reduction dimension share one E8M0 scale):
 *   y[r][n] = sum_k (x[r][k] * 2^(xs[r][k/32] - 127)) * (W[e][n][k] * 2^(ws[e][n][k/32] - 127))
 * with k ascending.  x (nrows, din) e4m3 codes, xs (nrows, din/32) E8M0;
 * W (E, F, din) e4m3 (output-major), ws (E, F, din/32) E8M0; din a multiple
 * of 32.  The page names the mode only; the block of 32 and E8M0 scales are
 * the MX format's own definition. */
int orc_expert_rows_mx(int nrows, const int32_t* row_expert, int E, int din, const uint8_t* x,
                       const uint8_t* xs, int F, const uint8_t* w, const uint8_t* ws, double* y) {
    if (nrows < 0 || !row_expert || !x || !xs || !w || !ws || !y || din <= 0 || F <= 0 ||
        din % 32 != 0)
        return ORC_ERR_ARG;
    for (int r = 0; r < nrows; ++r)
        if (row_expert[r] >= E) return ORC_ERR_INDEX;
    const int nb = din / 32;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)din);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            int e = row_expert[r];
            if (e < 0) continue;
            for (int k = 0; k < din; ++k)
                xr[k] = orc_e4m3_to_f64(x[(int64_t)r * din + k]) *
                        orc_e8m0_to_f64(xs[(int64_t)r * nb + k / 32]);
            for (int n = 0; n < F; ++n) {
                int64_t wrow = (int64_t)e * F + n;
                double acc = 0.0;
                for (int k = 0; k < din; ++k)
                    acc += xr[k] * (orc_e4m3_to_f64(w[wrow * din + k]) *
                                    orc_e8m0_to_f64(ws[wrow * nb + k / 32]));
                y[(int64_t)r * F + n] = acc;
            }
        }
        free(xr);
    }
    return ORC_OK;
}

/* Single-matrix experts with fp32 scales per group of 128 elements of K
 * (Ascend quant modes 4 "pergroup" and 5 "perblock"; the page names the
 * modes only, the group of 128 along the reduction dimension is this
 * layer's reading):
 *   y[r][n] = sum_g xs[r][g] * ws[e][n][g] * (sum_{k in group g} x[r][k] * W[e][n][k])
 * groups g = 0 .. din/128 - 1 ascending, k ascending inside a group.
 * xs (nrows, din/128): the activation scale of each row and group (NULL:
 * x_scale for all); ws (E, F, din/128): the weight scale of each output
 * channel and group.  Per-group weights (mode 4) give ws directly; 128 x 128
 * weight blocks (mode 5) repeat one scale over the 128 channels of a block. */
int orc_expert_rows_kscaled(int nrows, const int32_t* row_expert, int E, int din, int x_dtype,
                            const void* xrows, const double* xs, double x_scale, int F,
                            int w_dtype, const void* w1, const double* ws, double* y) {
    if (nrows < 0 || !row_expert || !xrows || !w1 || !ws || !y || din <= 0 || F <= 0 ||
        din % 128 != 0)
        return ORC_ERR_ARG;
    for (int r = 0; r < nrows; ++r)
        if (row_expert[r] >= E) return ORC_ERR_INDEX;
    const int ng = din / 128;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)din);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            int e = row_expert[r];
            if (e < 0) continue;
            orc_to_f64(xrows, x_dtype, (int64_t)r * din, din, xr);
            for (int n = 0; n < F; ++n) {
                int64_t wrow = (int64_t)e * F + n;
                double acc = 0.0;
                for (int g = 0; g < ng; ++g) {
                    double part = 0.0;
                    for (int k = 128 * g; k < 128 * g + 128; ++k)
                        part += xr[k] * load_elem(w1, w_dtype, wrow * din + k);
                    double sx = xs ? xs[(int64_t)r * ng + g] : x_scale;
                    acc += sx * ws[wrow * ng + g] * part;
                }
                y[(int64_t)r * F + n] = acc;
            }
        }
        free(xr);
    }
    return ORC_OK;
}

/* Per-token dynamic quantization (Ascend quant mode 7, "pertoken dynamic
 * quantization", parameter section): each token row of bf16 activations gets
 * its own scale amax(|row|) / 448 (448 = the largest e4m3 value; 1 for an
 * all-zero row) and codes e4m3(x / scale), rounded to nearest even and
 * saturated.  The page fixes no precision for this step; the layer takes it
 * in fp32, and since the codes are integers decided by that arithmetic, the
 * oracle takes the same decisions: the amax is exact, the two divisions are
 * IEEE binary32 divisions (this file is compiled without fast-math or
 * contraction), and the binary32 quotient is then rounded to e4m3 by the
 * encoder above. */
int orc_quantize_rows_dynamic(int n, int d, const uint16_t* x, uint8_t* codes, float* scales) {
    if (n < 0 || d <= 0 || !x || !codes || !scales) return ORC_ERR_ARG;
    for (int r = 0; r < n; ++r) {
        const uint16_t* row = x + (int64_t)r * d;
        float amax = 0.0f;
        for (int k = 0; k < d; ++k) {
            float v = fabsf((float)orc_bf16_to_f64(row[k]));
            if (v > amax) amax = v;
        }
        volatile float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
        scales[r] = scale;
        for (int k = 0; k < d; ++k) {
            volatile float q = (float)orc_bf16_to_f64(row[k]) / scale;
            codes[(int64_t)r * d + k] = orc_f64_to_e4m3((double)q);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* unpermute / combine                                                      */
/* ------------------------------------------------------------------------ */

/* gates != NULL: y[t] = sum_{j=0..K-1} gates[t][j] * y_perm[pos[t][j]]  (N, dout)
 * gates == NULL: y[t*K + j] = y_perm[pos[t][j]]                          (N*K, dout) */
int orc_combine(int N, int K, int dout, const int32_t* pos, const double* gates,
                const double* y_perm, double* y) {
    if (N < 0 || K <= 0 || dout <= 0 || !pos || !y_perm || !y) return ORC_ERR_ARG;
    for (int t = 0; t < N; ++t) {
        if (gates) {
            double* yt = y + (int64_t)t * dout;
            for (int n = 0; n < dout; ++n) yt[n] = 0.0;
            for (int j = 0; j < K; ++j) {
                double g = gates[(int64_t)t * K + j];
                const double* src = y_perm + (int64_t)pos[(int64_t)t * K + j] * dout;
                for (int n = 0; n < dout; ++n) yt[n] += g * src[n];
            }
        } else {
            for (int j = 0; j < K; ++j)
                memcpy(y + ((int64_t)t * K + j) * dout,
                       y_perm + (int64_t)pos[(int64_t)t * K + j] * dout, sizeof(double) * (size_t)dout);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* whole layer, token by token (no permutation involved)                    */
/* ------------------------------------------------------------------------ */

/* For each listed token t = tok[i]: route it (router weights, or the given
 * ids when w_r is NULL, with gates then taken from `given_gates` or 1), run
 * its K experts on x[t] and form
 *   gates_mode 1: y[i] = sum_j g[t][j] * E_{ids[t][j]}(x[t])          (ntok, dout)
 *   gates_mode 0: y[i*K + j] = E_{ids[t][j]}(x[t])                       (ntok*K, dout)
 * Outputs ids_out (ntok, K), gates_out (ntok, K), margin_out (ntok) may be NULL. */
int orc_forward_tokens(int ntok, const int32_t* tok, int N, int d, int E, int K, int x_dtype,
                       const void* x, const float* w_r, const float* bias, const int32_t* given_ids,
                       int act, int F, int w_dtype, const void* w1, const void* w3, const void* w2,
                       double x_scale, double w_scale, int gates_mode, double* y, int32_t* ids_out,
                       double* gates_out, double* margin_out) {
    if (ntok < 0 || !tok || d <= 0 || E <= 0 || K <= 0 || K > E || K > 64 || !x || !y)
        return ORC_ERR_ARG;
    if (!w_r && !given_ids) return ORC_ERR_ARG;
    if (!ffn_args_ok(d, F, act, w1, w3, w2)) return ORC_ERR_ARG;
    for (int i = 0; i < ntok; ++i)
        if (tok[i] < 0 || tok[i] >= N) return ORC_ERR_INDEX;
    if (given_ids)
        for (int i = 0; i < ntok; ++i)
            for (int j = 0; j < K; ++j) {
                int32_t e = given_ids[(int64_t)tok[i] * K + j];
                if (e < 0 || e >= E) return ORC_ERR_INDEX;
            }
    int dout = act == ORC_ACT_NONE ? F : d;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)d);
        double* L = (double*)malloc(sizeof(double) * (size_t)E);
        double* h = (double*)malloc(sizeof(double) * (size_t)F);
        double* ye = (double*)malloc(sizeof(double) * (size_t)dout);
        unsigned char* taken = (unsigned char*)malloc((size_t)E);
        int32_t ids[64];
        double g[64], margin = INFINITY;
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < ntok; ++i) {
            int t = tok[i];
            orc_to_f64(x, x_dtype, (int64_t)t * d, d, xr);
            if (w_r) {
                token_logits(d, E, xr, w_r, bias, L);
                token_topk(E, K, L, ids, g, &margin, taken);
            } else {
                for (int j = 0; j < K; ++j) { ids[j] = given_ids[(int64_t)t * K + j]; g[j] = 1.0; }
                margin = INFINITY;
            }
            if (gates_mode) {
                double* yt = y + (int64_t)i * dout;
                for (int n = 0; n < dout; ++n) yt[n] = 0.0;
                for (int j = 0; j < K; ++j) {
                    expert_row(ids[j], d, F, act, w_dtype, w1, w3, w2, x_scale, w_scale, xr, h, ye);
                    for (int n = 0; n < dout; ++n) yt[n] += g[j] * ye[n];
                }
            } else {
                for (int j = 0; j < K; ++j)
                    expert_row(ids[j], d, F, act, w_dtype, w1, w3, w2, x_scale, w_scale, xr, h,
                               y + ((int64_t)i * K + j) * dout);
            }
            for (int j = 0; j < K; ++j) {
                if (ids_out) ids_out[(int64_t)i * K + j] = ids[j];
                if (gates_out) gates_out[(int64_t)i * K + j] = g[j];
            }
            if (margin_out) margin_out[i] = margin;
        }
        free(xr); free(L); free(h); free(ye); free(taken);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* dense masked reference (every expert on every token)                     */
/* ------------------------------------------------------------------------ */

/* G: (N, E) gate matrix (zero where an expert is not selected).
 * y[t] = sum_{e=0..E-1} G[t][e] * E_e(x[t]), every expert evaluated. */
int orc_dense_masked(int N, int d, int E, int x_dtype, const void* x, const double* G, int act,
                     int F, int w_dtype, const void* w1, const void* w3, const void* w2,
                     double x_scale, double w_scale, double* y) {
    if (N < 0 || !x || !G || !y || !ffn_args_ok(d, F, act, w1, w3, w2)) return ORC_ERR_ARG;
    int dout = act == ORC_ACT_NONE ? F : d;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)d);
        double* h = (double*)malloc(sizeof(double) * (size_t)F);
        double* ye = (double*)malloc(sizeof(double) * (size_t)dout);
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < N; ++t) {
            orc_to_f64(x, x_dtype, (int64_t)t * d, d, xr);
            double* yt = y + (int64_t)t * dout;
            for (int n = 0; n < dout; ++n) yt[n] = 0.0;
            for (int e = 0; e < E; ++e) {
                expert_row(e, d, F, act, w_dtype, w1, w3, w2, x_scale, w_scale, xr, h, ye);
                double g = G[(int64_t)t * E + e];
                for (int n = 0; n < dout; ++n) yt[n] += g * ye[n];
            }
        }
        free(xr); free(h); free(ye);
    }
    return ORC_OK;
}

/* Plain matmul C (n, m) = A (n, k) @ B (k, m), double, naive (SpMM page's
 * dense C = A @ B). */
void orc_matmul(int n, int k, int m, const double* A, const double* B, double* C) {
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < m; ++j) {
            double acc = 0.0;
            for (int p = 0; p < k; ++p) acc += A[(int64_t)i * k + p] * B[(int64_t)p * m + j];
            C[(int64_t)i * m + j] = acc;
        }
}

int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
