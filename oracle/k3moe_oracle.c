/*
 * ORACLE -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar fp64 CPU statement of the MXFP4 routed-expert MoE
 * layer.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load it; the library's product path never does.  It shares no code
 * with the CUDA library.
 *
 * What it computes, per token t, in the order the sources give it:
 *   logits   l_e = sum_j x_j W_r[e,j] + b_e                  (router GEMV)
 *   softmax  p_e = exp(l_e - max l) / sum_e' exp(l_e' - max l) over all E
 *   top-k    the k experts with the largest l (same order as p), ties to the
 *            lower index, listed in descending order; w_j = p_idx_j, no
 *            renormalisation over the k picks
 *   experts  o_e = W_d,e (silu(W_g,e x) * W_u,e x), silu(z) = z / (1 + e^-z)
 *   shared   S = W_d,s (silu(W_g,s x) * W_u,s x), bf16 weights, weight 1
 *   combine  y = S + sum_j w_j o_idx_j
 * Sources: "Kimi K3 纯 C 语言 CPU 推理实战" (chenxutan.com), section 1.2 (the
 * routing formula y = sum g_i E_i, g = TopK(Softmax(W_gate x)), K = 16, 896
 * experts plus a shared expert) and section 2.4 (gate scores as a GEMV,
 * numerically stable softmax over all experts, top-k selection, weighted
 * combine); the kimi-k3-in-c project card ("P053"), core features (experts
 * multiplied directly on packed nibbles; MXFP4 = 4-bit E2M1 nibble plus a
 * shared E8M0 scale, 0.53125 bytes per weight).
 *
 * MXFP4 element (r, c) of a [rows][cols] matrix: nibble at byte
 * r*cols/2 + c/2, low nibble (bits 0-3) for even c, high nibble for odd c;
 * value E2M1(nibble) * 2^(scale[r][c/32] - 127).  E2M1 bit layout (sign bit 3,
 * 2 exponent bits with bias 1, 1 mantissa bit) and E8M0 (2^(e-127), 255 = NaN)
 * follow the OCP Microscaling Formats (MX) v1.0 specification, since the
 * pages only name the formats.
 *
 * All arithmetic is fp64; every sum runs in ascending index order, so the
 * result does not depend on the OpenMP thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* E2M1 magnitudes for codes 0..7: exponent field e (bits 2-1), mantissa m
 * (bit 0): e == 0 -> m * 0.5 (subnormal), else 2^(e-1) * (1 + m/2). */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1(unsigned nib) {
    double v = kE2M1[nib & 7u];
    return (nib & 8u) ? -v : v;
}

double oracle_e8m0(unsigned e) {
    if ((e & 0xFFu) == 255u) return NAN;
    return ldexp(1.0, (int)(e & 0xFFu) - 127);
}

double oracle_bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* bfloat16 nearest to v, ties to even, as bits (normal range; inf/nan kept) */
uint16_t oracle_bf16_rne(double v) {
    if (v == 0.0 || isnan(v) || isinf(v)) {
        float f = (float)v;
        uint32_t u;
        memcpy(&u, &f, 4);
        if (isnan(v)) return 0x7FC0u;
        return (uint16_t)(u >> 16);
    }
    int e;
    double m = frexp(fabs(v), &e);
    double r = nearbyint(ldexp(m, 8));
    double q = ldexp(r, e - 8);
    float f = (float)q;
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t h = (uint16_t)(u >> 16);
    if (v < 0) h |= 0x8000u;
    return h;
}

double oracle_mxfp4_weight(const uint8_t *nib, const uint8_t *scale, int64_t cols, int64_t r,
                           int64_t c) {
    uint8_t byte = nib[r * (cols / 2) + c / 2];
    unsigned code = (c & 1) ? (byte >> 4) : (byte & 0xFu);
    return oracle_e2m1(code) * oracle_e8m0(scale[r * (cols / 32) + c / 32]);
}

/* out[r] = sum_c W[r,c] v[c], W MXFP4 [rows][cols] */
void oracle_mxfp4_matvec(const uint8_t *nib, const uint8_t *scale, int64_t rows, int64_t cols,
                         const double *v, double *out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int64_t c = 0; c < cols; ++c) s += oracle_mxfp4_weight(nib, scale, cols, r, c) * v[c];
        out[r] = s;
    }
}

/* out[r] = sum_c W[r,c] v[c], W bf16 [rows][cols] */
void oracle_bf16_matvec(const uint16_t *w, int64_t rows, int64_t cols, const double *v,
                        double *out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int64_t c = 0; c < cols; ++c) s += oracle_bf16_value(w[r * cols + c]) * v[c];
        out[r] = s;
    }
}

/* logits[t][e] = sum_j x[t][j] W_r[e][j] + bias[e] (bias may be NULL) */
void oracle_router_logits(const uint16_t *x, int64_t T, const float *w, const float *bias,
                          int64_t d, int64_t E, double *logits) {
    for (int64_t t = 0; t < T; ++t) {
#pragma omp parallel for schedule(static)
        for (int64_t e = 0; e < E; ++e) {
            double s = 0.0;
            for (int64_t j = 0; j < d; ++j)
                s += oracle_bf16_value(x[t * d + j]) * (double)w[e * d + j];
            if (bias) s += (double)bias[e];
            logits[t * E + e] = s;
        }
    }
}

/* numerically stable softmax over all E entries */
void oracle_softmax(const double *l, int64_t E, double *p) {
    double m = l[0];
    for (int64_t e = 1; e < E; ++e)
        if (l[e] > m) m = l[e];
    double z = 0.0;
    for (int64_t e = 0; e < E; ++e) z += exp(l[e] - m);
    for (int64_t e = 0; e < E; ++e) p[e] = exp(l[e] - m) / z;
}

static const double *g_sort_keys;
static int cmp_desc_then_index(const void *a, const void *b) {
    int32_t i = *(const int32_t *)a, j = *(const int32_t *)b;
    double li = g_sort_keys[i], lj = g_sort_keys[j];
    if (li > lj) return -1;
    if (li < lj) return 1;
    return (i > j) - (i < j);
}

/* first k of all experts sorted by (-l_e, e): a full sort, then truncate */
void oracle_topk(const double *l, int64_t E, int64_t k, int32_t *idx) {
    int32_t *all = (int32_t *)malloc((size_t)E * sizeof(int32_t));
    for (int64_t e = 0; e < E; ++e) all[e] = (int32_t)e;
    g_sort_keys = l;
    qsort(all, (size_t)E, sizeof(int32_t), cmp_desc_then_index);
    for (int64_t j = 0; j < k; ++j) idx[j] = all[j];
    free(all);
}

/* router + softmax + top-k for T tokens; logits / probs may be NULL */
void oracle_route(const uint16_t *x, int64_t T, const float *w, const float *bias, int64_t d,
                  int64_t E, int64_t k, double *logits_out, double *probs_out, int32_t *idx,
                  double *weight) {
    double *l = (double *)malloc((size_t)(T * E) * sizeof(double));
    double *p = (double *)malloc((size_t)E * sizeof(double));
    oracle_router_logits(x, T, w, bias, d, E, l);
    for (int64_t t = 0; t < T; ++t) {
        oracle_softmax(l + t * E, E, p);
        oracle_topk(l + t * E, E, k, idx + t * k);
        for (int64_t j = 0; j < k; ++j) weight[t * k + j] = p[idx[t * k + j]];
        if (probs_out) memcpy(probs_out + t * E, p, (size_t)E * sizeof(double));
    }
    if (logits_out) memcpy(logits_out, l, (size_t)(T * E) * sizeof(double));
    free(p);
    free(l);
}

/*
 * Two routing variants the pages leave open (their routing formula uses the
 * raw softmax probability of each pick and adds no bias), written out for
 * parity with the library's flags:
 *   bias_select_only: the bias moves only the selection -- the top-k is taken
 *     on s_e = l_e + b_e, while p is the softmax of the unbiased l;
 *   renorm: the k weights are rescaled to sum to one over the picks,
 *     w_j = p_idx_j / sum_j' p_idx_j' (the sum in pick order).
 * With both off this is oracle_route.  logits_out receives l (unbiased when
 * bias_select_only, else l + b); probs_out the softmax p.
 */
void oracle_route_variant(const uint16_t *x, int64_t T, const float *w, const float *bias,
                          int64_t d, int64_t E, int64_t k, int renorm, int bias_select_only,
                          double *logits_out, double *probs_out, int32_t *idx, double *weight) {
    double *l = (double *)malloc((size_t)(T * E) * sizeof(double));
    double *sel = (double *)malloc((size_t)E * sizeof(double));
    double *p = (double *)malloc((size_t)E * sizeof(double));
    oracle_router_logits(x, T, w, bias_select_only ? NULL : bias, d, E, l);
    for (int64_t t = 0; t < T; ++t) {
        const double *lt = l + t * E;
        for (int64_t e = 0; e < E; ++e) sel[e] = lt[e] + ((bias_select_only && bias) ? (double)bias[e] : 0.0);
        oracle_softmax(lt, E, p);
        oracle_topk(sel, E, k, idx + t * k);
        double z = 0.0;
        for (int64_t j = 0; j < k; ++j) z += p[idx[t * k + j]];
        for (int64_t j = 0; j < k; ++j) {
            const double pj = p[idx[t * k + j]];
            weight[t * k + j] = renorm ? pj / z : pj;
        }
        if (probs_out) memcpy(probs_out + t * E, p, (size_t)E * sizeof(double));
    }
    if (logits_out) memcpy(logits_out, l, (size_t)(T * E) * sizeof(double));
    free(p);
    free(sel);
    free(l);
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Byte offsets of the six planes of a routed expert's blob:
 * [W_g nib | W_g scale | W_u nib | W_u scale | W_d nib | W_d scale]. */
static void blob_planes(const uint8_t *blob, int64_t d, int64_t ff, const uint8_t **p) {
    int64_t mat = d * ff;
    const uint8_t *q = blob;
    for (int m = 0; m < 3; ++m) {
        p[2 * m] = q;
        q += mat / 2;
        p[2 * m + 1] = q;
        q += mat / 32;
    }
}

/* one routed expert on one token, x given in fp64: out[d] = W_d(silu(W_g x) * W_u x) */
void oracle_expert_ffn_vec(const double *xv, const uint8_t *blob, int64_t d, int64_t ff,
                           double *out) {
    const uint8_t *p[6];
    blob_planes(blob, d, ff, p);
    double *g = (double *)malloc((size_t)ff * sizeof(double));
    double *u = (double *)malloc((size_t)ff * sizeof(double));
    oracle_mxfp4_matvec(p[0], p[1], ff, d, xv, g);
    oracle_mxfp4_matvec(p[2], p[3], ff, d, xv, u);
    for (int64_t i = 0; i < ff; ++i) g[i] = silu(g[i]) * u[i];
    oracle_mxfp4_matvec(p[4], p[5], d, ff, g, out);
    free(u);
    free(g);
}

/* one routed expert on T bf16 tokens: out[T][d] */
void oracle_expert_ffn(const uint16_t *x, int64_t T, const uint8_t *blob, int64_t d, int64_t ff,
                       double *out) {
    double *xv = (double *)malloc((size_t)d * sizeof(double));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < d; ++j) xv[j] = oracle_bf16_value(x[t * d + j]);
        oracle_expert_ffn_vec(xv, blob, d, ff, out + t * d);
    }
    free(xv);
}

/* shared expert (bf16 weights) on T tokens: out[T][d] */
void oracle_shared_ffn(const uint16_t *x, int64_t T, const uint16_t *wg, const uint16_t *wu,
                       const uint16_t *wd, int64_t d, int64_t ffs, double *out) {
    double *xv = (double *)malloc((size_t)d * sizeof(double));
    double *g = (double *)malloc((size_t)ffs * sizeof(double));
    double *u = (double *)malloc((size_t)ffs * sizeof(double));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < d; ++j) xv[j] = oracle_bf16_value(x[t * d + j]);
        oracle_bf16_matvec(wg, ffs, d, xv, g);
        oracle_bf16_matvec(wu, ffs, d, xv, u);
        for (int64_t i = 0; i < ffs; ++i) g[i] = silu(g[i]) * u[i];
        oracle_bf16_matvec(wd, d, ffs, g, out + t * d);
    }
    free(u);
    free(g);
    free(xv);
}

/*
 * y[t] = S(x_t) + sum_j weight[t][j] * o_{expert of slot (t,j)}(x_t), fp64.
 * slot_blobs[t*k + j] is the blob of the expert in slot j of token t (the
 * caller resolves idx -> blob, so only the selected experts need to exist in
 * host memory).  wg/wu/wd == NULL: no shared expert.
 */
void oracle_combine(const uint16_t *x, int64_t T, const double *weight, int64_t k,
                    const uint8_t *const *slot_blobs, const uint16_t *wg, const uint16_t *wu,
                    const uint16_t *wd, int64_t d, int64_t ff, int64_t ffs, double *y) {
    double *xv = (double *)malloc((size_t)d * sizeof(double));
    double *o = (double *)malloc((size_t)d * sizeof(double));
    if (wg && wu && wd && ffs > 0)
        oracle_shared_ffn(x, T, wg, wu, wd, d, ffs, y);
    else
        memset(y, 0, (size_t)(T * d) * sizeof(double));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < d; ++j) xv[j] = oracle_bf16_value(x[t * d + j]);
        for (int64_t s = 0; s < k; ++s) {
            oracle_expert_ffn_vec(xv, slot_blobs[t * k + s], d, ff, o);
            double w = weight[t * k + s];
            for (int64_t i = 0; i < d; ++i) y[t * d + i] += w * o[i];
        }
    }
    free(o);
    free(xv);
}

/*
 * The steps on either side of the layer in a pre-norm transformer block (the
 * kimi-k3-in-c project card names RMSNorm among its k3_ops.c kernels and the
 * dense trunk's normalisation parameters; the pages give no formula, so the
 * standard one is taken):
 *   x_j = RNE_bf16( h_j g_j / sqrt(mean_j h_j^2 + eps) )   (the layer's input)
 *   out = h + y                                            (the residual add)
 * h, g bf16; the norm in fp64, rounded once to bf16 (the layer takes bf16).
 */
void oracle_rmsnorm(const uint16_t *h, int64_t T, const uint16_t *g, double eps, int64_t d,
                    uint16_t *x_out) {
    for (int64_t t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int64_t j = 0; j < d; ++j) {
            const double v = oracle_bf16_value(h[t * d + j]);
            ss += v * v;
        }
        const double r = 1.0 / sqrt(ss / (double)d + eps);
        for (int64_t j = 0; j < d; ++j)
            x_out[t * d + j] =
                oracle_bf16_rne(oracle_bf16_value(h[t * d + j]) * r * oracle_bf16_value(g[j]));
    }
}

/* out[t][j] = h[t][j] + y[t][j] in fp64 */
void oracle_residual_add(const uint16_t *h, int64_t T, int64_t d, const double *y, double *out) {
    for (int64_t i = 0; i < T * d; ++i) out[i] = oracle_bf16_value(h[i]) + y[i];
}

/* the whole layer; blobs[e] is expert e's blob (all E present) */
void oracle_layer(const uint16_t *x, int64_t T, const float *w_router, const float *bias,
                  const uint8_t *const *blobs, const uint16_t *wg, const uint16_t *wu,
                  const uint16_t *wd, int64_t d, int64_t ff, int64_t E, int64_t k, int64_t ffs,
                  double *y, int32_t *idx, double *weight) {
    oracle_route(x, T, w_router, bias, d, E, k, NULL, NULL, idx, weight);
    const uint8_t **slot = (const uint8_t **)malloc((size_t)(T * k) * sizeof(void *));
    for (int64_t i = 0; i < T * k; ++i) slot[i] = blobs[idx[i]];
    oracle_combine(x, T, weight, k, slot, wg, wu, wd, d, ff, ffs, y);
    free(slot);
}
