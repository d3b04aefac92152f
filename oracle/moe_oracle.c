/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of the routed Mixture-of-Experts FFN
 * layer (softmax top-k router, GEGLU experts, weighted combine).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library calls, links or loads this file:
 * only the tests, the package smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes (the plain definition, written out):
 *   The pages name the layer and its parts but print no formula, so each step below
 *   takes the plainest reading of the names they give:
 *   - router logits L[t,e] = sum_h x[t,h] * Wr[h,e] (+ b_e), the linear gate feeding the
 *     fused "gating top-k softmax" router op (cann-recipes-infer "Gemma-4-26B-A4B 模型优化报告"
 *     §5 阶段3 融合算子, MoE Router npu_moe_gating_top_k_softmax; 128 experts on a 2816
 *     hidden, §1 模型概况 and the NVFP4 verification report §2.1 模型架构参数);
 *   - selection: the k experts with the largest logits, slot 0 = largest, equal logits
 *     ordered by the lower expert id (top-8 of 128, §1 模型概况);
 *   - weights: softmax over all E logits, then the k selected probabilities renormalised to
 *     sum to one (or left as they are when renorm == 0);
 *   - dispatch: per-expert counts, exclusive-scan offsets, and a stable permutation that
 *     lists, expert by expert, the (token, slot) pairs in ascending token order (the
 *     per-expert "split sizes" of the double_routing dispatch, §6.1 方案);
 *   - expert e: h = gelu_tanh(x Wg_e) * (x Wu_e), o = h Wd_e  (GEGLU with intermediate 704,
 *     §1 模型概况; activation gelu_pytorch_tanh, verification report §2.1);
 *   - combine: y[t] = sum_j w[t,j] * o_{t,j}.
 *
 * Precision: every bf16 input is widened exactly to double; each bf16*bf16 product is
 * exact in double; sums run in ascending index order with plain double additions (build
 * WITHOUT -ffast-math / reassociation; contraction to FMA is harmless because the products
 * are exact).  No intermediate result is rounded to a narrower type.
 *
 * Inputs must be finite.  Shapes are trusted (the caller checks them).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_VERSION 1

int oracle_version(void) { return ORACLE_VERSION; }

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* bf16 bit pattern -> double (exact). */
static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* The tanh form of GELU: 0.5 a (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3))). */
double oracle_gelu_tanh(double a) {
    const double c = sqrt(2.0 / M_PI);
    return 0.5 * a * (1.0 + tanh(c * (a + 0.044715 * a * a * a)));
}

/* L[t,e] = sum_{h ascending} x[t,h] * Wr[h,e], then + bias[e] (bias may be NULL).
 * x: [T,H] bf16, wr: [H,E] bf16, logits: [T,E] double. */
void oracle_router_logits(const uint16_t *x, const uint16_t *wr, const float *bias,
                          int64_t T, int H, int E, double *logits) {
#pragma omp parallel
    {
        double *acc = (double *)malloc(sizeof(double) * (size_t)E);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            for (int e = 0; e < E; ++e) acc[e] = 0.0;
            for (int h = 0; h < H; ++h) {
                const double xv = bf16_to_double(x[t * H + h]);
                const uint16_t *wrow = wr + (int64_t)h * E;
                for (int e = 0; e < E; ++e) acc[e] += xv * bf16_to_double(wrow[e]);
            }
            for (int e = 0; e < E; ++e)
                logits[t * E + e] = bias ? acc[e] + (double)bias[e] : acc[e];
        }
        free(acc);
    }
}

/* Per token: pick the k largest logits (ties -> lower id), slot 0 = largest; weights from
 * the softmax over all E logits, renormalised over the k selected when renorm != 0. */
void oracle_select(const double *logits, int64_t T, int E, int k, int renorm,
                   int32_t *ids, double *weights) {
#pragma omp parallel
    {
        char *taken = (char *)malloc((size_t)E);
        double *p = (double *)malloc(sizeof(double) * (size_t)E);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            const double *L = logits + t * E;
            memset(taken, 0, (size_t)E);
            for (int j = 0; j < k; ++j) {
                int best = -1;
                for (int e = 0; e < E; ++e)
                    if (!taken[e] && (best < 0 || L[e] > L[best])) best = e;
                taken[best] = 1;
                ids[t * k + j] = best;
            }
            double m = L[0];
            for (int e = 1; e < E; ++e)
                if (L[e] > m) m = L[e];
            double z = 0.0;
            for (int e = 0; e < E; ++e) {
                p[e] = exp(L[e] - m);
                z += p[e];
            }
            for (int e = 0; e < E; ++e) p[e] /= z;
            double s = 0.0;
            for (int j = 0; j < k; ++j) s += p[ids[t * k + j]];
            for (int j = 0; j < k; ++j) {
                const double pj = p[ids[t * k + j]];
                weights[t * k + j] = renorm ? pj / s : pj;
            }
        }
        free(taken);
        free(p);
    }
}

/* counts[e] = #pairs routed to e; offsets = exclusive scan (E+1 entries);
 * perm[sorted position] = t*k + j, expert by expert, ascending t within an expert;
 * inv[t*k + j] = sorted position. */
void oracle_dispatch(const int32_t *ids, int64_t T, int k, int E,
                     int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t q = 0; q < T * k; ++q) counts[ids[q]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            const int64_t q = t * k + j;
            const int32_t pos = fill[ids[q]]++;
            perm[pos] = (int32_t)q;
            inv[q] = pos;
        }
    free(fill);
}

/* One expert on one token row: out[n] = sum_i gelu_tanh(g_i) u_i Wd[i,n],
 * g_i = sum_h x_h Wg[h,i], u_i = sum_h x_h Wu[h,i].
 * xrow [H] bf16; wg, wu: this expert's [H,I] bf16; wd: this expert's [I,H] bf16;
 * work: 3*I doubles of scratch; out [H] double. */
static void expert_ffn(const uint16_t *xrow, const uint16_t *wg, const uint16_t *wu,
                       const uint16_t *wd, int H, int I, double *work, double *out) {
    double *g = work, *u = work + I, *hh = work + 2 * I;
    for (int i = 0; i < I; ++i) g[i] = u[i] = 0.0;
    for (int h = 0; h < H; ++h) {
        const double xv = bf16_to_double(xrow[h]);
        const uint16_t *gr = wg + (int64_t)h * I, *ur = wu + (int64_t)h * I;
        for (int i = 0; i < I; ++i) {
            g[i] += xv * bf16_to_double(gr[i]);
            u[i] += xv * bf16_to_double(ur[i]);
        }
    }
    for (int i = 0; i < I; ++i) hh[i] = oracle_gelu_tanh(g[i]) * u[i];
    for (int n = 0; n < H; ++n) out[n] = 0.0;
    for (int i = 0; i < I; ++i) {
        const uint16_t *dr = wd + (int64_t)i * H;
        for (int n = 0; n < H; ++n) out[n] += hh[i] * bf16_to_double(dr[n]);
    }
}

/* Public single-expert entry (for pins): expert index e of the stacked weights. */
void oracle_expert_ffn(const uint16_t *xrow, const uint16_t *w_gate, const uint16_t *w_up,
                       const uint16_t *w_down, int e, int H, int I, double *out) {
    double *work = (double *)malloc(sizeof(double) * 3 * (size_t)I);
    const int64_t hi = (int64_t)H * I;
    expert_ffn(xrow, w_gate + e * hi, w_up + e * hi, w_down + e * hi, H, I, work, out);
    free(work);
}

/* Whole layer.  Routes all T tokens (ids, weights, logits for every token), then for the
 * n_tok tokens listed in `tokens` (all T when tokens == NULL) writes
 * y[r, :] = sum_{j ascending} w[t,j] * o_{t,j}, r = row in the list. */
void oracle_forward(const uint16_t *x, const uint16_t *w_router, const float *bias,
                    const uint16_t *w_gate, const uint16_t *w_up, const uint16_t *w_down,
                    int64_t T, int H, int E, int I, int k, int renorm,
                    const int64_t *tokens, int64_t n_tok,
                    int32_t *ids, double *weights, double *logits, double *y) {
    oracle_router_logits(x, w_router, bias, T, H, E, logits);
    oracle_select(logits, T, E, k, renorm, ids, weights);
    if (!tokens) n_tok = T;
    const int64_t hi = (int64_t)H * I;
#pragma omp parallel
    {
        double *work = (double *)malloc(sizeof(double) * 3 * (size_t)I);
        double *o = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_tok; ++r) {
            const int64_t t = tokens ? tokens[r] : r;
            double *yr = y + r * H;
            for (int n = 0; n < H; ++n) yr[n] = 0.0;
            for (int j = 0; j < k; ++j) {
                const int64_t e = ids[t * k + j];
                expert_ffn(x + t * H, w_gate + e * hi, w_up + e * hi, w_down + e * hi, H, I,
                           work, o);
                const double w = weights[t * k + j];
                for (int n = 0; n < H; ++n) yr[n] += w * o[n];
            }
        }
        free(work);
        free(o);
    }
}
