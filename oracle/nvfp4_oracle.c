/*
 * nvfp4_oracle.c -- plain CPU oracle of NVFP4 quantisation (4-bit float elements, one 8-bit
 * float scale per group of 16) and of the routed MoE FFN layer with NVFP4 expert weights
 * and activations.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library calls, links or loads this file; it
 * shares no code, table or helper with the CUDA path.
 *
 * What the pages fix: the Gemma-4-26B-A4B-NVFP4 checkpoint quantises weights AND activations
 * to "4-bit float, group_size=16, per-group NVFP4" (Gemma-4-26B-A4B-NVFP4 Ascend verification
 * report, §2.3 量化配置 (NVFP4)).  What they leave open is taken from the format's published
 * definition:
 *   element       E2M1: sign bit, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
 *                 0, 0.5, 1, 1.5, 2, 3, 4, 6 (exponent 0 is subnormal: 0 and 0.5); no inf, nan.
 *   block scale   E4M3 ("fn": sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0
 *                 subnormal; the all-ones exponent with all-ones mantissa is nan, no inf;
 *                 largest finite 448), one per 16 consecutive elements along the reduction
 *                 axis (K).
 *   tensor scale  one fp32 per tensor (per expert and projection for weights; a fixed value
 *                 per activation tensor, set ahead of time).
 *   value         e2m1 * e4m3 * tensor_scale.
 * Quantisation of a group v[0..15] (fp32 inputs; every step one IEEE fp32 operation with
 * round-to-nearest-even, in this order):
 *   amax = max |v_i|;  s = (amax / 6) / ts;  s8 = E4M3(s) (nearest, ties to even code, values
 *   beyond 448 saturate to 448);  S = value(s8) * ts;
 *   code_i = 0 if S == 0, else E2M1(v_i / S) (nearest, ties to even code, saturating at 6;
 *   the sign bit is the input's, also when the magnitude rounds to zero).
 * Weight tensor scale: ts = amax over the tensor / (6 * 448), one fp32 division.
 * Dequantised values are exact in double (each is a product of at most 2 + 4 + 24 significant
 * bits).  One expert on one row computes in double with no rounding, except that its
 * intermediate h is quantised as an activation: h is rounded to fp32 first (the precision the
 * quantisation decisions are taken in).  The layer (routing, the weighted sum over the k
 * experts in slot order) is composed in oracle/__init__.py from the routing functions of
 * moe_oracle.c and this file's expert.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* E2M1 magnitude of a 3-bit code, from the bit-level definition. */
static double e2m1_mag(int c) {
    const int e = (c >> 1) & 3, m = c & 1;
    if (e == 0) return m ? 0.5 : 0.0;                   /* subnormal: m * 2^(1-1) / 2 */
    return ldexp(1.0 + 0.5 * m, e - 1);
}

double oracle_e2m1_value(int code) {
    const double v = e2m1_mag(code & 7);
    return (code & 8) ? -v : v;
}

/* E4M3 (fn) magnitude of a 7-bit code; NAN for the nan encoding. */
static double e4m3_mag(int c) {
    const int e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) return ldexp(m / 8.0, -6);
    return ldexp(1.0 + m / 8.0, e - 7);
}

double oracle_e4m3_value(int code) {
    const double v = e4m3_mag(code & 127);
    return (code & 128) ? -v : v;
}

/* Nearest code of a magnitude table (codes 0..n-1 ascending in value), ties to the even
 * code, beyond the largest value saturating to it.  a >= 0. */
static int nearest_code(double a, int n, double (*mag)(int)) {
    int best = 0;
    double bd = fabs(a - mag(0));
    for (int c = 1; c < n; ++c) {
        const double d = fabs(a - mag(c));
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return best;
}

/* The sign bit follows the input's sign, also when the magnitude rounds to zero (a
 * negative value that rounds to zero gives code 8, "-0"). */
int oracle_e2m1_round(float v) {
    const int c = nearest_code(fabs((double)v), 8, e2m1_mag);
    return signbit(v) ? (c | 8) : c;
}

int oracle_e4m3_round(float v) {
    const int c = nearest_code(fabs((double)v), 127, e4m3_mag);   /* 127 = nan, excluded */
    return (v < 0 && c != 0) ? (c | 128) : c;
}

float oracle_nvfp4_weight_scale(const float *v, int64_t n) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        const float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    return amax / 2688.0f;   /* 6 * 448 */
}

/* One group of 16: codes (one 4-bit code per byte) and its scale code. */
static void quantize_group(const float *v, float ts, uint8_t *codes, uint8_t *scale) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        const float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    const float s = (amax / 6.0f) / ts;
    const int s8 = oracle_e4m3_round(s);
    const float S = (float)e4m3_mag(s8) * ts;
    *scale = (uint8_t)s8;
    for (int i = 0; i < 16; ++i) codes[i] = (uint8_t)(S == 0.0f ? 0 : oracle_e2m1_round(v[i] / S));
}

/* v [rows][K] (K % 16 == 0) -> codes [rows][K] (one per byte), scales [rows][K/16]. */
void oracle_nvfp4_quantize(const float *v, int64_t rows, int K, float ts, uint8_t *codes,
                           uint8_t *scales) {
    for (int64_t r = 0; r < rows; ++r)
        for (int g = 0; g < K / 16; ++g)
            quantize_group(v + r * K + 16 * g, ts, codes + r * K + 16 * g,
                           scales + r * (K / 16) + g);
}

void oracle_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int K,
                             float ts, double *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int kk = 0; kk < K; ++kk)
            out[r * K + kk] = oracle_e2m1_value(codes[r * K + kk]) *
                              oracle_e4m3_value(scales[r * (K / 16) + kk / 16]) * (double)ts;
}

static double bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double oracle_gelu_tanh(double a);

/* Activation quantisation of one row: v (fp32) [K] -> dequantised values [K]. */
static void act_qdq(const float *v, int K, float ts, uint8_t *codes, uint8_t *sc, double *out) {
    oracle_nvfp4_quantize(v, 1, K, ts, codes, sc);
    oracle_nvfp4_dequantize(codes, sc, 1, K, ts, out);
}

/* One expert on one token row with NVFP4 weights and activations:
 * xq = qdq(x), g_i = sum_h xq_h Wg[i,h], u_i = sum_h xq_h Wu[i,h], hh = gelu_tanh(g) u,
 * hq = qdq(float(hh)), o_n = sum_i hq_i Wd[n,i].  Weights are given dequantised:
 * wg, wu [I][H], wd [H][I] (doubles). */
static void expert_ffn_q(const uint16_t *xrow, const double *wg, const double *wu,
                         const double *wd, int H, int I, float sx, float sh, double *out) {
    float *xf = (float *)calloc((size_t)H, sizeof(float));
    float *hf = (float *)calloc((size_t)I, sizeof(float));
    double *xq = (double *)malloc(sizeof(double) * (size_t)H);
    double *hq = (double *)malloc(sizeof(double) * (size_t)I);
    uint8_t *cb = (uint8_t *)malloc((size_t)(H > I ? H : I));
    uint8_t *sb = (uint8_t *)malloc((size_t)(H > I ? H : I) / 16 + 1);
    for (int h = 0; h < H; ++h) xf[h] = (float)bf16_value(xrow[h]);
    act_qdq(xf, H, sx, cb, sb, xq);
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            g += xq[h] * wg[(int64_t)i * H + h];
            u += xq[h] * wu[(int64_t)i * H + h];
        }
        hf[i] = (float)(oracle_gelu_tanh(g) * u);
    }
    act_qdq(hf, I, sh, cb, sb, hq);
    for (int n = 0; n < H; ++n) {
        double o = 0.0;
        for (int i = 0; i < I; ++i) o += hq[i] * wd[(int64_t)n * I + i];
        out[n] = o;
    }
    free(xf);
    free(hf);
    free(xq);
    free(hq);
    free(cb);
    free(sb);
}

/* Public single-expert entry (for pins). */
void oracle_expert_ffn_nvfp4(const uint16_t *xrow, const double *wg, const double *wu,
                             const double *wd, int H, int I, float sx, float sh, double *out) {
    expert_ffn_q(xrow, wg, wu, wd, H, I, sx, sh, out);
}
