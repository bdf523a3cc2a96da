/*
 * wlq_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of what the weight-only quantized Linear
 * computes.  It exists so that the CUDA library can be checked against it; it
 * shares no code, header, table or helper with the CUDA path, and nothing in
 * the product may call it.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg load it.
 *
 * Sources (web pages, cited by title and section):
 *  [JFC]  "Joy-face_change_optimized" model card (README), section
 *         "what this branch does" (files table): weight-only Linear with int4
 *         weights grouped along the input dimension, or int8 weights with one
 *         scale per output channel; tools row: RTN int4 with group size 64,
 *         RTN int8, and attention-int8 / MLP-int4 with group size 16.
 *  [NL]   "Nunchaku Lite: loading and running 4-bit SVDQuant" (news article),
 *         section "why it matters": the hardest part of the weights is handled
 *         by a low-rank correction kept in 16-bit precision; section "how it
 *         works": the W4A16 family keeps activations in 16 bits.
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes):
 *  - symmetric quantization, qmax = 2^(bits-1) - 1 (127 for int8, 7 for
 *    int4); codes lie in [-qmax, qmax];
 *  - "RTN" = round to nearest, ties to even, of W / s, with s the fp32 scale
 *    that is stored;
 *  - s = fp32(absmax / qmax), absmax over the group (the whole row for int8
 *    per-channel, `group` contiguous inputs for int4);
 *  - an all-zero group has s = 0 and codes 0 (no division is made);
 *  - non-finite weights are rejected;
 *  - the low-rank branch follows y += (x L1) L2 with L1 [K, r], L2 [r, N].
 *
 * Arithmetic: every step is done in fp64 on the exact values of its
 * operands; the only roundings are the one that produces the fp32 scale and
 * those of the fp64 sums.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NONFINITE 2

/* bf16 is the upper half of an IEEE binary32: widen by shifting. */
static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a real (held exactly in fp64) to the nearest integer, ties to even.
 * t - floor(t) is exact for |t| < 2^52, far beyond any code range. */
static double round_half_even(double t) {
    double f = floor(t);
    double d = t - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    /* exact tie: keep the even neighbour */
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/*
 * RTN symmetric quantization [JFC files table / tools row].
 * W      : fp32 [N, K] row-major
 * group  : 0 = one group per output row (per-channel), else the group size
 *          along K (K % group == 0)
 * codes  : int8 [N, K]
 * scales : fp32 [N, K / g]  (g = K for per-channel)
 */
int oracle_quantize(const float* W, int64_t N, int64_t K, int bits, int group,
                    int8_t* codes, float* scales) {
    if (N < 0 || K <= 0 || (bits != 8 && bits != 4) || group < 0) return ORACLE_ERR_ARG;
    const int64_t g = (group == 0) ? K : group;
    if (K % g != 0) return ORACLE_ERR_ARG;
    const int64_t G = K / g;
    const double qmax = (double)((1 << (bits - 1)) - 1);
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(W[i])) return ORACLE_ERR_NONFINITE;

#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t gi = 0; gi < G; ++gi) {
            const float* w = W + n * K + gi * g;
            int8_t* q = codes + n * K + gi * g;
            /* step 1: group absmax (exact) */
            double a = 0.0;
            for (int64_t k = 0; k < g; ++k) {
                double v = fabs((double)w[k]);
                if (v > a) a = v;
            }
            /* step 2: the stored scale is the fp32 nearest to a / qmax.  The
             * fp64 quotient rounded to fp32 is that value: fp64 carries more
             * than 2*24+2 bits, so the second rounding cannot differ from a
             * direct one. */
            const float s = (float)(a / qmax);
            scales[n * G + gi] = s;
            /* step 3: codes */
            for (int64_t k = 0; k < g; ++k) {
                double c = 0.0;
                if (s != 0.0f) {
                    /* For fp32 operands the exact quotient is never within an
                     * fp64 half-ulp of a half-integer unless it is one, so
                     * this fp64 quotient rounds like the exact real. */
                    double t = (double)w[k] / (double)s;
                    c = round_half_even(t);
                    if (c > qmax) c = qmax;
                    if (c < -qmax) c = -qmax;
                }
                q[k] = (int8_t)c;
            }
        }
    }
    return ORACLE_OK;
}

/* Dequantized weights, exact in fp64: deq[n,k] = q[n,k] * s[n, k / g]. */
int oracle_dequantize(const int8_t* codes, const float* scales, int64_t N, int64_t K,
                      int group, double* deq) {
    if (N < 0 || K <= 0 || group < 0) return ORACLE_ERR_ARG;
    const int64_t g = (group == 0) ? K : group;
    if (K % g != 0) return ORACLE_ERR_ARG;
    const int64_t G = K / g;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            deq[n * K + k] = (double)codes[n * K + k] * (double)scales[n * G + k / g];
    return ORACLE_OK;
}

/*
 * Weight-only quantized Linear [JFC files table; NL "how it works": 16-bit
 * activations, quantized weights; NL "why it matters": 16-bit low-rank
 * correction]:
 *
 *   y[m,n] = sum_k x[m,k] * q[n,k] * s[n, k/g]
 *          + sum_j ( sum_k x[m,k] * L1[k,j] ) * L2[j,n]      (if r > 0)
 *          + b[n]                                              (if bias)
 *
 * x: bf16 bits [M, K]; bias: bf16 bits [N] or NULL; L1: bf16 bits [K, r];
 * L2: bf16 bits [r, N]; y: fp64 [M, N].  A naive triple loop, no blocking.
 */
int oracle_linear(const uint16_t* x, int64_t M, int64_t K,
                  const int8_t* codes, const float* scales, int64_t N, int group,
                  const uint16_t* bias, const uint16_t* L1, const uint16_t* L2, int r,
                  double* y) {
    if (M < 0 || N < 0 || K <= 0 || group < 0 || r < 0 || r > 256) return ORACLE_ERR_ARG;
    if (r > 0 && (L1 == 0 || L2 == 0)) return ORACLE_ERR_ARG;
    const int64_t g = (group == 0) ? K : group;
    if (K % g != 0) return ORACLE_ERR_ARG;
    const int64_t G = K / g;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* xm = x + m * K;
        double T[256];
        /* low-rank prologue T = x L1 */
        for (int j = 0; j < r; ++j) {
            double t = 0.0;
            for (int64_t k = 0; k < K; ++k)
                t += bf16_value(xm[k]) * bf16_value(L1[k * r + j]);
            T[j] = t;
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double w = (double)codes[n * K + k] * (double)scales[n * G + k / g];
                acc += bf16_value(xm[k]) * w;
            }
            for (int j = 0; j < r; ++j)
                acc += T[j] * bf16_value(L2[(int64_t)j * N + n]);
            if (bias) acc += bf16_value(bias[n]);
            y[m * N + n] = acc;
        }
    }
    return ORACLE_OK;
}
