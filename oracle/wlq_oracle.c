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

/*
 * Round a non-negative real held exactly in fp64 to the nearest value of a
 * binary floating-point format with `p` significand bits (implicit bit
 * included) and minimum normal exponent `emin` (subnormals below 2^emin with
 * the fixed spacing 2^(emin - p + 1)), ties to even.  Returns +inf when the
 * rounded value exceeds `maxv`.  The spacing is a power of two, so x / spacing
 * is exact and the rounding is a single one.
 */
static double round_to_format(double x, int p, int emin, double maxv) {
    if (x == 0.0) return 0.0;
    int E;
    frexp(x, &E); /* x in [2^(E-1), 2^E) */
    int lead = E - 1;
    if (lead < emin) lead = emin;
    const double spacing = ldexp(1.0, lead - (p - 1));
    const double r = round_half_even(x / spacing) * spacing;
    return (r > maxv) ? INFINITY : r;
}

/* a weight of an fp32 or bf16 input array, exactly */
static double in_value(const void* W, int w_dtype, int64_t i) {
    if (w_dtype == 0) return (double)((const float*)W)[i];
    return bf16_value(((const uint16_t*)W)[i]);
}

/*
 * RTN symmetric quantization for any width of 2..8 bits, an fp32 or bf16
 * input, and a 32- or 16-bit stored scale ([JFC] tools row and files table:
 * RTN with per-channel or grouped scales; [JFC] section 1, the KV-dtype
 * setting: cached image K/V held as int8 with one scale per token and head,
 * i.e. one group per (token, head) row of head_dim inputs; [JFC] section 2:
 * a 5-bit MLP proposed as a further width).
 * w_dtype     : 0 fp32, 1 bf16 (bit patterns)
 * bits        : 2..8, qmax = 2^(bits-1) - 1
 * group       : 0 = whole row, else the group size along K
 * scale_dtype : 0 fp32, 1 fp16, 2 bf16 -- the stored scale is the value of
 *               that format nearest to a / qmax (ties to even); the codes are
 *               RTN of W / s with that stored s, clamped to +-qmax (a 16-bit
 *               scale may round below a / qmax)
 * codes       : int8 [N, K];  scale_values : fp32 [N, K / g], the stored
 *               scales' values (16-bit values are exact in fp32)
 * A stored scale that overflows its format is reported as non-finite.
 */
int oracle_quantize_ex(const void* W, int w_dtype, int64_t N, int64_t K, int bits, int group,
                       int scale_dtype, int8_t* codes, float* scale_values) {
    if (N < 0 || K <= 0 || bits < 2 || bits > 8 || group < 0 || w_dtype < 0 || w_dtype > 1 ||
        scale_dtype < 0 || scale_dtype > 2)
        return ORACLE_ERR_ARG;
    const int64_t g = (group == 0) ? K : group;
    if (K % g != 0) return ORACLE_ERR_ARG;
    const int64_t G = K / g;
    const double qmax = ldexp(1.0, bits - 1) - 1.0;
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(in_value(W, w_dtype, i))) return ORACLE_ERR_NONFINITE;
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t gi = 0; gi < G; ++gi) {
            double a = 0.0;
            for (int64_t k = 0; k < g; ++k) {
                double v = fabs(in_value(W, w_dtype, n * K + gi * g + k));
                if (v > a) a = v;
            }
            /* the stored scale: nearest value of the format to a / qmax (the
             * fp64 quotient is within 2^-53 relative of a / qmax, and a, qmax
             * are short enough that no tie of a 24-bit or shorter format lies
             * that close unless the quotient is exact) */
            const double qd = a / qmax;
            double s;
            if (scale_dtype == 0) s = (double)(float)qd;
            else if (scale_dtype == 1) s = round_to_format(qd, 11, -14, 65504.0);
            else s = round_to_format(qd, 8, -126, ldexp(255.0, 127 - 7));
            if (isinf(s)) { overflow = 1; s = 0.0; }
            scale_values[n * G + gi] = (float)s;
            for (int64_t k = 0; k < g; ++k) {
                double c = 0.0;
                if (s != 0.0) {
                    /* s is exactly an fp32 value; as in oracle_quantize the
                     * fp64 quotient rounds like the exact real */
                    c = round_half_even(in_value(W, w_dtype, n * K + gi * g + k) / s);
                    if (c > qmax) c = qmax;
                    if (c < -qmax) c = -qmax;
                }
                codes[n * K + gi * g + k] = (int8_t)c;
            }
        }
    }
    return overflow ? ORACLE_ERR_NONFINITE : ORACLE_OK;
}

/*
 * fp8 (e4m3, the "fn" variant: no infinity, largest finite 448) block
 * quantization along K ([JFC] section 1.1: DiT blocks streamed to 8 GB cards
 * in fp8, quantized on the GPU, the card noting that a CPU rounding differed
 * from CUDA's on a small fraction of elements -- here both sides round once,
 * to nearest even, from the same fp32 quotient).  The scale granularity is
 * not given; the reading is one fp32 scale per group of g inputs of a row
 * (g = K: per row): per group, s = fp32(a / 448); each
 * weight becomes the e4m3 value nearest to t = fp32(W / s) (ties to an even
 * significand), saturated to +-448; an all-zero group has s = 0 and codes 0.
 * codes : uint8 [N, K] e4m3 bit patterns (sign, 4 exponent bits with bias 7,
 *         3 significand bits; exponent field 0 = subnormals of spacing 2^-9)
 * scales: fp32 [N, K / g]
 */
static uint8_t e4m3_encode(double t) {
    const int neg = signbit(t) ? 1 : 0;
    double x = fabs(t);
    /* nearest e4m3 magnitude, ties to even: spacing 2^-9 below 2^-6, else
     * 2^(exponent - 3) */
    double r = round_to_format(x, 4, -6, 448.0);
    if (isinf(r)) r = 448.0; /* saturate */
    uint8_t bits;
    if (r < ldexp(1.0, -6)) {
        bits = (uint8_t)(r / ldexp(1.0, -9)); /* subnormal (or zero): m / 8 * 2^-6 */
    } else {
        int E;
        const double m = frexp(r, &E); /* r = m 2^E, m in [0.5, 1) */
        const int e = (E - 1) + 7;     /* biased exponent */
        const int man = (int)((m * 2.0 - 1.0) * 8.0);
        bits = (uint8_t)((e << 3) | man);
    }
    return (uint8_t)(bits | (neg << 7));
}

int oracle_quantize_fp8(const void* W, int w_dtype, int64_t N, int64_t K, int group, uint8_t* codes,
                        float* scales) {
    if (N < 0 || K <= 0 || group < 0 || w_dtype < 0 || w_dtype > 1) return ORACLE_ERR_ARG;
    const int64_t g = (group == 0) ? K : group;
    if (K % g != 0) return ORACLE_ERR_ARG;
    const int64_t G = K / g;
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(in_value(W, w_dtype, i))) return ORACLE_ERR_NONFINITE;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t gi = 0; gi < G; ++gi) {
            double a = 0.0;
            for (int64_t k = 0; k < g; ++k) {
                double v = fabs(in_value(W, w_dtype, n * K + gi * g + k));
                if (v > a) a = v;
            }
            const float s = (float)(a / 448.0);
            scales[n * G + gi] = s;
            for (int64_t k = 0; k < g; ++k) {
                uint8_t c = 0;
                if (s != 0.0f) {
                    /* t = the fp32 nearest to W / s: the fp64 quotient of two
                     * fp32 values rounds to fp32 like the exact one */
                    const float t = (float)(in_value(W, w_dtype, n * K + gi * g + k) / (double)s);
                    c = e4m3_encode((double)t);
                }
                codes[n * K + gi * g + k] = c;
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

/*
 * Residual of the low-rank split [NL "why it matters": the hard part of W is
 * carried by the 16-bit low-rank branch, the rest R is quantized].  With the
 * Linear y = x W^T and the branch y += (x L1) L2, L1 [K, r] and L2 [r, N]
 * stand for W^T's best rank-r part, so
 *   R[n][k] = fp32( W[n][k] - sum_{j=0}^{r-1} L1[k][j] * L2[j][n] )
 * with the sum taken in fp64 over j in increasing order (each product and
 * each addition rounded on its own), then one rounding to fp32.
 * W: fp32 [N, K]; L1, L2: bf16 bits; R: fp32 [N, K].
 */
int oracle_lowrank_residual(const float* W, const uint16_t* L1, const uint16_t* L2,
                            int64_t N, int64_t K, int r, float* R) {
    if (N < 0 || K <= 0 || r < 0 || (r > 0 && (L1 == 0 || L2 == 0))) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double p = 0.0;
            for (int j = 0; j < r; ++j) {
                const double prod = bf16_value(L1[k * r + j]) * bf16_value(L2[(int64_t)j * N + n]);
                p = p + prod;
            }
            const double d = (double)W[n * K + k] - p;
            R[n * K + k] = (float)d;
        }
    }
    return ORACLE_OK;
}

/*
 * NVFP4, the 4-bit format of the W4A4 path's Blackwell kernels [NL, section
 * "hardware and precision support": the NVFP4 variant of svdq_w4a4 runs on
 * Blackwell; section "how it works": W4A4 quantizes weights and activations
 * to 4 bits and keeps a 16-bit low-rank branch].  The pages name the format
 * without defining it; it is read as NVIDIA's NVFP4: E2M1 elements (sign,
 * magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one E4M3 scale per 16 consecutive
 * inputs of a row, one fp32 scale per tensor:
 *   g   = fp32(amax(X) / (6 * 448))            (0 for an all-zero tensor)
 *   s_b = E4M3 nearest to a_b / (6 g)          (a_b = max |x| over the block;
 *                                                ties to even, saturated at 448)
 *   q   = E2M1 nearest to x / (s_b g)          (ties to an even significand,
 *                                                saturated at 6; 0 when s_b = 0)
 *   x^  = q s_b g
 * The quotients are taken in fp64 from the exact operands: s_b g has at most
 * 28 significant bits, so it is exact, and a quotient of fp32 values cannot
 * come within fp64's rounding error of a midpoint of these short formats
 * without lying on it (the same argument as for the scales above).
 * X: fp32 or bf16 [rows, K], K % 16 == 0; codes: E2M1 bits (sign in bit 3)
 * [rows, K]; scales: E4M3 bits [rows, K / 16]; *gscale: g.
 */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static double e4m3_value(uint8_t bits) {
    const int e = (bits >> 3) & 15, m = bits & 7;
    const double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (bits & 0x80) ? -v : v;
}

static uint8_t e2m1_encode(double t) {
    const int neg = signbit(t) ? 1 : 0;
    double r = round_to_format(fabs(t), 2, 0, 6.0);
    if (isinf(r)) r = 6.0; /* saturate */
    uint8_t code = 0;
    for (int i = 0; i < 8; ++i)
        if (E2M1_MAG[i] == r) code = (uint8_t)i;
    return (uint8_t)(code | (neg << 3));
}

static double e2m1_value(uint8_t code) {
    const double v = E2M1_MAG[code & 7];
    return (code & 8) ? -v : v;
}

int oracle_nvfp4_quantize(const void* X, int x_dtype, int64_t rows, int64_t K, uint8_t* codes,
                          uint8_t* scales, float* gscale) {
    if (rows < 0 || K <= 0 || K % 16 != 0 || (x_dtype != 0 && x_dtype != 1)) return ORACLE_ERR_ARG;
    double amax = 0.0;
    for (int64_t i = 0; i < rows * K; ++i) {
        const double v = in_value(X, x_dtype, i);
        if (!isfinite(v)) return ORACLE_ERR_NONFINITE;
        if (fabs(v) > amax) amax = fabs(v);
    }
    const float g = (float)(amax / (6.0 * 448.0));
    *gscale = g;
    for (int64_t row = 0; row < rows; ++row) {
        for (int64_t b = 0; b < K / 16; ++b) {
            const int64_t base = row * K + b * 16;
            double ab = 0.0;
            for (int j = 0; j < 16; ++j) {
                const double v = fabs(in_value(X, x_dtype, base + j));
                if (v > ab) ab = v;
            }
            uint8_t sb = 0;
            if (g > 0.0f) sb = e4m3_encode(ab / (6.0 * (double)g));
            scales[row * (K / 16) + b] = sb;
            const double d = e4m3_value(sb) * (double)g; /* exact: <= 28 significant bits */
            for (int j = 0; j < 16; ++j)
                codes[base + j] = (d > 0.0) ? e2m1_encode(in_value(X, x_dtype, base + j) / d) : 0;
        }
    }
    return ORACLE_OK;
}

/* x^ = q s_b g for every element: fp64 [rows, K] (exact). */
int oracle_nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, float g, int64_t rows, int64_t K,
                            double* out) {
    if (rows < 0 || K <= 0 || K % 16 != 0) return ORACLE_ERR_ARG;
    for (int64_t row = 0; row < rows; ++row)
        for (int64_t k = 0; k < K; ++k)
            out[row * K + k] = e2m1_value(codes[row * K + k]) * e4m3_value(scales[row * (K / 16) + k / 16]) *
                               (double)g;
    return ORACLE_OK;
}

/*
 * The W4A4 Linear [NL, "how it works": 4-bit weights and activations with a
 * 16-bit low-rank correction]:
 *   y[m,n] = sum_k x^[m,k] w^[n,k] + sum_j (sum_k x[m,k] L1[k,j]) L2[j,n] + b[n]
 * x^, w^: NVFP4 dequantized activations [M, K] and weights [N, K]; the
 * low-rank branch takes the 16-bit x (bf16 bits) as it is.  fp64, naive loops.
 */
int oracle_nvfp4_linear(const uint8_t* xq, const uint8_t* xs, float xg, const uint16_t* x, int64_t M, int64_t K,
                        const uint8_t* wq, const uint8_t* ws, float wg, int64_t N, const uint16_t* bias,
                        const uint16_t* L1, const uint16_t* L2, int r, double* y) {
    if (M < 0 || N < 0 || K <= 0 || K % 16 != 0 || r < 0 || r > 256) return ORACLE_ERR_ARG;
    if (r > 0 && (L1 == 0 || L2 == 0 || x == 0)) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        double T[256];
        for (int j = 0; j < r; ++j) {
            double t = 0.0;
            for (int64_t k = 0; k < K; ++k) t += bf16_value(x[m * K + k]) * bf16_value(L1[k * r + j]);
            T[j] = t;
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const double a = e2m1_value(xq[m * K + k]) * e4m3_value(xs[m * (K / 16) + k / 16]) * (double)xg;
                const double w = e2m1_value(wq[n * K + k]) * e4m3_value(ws[n * (K / 16) + k / 16]) * (double)wg;
                acc += a * w;
            }
            double lr = 0.0;
            for (int j = 0; j < r; ++j) lr += T[j] * bf16_value(L2[(int64_t)j * N + n]);
            const double b = bias ? bf16_value(bias[n]) : 0.0;
            y[m * N + n] = acc + lr + b;
        }
    }
    return ORACLE_OK;
}
