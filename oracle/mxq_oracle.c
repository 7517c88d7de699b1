/*
 * mxq_oracle.c -- CPU oracle for the DuQuant++ online smooth-rotate-MXFP4 step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this.  The CUDA path never calls it,
 * and the two share no code, headers or tables.
 *
 * It is a plain, slow statement of what the path computes, in double
 * precision.  It follows the DuQuant++ write-up "DuQuant++: block-aligned
 * rotation quantisation for MXFP4 activation outliers" (jsqmd.com/news/928156):
 *
 *   smoothing  X -> X * Lambda^-1, a per-channel division          (§3.1, §3.3)
 *   rotation   each 32-element group times one shared 32x32 R^ (X -> X * R^);
 *              the block-diagonal operator is never formed          (§2.3, §3.2, §3.3)
 *   MXFP4      absmax of the group -> shared power-of-two scale s_j ->
 *              divide -> round to the nearest 4-bit float           (§2.1, §5.1 item 5)
 *
 * The write-up leaves the exact MXFP4 rule open.  This file takes the OCP
 * Microscaling (MX) v1.0 reading:
 *   - E8M0 exponent e = floor(log2(amax)) - 2, clamped to [-127, 127];
 *   - code = E2M1 round-to-nearest with ties to the even code, |u| > 6 -> 6,
 *     sign kept (so -0 and tiny negatives give code 0x8);
 *   - amax NaN/Inf -> scale byte 0xFF and all codes 0;
 *   - two codes per byte, the even column in the low nibble.
 * The rotated values are rounded to fp32 before the scale and code decisions,
 * the precision the CUDA kernel decides them in (the pages name none).
 *
 * Boundary flags (used by the parity tests to tell unique results from
 * rounding-order ties):
 *   element flag  ||u| - m| < 1e-3 * step(m) for a code midpoint m in
 *                 {0, .25, .75, 1.25, 1.75, 2.5, 3.5, 5} (steps .5,.5,.5,.5,.5,1,1,2);
 *                 the midpoint 0 separates +0 from -0;
 *   group flag    |amax - 2^k| < 2.5e-4 * 2^k for the nearest power of two.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GROUP 32

/* Planted mistakes: test infrastructure for the pins themselves.  A normal build
 * has MXQ_MUTANT 0 and none of them.  The pin-sensitivity test builds this file
 * with -DMXQ_MUTANT=k and checks that at least one pin fails for every k:
 *    1  E8M0 exponent floor(log2 amax) - 1 instead of - 2
 *    2  E2M1 ties away from zero instead of to the even code
 *    3  no saturation: |u| >= 7 wraps to code 0
 *    4  the sign of negative values dropped
 *    5  the rotation transposed (R[n][k] instead of R[k][n])
 *    6  Lambda multiplies the activations instead of dividing them
 *    7  nibble order swapped (odd column in the low nibble)
 *    8  scale and codes decided on the double values, not on fp32
 *    9  a NaN/Inf group gets scale byte 0 instead of 0xFF
 *   10  an E8M0 byte's value taken as 2^(byte - 126)
 *   11  the rotation sums only 31 of the 32 terms
 *   12  the search updates R <- G R instead of R <- R G
 *   13  the inverse rotation of the dequantiser uses R instead of R^T
 *   14  NVFP4: r_t = 1 / s_t (the 6 dropped)
 *   15  an all-zero group gets scale byte 127 instead of 0
 *   16  the MXFP4 GEMM ignores B's E8M0 scales
 *   17  the NVFP4 GEMM drops B's tensor scale
 *   18  E4M3 ties go to the odd code
 *   19  the group error without its square root (a ratio of squared norms)
 *   20  the B x B block rotation transposed
 *   21  scale atoms with the roles of r % 32 and r / 32 swapped
 *   22  the dequantiser divides by Lambda instead of multiplying */
#ifndef MXQ_MUTANT
#define MXQ_MUTANT 0
#endif
#define PLANTED(k) (MXQ_MUTANT == (k))
/* R^[k][n] of a row-major 32x32 matrix (transposed under planted mistake 5) */
#define RKN(R, k, n) (PLANTED(5) ? (R)[(n) * GROUP + (k)] : (R)[(k) * GROUP + (n)])

/* ---------------------------------------------------------------- formats */

/* bf16 bit pattern -> double (exact: bf16 is the top half of an IEEE single). */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* double -> bf16 bit pattern, one round-to-nearest-even step, overflow to Inf. */
static uint16_t double_to_bf16(double v)
{
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int ex;
    frexp(a, &ex);                          /* a = f * 2^ex, f in [0.5, 1) */
    int lead = ex - 1;                      /* a in [2^lead, 2^(lead+1)) */
    if (lead < -126) lead = -126;           /* bf16 subnormals share fp32's floor */
    double quantum = ldexp(1.0, lead - 7);  /* 8 significant bits */
    double q = nearbyint(a / quantum) * quantum;   /* default mode: ties to even */
    if (q >= ldexp(1.0, 128)) return sign | 0x7F80;
    float f = (float)q;                     /* exact: q has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

/* E2M1 magnitudes of codes 0..7 (1 sign, 2 exponent, 1 mantissa bit; bias 1). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Midpoints between neighbouring magnitudes, the grid step there, and the two
 * codes on either side.  Midpoint 0 separates +0 and -0. */
static const double MID[8]  = {0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
static const double STEP[8] = {0.5, 0.5, 0.5, 0.5, 0.5, 1.0, 1.0, 2.0};

/* Round u to the nearest E2M1 value: nearest magnitude, ties to the even code,
 * saturate above 6, keep the sign.  Returns the 4-bit code. */
int mxq_oracle_e2m1_code(double u)
{
    int neg = (signbit(u) && !PLANTED(4)) ? 1 : 0;
    double a = fabs(u);
    int best = 0;
    if (isnan(u)) return 0;
    if (PLANTED(3) && a >= 7.0) {
        best = 0;
    } else if (a >= E2M1_MAG[7]) {
        best = 7;
    } else {
        double bestd = a;                   /* distance to magnitude 0 */
        for (int c = 1; c < 8; ++c) {
            double d = fabs(a - E2M1_MAG[c]);
            /* strictly nearer wins; an exact tie goes to the even code */
            if (d < bestd || (d == bestd && (PLANTED(2) || (c & 1) == 0))) {
                best = c;
                bestd = d;
            }
        }
    }
    return (neg << 3) | best;
}

/* Value of a 4-bit code. */
double mxq_oracle_e2m1_value(int code)
{
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Shared E8M0 byte for a group absmax (finite, >= 0): e = floor(log2 amax) - 2,
 * clamped to [-127, 127]; byte = e + 127.  amax == 0 -> byte 0.  NaN/Inf -> 0xFF. */
int mxq_oracle_e8m0_byte(double amax)
{
    if (isnan(amax) || isinf(amax)) return 0xFF;
    if (amax == 0.0) return PLANTED(15) ? 127 : 0;
    int ex;
    frexp(amax, &ex);                       /* floor(log2 amax) = ex - 1 */
    int e = (ex - 1) - (PLANTED(1) ? 1 : 2);
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e + 127;
}

/* Value 2^(byte - 127) of a scale byte (byte 0xFF is NaN). */
double mxq_oracle_e8m0_value(int byte)
{
    if (byte == 0xFF) return NAN;
    return ldexp(1.0, byte - (PLANTED(10) ? 126 : 127));
}

/* ------------------------------------------------------ one group, step by step */

/* Quantise 32 rotated values y (already rounded to fp32) with a given scale
 * byte.  Writes 32 unpacked codes and, if requested, the element boundary flag
 * and the code on the other side of the flagged midpoint. */
int mxq_oracle_quantize_group_at(const double *y, int byte, uint8_t *codes,
                                 uint8_t *flags, uint8_t *alt)
{
    if (byte == 0xFF) {
        for (int n = 0; n < GROUP; ++n) {
            codes[n] = 0;
            if (flags) flags[n] = 0;
            if (alt) alt[n] = 0;
        }
        return 0;
    }
    int e = byte - 127;
    for (int n = 0; n < GROUP; ++n) {
        double u = ldexp(y[n], -e);         /* exact power-of-two scaling */
        int c = mxq_oracle_e2m1_code(u);
        codes[n] = (uint8_t)c;
        if (flags || alt) {
            double a = fabs(u);
            int f = 0, other = c;
            for (int m = 0; m < 8; ++m) {
                if (fabs(a - MID[m]) < 1e-3 * STEP[m]) {
                    f = 1;
                    if (m == 0) {
                        other = c ^ 8;      /* +0 <-> -0 */
                    } else {
                        int lo = m - 1, hi = m;   /* magnitudes either side */
                        int mag = c & 7;
                        other = (c & 8) | (mag == lo ? hi : lo);
                    }
                }
            }
            if (flags) flags[n] = (uint8_t)f;
            if (alt) alt[n] = (uint8_t)other;
        }
    }
    return 0;
}

/* Steps 4-8 for one group of double y: round to fp32, absmax, E8M0, codes,
 * plus the boundary information. */
static void quantize_group(const double *yin, uint8_t *codes_unpacked, uint8_t *byte_out,
                           uint8_t *eflags, uint8_t *alt, uint8_t *gflag, uint8_t *alt_byte)
{
    double y[GROUP];
    double amax = 0.0;
    int bad = 0;
    for (int n = 0; n < GROUP; ++n) {
        y[n] = PLANTED(8) ? yin[n] : (double)(float)yin[n];   /* the decision precision: fp32 */
        if (isnan(y[n]) || isinf(y[n])) bad = 1;
        double a = fabs(y[n]);
        if (a > amax) amax = a;
    }
    int byte = bad ? (PLANTED(9) ? 0 : 0xFF) : mxq_oracle_e8m0_byte(amax);
    *byte_out = (uint8_t)byte;
    mxq_oracle_quantize_group_at(y, byte, codes_unpacked, eflags, alt);

    if (gflag || alt_byte) {
        int f = 0, other = byte;
        if (!bad && amax > 0.0) {
            int ex;
            frexp(amax, &ex);
            double below = ldexp(1.0, ex - 1);      /* 2^floor(log2 amax) <= amax */
            double above = ldexp(1.0, ex);          /* > amax */
            if (amax - below < 2.5e-4 * below) {
                f = 1;
                other = mxq_oracle_e8m0_byte(below * (1.0 - 1e-9));
            } else if (above - amax < 2.5e-4 * above) {
                f = 1;
                other = mxq_oracle_e8m0_byte(above);
            }
        }
        if (gflag) *gflag = (uint8_t)f;
        if (alt_byte) *alt_byte = (uint8_t)other;
    }
}

/* ------------------------------------------------------------ whole matrices */

/* Steps 2-3 on doubles: Y[r, 32g+n] = sum_k (X[r, 32g+k] / lam[32g+k]) * R[k][n].
 * lam may be NULL (no smoothing).  R is row-major [k][n]. */
int mxq_oracle_rotate_f64(const double *X, int64_t rows, int64_t cols, const double *R,
                          const double *lam, double *Y, int nthreads)
{
    if (rows < 0 || cols < 0 || cols % GROUP) return 1;
    int64_t G = cols / GROUP;
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            double x[GROUP];
            for (int k = 0; k < GROUP; ++k) {
                x[k] = X[r * cols + g * GROUP + k];
                if (lam) x[k] = PLANTED(6) ? x[k] * lam[g * GROUP + k] : x[k] / lam[g * GROUP + k];
            }
            for (int n = 0; n < GROUP; ++n) {
                double acc = 0.0;
                for (int k = 0; k < GROUP - (PLANTED(11) ? 1 : 0); ++k) acc += x[k] * RKN(R, k, n);
                Y[r * cols + g * GROUP + n] = acc;
            }
        }
    }
    return 0;
}

/* Steps 4-8 for a whole matrix of rotated values.  Every output except codes
 * and scales may be NULL.  codes: [rows, cols/2] packed (even column in the low
 * nibble); scales: [rows, cols/32]; eflags/alt: [rows, cols] unpacked;
 * gflags/alt_scales: [rows, cols/32]. */
int mxq_oracle_quantize(const double *Y, int64_t rows, int64_t cols, uint8_t *codes,
                        uint8_t *scales, uint8_t *eflags, uint8_t *alt, uint8_t *gflags,
                        uint8_t *alt_scales, int nthreads)
{
    if (rows < 0 || cols < 0 || cols % GROUP) return 1;
    int64_t G = cols / GROUP;
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            int64_t e0 = r * cols + g * GROUP;
            uint8_t c[GROUP];
            quantize_group(Y + e0, c, scales + r * G + g, eflags ? eflags + e0 : NULL,
                           alt ? alt + e0 : NULL, gflags ? gflags + r * G + g : NULL,
                           alt_scales ? alt_scales + r * G + g : NULL);
            for (int i = 0; i < GROUP / 2; ++i)
                codes[e0 / 2 + i] = PLANTED(7) ? (uint8_t)(c[2 * i + 1] | (c[2 * i] << 4))
                                               : (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
    return 0;
}

/* The whole path from bf16 inputs, one row at a time (no full-size double
 * buffers): X bf16 [rows, cols], R bf16 [32][32] row-major [k][n], lam fp32
 * [cols] or NULL.  Y (double [rows, cols]) and the flag outputs may be NULL.
 * lam_mul = 0 divides by lam (the activations, X·Λ⁻¹); 1 multiplies (the
 * weights' side of §3.3's absorption, Wᵀ·Λ). */
static int rotate_quantize_rows(const uint16_t *X, int64_t rows, int64_t cols, const uint16_t *Rb,
                                const float *lam, int lam_mul, uint8_t *codes, uint8_t *scales,
                                double *Y, uint8_t *eflags, uint8_t *alt, uint8_t *gflags,
                                uint8_t *alt_scales, int nthreads)
{
    if (rows < 0 || cols < 0 || cols % GROUP) return 1;
    int64_t G = cols / GROUP;
    double R[GROUP * GROUP];
    for (int i = 0; i < GROUP * GROUP; ++i) R[i] = bf16_to_double(Rb[i]);
#pragma omp parallel for schedule(dynamic, 4) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            double x[GROUP], y[GROUP];
            uint8_t c[GROUP];
            int64_t e0 = r * cols + g * GROUP;
            /* step 1-2: exact bf16 -> double, then the per-channel division
             * (or, for weights, multiplication) */
            for (int k = 0; k < GROUP; ++k) {
                x[k] = bf16_to_double(X[e0 + k]);
                if (lam) x[k] = (lam_mul || PLANTED(6)) ? x[k] * (double)lam[g * GROUP + k] : x[k] / (double)lam[g * GROUP + k];
            }
            /* step 3: y = x * R^ */
            for (int n = 0; n < GROUP; ++n) {
                double acc = 0.0;
                for (int k = 0; k < GROUP - (PLANTED(11) ? 1 : 0); ++k) acc += x[k] * RKN(R, k, n);
                y[n] = acc;
                if (Y) Y[e0 + n] = acc;
            }
            /* steps 4-8 */
            quantize_group(y, c, scales + r * G + g, eflags ? eflags + e0 : NULL,
                           alt ? alt + e0 : NULL, gflags ? gflags + r * G + g : NULL,
                           alt_scales ? alt_scales + r * G + g : NULL);
            for (int i = 0; i < GROUP / 2; ++i)
                codes[e0 / 2 + i] = PLANTED(7) ? (uint8_t)(c[2 * i + 1] | (c[2 * i] << 4))
                                               : (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
    return 0;
}

int mxq_oracle_smooth_rotate_quantize(const uint16_t *X, int64_t rows, int64_t cols,
                                      const uint16_t *Rb, const float *lam, uint8_t *codes,
                                      uint8_t *scales, double *Y, uint8_t *eflags, uint8_t *alt,
                                      uint8_t *gflags, uint8_t *alt_scales, int nthreads)
{
    return rotate_quantize_rows(X, rows, cols, Rb, lam, 0, codes, scales, Y, eflags, alt, gflags,
                                alt_scales, nthreads);
}

/* The weights' side of the write-up's §3.3 (Ŵ = R̂ᵀ·Λ·W, absorbed offline):
 * with W stored transposed, Wt = Wᵀ [n_out, k_in], each row of Ŵᵀ = (Wt row · Λ)
 * · R̂ per 32-column group, then MXFP4 along k_in like the activations. */
int mxq_oracle_weight_rotate_quantize(const uint16_t *Wt, int64_t rows, int64_t cols,
                                      const uint16_t *Rb, const float *lam, uint8_t *codes,
                                      uint8_t *scales, double *Y, uint8_t *eflags, uint8_t *alt,
                                      uint8_t *gflags, uint8_t *alt_scales, int nthreads)
{
    return rotate_quantize_rows(Wt, rows, cols, Rb, lam, 1, codes, scales, Y, eflags, alt, gflags,
                                alt_scales, nthreads);
}

/* The consumer GEMM on MXFP4 operands (the write-up's §3.3 inference step on
 * Blackwell's native MXFP4 tensor cores, §1/§5.4): both operands K-major, codes
 * packed two per byte (even k in the low nibble), one E8M0 scale per 32 k.
 *   Y[m][n] = sum_k deq(A)[m][k] * deq(B)[n][k],  deq = E2M1 value * 2^(byte - 127)
 * in double, k ascending.  A: codes [M, K/2], scales [M, K/32]; B: codes [N, K/2],
 * scales [N, K/32]; Y: double [M, N].  A 0xFF scale makes its products NaN. */
int mxq_oracle_mxfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *b_codes,
                          const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, double *Y,
                          int nthreads)
{
    if (M < 0 || N < 0 || K < 0 || K % GROUP) return 1;
    int64_t G = K / GROUP;
    double *bd = (double *)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    if (!bd) return 1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int code = (b_codes[n * (K / 2) + k / 2] >> (4 * (k & 1))) & 0xF;
            bd[n * K + k] = mxq_oracle_e2m1_value(code) *
                            (PLANTED(16) ? 1.0 : mxq_oracle_e8m0_value(b_scales[n * G + k / GROUP]));
        }
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *ad = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t m = 0; m < M; ++m) {
            if (!ad) continue;
            for (int64_t k = 0; k < K; ++k) {
                int code = (a_codes[m * (K / 2) + k / 2] >> (4 * (k & 1))) & 0xF;
                ad[k] = mxq_oracle_e2m1_value(code) * mxq_oracle_e8m0_value(a_scales[m * G + k / GROUP]);
            }
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += ad[k] * bd[n * K + k];
                Y[m * N + n] = acc;
            }
        }
        free(ad);
    }
    free(bd);
    return 0;
}

/* --------------------------------------------------------------- NVFP4 variant */

/* The write-up's §5.3 names NVFP4 as another block-scaled format the method
 * suits; it gives no rule for it.  The reading taken is the public NVFP4 format:
 * blocks of 16 E2M1 values, one E4M3 scale per block and one fp32 scale s_t per
 * tensor, supplied by the caller.  Every decision is made in fp32 with this
 * sequence of correctly rounded single-precision operations:
 *   r_t = 1 / (6 * s_t)                         once per tensor
 *   v   = amax(block) * r_t;  s_b = E4M3(v)     round to nearest even, saturating at 448
 *   s   = s_b * s_t;          r   = 1 / s       (s == 0: all codes 0)
 *   u_n = y_n * r;            code_n = E2M1(u_n) as for MXFP4
 * A block holding NaN or Inf gets scale byte 0x7F (E4M3 NaN) and codes 0.     */

/* Value of an E4M3 code (OCP FP8, the variant without infinities: sign bit 7,
 * exponent bits 6-3 with bias 7, mantissa bits 2-0; exponent 0 is subnormal,
 * 0x7F and 0xFF are NaN, the largest value is 448). */
double mxq_oracle_e4m3_value(int code)
{
    int sgn = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* Nearest non-negative E4M3 code of v >= 0 by search over every code: ties go
 * to the even code, values past 448 to 448 (its nearest code), NaN to 0x7F. */
int mxq_oracle_e4m3_code(double v)
{
    if (isnan(v)) return 0x7F;
    int best = 0;
    double bd = fabs(v);
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(v - mxq_oracle_e4m3_value(c));
        if (d < bd || (d == bd && (c & 1) == (PLANTED(18) ? 1 : 0))) {
            best = c;
            bd = d;
        }
    }
    return best;
}

/* Codes of one 16-value block (values already fp32) under scale byte sb, with the
 * same element boundary flags as the MXFP4 quantiser. */
int mxq_oracle_nvfp4_block_at(const double *y, int sb, float s_t, uint8_t *codes, uint8_t *flags, uint8_t *alt)
{
    float s = (float)mxq_oracle_e4m3_value(sb) * s_t;
    int zero = sb == 0x7F || sb == 0xFF || s == 0.0f;
    float r = zero ? 0.0f : 1.0f / s;
    for (int n = 0; n < 16; ++n) {
        double u = zero ? 0.0 : (double)((float)y[n] * r);
        int c = zero ? 0 : mxq_oracle_e2m1_code(u);
        codes[n] = (uint8_t)c;
        if (flags || alt) {
            double a = fabs(u);
            int f = 0, other = c;
            for (int m = 0; m < 8 && !zero; ++m) {
                if (fabs(a - MID[m]) < 1e-3 * STEP[m]) {
                    f = 1;
                    if (m == 0) {
                        other = c ^ 8;
                    } else {
                        int lo = m - 1, hi = m, mag = c & 7;
                        other = (c & 8) | (mag == lo ? hi : lo);
                    }
                }
            }
            if (flags) flags[n] = (uint8_t)f;
            if (alt) alt[n] = (uint8_t)other;
        }
    }
    return 0;
}

/* X bf16 [rows, cols] -> y = (X / lam) * R per 32-column group (R bf16 [32][32], as
 * mxq_oracle_smooth_rotate_quantize) -> NVFP4 of every 16 columns of y.
 * codes [rows, cols/2] (even column in the low nibble); scales [rows, cols/16] E4M3;
 * Y, eflags/alt [rows, cols], bflags/alt_scales [rows, cols/16] may be NULL.
 * A block is flagged when v lies within 2.5e-4 (relative) of an E4M3 rounding midpoint;
 * alt_scales then holds the code on the other side. */
int mxq_oracle_nvfp4_quantize(const uint16_t *X, int64_t rows, int64_t cols, const uint16_t *Rb, const float *lam,
                              float s_t, uint8_t *codes, uint8_t *scales, double *Y, uint8_t *eflags, uint8_t *alt,
                              uint8_t *bflags, uint8_t *alt_scales, int nthreads)
{
    if (rows < 0 || cols < 0 || cols % GROUP) return 1;
    int64_t G = cols / GROUP, NB = cols / 16;
    double R[GROUP * GROUP];
    for (int i = 0; i < GROUP * GROUP; ++i) R[i] = bf16_to_double(Rb[i]);
    const float d6 = PLANTED(14) ? s_t : 6.0f * s_t;
    const float r_t = 1.0f / d6;
#pragma omp parallel for schedule(dynamic, 4) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            double x[GROUP], y[GROUP];
            int64_t e0 = r * cols + g * GROUP;
            for (int k = 0; k < GROUP; ++k) {
                x[k] = bf16_to_double(X[e0 + k]);
                if (lam) x[k] = x[k] / (double)lam[g * GROUP + k];
            }
            for (int n = 0; n < GROUP; ++n) {
                double acc = 0.0;
                for (int k = 0; k < GROUP; ++k) acc += x[k] * R[k * GROUP + n];
                if (Y) Y[e0 + n] = acc;
                y[n] = (double)(float)acc;          /* the decision precision: fp32 */
            }
            for (int h = 0; h < 2; ++h) {
                const double *yb = y + 16 * h;
                int64_t b = r * NB + g * 2 + h, eb = e0 + 16 * h;
                uint8_t c[16];
                float amax = 0.0f;
                int bad = 0;
                for (int n = 0; n < 16; ++n) {
                    if (isnan(yb[n]) || isinf(yb[n])) bad = 1;
                    float a = fabsf((float)yb[n]);
                    if (a > amax) amax = a;
                }
                int sb;
                if (bad) {
                    sb = 0x7F;
                    for (int n = 0; n < 16; ++n) {
                        c[n] = 0;
                        if (eflags) eflags[eb + n] = 0;
                        if (alt) alt[eb + n] = 0;
                    }
                } else {
                    float v = amax * r_t;
                    sb = mxq_oracle_e4m3_code((double)v);
                    mxq_oracle_nvfp4_block_at(yb, sb, s_t, c, eflags ? eflags + eb : NULL, alt ? alt + eb : NULL);
                }
                scales[b] = (uint8_t)sb;
                if (bflags || alt_scales) {
                    int f = 0, other = sb;
                    if (!bad) {
                        double v = (double)(amax * r_t), sv = mxq_oracle_e4m3_value(sb);
                        for (int dc = -1; dc <= 1; dc += 2) {
                            int cn = sb + dc;
                            if (cn < 0 || cn > 0x7E) continue;
                            double mid = 0.5 * (sv + mxq_oracle_e4m3_value(cn));
                            if (fabs(v - mid) < 2.5e-4 * mid) {
                                f = 1;
                                other = cn;
                            }
                        }
                    }
                    if (bflags) bflags[b] = (uint8_t)f;
                    if (alt_scales) alt_scales[b] = (uint8_t)other;
                }
                for (int i = 0; i < 8; ++i) codes[eb / 2 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
            }
        }
    }
    return 0;
}

/* The consumer GEMM on NVFP4 operands (the NVFP4 reading of the write-up's
 * §5.3, fed to the block-scaled tensor cores of §1/§5.4): both operands K-major,
 * codes packed two per byte (even k in the low nibble), one E4M3 scale per 16 k
 * and one fp32 tensor scale per operand:
 *   Y[m][n] = sum_k deq(A)[m][k] * deq(B)[n][k],
 *   deq = E2M1 value * E4M3 value of the block's scale * tensor scale,
 * in double, k ascending.  A: codes [M, K/2], scales [M, K/16]; B: codes [N, K/2],
 * scales [N, K/16]; Y: double [M, N].  A NaN scale (0x7F, 0xFF) makes its products NaN. */
int mxq_oracle_nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, float a_tscale, const uint8_t *b_codes,
                          const uint8_t *b_scales, float b_tscale, int64_t M, int64_t N, int64_t K, double *Y,
                          int nthreads)
{
    if (M < 0 || N < 0 || K < 0 || K % GROUP) return 1;
    int64_t NB = K / 16;
    double *bd = (double *)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    if (!bd) return 1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int code = (b_codes[n * (K / 2) + k / 2] >> (4 * (k & 1))) & 0xF;
            bd[n * K + k] = mxq_oracle_e2m1_value(code) * mxq_oracle_e4m3_value(b_scales[n * NB + k / 16]) *
                            (PLANTED(17) ? 1.0 : (double)b_tscale);
        }
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *ad = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t m = 0; m < M; ++m) {
            if (!ad) continue;
            for (int64_t k = 0; k < K; ++k) {
                int code = (a_codes[m * (K / 2) + k / 2] >> (4 * (k & 1))) & 0xF;
                ad[k] = mxq_oracle_e2m1_value(code) * mxq_oracle_e4m3_value(a_scales[m * NB + k / 16]) *
                        (double)a_tscale;
            }
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += ad[k] * bd[n * K + k];
                Y[m * N + n] = acc;
            }
        }
        free(ad);
    }
    free(bd);
    return 0;
}

/* Row-major E8M0 scales [rows, G] (G = K/32) in the layout Blackwell's
 * block-scaled MMA reads them in: 512-byte atoms, one per 128 rows x 4
 * k-blocks, atoms ordered by row block then k-block; inside an atom the scale
 * of row r (0..127) and k-block j (0..3) is byte 16 * (r % 32) + 4 * (r / 32) + j.
 * Rows and k-blocks past the matrix are 0.  out: ceil(rows/128) * ceil(G/4) * 512 bytes. */
int mxq_oracle_scales_to_mma(const uint8_t *scales, int64_t rows, int64_t G, uint8_t *out)
{
    if (rows < 0 || G < 0) return 1;
    int64_t RB = (rows + 127) / 128, CB = (G + 3) / 4;
    for (int64_t rb = 0; rb < RB; ++rb)
        for (int64_t cb = 0; cb < CB; ++cb)
            for (int r = 0; r < 128; ++r)
                for (int j = 0; j < 4; ++j) {
                    int64_t row = rb * 128 + r, kb = cb * 4 + j;
                    uint8_t v = (row < rows && kb < G) ? scales[row * G + kb] : 0;
                    int64_t at = PLANTED(21) ? 16 * (r / 32) + 4 * (r % 32) + j : 16 * (r % 32) + 4 * (r / 32) + j;
                    out[(rb * CB + cb) * 512 + at] = v;
                }
    return 0;
}

/* The rotation-block-size variant of the write-up's §4.3 ablation: blocks of
 * B = 16, 32, 64 or 128 columns are rotated by one shared B x B matrix, and
 * the MXFP4 groups stay at 32 columns.  For each row and each block of B
 * columns:
 *   1. x = the block's bf16 values in double, divided by Λ per channel;
 *   2. y = x * R_B (R_B bf16 [B][B], row-major [k][n]);
 *   3. every 32 consecutive columns of y (in the row) form one MXFP4 group,
 *      quantised as in mxq_oracle_smooth_rotate_quantize.
 * Outputs and flags have the layouts of mxq_oracle_smooth_rotate_quantize.
 * cols must be a multiple of both B and 32. */
int mxq_oracle_block_rotate_quantize(const uint16_t *X, int64_t rows, int64_t cols, int blk,
                                     const uint16_t *Rb, const float *lam, uint8_t *codes,
                                     uint8_t *scales, double *Y, uint8_t *eflags, uint8_t *alt,
                                     uint8_t *gflags, uint8_t *alt_scales, int nthreads)
{
    if (rows < 0 || cols < 0 || cols % GROUP || blk < 1 || blk > 128 || cols % blk) return 1;
    int64_t G = cols / GROUP;
    double *R = (double *)malloc(sizeof(double) * (size_t)(blk * blk));
    if (!R) return 1;
    for (int i = 0; i < blk * blk; ++i) R[i] = bf16_to_double(Rb[i]);
    int rc = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *yrow = (double *)malloc(sizeof(double) * (size_t)cols);
        double *x = (double *)malloc(sizeof(double) * (size_t)blk);
        if (!yrow || !x) {
#pragma omp atomic write
            rc = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < rows; ++r) {
                /* steps 1-2, block by block */
                for (int64_t b0 = 0; b0 < cols; b0 += blk) {
                    for (int k = 0; k < blk; ++k) {
                        x[k] = bf16_to_double(X[r * cols + b0 + k]);
                        if (lam) x[k] = x[k] / (double)lam[b0 + k];
                    }
                    for (int n = 0; n < blk; ++n) {
                        double acc = 0.0;
                        for (int k = 0; k < blk; ++k) acc += x[k] * (PLANTED(20) ? R[n * blk + k] : R[k * blk + n]);
                        yrow[b0 + n] = acc;
                    }
                }
                if (Y) memcpy(Y + r * cols, yrow, sizeof(double) * (size_t)cols);
                /* step 3: 32-column groups of the rotated row */
                for (int64_t g = 0; g < G; ++g) {
                    uint8_t c[GROUP];
                    int64_t e0 = r * cols + g * GROUP;
                    quantize_group(yrow + g * GROUP, c, scales + r * G + g, eflags ? eflags + e0 : NULL,
                                   alt ? alt + e0 : NULL, gflags ? gflags + r * G + g : NULL,
                                   alt_scales ? alt_scales + r * G + g : NULL);
                    for (int i = 0; i < GROUP / 2; ++i)
                        codes[e0 / 2 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
                }
            }
        }
        free(yrow);
        free(x);
    }
    free(R);
    return rc;
}

/* Dequantise: v = E2M1(code) * 2^(byte-127).  With R (bf16 [k][n]) the
 * rotation is undone, x_k = sum_n v_n R[k][n], and with lam the smoothing too,
 * x_k *= lam[k].  The exact double result is rounded once to bf16.  out_f64
 * (optional) receives the double before rounding. */
int mxq_oracle_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows,
                          int64_t cols, const uint16_t *Rb, const float *lam, uint16_t *out,
                          double *out_f64, int nthreads)
{
    if (rows < 0 || cols < 0 || cols % GROUP) return 1;
    int64_t G = cols / GROUP;
    double R[GROUP * GROUP];
    if (Rb)
        for (int i = 0; i < GROUP * GROUP; ++i) R[i] = bf16_to_double(Rb[i]);
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            int64_t e0 = r * cols + g * GROUP;
            double s = mxq_oracle_e8m0_value(scales[r * G + g]);
            double v[GROUP], x[GROUP];
            for (int n = 0; n < GROUP; ++n) {
                int byte = codes[(e0 + n) / 2];
                int code = (n & 1) ? (byte >> 4) : (byte & 15);
                v[n] = mxq_oracle_e2m1_value(code) * s;
            }
            for (int k = 0; k < GROUP; ++k) {
                if (Rb) {
                    double acc = 0.0;
                    for (int n = 0; n < GROUP; ++n) acc += v[n] * (PLANTED(13) ? R[n * GROUP + k] : R[k * GROUP + n]);
                    x[k] = acc;
                } else {
                    x[k] = v[k];
                }
                if (lam) x[k] = PLANTED(22) ? x[k] / (double)lam[g * GROUP + k] : x[k] * (double)lam[g * GROUP + k];
                out[e0 + k] = double_to_bf16(x[k]);
                if (out_f64) out_f64[e0 + k] = x[k];
            }
        }
    }
    return 0;
}

/* The per-group MXFP4 quantisation error of the write-up's §4.1 (Figure 1):
 * e_g = ||Q(y) - y||_2 / ||y||_2, where y is the group's rotated values
 * rounded to fp32 (the values the quantiser decides on) and Q(y) the group
 * dequantised from its own codes and scale.  An all-zero group has error 0 and a
 * NaN/Inf group NaN.  err [rows, cols/32] may be NULL; *mean gets the plain
 * average over all groups, summed in row-major order. */
int mxq_oracle_group_error(const uint16_t *X, int64_t rows, int64_t cols, const uint16_t *Rb,
                           const float *lam, double *err, double *mean, int nthreads)
{
    if (rows <= 0 || cols <= 0 || cols % GROUP) return 1;
    int64_t G = cols / GROUP;
    double R[GROUP * GROUP];
    for (int i = 0; i < GROUP * GROUP; ++i) R[i] = bf16_to_double(Rb[i]);
    double *e_all = err ? err : (double *)malloc(sizeof(double) * (size_t)(rows * G));
    if (!e_all) return 2;
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            double x[GROUP], y[GROUP];
            uint8_t c[GROUP], byte;
            int64_t e0 = r * cols + g * GROUP;
            for (int k = 0; k < GROUP; ++k) {
                x[k] = bf16_to_double(X[e0 + k]);
                if (lam) x[k] = x[k] / (double)lam[g * GROUP + k];
            }
            for (int n = 0; n < GROUP; ++n) {
                double acc = 0.0;
                for (int k = 0; k < GROUP; ++k) acc += x[k] * R[k * GROUP + n];
                y[n] = (double)(float)acc;          /* fp32, as in quantize_group */
            }
            quantize_group(y, c, &byte, NULL, NULL, NULL, NULL);
            double num = 0.0, den = 0.0;
            double s = mxq_oracle_e8m0_value(byte);
            for (int n = 0; n < GROUP; ++n) {
                double v = mxq_oracle_e2m1_value(c[n]) * s;
                num += (v - y[n]) * (v - y[n]);
                den += y[n] * y[n];
            }
            double e;
            if (byte == 0xFF) e = NAN;
            else e = den > 0.0 ? (PLANTED(19) ? num / den : sqrt(num / den)) : 0.0;
            e_all[r * G + g] = e;
        }
    }
    double total = 0.0;
    for (int64_t i = 0; i < rows * G; ++i) total += e_all[i];
    *mean = total / (double)(rows * G);
    if (!err) free(e_all);
    return 0;
}

/* ------------------------------------------------------- offline rotation search */

/* The Givens angle grid.  The write-up's §3.2 does not give the angle of each
 * candidate rotation.  Here angle a (0 <= a < 2n, skipping t = 0) is
 * t = tan(theta/2) = (a' - n)/n, with a' = a < n ? a : a + 1, and
 * c = (1 - t^2)/(1 + t^2), s = 2t/(1 + t^2): plain IEEE double operations, so any
 * implementation that follows them gets the same bits. */
void mxq_oracle_givens(int a, int n, double *c, double *s)
{
    int ap = a < n ? a : a + 1;
    double t = (double)(ap - n) / (double)n;
    double t2 = t * t;
    double den = 1.0 + t2;
    *c = (1.0 - t2) / den;
    *s = (2.0 * t) / den;
}

/* The outlier-aware rotation search of the write-up's §3.2, step by step.
 *   1. Locate the worst group: among the cols/32 channel groups, the [rows, 32]
 *      block of X / Lambda with the largest L-infinity norm (the first on ties).
 *   2. Start from R = I (32 x 32).
 *   3. Up to K steps:
 *      a. d = the column of the block holding its largest |value| (first on ties);
 *      b. for every other column j and every grid angle, the Givens rotation
 *         G(d, j): column d -> c*x_d - s*x_j, column j -> s*x_d + c*x_j;
 *      c. evaluate the L-infinity norm of the rotated block;
 *      d. keep the (j, angle) that lowers it most (the first on ties); stop if
 *         none lowers it;
 *      e. R <- R * G;
 *      f. block <- block * G.
 *   4. R is shared by every group (§3.2 step 4).
 * Rotations act on the right (X * R), the side the online step uses (§3.3).
 * R_out: 32 x 32 double, row-major [k][n].  group_out (optional): the worst group.
 * trace (optional): per step d, j, a.
 * linf (optional, K + 1 entries): the block's L-infinity norm before each step.
 * Returns the number of steps taken, or -1 on a bad argument. */
int mxq_oracle_rotation_search(const uint16_t *X, int64_t rows, int64_t cols, const float *lam, int K,
                               int n_angle, double *R_out, int64_t *group_out, int *trace, double *linf,
                               int nthreads)
{
    if (rows <= 0 || cols <= 0 || cols % GROUP || K < 0 || n_angle < 1) return -1;
    int64_t G = cols / GROUP;
    /* 1. the worst group */
    int64_t gw = 0;
    double best = -1.0;
    for (int64_t g = 0; g < G; ++g) {
        double m = 0.0;
        for (int64_t r = 0; r < rows; ++r)
            for (int k = 0; k < GROUP; ++k) {
                double v = bf16_to_double(X[r * cols + g * GROUP + k]);
                if (lam) v = v / (double)lam[g * GROUP + k];
                if (fabs(v) > m) m = fabs(v);
            }
        if (m > best) {
            best = m;
            gw = g;
        }
    }
    double *B = (double *)malloc(sizeof(double) * (size_t)(rows * GROUP));
    if (!B) return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int k = 0; k < GROUP; ++k) {
            double v = bf16_to_double(X[r * cols + gw * GROUP + k]);
            if (lam) v = v / (double)lam[gw * GROUP + k];
            B[r * GROUP + k] = v;
        }
    /* 2. R = I */
    double R[GROUP * GROUP];
    for (int i = 0; i < GROUP * GROUP; ++i) R[i] = (i / GROUP == i % GROUP) ? 1.0 : 0.0;
    double colmax[GROUP];
    int steps = 0;
    int n_cand = 2 * n_angle;
    double *cand = (double *)malloc(sizeof(double) * GROUP * (size_t)n_cand);
    if (!cand) {
        free(B);
        return -1;
    }
    for (int step = 0;; ++step) {
        for (int k = 0; k < GROUP; ++k) colmax[k] = 0.0;
        for (int64_t r = 0; r < rows; ++r)
            for (int k = 0; k < GROUP; ++k)
                if (fabs(B[r * GROUP + k]) > colmax[k]) colmax[k] = fabs(B[r * GROUP + k]);
        /* a. the column of the largest value */
        int d = 0;
        for (int k = 1; k < GROUP; ++k)
            if (colmax[k] > colmax[d]) d = k;
        double cur = colmax[d];
        if (linf) linf[step] = cur;
        if (step == K) break;
        /* b, c. every candidate's L-infinity norm */
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
        for (int ci = 0; ci < GROUP * n_cand; ++ci) {
            int j = ci / n_cand, a = ci % n_cand;
            if (j == d) {
                cand[ci] = INFINITY;
                continue;
            }
            double c, s;
            mxq_oracle_givens(a, n_angle, &c, &s);
            double m = 0.0;
            for (int k = 0; k < GROUP; ++k)
                if (k != d && k != j && colmax[k] > m) m = colmax[k];
            for (int64_t r = 0; r < rows; ++r) {
                double xd = B[r * GROUP + d], xj = B[r * GROUP + j];
                double u = c * xd - s * xj;
                double w = s * xd + c * xj;
                if (fabs(u) > m) m = fabs(u);
                if (fabs(w) > m) m = fabs(w);
            }
            cand[ci] = m;
        }
        /* d. the largest decrease */
        int bi = -1;
        for (int ci = 0; ci < GROUP * n_cand; ++ci)
            if (cand[ci] < cur && (bi < 0 || cand[ci] < cand[bi])) bi = ci;
        if (bi < 0) break;
        int j = bi / n_cand, a = bi % n_cand;
        double c, s;
        mxq_oracle_givens(a, n_angle, &c, &s);
        /* e. R <- R * G */
        for (int r = 0; r < GROUP; ++r) {
            if (PLANTED(12)) {   /* G * R: rows d and j instead of columns */
                double rd = R[d * GROUP + r], rj = R[j * GROUP + r];
                R[d * GROUP + r] = c * rd - s * rj;
                R[j * GROUP + r] = s * rd + c * rj;
                continue;
            }
            double rd = R[r * GROUP + d], rj = R[r * GROUP + j];
            R[r * GROUP + d] = c * rd - s * rj;
            R[r * GROUP + j] = s * rd + c * rj;
        }
        /* f. block <- block * G */
        for (int64_t r = 0; r < rows; ++r) {
            double xd = B[r * GROUP + d], xj = B[r * GROUP + j];
            B[r * GROUP + d] = c * xd - s * xj;
            B[r * GROUP + j] = s * xd + c * xj;
        }
        if (trace) {
            trace[3 * step] = d;
            trace[3 * step + 1] = j;
            trace[3 * step + 2] = a;
        }
        ++steps;
    }
    memcpy(R_out, R, sizeof R);
    if (group_out) *group_out = gw;
    free(cand);
    free(B);
    return steps;
}

/* Exposed for the pins: exact bf16 <-> double conversions. */
void mxq_oracle_bf16_to_double(const uint16_t *b, double *d, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) d[i] = bf16_to_double(b[i]);
}

void mxq_oracle_double_to_bf16(const double *d, uint16_t *b, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) b[i] = double_to_bf16(d[i]);
}
