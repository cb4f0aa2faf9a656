/*
 * w4a16_oracle.c -- plain, slow CPU oracle for the A16W4 per-group matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant
 * generator with the CUDA library; both sides are written independently from
 * the same source text.
 *
 * Source of every step: the page "WeightQuantBatchMatmulExperiment 算子深度解析"
 * (bjdmk.com.cn/news/4847346), section 4.1 "算子功能：MSD 伪量化算法",
 * equations 1-11, and section 4.2 (operator spec: x fp16, weight int4,
 * antiquant_scale fp16, y fp16, all 2-D).  The direct-dequant result is the
 * plain definition y = x . (antiquant_scale (.) W) of the same operator.
 *
 * Readings taken where the page is silent or garbled (each is stated again at
 * the function that uses it):
 *   R1  eq. 10 prints the denominators as "7.4914.98" and "7.4914.98*14.98";
 *       the multiplication sign was lost, so they are 7.49*14.98 and
 *       7.49*14.98*14.98 (each residual step rescales by 14.98, eq. 4 and 6).
 *   R2  A_max = rowMax(|A_group|) is taken per row m and per group of g
 *       consecutive K entries (eq. 1, "PerGroup").
 *   R3  round() is round-half-to-even.
 *   R4  tmp1..tmp3 are evaluated in IEEE binary32 with the constants 7.49f
 *       and 14.98f (the kernel-side constant table of section 4.1), in the
 *       literal operation order of eq. 2/4/6: (7.49*x)/A_max, (tmp-A)*14.98.
 *       A second mode evaluates the same steps in binary64 (used only for the
 *       truncation-bound pin).
 *   R5  A_max == 0 (an all-zero group) gives A1 = A2 = A3 = 0: the group
 *       contributes nothing and no division is performed.
 *   R6  the logical weight input is bytes [K/2][N]; byte (i, n) holds W[2i][n]
 *       in its low nibble and W[2i+1][n] in its high nibble, two's complement
 *       (section 4.3: "each byte stores two int4").
 *   R7  eq. 10-11 are evaluated in binary64, groups added in increasing order,
 *       and y is rounded to binary16 (round-to-nearest-even) once at the end.
 *   R13, R14  the routing prep of the grouped form (see oracle_moe_align).
 *   R15  bf16 activations for the dequant form (see oracle_dequant_bf16).
 *   R16  MSD with S = 2..4 unfold steps (see expand_row_steps).
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -fPIC -shared
 * (binary32 arithmetic must stay IEEE single with no FMA contraction).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------------- */
/* binary16 <-> binary64, from the IEEE 754 binary16 format definition      */
/* (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits).            */
/* ---------------------------------------------------------------------- */

double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f + 1024), e - 25);     /* (1.f) * 2^(e-15) */
    return sign ? -v : v;
}

/* Round a binary64 value to the nearest binary16, ties to even. */
uint16_t oracle_double_to_half(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return 0x7e00;
    if (a == 0.0) return sign;
    int E;
    frexp(a, &E);                 /* a = m * 2^E, m in [0.5, 1) */
    int e = E - 1;                /* a in [2^e, 2^(e+1)) */
    if (e < -14) {
        /* subnormal range: quantum 2^-24 */
        double q = rint(ldexp(a, 24));            /* exact scaling, RNE */
        return (uint16_t)(sign | (uint16_t)q);    /* q == 1024 -> min normal */
    }
    double q = rint(ldexp(a, 10 - e));            /* q in [1024, 2048] */
    if (q >= 2048.0) { q = 1024.0; e += 1; }
    if (e > 15) return (uint16_t)(sign | 0x7c00); /* overflow -> inf */
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(q - 1024.0));
}

void oracle_halves_to_double(const uint16_t* h, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_half_to_double(h[i]);
}

void oracle_doubles_to_half(const double* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_double_to_half(v[i]);
}

/* ---------------------------------------------------------------------- */
/* Weight decode (reading R6).                                              */
/* ---------------------------------------------------------------------- */

static int decode_nibble(unsigned v)
{
    v &= 0xf;
    return v >= 8 ? (int)v - 16 : (int)v;   /* two's complement int4 */
}

static int weight_at(const uint8_t* wp, int N, int k, int n)
{
    uint8_t b = wp[(size_t)(k >> 1) * N + n];
    return decode_nibble((k & 1) ? (b >> 4) : b);
}

void oracle_unpack_w(const uint8_t* wp, int K, int N, int8_t* w)
{
    for (int k = 0; k < K; ++k)
        for (int n = 0; n < N; ++n)
            w[(size_t)k * N + n] = (int8_t)weight_at(wp, N, k, n);
}

/* ---------------------------------------------------------------------- */
/* MSD eq. 1-7 for one row: A_max per group and the three residual digits.  */
/* ---------------------------------------------------------------------- */

/* mode 0: binary32 (reading R4); mode 1: binary64. */
static void expand_row(const uint16_t* xrow, int K, int g, int mode,
                       double* amax_row, int8_t* a1, int8_t* a2, int8_t* a3)
{
    int G = K / g;
    for (int gi = 0; gi < G; ++gi) {
        const uint16_t* xg = xrow + (size_t)gi * g;
        /* eq. 1: A_max = rowMax(|A_group|) (reading R2); exact on fp16 values */
        double am = 0.0;
        for (int j = 0; j < g; ++j) {
            double v = fabs(oracle_half_to_double(xg[j]));
            if (v > am) am = v;
        }
        amax_row[gi] = am;
        for (int j = 0; j < g; ++j) {
            int k = gi * g + j;
            if (am == 0.0) {                    /* reading R5 */
                a1[k] = a2[k] = a3[k] = 0;
                continue;
            }
            if (mode == 0) {
                float xf = (float)oracle_half_to_double(xg[j]);  /* exact */
                float amf = (float)am;                           /* exact */
                float tmp1 = (7.49f * xf) / amf;                 /* eq. 2 */
                float A1 = rintf(tmp1);                          /* eq. 3 */
                float tmp2 = (tmp1 - A1) * 14.98f;               /* eq. 4 */
                float A2 = rintf(tmp2);                          /* eq. 5 */
                float tmp3 = (tmp2 - A2) * 14.98f;               /* eq. 6 */
                float A3 = rintf(tmp3);                          /* eq. 7 */
                a1[k] = (int8_t)A1; a2[k] = (int8_t)A2; a3[k] = (int8_t)A3;
            } else {
                double xd = oracle_half_to_double(xg[j]);
                double tmp1 = (7.49 * xd) / am;
                double A1 = rint(tmp1);
                double tmp2 = (tmp1 - A1) * 14.98;
                double A2 = rint(tmp2);
                double tmp3 = (tmp2 - A2) * 14.98;
                double A3 = rint(tmp3);
                a1[k] = (int8_t)A1; a2[k] = (int8_t)A2; a3[k] = (int8_t)A3;
            }
        }
    }
}

/* eq. 1-8 for all rows.  amax: [M][G] (binary64, exact fp16 values).
 * a: A_int of eq. 8, the residual matrices stacked along M: [3][M][K]. */
int oracle_msd_expand(const uint16_t* x, int M, int K, int g, int mode,
                      double* amax, int8_t* a)
{
    if (g <= 0 || K % g) return -1;
    int G = K / g;
    for (int m = 0; m < M; ++m)
        expand_row(x + (size_t)m * K, K, g, mode, amax + (size_t)m * G,
                   a + (size_t)m * K, a + ((size_t)M + m) * K,
                   a + (2 * (size_t)M + m) * K);
    return 0;
}

/* eq. 9: Y_int = A_int . Weight_group, per group, exact in int64.
 * a: [3][M][K]; yint: [3][M][G][N]. */
int oracle_msd_yint(const int8_t* a, const uint8_t* wp, int M, int K, int N,
                    int g, int64_t* yint)
{
    if (g <= 0 || K % g) return -1;
    int G = K / g;
    for (int r = 0; r < 3; ++r)
        for (int m = 0; m < M; ++m) {
            const int8_t* ar = a + ((size_t)r * M + m) * K;
            for (int gi = 0; gi < G; ++gi) {
                int64_t* out = yint + (((size_t)r * M + m) * G + gi) * N;
#pragma omp parallel for schedule(static)
                for (int n = 0; n < N; ++n) {
                    int64_t s = 0;
                    for (int k = gi * g; k < (gi + 1) * g; ++k)
                        s += (int64_t)ar[k] * weight_at(wp, N, k, n);
                    out[n] = s;
                }
            }
        }
    return 0;
}

/* eq. 10 for one (row, group, column), reading R1, evaluated as printed. */
static double merge_y(int64_t y1, int64_t y2, int64_t y3, double amax, double scale)
{
    double yg = ((double)y1 / 7.49 + (double)y2 / (7.49 * 14.98)
                 + (double)y3 / (7.49 * 14.98 * 14.98)) * amax;
    return yg * scale;
}

/* eq. 10-11 from stored Y_int: y[M][N] in binary64 (reading R7). */
int oracle_msd_combine(const int64_t* yint, const double* amax,
                       const uint16_t* scale, int M, int K, int N, int g,
                       double* y)
{
    if (g <= 0 || K % g) return -1;
    int G = K / g;
    for (int m = 0; m < M; ++m)
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;                              /* Y^0 = 0 */
            for (int gi = 0; gi < G; ++gi) {
                size_t i1 = (((size_t)0 * M + m) * G + gi) * N + n;
                size_t i2 = (((size_t)1 * M + m) * G + gi) * N + n;
                size_t i3 = (((size_t)2 * M + m) * G + gi) * N + n;
                double s = oracle_half_to_double(scale[(size_t)gi * N + n]);
                acc = merge_y(yint[i1], yint[i2], yint[i3],
                              amax[(size_t)m * G + gi], s) + acc;  /* eq. 11 */
            }
            y[(size_t)m * N + n] = acc;
        }
    return 0;
}

/* All eleven steps for every output, row by row (the per-row Y_int is kept
 * only for the row being processed).  y: [M][N] binary64. */
int oracle_msd(const uint16_t* x, const uint8_t* wp, const uint16_t* scale,
               int M, int K, int N, int g, int mode, double* y)
{
    if (g <= 0 || K % g) return -1;
    int G = K / g;
    double* amax = (double*)malloc(sizeof(double) * (size_t)G);
    int8_t* a = (int8_t*)malloc(3 * (size_t)K);
    if (!amax || !a) { free(amax); free(a); return -2; }
    for (int m = 0; m < M; ++m) {
        expand_row(x + (size_t)m * K, K, g, mode, amax, a, a + K, a + 2 * (size_t)K);
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int gi = 0; gi < G; ++gi) {
                int64_t y1 = 0, y2 = 0, y3 = 0;
                for (int k = gi * g; k < (gi + 1) * g; ++k) {
                    int w = weight_at(wp, N, k, n);
                    y1 += (int64_t)a[k] * w;
                    y2 += (int64_t)a[K + k] * w;
                    y3 += (int64_t)a[2 * (size_t)K + k] * w;
                }
                double s = oracle_half_to_double(scale[(size_t)gi * N + n]);
                acc = merge_y(y1, y2, y3, amax[gi], s) + acc;
            }
            y[(size_t)m * N + n] = acc;
        }
    }
    free(amax);
    free(a);
    return 0;
}

/* The same eleven steps, only at the listed (row, column) pairs. */
int oracle_msd_at(const uint16_t* x, const uint8_t* wp, const uint16_t* scale,
                  int M, int K, int N, int g, int mode,
                  const int32_t* rows, const int32_t* cols, int count, double* y)
{
    if (g <= 0 || K % g) return -1;
    int G = K / g;
    int bad = 0;
#pragma omp parallel
    {
        double* amax = (double*)malloc(sizeof(double) * (size_t)G);
        int8_t* a = (int8_t*)malloc(3 * (size_t)K);
        int last_row = -1;
#pragma omp for schedule(static)
        for (int i = 0; i < count; ++i) {
            int m = rows[i], n = cols[i];
            if (!amax || !a || m < 0 || m >= M || n < 0 || n >= N) {
                y[i] = NAN;
#pragma omp atomic write
                bad = 1;
                continue;
            }
            if (m != last_row) {
                expand_row(x + (size_t)m * K, K, g, mode, amax, a, a + K, a + 2 * (size_t)K);
                last_row = m;
            }
            double acc = 0.0;
            for (int gi = 0; gi < G; ++gi) {
                int64_t y1 = 0, y2 = 0, y3 = 0;
                for (int k = gi * g; k < (gi + 1) * g; ++k) {
                    int w = weight_at(wp, N, k, n);
                    y1 += (int64_t)a[k] * w;
                    y2 += (int64_t)a[K + k] * w;
                    y3 += (int64_t)a[2 * (size_t)K + k] * w;
                }
                double s = oracle_half_to_double(scale[(size_t)gi * N + n]);
                acc = merge_y(y1, y2, y3, amax[gi], s) + acc;
            }
            y[i] = acc;
        }
        free(amax);
        free(a);
    }
    return bad ? -3 : 0;
}

/* ---------------------------------------------------------------------- */
/* MSD with S unfold steps.  Section 7 of the same page ("性能分析") notes    */
/* that the gain varies with the number of MSD unfold steps; section 4.1    */
/* gives three.  Reading R16: an S-step expansion runs the same residual     */
/* recursion (eq. 2-7) for S digits, tmp_{i+1} = (tmp_i - A_i) * 14.98 and   */
/* A_{i+1} = round(tmp_{i+1}), so its digits are the first S digits of any   */
/* longer expansion; eq. 10 gets one term per digit, Y_i divided by          */
/* 7.49 * 14.98^(i-1) (extending R1).  A_max, R2-R7 are unchanged.  These    */
/* functions stand beside the three-step ones above and do not replace them. */
/* ---------------------------------------------------------------------- */

#define ORACLE_MAX_STEPS 8

/* eq. 1-7 with S digits for one row (mode 0 binary32, 1 binary64).
 * a: digit i of element k at a[i * plane + k]. */
static void expand_row_steps(const uint16_t* xrow, int K, int g, int mode, int S,
                             double* amax_row, int8_t* a, size_t plane)
{
    int G = K / g;
    for (int gi = 0; gi < G; ++gi) {
        const uint16_t* xg = xrow + (size_t)gi * g;
        double am = 0.0;                                   /* eq. 1, R2 */
        for (int j = 0; j < g; ++j) {
            double v = fabs(oracle_half_to_double(xg[j]));
            if (v > am) am = v;
        }
        amax_row[gi] = am;
        for (int j = 0; j < g; ++j) {
            int k = gi * g + j;
            if (am == 0.0) {                               /* R5 */
                for (int i = 0; i < S; ++i) a[(size_t)i * plane + k] = 0;
                continue;
            }
            if (mode == 0) {
                float xf = (float)oracle_half_to_double(xg[j]);
                float amf = (float)am;
                float t = (7.49f * xf) / amf;              /* eq. 2 */
                for (int i = 0; i < S; ++i) {
                    float A = rintf(t);                    /* eq. 3, 5, 7, ... */
                    a[(size_t)i * plane + k] = (int8_t)A;
                    t = (t - A) * 14.98f;                  /* eq. 4, 6, ... */
                }
            } else {
                double t = (7.49 * oracle_half_to_double(xg[j])) / am;
                for (int i = 0; i < S; ++i) {
                    double A = rint(t);
                    a[(size_t)i * plane + k] = (int8_t)A;
                    t = (t - A) * 14.98;
                }
            }
        }
    }
}

/* a: [S][M][K]; amax: [M][G]. */
int oracle_msd_expand_steps(const uint16_t* x, int M, int K, int g, int mode, int S,
                            double* amax, int8_t* a)
{
    if (g <= 0 || K % g || S < 1 || S > ORACLE_MAX_STEPS) return -1;
    int G = K / g;
    for (int m = 0; m < M; ++m)
        expand_row_steps(x + (size_t)m * K, K, g, mode, S, amax + (size_t)m * G,
                         a + (size_t)m * K, (size_t)M * K);
    return 0;
}

/* eq. 9 for S planes: a [S][M][K] -> yint [S][M][G][N], exact in int64. */
int oracle_msd_yint_planes(const int8_t* a, int S, const uint8_t* wp, int M, int K, int N,
                           int g, int64_t* yint)
{
    if (g <= 0 || K % g || S < 1) return -1;
    int G = K / g;
    for (int r = 0; r < S; ++r)
        for (int m = 0; m < M; ++m) {
            const int8_t* ar = a + ((size_t)r * M + m) * K;
            for (int gi = 0; gi < G; ++gi) {
                int64_t* out = yint + (((size_t)r * M + m) * G + gi) * N;
#pragma omp parallel for schedule(static)
                for (int n = 0; n < N; ++n) {
                    int64_t s = 0;
                    for (int k = gi * g; k < (gi + 1) * g; ++k)
                        s += (int64_t)ar[k] * weight_at(wp, N, k, n);
                    out[n] = s;
                }
            }
        }
    return 0;
}

/* eq. 10 with S terms (R16): (sum_i Y_i / (7.49 * 14.98^(i-1))) * A_max *
 * scale, the terms added in increasing i. */
static double merge_y_steps(const int64_t* yi, int S, double amax, double scale)
{
    double den = 7.49, sum = 0.0;
    for (int i = 0; i < S; ++i) {
        sum = sum + (double)yi[i] / den;
        den = den * 14.98;
    }
    return sum * amax * scale;
}

/* One output (m, n) from a row's digits a [S][K] (plane stride K). */
static double msd_out_steps(const int8_t* a, int S, const double* amax, const uint8_t* wp,
                            const uint16_t* scale, int K, int N, int g, int n)
{
    int G = K / g;
    double acc = 0.0;
    for (int gi = 0; gi < G; ++gi) {
        int64_t yi[ORACLE_MAX_STEPS];
        for (int i = 0; i < S; ++i) yi[i] = 0;
        for (int k = gi * g; k < (gi + 1) * g; ++k) {
            int w = weight_at(wp, N, k, n);
            for (int i = 0; i < S; ++i) yi[i] += (int64_t)a[(size_t)i * K + k] * w;
        }
        double s = oracle_half_to_double(scale[(size_t)gi * N + n]);
        acc = merge_y_steps(yi, S, amax[gi], s) + acc;     /* eq. 11 */
    }
    return acc;
}

/* All steps with S digits: y [M][N] binary64. */
int oracle_msd_steps(const uint16_t* x, const uint8_t* wp, const uint16_t* scale,
                     int M, int K, int N, int g, int mode, int S, double* y)
{
    if (g <= 0 || K % g || S < 1 || S > ORACLE_MAX_STEPS) return -1;
    int G = K / g;
    double* amax = (double*)malloc(sizeof(double) * (size_t)G);
    int8_t* a = (int8_t*)malloc((size_t)S * K);
    if (!amax || !a) { free(amax); free(a); return -2; }
    for (int m = 0; m < M; ++m) {
        expand_row_steps(x + (size_t)m * K, K, g, mode, S, amax, a, (size_t)K);
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n)
            y[(size_t)m * N + n] = msd_out_steps(a, S, amax, wp, scale, K, N, g, n);
    }
    free(amax);
    free(a);
    return 0;
}

/* The same, only at the listed (row, column) pairs. */
int oracle_msd_at_steps(const uint16_t* x, const uint8_t* wp, const uint16_t* scale,
                        int M, int K, int N, int g, int mode, int S,
                        const int32_t* rows, const int32_t* cols, int count, double* y)
{
    if (g <= 0 || K % g || S < 1 || S > ORACLE_MAX_STEPS) return -1;
    int G = K / g;
    int bad = 0;
#pragma omp parallel
    {
        double* amax = (double*)malloc(sizeof(double) * (size_t)G);
        int8_t* a = (int8_t*)malloc((size_t)S * K);
        int last_row = -1;
#pragma omp for schedule(static)
        for (int i = 0; i < count; ++i) {
            int m = rows[i], n = cols[i];
            if (!amax || !a || m < 0 || m >= M || n < 0 || n >= N) {
                y[i] = NAN;
#pragma omp atomic write
                bad = 1;
                continue;
            }
            if (m != last_row) {
                expand_row_steps(x + (size_t)m * K, K, g, mode, S, amax, a, (size_t)K);
                last_row = m;
            }
            y[i] = msd_out_steps(a, S, amax, wp, scale, K, N, g, n);
        }
        free(amax);
        free(a);
    }
    return bad ? -3 : 0;
}

/* ---------------------------------------------------------------------- */
/* Direct dequant: the plain definition y = x . (scale (.) W), binary64.     */
/* Every product x*scale*W is exact in binary64 (11+11+4 significant bits);  */
/* only the K-sum rounds, in increasing k.                                   */
/* ---------------------------------------------------------------------- */

int oracle_dequant(const uint16_t* x, const uint8_t* wp, const uint16_t* scale,
                   int M, int K, int N, int g, double* y)
{
    if (g <= 0 || K % g) return -1;
    for (int m = 0; m < M; ++m)
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) {
                double xv = oracle_half_to_double(x[(size_t)m * K + k]);
                double s = oracle_half_to_double(scale[(size_t)(k / g) * N + n]);
                acc += xv * s * (double)weight_at(wp, N, k, n);
            }
            y[(size_t)m * N + n] = acc;
        }
    return 0;
}

int oracle_dequant_at(const uint16_t* x, const uint8_t* wp, const uint16_t* scale,
                      int M, int K, int N, int g,
                      const int32_t* rows, const int32_t* cols, int count, double* y)
{
    if (g <= 0 || K % g) return -1;
    int bad = 0;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < count; ++i) {
        int m = rows[i], n = cols[i];
        if (m < 0 || m >= M || n < 0 || n >= N) {
            y[i] = NAN;
#pragma omp atomic write
            bad = 1;
            continue;
        }
        double acc = 0.0;
        for (int k = 0; k < K; ++k) {
            double xv = oracle_half_to_double(x[(size_t)m * K + k]);
            double s = oracle_half_to_double(scale[(size_t)(k / g) * N + n]);
            acc += xv * s * (double)weight_at(wp, N, k, n);
        }
        y[i] = acc;
    }
    return bad ? -3 : 0;
}

/* ---------------------------------------------------------------------- */
/* bf16 activations for the dequant form (the INT4 + BF16 pairing of the    */
/* Humming article, aihirek.info).  bfloat16 is the upper half of binary32: */
/* 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits.  Reading R15:   */
/* x, scale and y are all bf16; y is the same exact binary64 definition     */
/* x . (scale (.) W), rounded to bf16 by the caller's tolerance check.      */
/* ---------------------------------------------------------------------- */

double oracle_bf16_to_double(uint16_t b)
{
    const int sign = (b >> 15) & 1;
    const int e = (b >> 7) & 0xff;
    const int f = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);                /* subnormal: f * 2^-126 * 2^-7 */
    else if (e == 0xff)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + f), e - 134);     /* (1 + f/128) * 2^(e-127) */
    return sign ? -v : v;
}

void oracle_bf16s_to_double(const uint16_t* b, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_double(b[i]);
}

int oracle_dequant_bf16(const uint16_t* x, const uint8_t* wp, const uint16_t* scale, int M, int K, int N,
                        int g, double* y)
{
    if (g <= 0 || K % g) return -1;
    for (int m = 0; m < M; ++m)
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) {
                const double xv = oracle_bf16_to_double(x[(size_t)m * K + k]);
                const double s = oracle_bf16_to_double(scale[(size_t)(k / g) * N + n]);
                acc += xv * s * (double)weight_at(wp, N, k, n);
            }
            y[(size_t)m * N + n] = acc;
        }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Routing prep for the grouped (per-expert) form.                          */
/*                                                                          */
/* The grouped matmul takes each expert's tokens as one contiguous segment  */
/* of rows (offsets[E+1]); the mixture-of-experts scheduling of the Humming */
/* article (aihirek.info, MoE section) and the moe_align_block_size step of */
/* the FlagGems operator list (pwwt.cn) both start from a router's          */
/* topk_ids [T][topk].  Reading R13: the routing prep is a stable grouping  */
/* of the entries i = t*topk + j (token t's j-th expert) by expert id, in   */
/* increasing i within an expert; an id outside [0, E) takes no row.  R14:   */
/* the un-permute adds token t's rows weighted by its gate weights,         */
/* slots in increasing j, in binary64, rounded to binary16 once.            */
/* ---------------------------------------------------------------------- */

/* offsets[e] = entries whose expert is below e; entry i of expert e gets row
 * pos = offsets[e] + (entries of expert e before i); sorted_token[pos] = t
 * (its token) and inv_pos[i] = pos.  Entries without an expert get
 * inv_pos[i] = -1 and rows offsets[E] .. T*topk-1 hold -1.  Returns the
 * number of such entries. */
int oracle_moe_align(const int32_t* ids, int T, int topk, int E, int32_t* offsets,
                     int32_t* sorted_token, int32_t* inv_pos)
{
    const int n = T * topk;
    int64_t* fill = (int64_t*)calloc((size_t)E + 1, sizeof(int64_t));
    if (!fill) return -1;
    int dropped = 0;
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int i = 0; i < n; ++i) {
        const int e = ids[i];
        if (e < 0 || e >= E) {
            ++dropped;
            continue;
        }
        ++offsets[e + 1];
    }
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    for (int i = 0; i < n; ++i) sorted_token[i] = -1;
    for (int i = 0; i < n; ++i) {
        const int e = ids[i];
        if (e < 0 || e >= E) {
            inv_pos[i] = -1;
            continue;
        }
        const int pos = offsets[e] + (int)fill[e]++;
        sorted_token[pos] = i / topk;
        inv_pos[i] = pos;
    }
    free(fill);
    return dropped;
}

/* y[t][n] = sum_j w[t][j] * y_sorted[inv_pos[t*topk+j]][n] (binary16 in and
 * out, binary64 sum, slots in increasing j, entries without a row skipped). */
int oracle_moe_combine(const uint16_t* y_sorted, const int32_t* inv_pos, const float* w, int T, int topk,
                       int N, uint16_t* y)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int j = 0; j < topk; ++j) {
                const int pos = inv_pos[t * topk + j];
                if (pos < 0) continue;
                acc += (double)w[t * topk + j] * oracle_half_to_double(y_sorted[(size_t)pos * N + n]);
            }
            y[(size_t)t * N + n] = oracle_double_to_half(acc);
        }
    return 0;
}

/* Threads an OpenMP parallel region will use (for the CPU-baseline report). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
