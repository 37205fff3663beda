/*
 * quant_oracle.c -- fp64 CPU oracle for fp8-e4m3 quantisation with incoherent processing.
 * TEST INFRASTRUCTURE: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark load this code.  It shares nothing with the CUDA library.
 *
 * What it computes follows the page "FlashAttention-3 (DE)", section "Niedrige
 * Praezision (FP8) mit reduziertem Quantisierungsfehler": before quantisation each
 * query / key vector is multiplied by a random orthogonal matrix, here the Hadamard
 * matrix with random column signs, R = diag(s) H / sqrt(d); because R is orthogonal,
 * (Q R)(K R)^T = Q K^T, so the scores are unchanged while outliers are spread over all
 * coordinates.  The quantisation itself is the per-(batch, head) amax scaling into the
 * OCP e4m3 format that the fp8 path uses: descale = amax / 448, code = nearest e4m3
 * value of y / descale.
 *
 * Every step is the plain definition in binary64: H from the doubling recursion, y as a
 * full matrix-vector product, the code as the nearest of the 127 non-negative finite
 * e4m3 values found by search.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

double oracle_decode_bf16(uint16_t h);
double oracle_decode_e4m3(uint8_t c);

#define ORACLE_QF64 0
#define ORACLE_QBF16 1
#define E4M3_MAX_FINITE 448.0

/*
 * Sylvester's Hadamard matrix of order d (a power of two), d x d row-major:
 * H_1 = [1] and H_{2n} = [[H_n, H_n], [H_n, -H_n]].  Returns 0, or -1 if d is not a
 * power of two >= 1.
 */
int oracle_hadamard(int64_t d, double *out) {
    if (d < 1 || (d & (d - 1)) != 0 || out == NULL) return -1;
    out[0] = 1.0;
    for (int64_t n = 1; n < d; n *= 2) {
        /* grow the leading n x n block (stored with row stride d) to 2n x 2n */
        for (int64_t i = 0; i < n; ++i)
            for (int64_t j = 0; j < n; ++j) {
                const double h = out[i * d + j];
                out[i * d + (j + n)] = h;
                out[(i + n) * d + j] = h;
                out[(i + n) * d + (j + n)] = -h;
            }
    }
    return 0;
}

/*
 * Nearest finite OCP e4m3 code to v, ties to the code with an even mantissa (the
 * round-to-nearest-even rule), magnitudes beyond 448 to 448 (saturation to the largest
 * finite value).  The sign bit is v's sign bit.  NaN input gives 0x7F.
 */
uint8_t oracle_encode_e4m3(double v) {
    if (isnan(v)) return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs(v);
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        const double err = fabs(a - oracle_decode_e4m3((uint8_t)c));
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

static double load_x(const void *x, int elem_type, int64_t idx) {
    if (elem_type == ORACLE_QBF16) return oracle_decode_bf16(((const uint16_t *)x)[idx]);
    return ((const double *)x)[idx];
}

/*
 * Quantise S independent slices of N rows of length d (x is [S, N, d], bf16 bits or
 * fp64 by elem_type).  With signs != NULL (d entries of +1 / -1) every row is first
 * rotated: y = x diag(s) H / sqrt(d); with signs == NULL, y = x.
 *
 * Per slice: amax = max |y|; descale = amax / 448 and code = encode(y * 448 / amax), or
 * descale = 1 and every code 0 when amax == 0.
 *
 * Outputs: codes [S, N, d] (may be NULL), descale [S] (may be NULL), y_out [S, N, d] in
 * fp64 (may be NULL).  nthreads > 0 sets the OpenMP thread count, 0 keeps the default.
 * Returns 0, -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_quantize_e4m3(const void *x, int elem_type, const int8_t *signs, int64_t S,
                         int64_t N, int64_t d, uint8_t *codes, double *descale,
                         double *y_out, int nthreads) {
    if (x == NULL || S < 0 || N < 0 || d < 1 ||
        (elem_type != ORACLE_QF64 && elem_type != ORACLE_QBF16))
        return -1;
    if (signs != NULL && (d & (d - 1)) != 0) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    double *H = NULL;
    if (signs != NULL) {
        for (int64_t t = 0; t < d; ++t)
            if (signs[t] != 1 && signs[t] != -1) return -1;
        H = (double *)malloc((size_t)(d * d) * sizeof(double));
        if (H == NULL) return -2;
        oracle_hadamard(d, H);
    }
    double *y = (double *)malloc((size_t)(N * d > 0 ? N * d : 1) * sizeof(double));
    if (y == NULL) {
        free(H);
        return -2;
    }
    for (int64_t s = 0; s < S; ++s) {
        const int64_t base = s * N * d;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < N; ++i) {
            for (int64_t j = 0; j < d; ++j) {
                if (H == NULL) {
                    y[i * d + j] = load_x(x, elem_type, base + i * d + j);
                } else {
                    double acc = 0.0;
                    for (int64_t t = 0; t < d; ++t)
                        acc += load_x(x, elem_type, base + i * d + t) * (double)signs[t] *
                               H[t * d + j];
                    y[i * d + j] = acc / sqrt((double)d);
                }
            }
        }
        double amax = 0.0;
        for (int64_t e = 0; e < N * d; ++e)
            if (fabs(y[e]) > amax) amax = fabs(y[e]);
        if (descale != NULL) descale[s] = amax > 0.0 ? amax / E4M3_MAX_FINITE : 1.0;
        if (codes != NULL) {
#pragma omp parallel for schedule(static)
            for (int64_t e = 0; e < N * d; ++e)
                codes[base + e] = amax > 0.0 ? oracle_encode_e4m3(y[e] * E4M3_MAX_FINITE / amax)
                                             : 0;
        }
        if (y_out != NULL) memcpy(y_out + base, y, (size_t)(N * d) * sizeof(double));
    }
    free(y);
    free(H);
    return 0;
}
