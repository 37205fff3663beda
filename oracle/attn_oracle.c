/*
 * Plain fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is called by tests/, by the smoke check in
 * __graft_entry__.py and by the CPU-baseline leg of bench.py.  The product path (the
 * CUDA library under exact_attention_101_b200/) never links, loads or calls it, and it
 * shares no code with that path.
 *
 * What it computes (one query row at a time, the score row S[i,:] materialised in full):
 *
 *   s_ij  = scale * sum_t q[i,t] * k[j,t]                       j admissible
 *   m_i   = max_j s_ij
 *   p_ij  = exp(s_ij - m_i)
 *   l_i   = sum_j p_ij
 *   O[i,:] = (sum_j p_ij * v[j,:]) / l_i
 *   LSE_i = m_i + ln(l_i)          (= ln sum_j exp(s_ij), natural log)
 *
 * This is the attention formula softmax(Q K^T / sqrt(d_k)) V of the page
 * "FlashAttention (DE)", section "Problematik der Standard-Attention", with the scale
 * passed explicitly and the usual max subtraction, which leaves softmax unchanged.
 * The same pages stress that FlashAttention returns exactly this result, not an
 * approximation ("Flash Attention" page, section "Zentrale technische Innovationen",
 * the bullet on exact computation), so the plain definition is the oracle.
 *
 * Causal masking ("Flash Attention" page, section "Zentrale technische Innovationen",
 * the bullet on autoregressive models): key j is admissible for query i iff
 * j <= i + (Nk - Nq).  With Nq == Nk that is j <= i.  With Nq != Nk the pages say nothing;
 * the queries are read as the last Nq positions of a sequence of Nk keys (bottom-right
 * alignment: each query sees every key up to its own position).  A query with no
 * admissible key (Nq > Nk) gets O = 0 and LSE = ln(empty sum) = -inf.
 *
 * Grouped/multi-query heads ("Flash Attention" page, same section, the MQA/GQA bullet; page
 * "FlashAttention 4: Praxisleitfaden ...", section "Kompatibilitaet und aktueller
 * Stand", which describes several query heads sharing one K/V projection): query
 * head hq reads K/V head hq / (Hq / Hkv).
 *
 * Inputs are decoded from their storage format to double here (bf16: the 16 high bits of
 * an IEEE binary32; e4m3: OCP 8-bit floating point E4M3, bias 7, no infinities, NaN =
 * S.1111.111), and e4m3 values are multiplied by a per-(batch, head) descale.  All
 * arithmetic after decoding is IEEE binary64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F64 = 0, ORACLE_BF16 = 1, ORACLE_E4M3 = 2 };

/* bf16 -> double: the bf16 bits are the upper half of a binary32. */
double oracle_decode_bf16(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP E4M3 -> double.  sign s, exponent e (4 bits, bias 7), mantissa m (3 bits).
 * e == 0: subnormal, value m/8 * 2^(1-7).  e == 15 && m == 7: NaN.  Otherwise
 * (1 + m/8) * 2^(e-7).  The largest finite magnitude is 1.75 * 2^8 = 448. */
double oracle_decode_e4m3(uint8_t c) {
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, 1 - 7);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

static double load_elem(const void *base, int elem_type, int64_t idx) {
    switch (elem_type) {
    case ORACLE_F64:
        return ((const double *)base)[idx];
    case ORACLE_BF16:
        return oracle_decode_bf16(((const uint16_t *)base)[idx]);
    default:
        return oracle_decode_e4m3(((const uint8_t *)base)[idx]);
    }
}

/*
 * Compute attention for a list of query rows.
 *
 * Layout: q, o are [B, Hq, Nq, d]; k, v are [B, Hkv, Nk, d]; lse is [B, Hq, Nq]; all
 * contiguous, row-major.  rows[r] is a flattened query-row index (b*Hq + hq)*Nq + i;
 * when rows == NULL all B*Hq*Nq rows are computed in order.  Outputs: o_out[r*d + t]
 * and lse_out[r] for the r-th requested row.
 *
 * descale_q / descale_k / descale_v: per-(batch, head) multipliers applied after
 * decoding ([B*Hq], [B*Hkv], [B*Hkv]); pass NULL for 1.0.
 *
 * Returns 0 on success, -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_attention_rows(const void *q, const void *k, const void *v, int elem_type,
                          const double *descale_q, const double *descale_k,
                          const double *descale_v, int64_t B, int64_t Hq, int64_t Hkv,
                          int64_t Nq, int64_t Nk, int64_t d, double scale, int causal,
                          const int64_t *rows, int64_t nrows, double *o_out, double *lse_out,
                          int nthreads) {
    if (!q || !k || !v || !o_out || !lse_out) return -1;
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || d < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    if (elem_type < ORACLE_F64 || elem_type > ORACLE_E4M3) return -1;
    const int64_t total_rows = B * Hq * Nq;
    if (rows == NULL) nrows = total_rows;
    if (nrows < 0) return -1;
    for (int64_t r = 0; rows && r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= total_rows) return -1;
    const int64_t group = Hq / Hkv;
    int failed = 0;

#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel
    {
        double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
        double *srow = (double *)malloc(sizeof(double) * (size_t)Nk);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        if (!qrow || !srow || !acc) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < nrows; ++r) {
                const int64_t flat = rows ? rows[r] : r;
                const int64_t i = flat % Nq;
                const int64_t bh = flat / Nq;   /* b*Hq + hq */
                const int64_t b = bh / Hq;
                const int64_t hq = bh % Hq;
                const int64_t hk = hq / group;
                const int64_t bhk = b * Hkv + hk;
                const double dq = descale_q ? descale_q[bh] : 1.0;
                const double dk = descale_k ? descale_k[bhk] : 1.0;
                const double dv = descale_v ? descale_v[bhk] : 1.0;
                const int64_t qoff = (bh * Nq + i) * d;
                const int64_t kvoff = bhk * Nk * d;
                for (int64_t t = 0; t < d; ++t) qrow[t] = load_elem(q, elem_type, qoff + t) * dq;

                /* Admissible keys: all of them, or j <= i + (Nk - Nq) under the causal
                 * mask. */
                int64_t nkeys = Nk;
                if (causal && i + 1 + (Nk - Nq) < nkeys) nkeys = i + 1 + (Nk - Nq);
                if (nkeys <= 0) {
                    for (int64_t t = 0; t < d; ++t) o_out[r * d + t] = 0.0;
                    lse_out[r] = -INFINITY;
                    continue;
                }

                /* Row i of S, materialised. */
                double m = -INFINITY;
                for (int64_t j = 0; j < nkeys; ++j) {
                    double dot = 0.0;
                    for (int64_t t = 0; t < d; ++t)
                        dot += qrow[t] * (load_elem(k, elem_type, kvoff + j * d + t) * dk);
                    srow[j] = scale * dot;
                    if (srow[j] > m) m = srow[j];
                }
                /* Softmax numerators, their sum, and the weighted sum of value rows. */
                double l = 0.0;
                for (int64_t t = 0; t < d; ++t) acc[t] = 0.0;
                for (int64_t j = 0; j < nkeys; ++j) {
                    const double p = exp(srow[j] - m);
                    l += p;
                    for (int64_t t = 0; t < d; ++t)
                        acc[t] += p * (load_elem(v, elem_type, kvoff + j * d + t) * dv);
                }
                for (int64_t t = 0; t < d; ++t) o_out[r * d + t] = acc[t] / l;
                lse_out[r] = m + log(l);
            }
        }
        free(qrow);
        free(srow);
        free(acc);
    }
    return failed ? -2 : 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
