/*
 * bwd_oracle.c -- fp64 CPU oracle for the gradients of exact attention.
 * TEST INFRASTRUCTURE: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark load this code.  It shares nothing with the CUDA library.
 *
 * The pages say that FlashAttention does not store the attention matrix for the
 * backward pass but computes it again ("Flash Attention" page, section "Zentrale
 * technische Innovationen", the bullet on recomputation, and its overview).  What the
 * backward pass computes is fixed by calculus: for O = P V with P = softmax(S) taken row
 * by row, S = scale * Q K^T over the admissible keys (j <= i + Nk - Nq under the causal
 * mask, aligned at the bottom right as in the forward oracle), and an upstream gradient dO,
 *
 *   dV     = P^T dO
 *   dP     = dO V^T
 *   dS_ij  = P_ij (dP_ij - sum_k P_ik dP_ik)       (the Jacobian of a row softmax)
 *   dQ     = scale * dS K
 *   dK     = scale * dS^T Q
 *
 * With grouped heads (query head hq reads K/V head hq / (Hq / Hkv)), the dK and dV of a
 * K/V head are the sums over the query heads that read it.  A query row without any
 * admissible key (causal, Nq > Nk) has the constant output O = 0, so its dQ row is zero
 * and it adds nothing to dK and dV.
 *
 * Evaluation, per (batch, K/V head) and all binary64: first the query rows (score row,
 * its maximum and sum, P row, dP row, the row term sum_k P_ik dP_ik, dQ row), keeping each
 * row's log-sum-exp and row term; then the key rows (dV and dK rows from the recomputed
 * column of P and dP).  Inputs are fp64 or bf16 bits.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

double oracle_decode_bf16(uint16_t h);

#define BWD_F64 0
#define BWD_BF16 1

static double ld(const void *p, int et, int64_t i) {
    return et == BWD_BF16 ? oracle_decode_bf16(((const uint16_t *)p)[i]) : ((const double *)p)[i];
}

static double dot_rows(const void *a, int64_t ia, const void *b, int64_t ib, int et, int64_t d) {
    double s = 0.0;
    for (int64_t t = 0; t < d; ++t) s += ld(a, et, ia + t) * ld(b, et, ib + t);
    return s;
}

/*
 * q, dout: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]; all of one element type.
 * Outputs dq [B, Hq, Nq, d], dk and dv [B, Hkv, Nk, d] in fp64.
 * Returns 0, -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_attention_bwd(const void *q, const void *k, const void *v, const void *dout,
                         int elem_type, int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                         int64_t Nk, int64_t d, double scale, int causal, double *dq,
                         double *dk, double *dv, int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || d < 1 || Hq % Hkv != 0) return -1;
    if (elem_type != BWD_F64 && elem_type != BWD_BF16) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int64_t group = Hq / Hkv;
    double *lse = (double *)malloc(sizeof(double) * (size_t)(group * Nq));
    double *rowterm = (double *)malloc(sizeof(double) * (size_t)(group * Nq));
    if (!lse || !rowterm) {
        free(lse);
        free(rowterm);
        return -2;
    }
    int failed = 0;
    for (int64_t b = 0; b < B && !failed; ++b)
        for (int64_t hk = 0; hk < Hkv && !failed; ++hk) {
            const int64_t kvoff = (b * Hkv + hk) * Nk * d;
            /* query rows of every query head that reads this K/V head */
#pragma omp parallel
            {
                double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
                double *dp = (double *)malloc(sizeof(double) * (size_t)Nk);
                if (!s || !dp) {
#pragma omp atomic write
                    failed = 1;
                } else {
#pragma omp for schedule(dynamic, 4)
                    for (int64_t gi = 0; gi < group * Nq; ++gi) {
                        const int64_t hq = hk * group + gi / Nq, i = gi % Nq;
                        const int64_t qoff = ((b * Hq + hq) * Nq + i) * d;
                        const int64_t last = i + (Nk - Nq); /* last key the mask admits */
                        const int64_t nkeys = !causal ? Nk : (last < Nk ? last + 1 : Nk);
                        if (nkeys <= 0) {
                            for (int64_t t = 0; t < d; ++t) dq[qoff + t] = 0.0;
                            lse[gi] = -INFINITY;
                            rowterm[gi] = 0.0;
                            continue;
                        }
                        double m = -INFINITY;
                        for (int64_t j = 0; j < nkeys; ++j) {
                            s[j] = scale * dot_rows(q, qoff, k, kvoff + j * d, elem_type, d);
                            if (s[j] > m) m = s[j];
                        }
                        double l = 0.0;
                        for (int64_t j = 0; j < nkeys; ++j) l += exp(s[j] - m);
                        double term = 0.0;
                        for (int64_t j = 0; j < nkeys; ++j) {
                            s[j] = exp(s[j] - m) / l;                      /* P_ij */
                            dp[j] = dot_rows(dout, qoff, v, kvoff + j * d, elem_type, d);
                            term += s[j] * dp[j];
                        }
                        lse[gi] = m + log(l);
                        rowterm[gi] = term;
                        for (int64_t t = 0; t < d; ++t) {
                            double acc = 0.0;
                            for (int64_t j = 0; j < nkeys; ++j)
                                acc += s[j] * (dp[j] - term) * ld(k, elem_type, kvoff + j * d + t);
                            dq[qoff + t] = scale * acc;
                        }
                    }
                }
                free(s);
                free(dp);
            }
            if (failed) break;
            /* key rows: dV_j = sum_i P_ij dO_i, dK_j = scale sum_i dS_ij q_i */
#pragma omp parallel for schedule(dynamic, 4)
            for (int64_t j = 0; j < Nk; ++j) {
                double *dvr = dv + kvoff + j * d, *dkr = dk + kvoff + j * d;
                for (int64_t t = 0; t < d; ++t) dvr[t] = dkr[t] = 0.0;
                for (int64_t gi = 0; gi < group * Nq; ++gi) {
                    const int64_t hq = hk * group + gi / Nq, i = gi % Nq;
                    if (causal && j > i + (Nk - Nq)) continue;
                    const int64_t qoff = ((b * Hq + hq) * Nq + i) * d;
                    const double sij = scale * dot_rows(q, qoff, k, kvoff + j * d, elem_type, d);
                    const double p = exp(sij - lse[gi]);
                    const double dpij = dot_rows(dout, qoff, v, kvoff + j * d, elem_type, d);
                    const double ds = p * (dpij - rowterm[gi]);
                    for (int64_t t = 0; t < d; ++t) {
                        dvr[t] += p * ld(dout, elem_type, qoff + t);
                        dkr[t] += scale * ds * ld(q, elem_type, qoff + t);
                    }
                }
            }
        }
    free(lse);
    free(rowterm);
    return failed ? -2 : 0;
}
