/*
 * dropout_oracle.c -- fp64 CPU oracle for attention with dropout on the attention weights.
 * TEST INFRASTRUCTURE: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark load this code.  It shares nothing with the CUDA library.
 *
 * The page "Flash Attention" (section "Zentrale technische Innovationen", the fusion
 * bullet) lists dropout among the operations fused with the softmax into one kernel.
 * Computed here, per query row i of (batch, query head) bh, over the admissible keys j:
 *
 *   p_j    = exp(s_j - m),  l = sum_j p_j            (s_j = scale * q_i . k_j)
 *   keep_j = 1 if byte_j >= thr else 0               (thr = dropout threshold, 0 .. 255)
 *   O      = sum_j p_j keep_j v_j / (l * (1 - thr/256))
 *   LSE    = m + ln l                                 (dropout does not change it)
 *
 * so that E[O] over the random bytes is the attention without dropout.  byte_j is byte
 * (j mod 32) -- little-endian within the four 64-bit words -- of the Philox4x64-10 block
 * (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11)
 * for counter (j / 32, i, bh, 0) and key (seed, offset): one block serves 32 consecutive
 * keys of one row.  The keep probability is 1 - thr/256.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

double oracle_decode_bf16(uint16_t h);

/* Philox4x64-10: ten rounds of two 64x64->128-bit products, the key bumped by the Weyl
 * increments after each round. */
void oracle_philox4x64(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
    const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
    uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        const unsigned __int128 p0 = (unsigned __int128)M0 * c0;
        const unsigned __int128 p1 = (unsigned __int128)M1 * c2;
        const uint64_t hi0 = (uint64_t)(p0 >> 64), lo0 = (uint64_t)p0;
        const uint64_t hi1 = (uint64_t)(p1 >> 64), lo1 = (uint64_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += W0;
        k1 += W1;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* The random byte deciding whether key j of row i of (batch, head) bh is kept. */
uint8_t oracle_dropout_byte(uint64_t seed, uint64_t offset, int64_t bh, int64_t i, int64_t j) {
    const uint64_t ctr[4] = {(uint64_t)(j >> 5), (uint64_t)i, (uint64_t)bh, 0};
    const uint64_t key[2] = {seed, offset};
    uint64_t o[4];
    oracle_philox4x64(ctr, key, o);
    const int t = (int)(j & 31);
    return (uint8_t)(o[t >> 3] >> (8 * (t & 7)));
}

static double ld(const void *p, int bf16, int64_t i) {
    return bf16 ? oracle_decode_bf16(((const uint16_t *)p)[i]) : ((const double *)p)[i];
}

/*
 * Attention with dropout for selected query rows (layout and rows as in
 * oracle_attention_rows; inputs fp64 (bf16 = 0) or bf16 bits (bf16 = 1)).  Causal masking
 * admits key j for query i iff j <= i + (Nk - Nq); a row with no admissible key gets O = 0
 * and LSE = -inf.  Returns 0, -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_attention_dropout_rows(const void *q, const void *k, const void *v, int bf16,
                                  int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk,
                                  int64_t d, double scale, int causal, int thr, uint64_t seed,
                                  uint64_t offset, const int64_t *rows, int64_t nrows,
                                  double *o_out, double *lse_out, int nthreads) {
    if (!q || !k || !v || !o_out || !lse_out) return -1;
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || d < 1 || Hq % Hkv != 0) return -1;
    if (thr < 0 || thr > 255) return -1;
    const int64_t total = B * Hq * Nq;
    if (rows == NULL) nrows = total;
    for (int64_t r = 0; rows && r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return -1;
    const int64_t group = Hq / Hkv;
    const double keep_scale = 1.0 / (1.0 - thr / 256.0);
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        if (!s || !acc) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < nrows; ++r) {
                const int64_t flat = rows ? rows[r] : r;
                const int64_t i = flat % Nq, bh = flat / Nq;
                const int64_t b = bh / Hq, hq = bh % Hq;
                const int64_t bhk = b * Hkv + hq / group;
                const int64_t qoff = (bh * Nq + i) * d, kvoff = bhk * Nk * d;
                int64_t n_adm = Nk; /* admissible keys, bottom-right causal */
                if (causal && i + 1 + (Nk - Nq) < n_adm) n_adm = i + 1 + (Nk - Nq);
                if (n_adm <= 0) {
                    for (int64_t t = 0; t < d; ++t) o_out[r * d + t] = 0.0;
                    lse_out[r] = -INFINITY;
                    continue;
                }
                double row_max = -INFINITY;
                for (int64_t j = 0; j < n_adm; ++j) {
                    double dot = 0.0;
                    for (int64_t t = 0; t < d; ++t)
                        dot += ld(q, bf16, qoff + t) * ld(k, bf16, kvoff + j * d + t);
                    s[j] = scale * dot;
                    if (s[j] > row_max) row_max = s[j];
                }
                double row_sum = 0.0;
                for (int64_t t = 0; t < d; ++t) acc[t] = 0.0;
                for (int64_t j = 0; j < n_adm; ++j) {
                    const double p = exp(s[j] - row_max);
                    row_sum += p;
                    if (oracle_dropout_byte(seed, offset, bh, i, j) >= thr)
                        for (int64_t t = 0; t < d; ++t) acc[t] += p * ld(v, bf16, kvoff + j * d + t);
                }
                for (int64_t t = 0; t < d; ++t) o_out[r * d + t] = acc[t] * keep_scale / row_sum;
                lse_out[r] = row_max + log(row_sum);
            }
        }
        free(s);
        free(acc);
    }
    return failed ? -2 : 0;
}
