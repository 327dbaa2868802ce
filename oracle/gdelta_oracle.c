/*
 * gdelta_oracle.c -- plain, slow fp64 CPU oracle for the recurrent memory
 * channel of ATMA: a gated-delta associative memory read and written token by
 * token.
 *
 * TEST INFRASTRUCTURE, like polar_oracle.c (compiled into the same library):
 * only the test-suite, the smoke check and the bench's CPU-baseline leg load
 * it; it shares nothing with the CUDA library.
 *
 * Source: "ATMA: Length-Invariant Language Modeling via Polar Attention and
 * Gated-Delta Compression Memory" (gist.science technical summary, section 2.1
 * "Recurrent Memory Channel": an additive third stream driven by a gated-delta
 * Titans-style memory, with L2-normalised keys and queries as the stability
 * mechanism; section 2.2 "In-Place Gated-Delta Step Kernel"; the v3 abstract
 * says the channel derives from Gated DeltaNet).  The pages name the rule but
 * print no formula; the reading taken is the published gated delta rule
 * (Yang, Kautz, Hatamizadeh, "Gated Delta Networks", ICLR 2025):
 *
 * Per (sequence, head), state S (Dv x Dk, starts at the given S_0), token t:
 *
 *   qh = q_t / |q_t| ,  kh = k_t / |k_t|     (a zero row stays zero)
 *   S_t = alpha_t * S_{t-1} * (I - beta_t kh kh^T) + beta_t v_t kh^T
 *   o_t = S_t qh                              (read after the write)
 *
 * alpha_t in [0, 1] is the decay gate and beta_t in [0, 1] the write strength,
 * one of each per (token, head), given as inputs.  The memory output o_t is
 * the third additive stream: out = content + count + memory.
 *
 * Two evaluation orders (both fp64):
 *   literal = 1: the definition above as written: M = I - beta kh kh^T
 *                materialised, S <- alpha (S M) + beta v kh^T by an explicit
 *                Dv x Dk x Dk product (O(D^3) a token, small cases only);
 *   literal = 0: the same update expanded as a rank-one correction,
 *                S[r][c] <- alpha S[r][c] + beta (v[r] - alpha (S kh)[r]) kh[c]
 *                (O(D^2) a token), for full-length sequences.
 *
 * ORACLE_MUTANT 13-17 plant mistakes that the memory pins must catch.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

typedef struct {
    int B, T, H, D; /* sequences, tokens, memory heads, head dim (Dk = Dv = D) */
} gdelta_cfg;

static inline double gd_ld(const void *p, int dtype, int64_t idx) {
    if (dtype == 0) return (double)((const float *)p)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* x / |x| for one row; a zero row stays zero. */
static void gd_unit(const void *src, int dtype, int64_t off, int D, double *dst) {
    double ss = 0.0;
    for (int d = 0; d < D; ++d) {
        dst[d] = gd_ld(src, dtype, off + d);
        ss += dst[d] * dst[d];
    }
#if ORACLE_MUTANT == 14
    (void)ss; /* mistake: the stability normalisation is skipped */
#else
    const double inv = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;
    for (int d = 0; d < D; ++d) dst[d] *= inv;
#endif
}

/*
 * q, k, v   [B, T, H, D] (dtype 0 fp32, 1 bf16 bits)
 * alpha     [B, T, H] fp64 (the exact fp32 inputs, widened)
 * beta      [B, T, H] fp64
 * state     [B, H, D, D] fp64, row r = value dim, column c = key dim: S_0 in,
 *           the state after the last token out
 * out       [B, T, H, D] fp64, o_t
 */
int oracle_gdelta(const gdelta_cfg *cfg, const void *q, const void *k, const void *v, int dtype,
                  const double *alpha, const double *beta, double *state, double *out,
                  int literal) {
    if (!cfg || cfg->B < 0 || cfg->T < 0 || cfg->H <= 0 || cfg->D <= 0) return -1;
    const int B = cfg->B, T = cfg->T, H = cfg->H, D = cfg->D;
    int rc = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *S = state + ((int64_t)b * H + h) * D * D;
            double *qh = malloc(sizeof(double) * D), *kh = malloc(sizeof(double) * D);
            double *vt = malloc(sizeof(double) * D), *Sk = malloc(sizeof(double) * D);
            double *M = literal ? malloc(sizeof(double) * D * D) : NULL;
            double *SM = literal ? malloc(sizeof(double) * D * D) : NULL;
            if (!qh || !kh || !vt || !Sk || (literal && (!M || !SM))) {
#pragma omp atomic write
                rc = -3;
                free(qh); free(kh); free(vt); free(Sk); free(M); free(SM);
                continue;
            }
            for (int t = 0; t < T; ++t) {
                const int64_t row = ((int64_t)b * T + t) * H + h;
                gd_unit(q, dtype, row * D, D, qh);
                gd_unit(k, dtype, row * D, D, kh);
                for (int d = 0; d < D; ++d) vt[d] = gd_ld(v, dtype, row * D + d);
                const double a = alpha[row], be = beta[row];
                double *o = out + row * D;
#if ORACLE_MUTANT == 15
                /* mistake: the readout takes the state before this token's write */
                for (int r = 0; r < D; ++r) {
                    double acc = 0.0;
                    for (int c = 0; c < D; ++c) acc += S[r * D + c] * qh[c];
                    o[r] = acc;
                }
#endif
                if (literal) {
                    for (int i = 0; i < D; ++i)
                        for (int j = 0; j < D; ++j)
                            M[i * D + j] = (i == j ? 1.0 : 0.0) - be * kh[i] * kh[j];
                    for (int r = 0; r < D; ++r)
                        for (int c = 0; c < D; ++c) {
                            double acc = 0.0;
#if ORACLE_MUTANT == 16
                            /* mistake: the operands of the product swapped, M S */
                            for (int i = 0; i < D; ++i) acc += M[r * D + i] * S[i * D + c];
#else
                            for (int i = 0; i < D; ++i) acc += S[r * D + i] * M[i * D + c];
#endif
                            SM[r * D + c] = acc;
                        }
                    for (int r = 0; r < D; ++r)
                        for (int c = 0; c < D; ++c)
                            S[r * D + c] = a * SM[r * D + c] + be * vt[r] * kh[c];
                } else {
                    for (int r = 0; r < D; ++r) {
                        double acc = 0.0;
                        for (int c = 0; c < D; ++c) acc += S[r * D + c] * kh[c];
                        Sk[r] = acc;
                    }
                    for (int r = 0; r < D; ++r) {
#if ORACLE_MUTANT == 13
                        /* mistake: the decay gate left off the erase term */
                        const double w = be * (vt[r] - Sk[r]);
#else
                        const double w = be * (vt[r] - a * Sk[r]);
#endif
                        for (int c = 0; c < D; ++c) S[r * D + c] = a * S[r * D + c] + w * kh[c];
                    }
                }
#if ORACLE_MUTANT != 15
                for (int r = 0; r < D; ++r) {
                    double acc = 0.0;
#if ORACLE_MUTANT == 17
                    /* mistake: the read takes the transposed state, S^T q */
                    for (int c = 0; c < D; ++c) acc += S[c * D + r] * qh[c];
#else
                    for (int c = 0; c < D; ++c) acc += S[r * D + c] * qh[c];
#endif
                    o[r] = acc;
                }
#endif
            }
            free(qh); free(kh); free(vt); free(Sk); free(M); free(SM);
        }
    }
    return rc;
}
