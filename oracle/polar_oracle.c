/*
 * polar_oracle.c -- plain, slow fp64 CPU oracle for the causal Polar Attention
 * mixing step (prefill) and its GQA-grouped paged-KV decode variant.
 *
 * TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the bench's
 * CPU-baseline leg load this library.  It shares no code, header, table or
 * helper with the CUDA library, and the CUDA library never calls it.
 *
 * Source: "ATMA: Length-Invariant Language Modeling via Polar Attention and
 * Gated-Delta Compression Memory" (H. Akbar, arXiv 2606.25156), as summarised
 * on gist.science ("Technical Summary", section 2.1 "Polar Attention: A
 * Three-Channel Decomposition" and section 2.2 "Hardware-Software Codesign"),
 * and the v3 abstract.  The pages give the method in words only; the explicit
 * parametric forms below are the ones the project specification fixes, and the
 * readings where the pages are silent are listed next to each step.
 *
 * Per query row (batch b, query head h, row i) with visible keys j in [0, n):
 *
 *   g     = h / (Hq / Hkv)             GQA: contiguous groups of query heads
 *                                      share one key/value head ("GQA-Grouped
 *                                      Paged Decode Kernel", section 2.2).
 *   n     = i + 1 (causal prefill)     reading: the length in the length
 *           | T (non-causal)           temperature is the number of keys the
 *           | seqlen (decode)          row can see, so row i never depends on
 *                                      the future.
 *   window W > 0 (sliding window, the ablation the results section names):
 *                                      the visible keys are the last W of
 *                                      those, j in [i - W + 1, i] (prefill) or
 *                                      [seqlen - W, seqlen) (decode), and n is
 *                                      their count, min(i + 1, W) / min(seqlen,
 *                                      W); every statistic below runs over
 *                                      that range.
 *   tau   = 1 + alpha*ln(n/L)  if n > L, else 1     length temperature,
 *                                      "sharpen distributions as context
 *                                      grows" (section 2.1, direction channel).
 *   c     = s * tau ;  z_j = c * <q_i, k_j>          logits.
 *   m     = max_j z_j
 *   mu    = mean_j z_j ; sigma = population std of z_j
 *   z0    = mu + sigma*sqrt(2 ln n)    extreme-value-corrected null floor: the
 *                                      expected maximum of n noise logits; it
 *                                      is an extra logit with a zero value
 *                                      vector (section 2.1).
 *   w_j   = exp(z_j - m) ; l = sum w ; l2 = sum w^2 ; acc = sum w_j v_j
 *   n_eff = l^2 / l2                   participation ratio / inverse Simpson
 *                                      index of p_j = w_j / l (section 2.1,
 *                                      magnitude channel).  Reading: the null
 *                                      slot is not part of n_eff (with a zero
 *                                      value it cannot move the direction, and
 *                                      including it would break "uniform
 *                                      logits give n_eff = n").
 *   content = acc / max(|acc|, 1e-30)  direction channel: the matched value
 *                                      sum projected onto the unit sphere.
 *   gate  = 1 / (1 + exp(-beta*(m - z0)))   "gated by the confidence of signal
 *                                      detection" (section 2.1).
 *   count = gate * tanh(ln(n_eff) / ln(L)) * u_h    "bounded, saturating
 *                                      monotonic function (tanh of log)".
 *   out   = content + count            the first two channels; the memory
 *                                      stream's oracle is gdelta_oracle.c.
 *
 * Modes (all fp64; inputs are the exact fp32 values or the exact bf16 bits
 * widened to fp64):
 *   0  two-pass definition (the formulas above, in that order);
 *   1  brute force: materialise the softmax p_j = e^{z_j} / sum e^{z} without a
 *      max shift, n_eff = 1 / sum p_j^2 -- an independent route to the same
 *      numbers, used only to pin modes 0 and 2 on small inputs;
 *   2  streaming: keys in blocks of `block`, running max, l and l2 rescaled on
 *      a max update by r and r^2 ("streaming accumulators and squared
 *      correction factors", section 2.2, fused Polar Attention kernel), one-pass
 *      sums S1 = sum <q,k>, S2 = sum <q,k>^2 for the null floor, and an
 *      optional lazy threshold theta (rescale only when a block max exceeds
 *      the reference max by more than theta, natural-log units).
 *
 * ORACLE_MUTANT (compile-time, default 0) plants one deliberate mistake; the
 * test-suite builds mutants to prove that its pins catch each of them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

#define ORACLE_PAGE 64 /* tokens per KV page */

typedef struct {
    int B, T, Hq, Hkv, D;
    double s;      /* logit scale */
    double alpha;  /* length-temperature coefficient */
    int L;         /* training length L_train */
    double beta;   /* gate slope */
    int causal;    /* prefill: 1 = row i sees keys 0..i */
    int window;    /* 0: all of them; W > 0: only the last W visible keys */
} oracle_cfg;

/* ---- input decoding (not method arithmetic) ------------------------------ */

static inline double ld(const void *p, int dtype, int64_t idx) {
    if (dtype == 0) return (double)((const float *)p)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Where key/value row j of one (sequence, kv head) lives. */
typedef struct {
    const void *kbase, *vbase; /* dense: k and v tensors; paged: the pool */
    int dtype, D, Hkv, g;
    int paged;
    int64_t dense_off;    /* dense: element offset of (b, j=0, g, d=0) */
    int64_t dense_stride; /* dense: elements between consecutive j */
    const int32_t *pt;    /* paged: page-table row of this sequence */
    int64_t j0;           /* position of the first visible key (row index j = 0) */
} key_src;

static inline int64_t kv_off(const key_src *ks, int64_t j, int which) {
    j += ks->j0;
    if (!ks->paged) return ks->dense_off + j * ks->dense_stride;
    int64_t page = ks->pt[j / ORACLE_PAGE];
#if ORACLE_MUTANT == 20
    which = 1 - which; /* mistake: the page's key and value planes swapped */
#endif
    return (((page * 2 + which) * ks->Hkv + ks->g) * ORACLE_PAGE + (j % ORACLE_PAGE)) * ks->D;
}

static inline double key_el(const key_src *ks, int64_t j, int d) {
    return ld(ks->kbase, ks->dtype, kv_off(ks, j, 0) + d);
}
static inline double val_el(const key_src *ks, int64_t j, int d) {
    return ld(ks->paged ? ks->kbase : ks->vbase, ks->dtype, kv_off(ks, j, 1) + d);
}

static double qk_dot(const double *q, const key_src *ks, int64_t j) {
    double acc = 0.0;
    for (int d = 0; d < ks->D; ++d) acc += q[d] * key_el(ks, j, d);
    return acc;
}

/* ---- the pieces every mode shares ---------------------------------------- */

/* Length temperature: tau = 1 + alpha*ln(n/L) for n > L, else 1. */
static double length_temperature(int64_t n, const oracle_cfg *cfg) {
#if ORACLE_MUTANT == 7
    if (n > cfg->L) return 1.0 + cfg->alpha * log2((double)n / cfg->L);
#else
    if (n > cfg->L) return 1.0 + cfg->alpha * log((double)n / cfg->L);
#endif
    return 1.0;
}

/* Null floor z0 = mu + sigma*sqrt(2 ln n). */
static double null_floor(double mu, double sigma, int64_t n) {
#if ORACLE_MUTANT == 8
    return mu + sigma * sqrt(log((double)n));
#else
    return mu + sigma * sqrt(2.0 * log((double)n));
#endif
}

/* Gate = sigmoid(beta*(m - z0)). */
static double confidence_gate(double m, double z0, double beta) {
#if ORACLE_MUTANT == 3
    return 1.0 / (1.0 + exp(-beta * (z0 - m)));
#else
    return 1.0 / (1.0 + exp(-beta * (m - z0)));
#endif
}

/* out = content + gate*tanh(ln n_eff / ln L)*u_h, content = acc/|acc|. */
static void emit(const double *acc, int D, double neff, double gate, const float *u_h, int L,
                 double *out) {
    double nrm = 0.0;
    for (int d = 0; d < D; ++d) nrm += acc[d] * acc[d];
    nrm = sqrt(nrm);
    if (nrm < 1e-30) nrm = 1e-30;
#if ORACLE_MUTANT == 9
    nrm = 1.0;
#endif
    double mag = gate * tanh(log(neff) / log((double)L));
    for (int d = 0; d < D; ++d) out[d] = acc[d] / nrm + mag * (double)u_h[d];
}

/* ---- mode 0: the two-pass definition ------------------------------------- */

static void row_two_pass(const double *q, const key_src *ks, int64_t n, const oracle_cfg *cfg,
                         const float *u_h, double *zbuf, double *out, double *neff_out,
                         double *st) {
    const int D = ks->D;
    const double c = cfg->s * length_temperature(n, cfg);
    double m = -INFINITY, sum = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        zbuf[j] = c * qk_dot(q, ks, j);
        if (zbuf[j] > m) m = zbuf[j];
        sum += zbuf[j];
    }
    double mu = sum / (double)n, var = 0.0;
    for (int64_t j = 0; j < n; ++j) var += (zbuf[j] - mu) * (zbuf[j] - mu);
#if ORACLE_MUTANT == 6
    double sigma = n > 1 ? sqrt(var / (double)(n - 1)) : 0.0;
#else
    double sigma = sqrt(var / (double)n);
#endif
    double z0 = null_floor(mu, sigma, n);

    double l = 0.0, l2 = 0.0, acc[256];
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double w = exp(zbuf[j] - m);
        l += w;
        l2 += w * w;
        for (int d = 0; d < D; ++d) acc[d] += w * val_el(ks, j, d);
    }
#if ORACLE_MUTANT == 2
    double neff = l / l2;
#else
    double neff = l * l / l2;
#endif
    double gate = confidence_gate(m, z0, cfg->beta);
    emit(acc, D, neff, gate, u_h, cfg->L, out);
    *neff_out = neff;
    if (st) {
        st[0] = m; st[1] = mu; st[2] = sigma; st[3] = z0;
        st[4] = gate; st[5] = l; st[6] = l2; st[7] = c;
    }
}

/* ---- mode 1: brute force (materialised softmax) --------------------------- */

static void row_brute(const double *q, const key_src *ks, int64_t n, const oracle_cfg *cfg,
                      const float *u_h, double *zbuf, double *out, double *neff_out, double *st) {
    const int D = ks->D;
    const double c = cfg->s * length_temperature(n, cfg);
    for (int64_t j = 0; j < n; ++j) zbuf[j] = c * qk_dot(q, ks, j);
    double Z = 0.0, m = -INFINITY, mu = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        Z += exp(zbuf[j]);
        m = zbuf[j] > m ? zbuf[j] : m;
        mu += zbuf[j];
    }
    mu /= (double)n;
    double sumsq = 0.0, var = 0.0, acc[256];
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double p = exp(zbuf[j]) / Z;
        sumsq += p * p;
        var += (zbuf[j] - mu) * (zbuf[j] - mu) / (double)n;
        for (int d = 0; d < D; ++d) acc[d] += p * val_el(ks, j, d);
    }
    double sigma = sqrt(var);
    double z0 = null_floor(mu, sigma, n);
    double neff = 1.0 / sumsq;
    double gate = confidence_gate(m, z0, cfg->beta);
    emit(acc, D, neff, gate, u_h, cfg->L, out);
    *neff_out = neff;
    if (st) {
        /* l and l2 relative to the true max, for comparison with mode 0 */
        double em = exp(m);
        st[0] = m; st[1] = mu; st[2] = sigma; st[3] = z0;
        st[4] = gate; st[5] = Z / em; st[6] = sumsq * (Z / em) * (Z / em); st[7] = c;
    }
}

/* ---- mode 2: streaming with squared correction factors -------------------- */

static void row_stream(const double *q, const key_src *ks, int64_t n, const oracle_cfg *cfg,
                       const float *u_h, int block, double theta, double *zbuf, double *out,
                       double *neff_out, double *st) {
    const int D = ks->D;
    const double c = cfg->s * length_temperature(n, cfg);
    double m_run = -INFINITY; /* true running max of the logits */
    double m_ref = -INFINITY; /* max the weights are currently relative to */
    double l = 0.0, l2 = 0.0, S1 = 0.0, S2 = 0.0, acc[256];
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    if (block < 1) block = 1;
    for (int64_t j0 = 0; j0 < n; j0 += block) {
        int64_t j1 = j0 + block < n ? j0 + block : n;
        double bm = -INFINITY;
        for (int64_t j = j0; j < j1; ++j) {
            double sdot = qk_dot(q, ks, j);
            S1 += sdot;
            S2 += sdot * sdot;
            zbuf[j - j0] = c * sdot;
            if (zbuf[j - j0] > bm) bm = zbuf[j - j0];
        }
        if (bm > m_run) m_run = bm;
        if (m_ref == -INFINITY || bm > m_ref + theta) {
            double r = m_ref == -INFINITY ? 0.0 : exp(m_ref - m_run);
            l *= r;
#if ORACLE_MUTANT == 1
            l2 *= r;
#else
            l2 *= r * r;
#endif
            for (int d = 0; d < D; ++d) acc[d] *= r;
            m_ref = m_run;
        }
        for (int64_t j = j0; j < j1; ++j) {
            double p = exp(zbuf[j - j0] - m_ref);
            l += p;
            l2 += p * p;
            for (int d = 0; d < D; ++d) acc[d] += p * val_el(ks, j, d);
        }
    }
    double mean_s = S1 / (double)n;
    double var_s = S2 / (double)n - mean_s * mean_s;
    if (var_s < 0.0) var_s = 0.0;
    double mu = c * mean_s, sigma = c * sqrt(var_s);
    double z0 = null_floor(mu, sigma, n);
    double neff = l * l / l2;
    double gate = confidence_gate(m_run, z0, cfg->beta);
    emit(acc, D, neff, gate, u_h, cfg->L, out);
    *neff_out = neff;
    if (st) {
        double f = exp(m_ref - m_run); /* re-express l, l2 relative to the true max */
        st[0] = m_run; st[1] = mu; st[2] = sigma; st[3] = z0;
        st[4] = gate; st[5] = l * f; st[6] = l2 * f * f; st[7] = c;
    }
}

static void eval_row(int mode, int block, double theta, const double *q, const key_src *ks,
                     int64_t n, const oracle_cfg *cfg, const float *u_h, double *zbuf,
                     double *out, double *neff, double *st) {
    if (mode == 1)
        row_brute(q, ks, n, cfg, u_h, zbuf, out, neff, st);
    else if (mode == 2)
        row_stream(q, ks, n, cfg, u_h, block, theta, zbuf, out, neff, st);
    else
        row_two_pass(q, ks, n, cfg, u_h, zbuf, out, neff, st);
}

static int kv_head_of(int h, int Hq, int Hkv) {
#if ORACLE_MUTANT == 5
    return h % Hkv;
#else
    return h / (Hq / Hkv);
#endif
}

/* ---- public entry points -------------------------------------------------- */

/*
 * Prefill.  q: [B,T,Hq,D]; k, v: [B,T,Hkv,D] (dtype 0 = fp32, 1 = bf16 bits);
 * u: [Hq,D] fp32.  rows: flat indices ((b*Hq + h)*T + i), or NULL for all
 * B*Hq*T rows in that order.  out: [nrows][D]; neff: [nrows]; stats
 * (optional): [nrows][8] = m, mu, sigma, z0, gate, l, l2, c.
 * Returns 0, or -1 on invalid arguments.
 */
int oracle_polar_fwd(const oracle_cfg *cfg, const void *q, const void *k, const void *v,
                     int dtype, const float *u, const int64_t *rows, int64_t nrows, int mode,
                     int block, double theta, double *out, double *neff, double *stats) {
    if (!cfg || cfg->D <= 0 || cfg->D > 256 || cfg->Hkv <= 0 || cfg->Hq % cfg->Hkv != 0 ||
        cfg->L < 2 || cfg->T < 0 || cfg->B < 0)
        return -1;
    const int64_t total = (int64_t)cfg->B * cfg->Hq * cfg->T;
    if (!rows) nrows = total;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t flat = rows ? rows[r] : r;
        if (flat < 0 || flat >= total) { bad = 1; continue; }
        const int D = cfg->D, T = cfg->T;
        int64_t i = flat % T, bh = flat / T;
        int h = (int)(bh % cfg->Hq), b = (int)(bh / cfg->Hq);
        int g = kv_head_of(h, cfg->Hq, cfg->Hkv);
        double qrow[256];
        for (int d = 0; d < D; ++d) qrow[d] = ld(q, dtype, (((int64_t)b * T + i) * cfg->Hq + h) * D + d);
#if ORACLE_MUTANT == 4
        int64_t n = cfg->causal ? (i > 0 ? i : 1) : T;
#else
        int64_t n = cfg->causal ? i + 1 : T;
#endif
        int64_t lo = 0; /* first visible key */
        if (cfg->causal && cfg->window > 0 && n > cfg->window) {
#if ORACLE_MUTANT == 21
            lo = n - cfg->window + 1; /* mistake: the window one key short */
            n = cfg->window - 1;
#else
            lo = n - cfg->window;
            n = cfg->window;
#endif
        }
        key_src ks = {k, v, dtype, D, cfg->Hkv, g, 0,
                      ((int64_t)b * T * cfg->Hkv + g) * D, (int64_t)cfg->Hkv * D, NULL, lo};
        double *zbuf = (double *)malloc(sizeof(double) * (size_t)(n > block ? n : block) + 8);
        if (!zbuf) { bad = 1; continue; }
#if ORACLE_MUTANT == 10
        const float *u_h = u;
#else
        const float *u_h = u + (int64_t)h * D;
#endif
        eval_row(mode, block, theta, qrow, &ks, n, cfg, u_h, zbuf, out + r * D, neff + r,
                 stats ? stats + r * 8 : NULL);
        free(zbuf);
    }
    return bad ? -1 : 0;
}

/*
 * Paged GQA decode.  q: [N,Hq,D]; kv_pages: [num_pages][2][Hkv][64][D] (K then
 * V, head-major, 64 tokens per page); page_table: [N][max_pages] int32;
 * seqlens: [N] (>= 1).  Query of sequence s sees its keys 0..seqlens[s]-1
 * (the last cfg->window of them when window > 0).
 * rows: flat (s*Hq + h) or NULL for all.  Outputs as for oracle_polar_fwd.
 * Returns 0, -1 on invalid arguments, -2 on a page id out of range.
 */
int oracle_polar_decode(const oracle_cfg *cfg, const void *q, const void *kv_pages,
                        int64_t num_pages, const int32_t *page_table, int max_pages,
                        const int32_t *seqlens, int num_seqs, int dtype, const float *u,
                        const int64_t *rows, int64_t nrows, int mode, int block, double theta,
                        double *out, double *neff, double *stats) {
    if (!cfg || cfg->D <= 0 || cfg->D > 256 || cfg->Hkv <= 0 || cfg->Hq % cfg->Hkv != 0 ||
        cfg->L < 2 || num_seqs < 0 || max_pages < 0)
        return -1;
    const int64_t total = (int64_t)num_seqs * cfg->Hq;
    if (!rows) nrows = total;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t flat = rows ? rows[r] : r;
        if (flat < 0 || flat >= total) { bad |= 1; continue; }
        const int D = cfg->D;
        int h = (int)(flat % cfg->Hq), sq = (int)(flat / cfg->Hq);
        int64_t n = seqlens[sq];
        if (n < 1 || n > (int64_t)max_pages * ORACLE_PAGE) { bad |= 1; continue; }
        const int32_t *pt = page_table + (int64_t)sq * max_pages;
        int64_t npg = (n + ORACLE_PAGE - 1) / ORACLE_PAGE;
        int badpage = 0;
        for (int64_t p = 0; p < npg; ++p)
            if (pt[p] < 0 || pt[p] >= num_pages) badpage = 1;
        if (badpage) { bad |= 2; continue; }
        int g = kv_head_of(h, cfg->Hq, cfg->Hkv);
        double qrow[256];
        for (int d = 0; d < D; ++d) qrow[d] = ld(q, dtype, ((int64_t)sq * cfg->Hq + h) * D + d);
        int64_t lo = 0; /* first visible position */
        if (cfg->window > 0 && n > cfg->window) {
            lo = n - cfg->window;
            n = cfg->window;
        }
        key_src ks = {kv_pages, kv_pages, dtype, D, cfg->Hkv, g, 1, 0, 0, pt, lo};
        double *zbuf = (double *)malloc(sizeof(double) * (size_t)(n > block ? n : block) + 8);
        if (!zbuf) { bad |= 1; continue; }
        eval_row(mode, block, theta, qrow, &ks, n, cfg, u + (int64_t)h * D, zbuf, out + r * D,
                 neff + r, stats ? stats + r * 8 : NULL);
        free(zbuf);
    }
    if (bad & 2) return -2;
    return bad ? -1 : 0;
}

/*
 * Backward of the prefill (NEXT: the training use of the step).  Given
 * g = dL/dout for every row, the gradients dL/dq, dL/dk, dL/dv (fp64, same
 * layouts as q, k, v) and dL/du ([Hq][D]).  Each row is recomputed by the
 * two-pass definition above; then, with w_j = e^{z_j - m}, A = sum w_j v_j,
 * content = A/|A|, T = tanh(ln n_eff / ln L):
 *   du_h   += gate*T*g
 *   gamma   = <g, u_h>;  dgate = gamma*T;  dT = gamma*gate
 *   dn_eff  = dT*(1 - T^2) / (n_eff ln L)
 *   dl      = 2 l/l2 * dn_eff;  dl2 = -(l/l2)^2 * dn_eff   (n_eff = l^2/l2)
 *   dA      = (g - content <content, g>) / |A|             (A/|A|)
 *   dm      = beta*gate*(1 - gate)*dgate;  dz0 = -dm       (gate on m - z0)
 *   dmu     = dz0;  dsigma = dz0*sqrt(2 ln n)              (z0 = mu + sigma sqrt(2 ln n))
 *   dz_j    = w_j (dl + 2 dl2 w_j + <dA, v_j>) + dmu/n + dsigma (z_j - mu)/(n sigma)
 *             + [j = argmax] dm          (the max's subgradient: its first index;
 *                                       sigma = 0 contributes nothing)
 *   dS_j    = c dz_j;  dq += dS_j k_j;  dk_j += dS_j q;  dv_j += w_j dA.
 * The shift m cancels from content and n_eff (both scale-invariant), so w may
 * be taken relative to any common reference.  Inputs as oracle_polar_fwd; g
 * is fp64 [B,T,Hq,D].  Returns 0, or -1 on invalid arguments.
 */
int oracle_polar_bwd(const oracle_cfg *cfg, const void *q, const void *k, const void *v,
                     int dtype, const float *u, const double *gout, double *dq, double *dk,
                     double *dv, double *du) {
    if (!cfg || cfg->D <= 0 || cfg->D > 256 || cfg->Hkv <= 0 || cfg->Hq % cfg->Hkv != 0 ||
        cfg->L < 2 || cfg->T < 0 || cfg->B < 0 || !cfg->causal)
        return -1;
    const int B = cfg->B, T = cfg->T, Hq = cfg->Hq, Hkv = cfg->Hkv, D = cfg->D;
    const int G = Hq / Hkv;
    memset(dq, 0, sizeof(double) * (size_t)B * T * Hq * D);
    memset(dk, 0, sizeof(double) * (size_t)B * T * Hkv * D);
    memset(dv, 0, sizeof(double) * (size_t)B * T * Hkv * D);
    double *du_part = (double *)calloc((size_t)B * Hq * D, sizeof(double));
    if (!du_part) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t task = 0; task < (int64_t)B * Hkv; ++task) {
        /* One (batch, kv head): every write to dk, dv of kv head g and to dq
           of its query heads stays inside this task. */
        const int b = (int)(task / Hkv), g = (int)(task % Hkv);
        double *z = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double *w = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        if (!z || !w) { bad = 1; free(z); free(w); continue; }
        for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            for (int64_t i = 0; i < T; ++i) {
                int64_t n = i + 1, lo = 0;
                if (cfg->window > 0 && n > cfg->window) { lo = n - cfg->window; n = cfg->window; }
                double qr[256], gr[256];
                const int64_t qo = (((int64_t)b * T + i) * Hq + h) * D;
                for (int d = 0; d < D; ++d) { qr[d] = ld(q, dtype, qo + d); gr[d] = gout[qo + d]; }
                const double c = cfg->s * length_temperature(n, cfg);
                /* forward, two-pass */
                double m = -INFINITY, mu = 0.0;
                int64_t jmax = 0;
                for (int64_t j = 0; j < n; ++j) {
                    const int64_t ko = (((int64_t)b * T + lo + j) * Hkv + g) * D;
                    double sd = 0.0;
                    for (int d = 0; d < D; ++d) sd += qr[d] * ld(k, dtype, ko + d);
                    z[j] = c * sd;
                    if (z[j] > m) { m = z[j]; jmax = j; }
                    mu += z[j];
                }
                mu /= (double)n;
                double var = 0.0;
                for (int64_t j = 0; j < n; ++j) var += (z[j] - mu) * (z[j] - mu);
                const double sigma = sqrt(var / (double)n);
                const double kn = sqrt(2.0 * log((double)n));
                const double z0 = mu + sigma * kn;
                const double gate = 1.0 / (1.0 + exp(-cfg->beta * (m - z0)));
                double l = 0.0, l2 = 0.0, A[256];
                for (int d = 0; d < D; ++d) A[d] = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    const int64_t vo = (((int64_t)b * T + lo + j) * Hkv + g) * D;
                    w[j] = exp(z[j] - m);
                    l += w[j];
                    l2 += w[j] * w[j];
                    for (int d = 0; d < D; ++d) A[d] += w[j] * ld(v, dtype, vo + d);
                }
                double nrm = 0.0;
                for (int d = 0; d < D; ++d) nrm += A[d] * A[d];
                nrm = sqrt(nrm);
                const double an = nrm > 1e-30 ? nrm : 1e-30;
                const double neff = l * l / l2;
                const double lnL = log((double)cfg->L);
                const double Tm = tanh(log(neff) / lnL);
                /* backward */
                const float *uh = u + (int64_t)h * D;
                double gamma = 0.0, cg = 0.0;
                for (int d = 0; d < D; ++d) {
                    du_part[((int64_t)b * Hq + h) * D + d] += gate * Tm * gr[d];
                    gamma += gr[d] * (double)uh[d];
                    cg += (A[d] / an) * gr[d];
                }
                const double dgate = gamma * Tm, dT = gamma * gate;
                const double dneff = dT * (1.0 - Tm * Tm) / (neff * lnL);
                const double dl = dneff * 2.0 * l / l2;
#if ORACLE_MUTANT == 12
                const double dl2 = dneff * (l / l2) * (l / l2);
#else
                const double dl2 = -dneff * (l / l2) * (l / l2);
#endif
                double dA[256];
                for (int d = 0; d < D; ++d) dA[d] = (gr[d] - (A[d] / an) * cg) / an;
                const double dm = cfg->beta * gate * (1.0 - gate) * dgate;
                const double dmu = -dm, dsigma = -dm * kn;
                for (int64_t j = 0; j < n; ++j) {
                    const int64_t ko = (((int64_t)b * T + lo + j) * Hkv + g) * D;
                    double av = 0.0;
                    for (int d = 0; d < D; ++d) av += dA[d] * ld(v, dtype, ko + d);
                    double dz = w[j] * (dl + 2.0 * dl2 * w[j] + av) + dmu / (double)n;
#if ORACLE_MUTANT != 11
                    if (sigma > 0.0) dz += dsigma * (z[j] - mu) / ((double)n * sigma);
#endif
#if ORACLE_MUTANT != 19
                    if (j == jmax) dz += dm;
#endif
                    const double dS = c * dz;
                    for (int d = 0; d < D; ++d) {
                        dq[qo + d] += dS * ld(k, dtype, ko + d);
                        dk[ko + d] += dS * qr[d];
#if ORACLE_MUTANT == 18
                        /* mistake: the direction's projection left out of dv */
                        dv[ko + d] += w[j] * gr[d] / an;
#else
                        dv[ko + d] += w[j] * dA[d];
#endif
                    }
                }
            }
        }
        free(z);
        free(w);
    }
    memset(du, 0, sizeof(double) * (size_t)Hq * D);
    for (int b = 0; b < B; ++b)
        for (int64_t e = 0; e < (int64_t)Hq * D; ++e) du[e] += du_part[(int64_t)b * Hq * D + e];
    free(du_part);
    return bad ? -1 : 0;
}

/* Compile-time mutant id, so a test can confirm which build it loaded. */
int oracle_mutant_id(void) { return ORACLE_MUTANT; }
