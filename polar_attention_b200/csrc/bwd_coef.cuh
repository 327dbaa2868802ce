// bwd_coef.cuh -- the per-row part of the prefill backward, shared by the
// tensor-core rows pass (fwd_tc.cu, which recomputes each row's streaming
// state) and the rows kernel that starts from a training forward's saved state
// (bwd_simt.cu).
//
// Method: "ATMA: Length-Invariant Language Modeling via Polar Attention and
// Gated-Delta Compression Memory", gist.science technical summary, section 2.1
// (magnitude channel: n_eff = l^2/l2, tanh-log of n_eff, the gate on the max
// logit over the null floor mu + sigma sqrt(2 ln n)) and section 2.2 (the fused
// kernel's streaming l, l2); the training use is section 3.
#pragma once

#include "polar_common.cuh"
#include "polar_internal.h"

namespace polar {

// Magnitude channel of one row from its streaming state: l, l2 (weights
// relative to any common reference), the max raw dot m_raw, the raw sums s1,
// s2, the logit scale c and the n visible keys.
struct RowMag {
    float gate, Tm;      // gate and tanh(ln n_eff / ln L); count = gate * Tm
    float ne;            // n_eff after the clamp to [1, n]
    bool clamped;        // the clamp was active (no gradient through n_eff)
    float mu, sigma, kn; // null floor z0 = mu + sigma * kn
};

__device__ __forceinline__ RowMag row_mag(float l, float l2, float m_raw, float s1, float s2,
                                          float c, float n, float beta, float inv_ln_L) {
    RowMag r;
    const float mean_s = s1 / n;
    const float sig_s = sqrtf(fmaxf(s2 / n - mean_s * mean_s, 0.0f));
    r.mu = c * mean_s;
    r.sigma = c * sig_s;
    r.kn = sqrtf(2.0f * logf(n));
    const float z0 = r.mu + r.sigma * r.kn;
    r.gate = 1.0f / (1.0f + expf(-beta * (c * m_raw - z0)));
    const float ne_raw = (l * l) / l2;
    r.ne = fminf(fmaxf(ne_raw, 1.0f), n);
    r.clamped = r.ne != ne_raw;
    r.Tm = tanhf(logf(r.ne) * inv_ln_L);
    return r;
}

// The row's coefficient record (BwdCoef layout) for the backward's dK/dV and
// dQ passes, given gu = <g, u_h> with g = dL/dout of the row: the chain rule
// through count = gate * Tm into l, l2 (via n_eff), the max logit and the null
// floor's mean and spread.  Weights are w = 2^(cl2 S - cl2) (the fixed
// reference cl2 = c log2e); jarg is the row's first argmax key, lo its first
// visible key.  Rows past the end (live = false) get a record whose weights and
// dS vanish.
__device__ __forceinline__ void store_coef_record(float *rec, bool live, const RowMag &m,
                                                  float gu, float l, float l2, float c,
                                                  float cl2, float n, float beta,
                                                  float inv_ln_L, int jarg, int lo) {
    float4 *cr = reinterpret_cast<float4 *>(rec);
    if (live) {
        const float dgate = gu * m.Tm, dT = gu * m.gate;
        const float dneff = m.clamped ? 0.0f : dT * (1.0f - m.Tm * m.Tm) * inv_ln_L / m.ne;
        const float dl = 2.0f * dneff * l / l2;
        const float dl2 = -dneff * (l / l2) * (l / l2);
        const float dm = beta * m.gate * (1.0f - m.gate) * dgate;
        const float dsigma = -dm * m.kn;
        const float cmu = -dm / n - (m.sigma > 0.0f ? dsigma * m.mu / (n * m.sigma) : 0.0f);
        const float csS = m.sigma > 0.0f ? dsigma * c / (n * m.sigma) : 0.0f;
        cr[0] = make_float4(cl2, -cl2, c, c * dl);
        cr[1] = make_float4(2.0f * c * dl2, c * csS, c * cmu, c * dm);
        cr[2] = make_float4(__int_as_float(jarg), __int_as_float(lo), m.gate * m.Tm, 0.f);
    } else {
        cr[0] = make_float4(0.f, -INFINITY, 0.f, 0.f);
        cr[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        cr[2] = make_float4(__int_as_float(-1), __int_as_float(0), 0.f, 0.f);
    }
    cr[3] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace polar
