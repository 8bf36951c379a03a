/*
 * fp32 canonical-order replicas for the oracle of EntmaxKV page selection.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by oracle/replica.py; never linked into,
 * and sharing nothing with, the CUDA library.
 *
 * Why: which pages are selected is an integer decision taken from fp32 page
 * scores (EntmaxKV pages, section 2.A: bounding-box bound and Gaussian page
 * statistics; section 2.B: top-k and Gaussian-aware selection).  For the two
 * sides to decide alike they must compute these scores in the same precision
 * and order.  This file is that order, written out:
 *
 *  - page metadata (Welford, fp32, token order):
 *        first token: mean = x, m2 = 0, kmin = kmax = x
 *        later token t (1-based n = t + 1):
 *            d1 = x - mean;  mean = mean + d1 / n;  d2 = x - mean;
 *            m2 = fmaf(d1, d2, m2);
 *            kmin = (x < kmin) ? x : kmin;  kmax = (x > kmax) ? x : kmax
 *  - dot products over d (the bound's sum and the Gaussian sums) split d into
 *    8 consecutive slices of d/8 coordinates; each slice is a chain of fmaf
 *    from 0 in ascending d, and the slice sums S0..S7 are combined as
 *        ((S0 + S1) + (S2 + S3)) + ((S4 + S5) + (S6 + S7))
 *  - bounding-box bound of one page for head h, with terms
 *        q[d] * (q[d] >= 0 ? kmax[d] : kmin[d]):
 *        UB_h = dot * scale;  UBg = max over the group's heads; -0 -> +0
 *  - Gaussian page estimate for head h:
 *        ma = dot of q[d] * mean[d];   va = dot of (q[d]*q[d]) * m2[d]
 *        m = ma * scale;  v = (va / n) * (scale * scale)
 *        est = fmaf(sqrtf(v), z[n], m)
 *
 * Built with -ffp-contract=off so that no other operation is fused; fmaf and
 * sqrtf are the correctly rounded C99 functions.
 */
#include <math.h>
#include <stdint.h>

/* Metadata of the P = ceil(L/ps) pages of one (sequence, kv-head).
 * keys: [L][d] fp32 (bf16 keys widened exactly).  Outputs [P][d]; count [P]. */
void replica_page_meta(const float* keys, int64_t L, int d, int ps,
                       float* kmin, float* kmax, float* mean, float* m2,
                       int32_t* count)
{
    int64_t P = (L + ps - 1) / ps;
    for (int64_t p = 0; p < P; ++p) {
        int64_t t0 = p * ps;
        int64_t t1 = t0 + ps < L ? t0 + ps : L;
        for (int j = 0; j < d; ++j) {
            float mu = 0.0f, s = 0.0f, lo = 0.0f, hi = 0.0f;
            for (int64_t t = t0; t < t1; ++t) {
                float x = keys[t * d + j];
                if (t == t0) {
                    mu = x; s = 0.0f; lo = x; hi = x;
                    continue;
                }
                float n = (float)(t - t0 + 1);
                float d1 = x - mu;
                mu = mu + d1 / n;
                float d2 = x - mu;
                s = fmaf(d1, d2, s);
                lo = (x < lo) ? x : lo;
                hi = (x > hi) ? x : hi;
            }
            kmin[p * d + j] = lo;
            kmax[p * d + j] = hi;
            mean[p * d + j] = mu;
            m2[p * d + j] = s;
        }
        count[p] = (int32_t)(t1 - t0);
    }
}

/* The fixed combination of the 8 slice sums. */
static float tree8(const float* s)
{
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

/* Bounding-box bounds of P pages for the G heads of one group.
 * q: [G][d]; kmin/kmax: [P][d]; ub: [G][P] (may be NULL); ubg: [P]. */
void replica_bound(const float* q, int G, int d,
                   const float* kmin, const float* kmax, int64_t P,
                   float scale, float* ub, float* ubg)
{
    const int w = d / 8;
    for (int64_t p = 0; p < P; ++p) {
        float best = 0.0f;
        for (int h = 0; h < G; ++h) {
            float s[8];
            for (int k = 0; k < 8; ++k) {
                float acc = 0.0f;
                for (int j = k * w; j < (k + 1) * w; ++j) {
                    float qd = q[h * d + j];
                    float sel = (qd >= 0.0f) ? kmax[p * d + j] : kmin[p * d + j];
                    acc = fmaf(qd, sel, acc);
                }
                s[k] = acc;
            }
            float u = tree8(s) * scale;
            if (ub) ub[h * P + p] = u;
            if (h == 0 || u > best) best = u;
        }
        if (best == 0.0f) best = 0.0f;   /* -0 -> +0 */
        ubg[p] = best;
    }
}

/* Gaussian page estimates of P pages for G heads.
 * mean/m2: [P][d]; count: [P] (>= 1); z: fp32 table indexed by count.
 * m, v, est: [G][P]. */
void replica_gauss(const float* q, int G, int d,
                   const float* mean, const float* m2, const int32_t* count,
                   int64_t P, float scale, const float* z,
                   float* m, float* v, float* est)
{
    float scale2 = scale * scale;
    const int w = d / 8;
    for (int h = 0; h < G; ++h) {
        for (int64_t p = 0; p < P; ++p) {
            float sm[8], sv[8];
            for (int k = 0; k < 8; ++k) {
                float ma = 0.0f, va = 0.0f;
                for (int j = k * w; j < (k + 1) * w; ++j) {
                    float qd = q[h * d + j];
                    float q2 = qd * qd;
                    ma = fmaf(qd, mean[p * d + j], ma);
                    va = fmaf(q2, m2[p * d + j], va);
                }
                sm[k] = ma;
                sv[k] = va;
            }
            int32_t n = count[p];
            float mm = tree8(sm) * scale;
            float vv = (tree8(sv) / (float)n) * scale2;
            m[h * P + p] = mm;
            v[h * P + p] = vv;
            est[h * P + p] = fmaf(sqrtf(vv), z[n], mm);
        }
    }
}
