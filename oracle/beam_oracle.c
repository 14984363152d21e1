/*
 * beam_oracle.c -- fp64 CPU oracle of the BEAM-masked MoE layer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY (see beam_oracle.h).  Plain loops in the order the
 * method states them; no blocking, no SIMD intrinsics, no reordering beyond
 * skipping terms that the definition multiplies by an exact zero.
 *
 * Source: "BEAM: Binary Expert Activation Masking for Dynamic Routing in MoE"
 * (arXiv 2605.14438, Chinese translation of the HTML version), §3.1 and §3.2.
 * Readings where the page is silent are marked READING below.
 */
#include "beam_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Widen one stored element to double.  bfloat16 is the upper half of an
 * IEEE binary32, so the widening is exact. */
static double load_elem(const void *base, int dtype, size_t i) {
    if (dtype == ORACLE_F32) return (double)((const float *)base)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* §3.2 step 1: r = R(x) = x W (the main router is a bias-free linear map).
 * §3.2 step 2 / Eq. (5): the mask router's pre-activation x W_m; the sigmoid
 * is applied in oracle_route, where the threshold of Eq. (6) is taken. */
int oracle_logits(int T, int d, int E, int dtype, const void *x, const void *W_gate,
                  const void *W_mask, double *r, double *z) {
    if (T < 0 || d <= 0 || E <= 0 || !x || !W_gate || !r) return -1;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_F32) return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += load_elem(x, dtype, (size_t)t * d + j) *
                       load_elem(W_gate, dtype, (size_t)e * d + j);
            r[(size_t)t * E + e] = acc;
            if (!isfinite(acc)) bad = 1;
            if (W_mask && z) {
                double accm = 0.0;
                for (int j = 0; j < d; ++j)
                    accm += load_elem(x, dtype, (size_t)t * d + j) *
                            load_elem(W_mask, dtype, (size_t)e * d + j);
                z[(size_t)t * E + e] = accm;
                if (!isfinite(accm)) bad = 1;
            }
        }
    }
    return bad ? -2 : 0;
}

/* Eq. (1)/(4): Top-K keeps the K largest logits and sets the rest to -inf
 * before the softmax.  READING: the page does not order the candidates nor
 * break ties; candidates are listed by descending logit and an exact tie goes
 * to the lower expert index, which makes the selection unique.
 *
 * Eq. (5)-(6): m = 1 iff sigmoid(z) >= tau, with tau = 0.5 in the method and
 * other values in the threshold ablation (news article, §8).  sigmoid is
 * increasing, so the test is taken on the pre-activation as z >= logit(tau),
 * which the caller passes as tau_logit (0 for tau = 0.5, where sigmoid(0) =
 * 0.5 exactly).  READING: the news article's "index becomes -1 when the raw
 * value is <= 0" contradicts both Eq. (6) and the zero-initialisation claim
 * that every candidate is kept, so Eq. (6) wins; -0.0 counts as >= 0.
 *
 * Eq. (7): w = g * m with no renormalisation after the mask. */
int oracle_route(int T, int E, int K, int renorm, double tau_logit, const double *r,
                 const double *z, int32_t *cand, double *g, int32_t *idx, double *w,
                 int32_t *counts, int32_t *hist) {
    if (T < 0 || E <= 0 || K <= 0 || K > E || !r || !idx) return -1;
    if (isnan(tau_logit)) return -1;
    if (counts) memset(counts, 0, sizeof(int32_t) * (size_t)E);
    if (hist) memset(hist, 0, sizeof(int32_t) * (size_t)(K + 1));
    char *taken = (char *)malloc((size_t)E);
    int32_t *c = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    double *gk = (double *)malloc(sizeof(double) * (size_t)K);
    if (!taken || !c || !gk) { free(taken); free(c); free(gk); return -1; }
    int rc = 0;
    for (int t = 0; t < T && rc == 0; ++t) {
        const double *rt = r + (size_t)t * E;
        for (int e = 0; e < E; ++e) {
            if (!isfinite(rt[e])) rc = -2;
        }
        if (rc) break;
        /* Top-K: K rounds of "largest remaining logit, lowest index on ties". */
        memset(taken, 0, (size_t)E);
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || rt[e] > rt[best]) best = e;
            }
            taken[best] = 1;
            c[k] = best;
        }
        /* Softmax of Top-K(r): entries outside the Top-K are -inf, so they add
         * nothing to the denominator (renorm = 1).  With renorm = 0 the
         * softmax runs over all E logits and is then restricted to the
         * candidates.  Shifted by the largest logit, which is rt[c[0]]. */
        double m = rt[c[0]];
        double denom = 0.0;
        if (renorm) {
            for (int k = 0; k < K; ++k) denom += exp(rt[c[k]] - m);
        } else {
            for (int e = 0; e < E; ++e) denom += exp(rt[e] - m);
        }
        for (int k = 0; k < K; ++k) gk[k] = exp(rt[c[k]] - m) / denom;
        /* Binary mask on the candidates, then aggregation. */
        int kept = 0;
        for (int k = 0; k < K; ++k) {
            int mk = 1;
            if (z) {
                double zz = z[(size_t)t * E + c[k]];
                mk = (zz >= tau_logit) ? 1 : 0; /* NaN compares false: not kept */
            }
            size_t o = (size_t)t * K + k;
            if (cand) cand[o] = c[k];
            if (g) g[o] = gk[k];
            idx[o] = mk ? c[k] : -1;
            if (w) w[o] = mk ? gk[k] : 0.0;
            if (mk) {
                ++kept;
                if (counts) counts[c[k]] += 1;
            }
        }
        if (hist) hist[kept] += 1;
    }
    free(taken);
    free(c);
    free(gk);
    return rc;
}

int oracle_route_f32(int T, int E, int K, int renorm, double tau_logit, const float *r,
                     const float *z, int32_t *cand, double *g, int32_t *idx, double *w,
                     int32_t *counts, int32_t *hist) {
    if (T < 0 || E <= 0 || !r) return -1;
    size_t n = (size_t)T * E;
    double *rd = (double *)malloc(sizeof(double) * (n ? n : 1));
    double *zd = z ? (double *)malloc(sizeof(double) * (n ? n : 1)) : NULL;
    if (!rd || (z && !zd)) { free(rd); free(zd); return -1; }
    for (size_t i = 0; i < n; ++i) {
        rd[i] = (double)r[i];
        if (z) zd[i] = (double)z[i];
    }
    int rc = oracle_route(T, E, K, renorm, tau_logit, rd, zd, cand, g, idx, w, counts, hist);
    free(rd);
    free(zd);
    return rc;
}

/* Expert-token batch grouping: masked entries (-1) are left out of the count,
 * so a masked pair is never scheduled (techwalker news article on BEAM, §5,
 * the second of the two vLLM kernel changes).  READING: pairs are listed by
 * expert, then by token. */
int oracle_permutation(int T, int K, int E, const int32_t *idx, int32_t *offsets,
                       int32_t *pairs) {
    if (T < 0 || K <= 0 || E <= 0 || !idx || !offsets || !pairs) return -1;
    int n = 0;
    for (int e = 0; e < E; ++e) {
        offsets[e] = n;
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k)
                if (idx[(size_t)t * K + k] == e) pairs[n++] = t * K + k;
    }
    offsets[E] = n;
    return 0;
}

/* Eq. (3): E_i(x) = (delta(x W_gate^(i)) (.) (x W_up^(i))) W_down^(i), with
 * delta = SiLU (READING: the page leaves delta unnamed; SwiGLU experts), and
 * Eq. (8): y = sum_i w_i E_i(x).  Terms with w_i = 0 are exact zeros and are
 * skipped; a token with no kept candidate therefore gets y = 0, i.e. it passes
 * the layer through the residual alone (news article, §5).  The sum runs over
 * the candidate slots in order k = 0..K-1. */
int oracle_experts(int T, int d, int E, int I, int K, int dtype, const void *x,
                   const void *W1, const void *W3, const void *W2, const int32_t *idx,
                   const double *w, int t_begin, int t_end, double *y, int nthreads) {
    if (T < 0 || d <= 0 || E <= 0 || I <= 0 || K <= 0) return -1;
    if (!x || !W1 || !W3 || !W2 || !idx || !w || !y) return -1;
    if (t_begin < 0 || t_end > T || t_begin > t_end) return -1;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_F32) return -1;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#else
    nthreads = 1;
#endif
    int bad = 0;
#pragma omp parallel num_threads(nthreads) reduction(| : bad)
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        if (!xt || !h) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int t = t_begin; t < t_end; ++t) {
            if (!xt || !h) continue;
            double *yt = y + (size_t)(t - t_begin) * d;
            for (int j = 0; j < d; ++j) yt[j] = 0.0;
            for (int j = 0; j < d; ++j) xt[j] = load_elem(x, dtype, (size_t)t * d + j);
            for (int k = 0; k < K; ++k) {
                int e = idx[(size_t)t * K + k];
                if (e < 0) continue; /* m_k = 0: expert skipped entirely */
                if (e >= E) { bad = 1; continue; }
                double wk = w[(size_t)t * K + k];
                /* h = SiLU(x W_gate) (.) (x W_up) */
                for (int i = 0; i < I; ++i) {
                    size_t row = ((size_t)e * I + i) * d;
                    double a = 0.0, b = 0.0;
                    for (int j = 0; j < d; ++j) {
                        a += xt[j] * load_elem(W1, dtype, row + j);
                        b += xt[j] * load_elem(W3, dtype, row + j);
                    }
                    h[i] = a / (1.0 + exp(-a)) * b;
                }
                /* y += w_k * (h W_down) */
                for (int j = 0; j < d; ++j) {
                    size_t row = ((size_t)e * d + j) * I;
                    double s = 0.0;
                    for (int i = 0; i < I; ++i) s += h[i] * load_elem(W2, dtype, row + i);
                    yt[j] += wk * s;
                }
            }
            for (int j = 0; j < d; ++j)
                if (!isfinite(yt[j])) bad = 2;
        }
        free(xt);
        free(h);
    }
    if (bad == 2 || bad == 3) return -2;
    return bad ? -1 : 0;
}

/* Shared experts: every token, weight 1, after the routed sum (see header). */
int oracle_shared_experts(int T, int d, int n_shared, int Is, int dtype, const void *x,
                          const void *W1s, const void *W3s, const void *W2s, int t_begin,
                          int t_end, double *y, int nthreads) {
    if (T < 0 || d <= 0 || n_shared < 0 || (n_shared > 0 && Is <= 0)) return -1;
    if (n_shared == 0) return 0;
    if (!x || !W1s || !W3s || !W2s || !y) return -1;
    if (t_begin < 0 || t_end > T || t_begin > t_end) return -1;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_F32) return -1;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#else
    nthreads = 1;
#endif
    int bad = 0;
#pragma omp parallel num_threads(nthreads) reduction(| : bad)
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *h = (double *)malloc(sizeof(double) * (size_t)Is);
        if (!xt || !h) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int t = t_begin; t < t_end; ++t) {
            if (!xt || !h) continue;
            double *yt = y + (size_t)(t - t_begin) * d;
            for (int j = 0; j < d; ++j) xt[j] = load_elem(x, dtype, (size_t)t * d + j);
            for (int s = 0; s < n_shared; ++s) {
                for (int i = 0; i < Is; ++i) {
                    size_t row = ((size_t)s * Is + i) * d;
                    double a = 0.0, b = 0.0;
                    for (int j = 0; j < d; ++j) {
                        a += xt[j] * load_elem(W1s, dtype, row + j);
                        b += xt[j] * load_elem(W3s, dtype, row + j);
                    }
                    h[i] = a / (1.0 + exp(-a)) * b;
                }
                for (int j = 0; j < d; ++j) {
                    size_t row = ((size_t)s * d + j) * Is;
                    double acc = 0.0;
                    for (int i = 0; i < Is; ++i) acc += h[i] * load_elem(W2s, dtype, row + i);
                    yt[j] += acc;
                }
            }
            for (int j = 0; j < d; ++j)
                if (!isfinite(yt[j])) bad = 2;
        }
        free(xt);
        free(h);
    }
    if (bad == 2 || bad == 3) return -2;
    return bad ? -1 : 0;
}
