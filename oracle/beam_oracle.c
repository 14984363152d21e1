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
            /* -inf is a logit of weight 0 (Eq. 1 writes it for the experts
             * outside the Top-K); NaN and +inf have no defined softmax. */
            if (isnan(rt[e]) || rt[e] == INFINITY) rc = -2;
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
        if (m == -INFINITY) {
            /* READING: every candidate's logit is -inf, so Eq. (4) is 0/0; the
             * candidates get weight 0 and the token contributes nothing, as an
             * all-masked token does. */
            for (int k = 0; k < K; ++k) gk[k] = 0.0;
        } else {
            if (renorm) {
                for (int k = 0; k < K; ++k) denom += exp(rt[c[k]] - m);
            } else {
                for (int e = 0; e < E; ++e) denom += exp(rt[e] - m);
            }
            for (int k = 0; k < K; ++k) gk[k] = exp(rt[c[k]] - m) / denom;
        }
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

/* Training-mode backward (see header).  Phase 1, per token: the forward of
 * every candidate (a = x W1^T, b = x W3^T, h = SiLU(a) (.) b, e = h W2^T), then
 *   u_k    = <dy, e_k>
 *   dm_k   = g_k u_k                         (through w = g m, Eq. 7; STE term)
 *   dz_k   = (dm_k + beta) s_k (1 - s_k)     (s = sigmoid(z), Eq. 5; dm/ds = 1)
 *   dg_k   = m_k u_k
 *   dr     = softmax backward of dg (over the candidates when renorm, Eq. 4;
 *            over all E logits otherwise)
 * and, for kept candidates, the expert backward with upstream w_k dy:
 *   dh = W2^T (w_k dy), da = dh (.) b (.) SiLU'(a), db = dh (.) SiLU(a),
 *   dx += W1^T da + W3^T db.
 * dx also gets W_gate^T dr and W_mask^T dz.  Phase 2 sums the weight
 * gradients over tokens (ascending) and slots (ascending). */
static double sigmoid_d(double v) { return 1.0 / (1.0 + exp(-v)); }

int oracle_backward(int T, int d, int E, int I, int K, int renorm, int dtype, double tau_logit,
                    double beta, int ste, const void *x, const void *W_gate, const void *W_mask,
                    const void *W1, const void *W3, const void *W2, const void *dy, int n_sel,
                    const int32_t *sel, const double *r_in, const double *z_in, double *dx,
                    double *dWg, double *dWm, double *dW1, double *dW3, double *dW2, double *u,
                    double *dz, int nthreads) {
    if (T < 0 || d <= 0 || E <= 0 || I <= 0 || K <= 0 || K > E) return -1;
    if (!x || !W_gate || !W1 || !W3 || !W2 || !dy || !dx || !dWg) return -1;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_F32) return -1;
    if (sel == NULL) n_sel = E;
    if (n_sel < 0) return -1;
    for (int s = 0; sel && s < n_sel; ++s)
        if (sel[s] < 0 || sel[s] >= E) return -1;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#else
    nthreads = 1;
#endif
    const size_t TK = (size_t)T * K, TE = (size_t)T * E;
    double *r = (double *)malloc(sizeof(double) * (TE ? TE : 1));
    double *zl = (double *)malloc(sizeof(double) * (TE ? TE : 1));
    int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * (TK ? TK : 1));
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (TK ? TK : 1));
    double *g = (double *)malloc(sizeof(double) * (TK ? TK : 1));
    double *w = (double *)malloc(sizeof(double) * (TK ? TK : 1));
    double *uk = (double *)malloc(sizeof(double) * (TK ? TK : 1));
    double *dzk = (double *)malloc(sizeof(double) * (TK ? TK : 1));
    double *dr = (double *)malloc(sizeof(double) * (TE ? TE : 1));
    double *hs = (double *)malloc(sizeof(double) * (TK ? TK : 1) * I);
    double *das = (double *)malloc(sizeof(double) * (TK ? TK : 1) * I);
    double *dbs = (double *)malloc(sizeof(double) * (TK ? TK : 1) * I);
    int rc = 0;
    if (!r || !zl || !cand || !idx || !g || !w || !uk || !dzk || !dr || !hs || !das || !dbs) {
        rc = -1;
        goto done;
    }
    if (r_in) {
        memcpy(r, r_in, sizeof(double) * TE);
        if (W_mask && z_in) memcpy(zl, z_in, sizeof(double) * TE);
        else if (W_mask) { rc = -1; goto done; }
    } else {
        rc = oracle_logits(T, d, E, dtype, x, W_gate, W_mask, r, W_mask ? zl : NULL);
        if (rc) goto done;
    }
    rc = oracle_route(T, E, K, renorm, tau_logit, r, W_mask ? zl : NULL, cand, g, idx, w, NULL,
                      NULL);
    if (rc) goto done;

    int bad = 0;
#pragma omp parallel num_threads(nthreads) reduction(| : bad)
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *dyt = (double *)malloc(sizeof(double) * (size_t)d);
        double *a = (double *)malloc(sizeof(double) * (size_t)I);
        double *b = (double *)malloc(sizeof(double) * (size_t)I);
        double *dh = (double *)malloc(sizeof(double) * (size_t)I);
        double *dg = (double *)malloc(sizeof(double) * (size_t)K);
        if (!xt || !dyt || !a || !b || !dh || !dg) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < T; ++t) {
            if (bad & 1) continue;
            for (int j = 0; j < d; ++j) {
                xt[j] = load_elem(x, dtype, (size_t)t * d + j);
                dyt[j] = load_elem(dy, dtype, (size_t)t * d + j);
            }
            double *dxt = dx + (size_t)t * d;
            for (int j = 0; j < d; ++j) dxt[j] = 0.0;
            for (int k = 0; k < K; ++k) {
                const size_t o = (size_t)t * K + k;
                const int e = cand[o];
                double *h = hs + o * I, *da = das + o * I, *db = dbs + o * I;
                for (int i = 0; i < I; ++i) {
                    size_t row = ((size_t)e * I + i) * d;
                    double ai = 0.0, bi = 0.0;
                    for (int j = 0; j < d; ++j) {
                        ai += xt[j] * load_elem(W1, dtype, row + j);
                        bi += xt[j] * load_elem(W3, dtype, row + j);
                    }
                    a[i] = ai;
                    b[i] = bi;
                    h[i] = ai * sigmoid_d(ai) * bi;
                }
                double uu = 0.0;
                for (int j = 0; j < d; ++j) {
                    size_t row = ((size_t)e * d + j) * I;
                    double ej = 0.0;
                    for (int i = 0; i < I; ++i) ej += h[i] * load_elem(W2, dtype, row + i);
                    uu += dyt[j] * ej;
                }
                uk[o] = uu;
                const int kept = idx[o] >= 0;
                dg[k] = kept ? uu : 0.0;
                if (W_mask) {
                    const double sg = sigmoid_d(zl[(size_t)t * E + e]);
                    const double dm = ste ? g[o] * uu : 0.0;
                    dzk[o] = (dm + beta) * sg * (1.0 - sg);
                } else {
                    dzk[o] = 0.0;
                }
                if (!kept) {
                    for (int i = 0; i < I; ++i) da[i] = db[i] = 0.0;
                    continue;
                }
                /* Expert backward with upstream w_k dy. */
                for (int i = 0; i < I; ++i) dh[i] = 0.0;
                for (int j = 0; j < d; ++j) {
                    size_t row = ((size_t)e * d + j) * I;
                    const double c = w[o] * dyt[j];
                    for (int i = 0; i < I; ++i) dh[i] += c * load_elem(W2, dtype, row + i);
                }
                for (int i = 0; i < I; ++i) {
                    const double sa = sigmoid_d(a[i]);
                    da[i] = dh[i] * b[i] * sa * (1.0 + a[i] * (1.0 - sa));
                    db[i] = dh[i] * a[i] * sa;
                }
                for (int i = 0; i < I; ++i) {
                    size_t row = ((size_t)e * I + i) * d;
                    for (int j = 0; j < d; ++j)
                        dxt[j] += da[i] * load_elem(W1, dtype, row + j) +
                                  db[i] * load_elem(W3, dtype, row + j);
                }
            }
            /* Softmax backward: g_k = p_{c_k}; dL/dr_e = p_e (dg_e - sum_k g_k dg_k). */
            double sdot = 0.0;
            for (int k = 0; k < K; ++k) sdot += g[(size_t)t * K + k] * dg[k];
            double *drt = dr + (size_t)t * E;
            for (int e = 0; e < E; ++e) drt[e] = 0.0;
            if (renorm) {
                for (int k = 0; k < K; ++k) {
                    const size_t o = (size_t)t * K + k;
                    drt[cand[o]] = g[o] * (dg[k] - sdot);
                }
            } else {
                const double *rt = r + (size_t)t * E;
                const double mx = rt[cand[(size_t)t * K]];
                double den = 0.0;
                for (int e = 0; e < E; ++e) den += exp(rt[e] - mx);
                for (int e = 0; e < E; ++e) drt[e] = -exp(rt[e] - mx) / den * sdot;
                for (int k = 0; k < K; ++k) {
                    const size_t o = (size_t)t * K + k;
                    drt[cand[o]] += g[o] * dg[k];
                }
            }
            for (int e = 0; e < E; ++e) {
                if (drt[e] == 0.0) continue;
                for (int j = 0; j < d; ++j)
                    dxt[j] += drt[e] * load_elem(W_gate, dtype, (size_t)e * d + j);
            }
            if (W_mask) {
                for (int k = 0; k < K; ++k) {
                    const size_t o = (size_t)t * K + k;
                    for (int j = 0; j < d; ++j)
                        dxt[j] += dzk[o] * load_elem(W_mask, dtype, (size_t)cand[o] * d + j);
                }
            }
            for (int j = 0; j < d; ++j)
                if (!isfinite(dxt[j])) bad |= 2;
        }
        free(xt);
        free(dyt);
        free(a);
        free(b);
        free(dh);
        free(dg);
    }
    if (bad & 1) { rc = -1; goto done; }
    if (bad) { rc = -2; goto done; }

    /* Router gradients: dWg[e] = sum_t dr[t][e] x_t; dWm[e] = sum over the
     * (t, k) with c = e of dz x_t. */
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int e = 0; e < E; ++e) {
        double *gw = dWg + (size_t)e * d;
        double *mw = W_mask && dWm ? dWm + (size_t)e * d : NULL;
        for (int j = 0; j < d; ++j) {
            gw[j] = 0.0;
            if (mw) mw[j] = 0.0;
        }
        for (int t = 0; t < T; ++t) {
            const double c = dr[(size_t)t * E + e];
            if (c != 0.0)
                for (int j = 0; j < d; ++j) gw[j] += c * load_elem(x, dtype, (size_t)t * d + j);
            if (!mw) continue;
            for (int k = 0; k < K; ++k) {
                const size_t o = (size_t)t * K + k;
                if (cand[o] != e) continue;
                for (int j = 0; j < d; ++j)
                    mw[j] += dzk[o] * load_elem(x, dtype, (size_t)t * d + j);
            }
        }
    }

    /* Expert weight gradients of the selected experts, kept pairs only. */
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int s = 0; s < n_sel; ++s) {
        const int e = sel ? sel[s] : s;
        double *g1 = dW1 ? dW1 + (size_t)s * I * d : NULL;
        double *g3 = dW3 ? dW3 + (size_t)s * I * d : NULL;
        double *g2 = dW2 ? dW2 + (size_t)s * d * I : NULL;
        if (g1) memset(g1, 0, sizeof(double) * (size_t)I * d);
        if (g3) memset(g3, 0, sizeof(double) * (size_t)I * d);
        if (g2) memset(g2, 0, sizeof(double) * (size_t)d * I);
        for (int t = 0; t < T; ++t) {
            for (int k = 0; k < K; ++k) {
                const size_t o = (size_t)t * K + k;
                if (idx[o] != e) continue; /* masked or another expert */
                const double *da = das + o * I, *db = dbs + o * I, *h = hs + o * I;
                for (int i = 0; i < I; ++i)
                    for (int j = 0; j < d; ++j) {
                        const double xj = load_elem(x, dtype, (size_t)t * d + j);
                        if (g1) g1[(size_t)i * d + j] += da[i] * xj;
                        if (g3) g3[(size_t)i * d + j] += db[i] * xj;
                    }
                if (g2)
                    for (int j = 0; j < d; ++j) {
                        const double c = w[o] * load_elem(dy, dtype, (size_t)t * d + j);
                        for (int i = 0; i < I; ++i) g2[(size_t)j * I + i] += c * h[i];
                    }
            }
        }
    }
    if (u) memcpy(u, uk, sizeof(double) * TK);
    if (dz) memcpy(dz, dzk, sizeof(double) * TK);
done:
    free(r); free(zl); free(cand); free(idx); free(g); free(w); free(uk); free(dzk); free(dr);
    free(hs); free(das); free(dbs);
    return rc;
}
