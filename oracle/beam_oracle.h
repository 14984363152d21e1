/*
 * beam_oracle.h -- fp64 CPU oracle of the BEAM-masked MoE layer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  This library is the slow, plain definition that
 * the CUDA path is checked against.  Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it.  It shares no code, header,
 * table or helper with the CUDA library, and never calls into it.
 *
 * Method source: "BEAM: Binary Expert Activation Masking for Dynamic Routing
 * in MoE" (arXiv 2605.14438, Chinese translation of the HTML version),
 * §3.1 Eq. (1)-(3) and §3.2 Eq. (4)-(8).
 *
 * Storage dtypes of the inputs: ORACLE_BF16 (raw bfloat16 bits in uint16) or
 * ORACLE_F32.  Every value is widened to double before any arithmetic.
 *
 * Return codes: 0 = ok, -1 = bad argument, -2 = non-finite value met in the
 * data the computation actually used (the oracle rejects such inputs).
 */
#ifndef BEAM_ORACLE_H
#define BEAM_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_BF16 = 0, ORACLE_F32 = 1 };

/* Router logits, §3.2 step 1 (r = R(x) = x W) and step 2 (pre-sigmoid x W_m).
 * x [T,d]; W_gate, W_mask [E,d] (row e holds column e of the paper's d x N
 * matrix).  r, z [T,E] fp64.  W_mask may be NULL, then z is not written. */
int oracle_logits(int T, int d, int E, int dtype, const void *x, const void *W_gate,
                  const void *W_mask, double *r, double *z);

/* Routing decisions and weights from given logits, Eq. (4)-(7).
 * r [T,E]; z [T,E] or NULL (mask disabled: every candidate kept).
 * tau_logit: the binarisation threshold tau of Eq. (6) given as its logit,
 * ln(tau / (1 - tau)); 0 is the paper's tau = 0.5.  sigmoid(z) >= tau holds
 * exactly when z >= tau_logit (sigmoid is increasing), so the test is taken on
 * z and both implementations compare against the same number.
 * renorm = 1: softmax over the Top-K entries (Eq. 4).  renorm = 0: softmax
 * over all E logits, restricted to the Top-K.
 * Outputs (any may be NULL except idx):
 *   cand [T,K]   candidate experts in descending logit order, ties -> lower id
 *   g    [T,K]   softmax weight of each candidate (before the mask)
 *   idx  [T,K]   cand, or -1 where the binary mask is 0
 *   w    [T,K]   g * m (Eq. 7, no renormalisation after the mask)
 *   counts [E]   kept (token, expert) pairs per expert
 *   hist [K+1]   tokens by number of kept candidates */
int oracle_route(int T, int E, int K, int renorm, double tau_logit, const double *r,
                 const double *z, int32_t *cand, double *g, int32_t *idx, double *w,
                 int32_t *counts, int32_t *hist);

/* Same decisions fed with fp32 logits (as exported by another implementation):
 * r, z are float [T,E]; they are widened exactly to double first. */
int oracle_route_f32(int T, int E, int K, int renorm, double tau_logit, const float *r,
                     const float *z, int32_t *cand, double *g, int32_t *idx, double *w,
                     int32_t *counts, int32_t *hist);

/* Expert-token grouping: kept pairs listed expert by expert (ascending), and
 * within an expert by token (ascending).  Each entry is t*K + k.
 * offsets [E+1] (unpadded), pairs [>= number of kept pairs]. */
int oracle_permutation(int T, int K, int E, const int32_t *idx, int32_t *offsets,
                       int32_t *pairs);

/* Masked weighted sum of SwiGLU experts, Eq. (3) with delta = SiLU and Eq. (8),
 * for tokens t in [t_begin, t_end).  x [T,d]; W1 (gate), W3 (up) [E,I,d];
 * W2 (down) [E,d,I]; idx, w [T,K] from oracle_route.  y [(t_end-t_begin), d].
 * Tokens with no kept candidate get y = 0.  nthreads <= 0 uses the OpenMP
 * default. */
int oracle_experts(int T, int d, int E, int I, int K, int dtype, const void *x,
                   const void *W1, const void *W3, const void *W2, const int32_t *idx,
                   const double *w, int t_begin, int t_end, double *y, int nthreads);

/* Shared experts (news article on BEAM, §5: models with always-on shared
 * experts keep running them for every token, all-masked ones included).
 * READING: each of the n_shared SwiGLU experts is added with weight 1 after
 * the routed sum.  W1s, W3s [n_shared, Is, d]; W2s [n_shared, d, Is].
 * Adds sum_s E_s(x_t) to y[t - t_begin] for t in [t_begin, t_end). */
int oracle_shared_experts(int T, int d, int n_shared, int Is, int dtype, const void *x,
                          const void *W1s, const void *W3s, const void *W2s, int t_begin,
                          int t_end, double *y, int nthreads);

/* Training-mode backward of the layer (news article on BEAM, §4: the
 * straight-through estimator and the sparsity penalty).  Objective:
 *   L = sum_t <dy_t, y_t> + beta * sum_t sum_{k<K} sigmoid(z_{t,c_k})
 * with y the forward of Eq. (8).  READINGS (the pages describe both terms in
 * words only): the estimator passes the gradient straight through the
 * threshold of Eq. (6), dm/dm_hat = 1, and keeps the sigmoid's derivative; the
 * penalty adds up the K candidates' m_hat of every token.  Every candidate's
 * expert is evaluated, kept or not, because u_{t,k} = <dy_t, E_{c_k}(x_t)>
 * enters the mask gradient of a masked candidate too.  ste = 0 leaves the
 * straight-through term out: the exact gradient of L with the candidates and
 * the mask held fixed, which finite differences can check.
 * Inputs in the storage dtype (dy too); W_mask may be NULL (no mask: m = 1,
 * no penalty).  Outputs fp64, overwritten: dx [T,d]; dWg, dWm [E,d] (dWm
 * untouched without a mask); u, dz [T,K] or NULL; the expert gradients of the
 * n_sel experts listed in sel (sel NULL: all E in order), each NULL-able:
 * dW1, dW3 [n_sel,I,d], dW2 [n_sel,d,I].  Returns -2 on a non-finite value.
 * r_in, z_in [T,E]: logits to route with instead of computing them (another
 * implementation's, widened), or NULL; z_in is used only with a mask. */
int oracle_backward(int T, int d, int E, int I, int K, int renorm, int dtype, double tau_logit,
                    double beta, int ste, const void *x, const void *W_gate, const void *W_mask,
                    const void *W1, const void *W3, const void *W2, const void *dy, int n_sel,
                    const int32_t *sel, const double *r_in, const double *z_in, double *dx,
                    double *dWg, double *dWm, double *dW1, double *dW3, double *dW2, double *u,
                    double *dz, int nthreads);

/* Threads the OpenMP runtime would use by default (for reporting). */
int oracle_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif
