// topk_token.cuh -- top-K, softmax, binary mask and aggregation of one token
// by one warp (BEAM §3.2 Eq. 4-7).  The calling warp must be converged (every
// shuffle below is full-mask).
#pragma once

#include <climits>

namespace beam {

// lg: the token's logits in shared memory, gate logits [0, E), mask
// pre-activations [E, 2E) (read only with a mask).  Lane l holds experts l,
// l+32, ...; K rounds of a warp arg-max (ties -> lower expert id) give the
// candidates in descending order.  renorm: softmax over the candidates
// (Eq. 4); else over all E.  Candidate k is kept iff its z >= thr = logit(tau)
// (Eq. 6; NaN is not kept); w = g * m (Eq. 7).  A -inf gate logit weighs 0,
// and a token whose candidates are all -inf gets weights 0 (its softmax is
// 0/0; it then contributes nothing).  Writes idx_t[k] / w_t[k] and,
// when given, cand_t[k] / gk_t[k]; adds to the shared counters.
template <int EPL>
__device__ __forceinline__ void topk_token(const float *lg, int E, int K, int renorm,
                                           int has_mask, float thr, int *idx_t, float *w_t,
                                           int *cand_t, float *gk_t, int *s_counts,
                                           int *s_counts_all, int *s_hist) {
    constexpr unsigned kAll = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    float r[EPL], z[EPL];
    unsigned taken = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int j = lane + 32 * i;
        r[i] = -INFINITY;
        z[i] = 0.0f;
        if (j < E) {
            const float rs = lg[j];
            r[i] = (rs != rs) ? -INFINITY : rs;  // NaN never wins a slot
            if (has_mask) z[i] = lg[E + j];
        } else {
            taken |= 1u << i;
        }
    }

    // Selection keys: larger logit -> larger unsigned key (-0 counts as +0,
    // since the two compare equal); 0 marks an entry that can no longer win.
    // Each round takes the largest key over the warp with one redux.sync and
    // the lowest expert id holding it with another (ties -> lower id).
    unsigned key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const float v = r[i] == 0.0f ? 0.0f : r[i];
        const unsigned b = __float_as_uint(v);
        key[i] = ((taken >> i) & 1u) ? 0u : ((b & 0x80000000u) ? ~b : (b | 0x80000000u));
    }
    int my_cand = -1;
    float my_e = 0.0f, my_z = 0.0f, rmax = 0.0f, denom = 0.0f;
    for (int k = 0; k < K; ++k) {
        unsigned bk = 0u;
        int bi = INT_MAX;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (key[i] > bk) {  // i ascending: the lowest id among equal keys
                bk = key[i];
                bi = lane + 32 * i;
            }
        const unsigned wk = __reduce_max_sync(kAll, bk);
        const int wi = int(__reduce_min_sync(kAll, bk == wk ? unsigned(bi) : 0xffffffffu));
        const float bv = __uint_as_float((wk & 0x80000000u) ? (wk & 0x7fffffffu) : ~wk);
        float oz = 0.0f;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (lane + 32 * i == wi) {
                oz = z[i];
                key[i] = 0u;
            }
        const float bz = __shfl_sync(kAll, oz, wi & 31);
        if (k == 0) rmax = bv;
        // a -inf logit has weight 0 (Eq. 1); this also keeps a row whose
        // every logit is -inf (rmax = -inf) free of inf - inf
        const float ek = bv == -INFINITY ? 0.0f : expf(bv - rmax);
        denom += ek;
        if (lane == k) {
            my_cand = wi;
            my_e = ek;
            my_z = bz;
        }
    }
    if (!renorm) {
        float part = 0.0f;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (lane + 32 * i < E && r[i] != -INFINITY) part += expf(r[i] - rmax);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(kAll, part, off);
        denom = part;  // identical on every lane (pairwise sums commute exactly)
    }
    const bool kept = (lane < K) && (!has_mask || my_z >= thr);
    if (lane < K) {
        const float g = denom > 0.0f ? my_e / denom : 0.0f;  // every logit -inf: weights 0
        idx_t[lane] = kept ? my_cand : -1;
        w_t[lane] = kept ? g : 0.0f;
        if (kept) atomicAdd(&s_counts[my_cand], 1);
        if (cand_t) cand_t[lane] = my_cand;
        if (gk_t) gk_t[lane] = g;
        if (s_counts_all) atomicAdd(&s_counts_all[my_cand], 1);
    }
    const int nkept = __popc(__ballot_sync(kAll, kept));
    if (lane == 0) atomicAdd(&s_hist[nkept], 1);
}

}  // namespace beam
