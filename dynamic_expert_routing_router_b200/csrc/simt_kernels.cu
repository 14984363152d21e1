// simt_kernels.cu -- the CUDA-core stages of the BEAM MoE layer:
//   topk_mask   Top-K, softmax, binary mask and aggregation per token
//               (BEAM §3.2 Eq. 4-7), per-expert counts and kept histogram
//   permute     expert-token grouping of the kept pairs only (masked pairs
//               are left out of the count, so they are never scheduled)
//   gather      token rows copied into expert order for the grouped GEMMs
//   combine     y = sum_k w_k * E_{c_k}(x) over kept candidates (Eq. 8)
// and the fp32 path (router and expert GEMMs on CUDA cores) for BEAM_F32.
#include <cuda_bf16.h>

#include <climits>

#include "beam_internal.h"
#include "beam_ptx.cuh"
#include "grouping.cuh"
#include "topk_token.cuh"

namespace beam {

namespace {


// ------------------------------------------------------------ top-K + mask --
//
// A block takes `tpb` tokens at a time.  Phase 1: all threads add the router's
// split-K partial logits for those tokens (independent float4 loads, summed in
// split order) into shared memory, and export them when asked.  Phase 2: one
// warp per token; lane l holds the logits of experts l, l+32, ...  K rounds of
// a warp arg-max (ties -> lower expert id) give the candidates in descending
// order.  renorm: softmax over the candidates (Eq. 4); else over all E.  The
// mask keeps candidate k iff its pre-sigmoid value z >= thr = logit(tau)
// (Eq. 6, tau = 0.5 <=> thr = 0; NaN is not kept); w = g * m (Eq. 7).  Counts and the histogram are gathered in shared
// memory and added to global memory once per block.
constexpr int kTopkMaxTok = 8;

template <int EPL>
__global__ void __launch_bounds__(256) topk_mask_kernel(const TopkArgs a, int tpb) {
    __shared__ int s_counts[kMaxE];
    __shared__ int s_counts_all[kMaxE];
    __shared__ int s_hist[kMaxK + 1];
    __shared__ __align__(16) float s_logit[kTopkMaxTok][2 * kMaxE];
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) s_counts[i] = s_counts_all[i] = 0;
    if (threadIdx.x <= a.K) s_hist[threadIdx.x] = 0;
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();
    if (a.hdr && blockIdx.x == 0 && threadIdx.x == 0) {
        // The whole router grid has finished: this call's error word starts
        // from the router's status, and the router word is reset.
        const int rs = a.hdr[kHdrErrRouter];
        a.hdr[kHdrErr] = rs == kRouterTimeoutTag ? DEV_ERR_TIMEOUT : DEV_OK;
        a.hdr[kHdrErrRouter] = 0;
    }

    const int warp = threadIdx.x >> 5;
    const int E2 = 2 * a.E;
    const int cols = a.has_mask ? E2 : a.E;  // columns that hold logits
    const long long slab = (long long)a.T * E2;
    const bool vec = (E2 % 4 == 0) && (cols % 4 == 0);

    for (int t0 = blockIdx.x * tpb; t0 < a.T; t0 += gridDim.x * tpb) {
        const int nt = min(tpb, a.T - t0);
        // ---- phase 1: split sums -> shared memory
        if (vec) {
            const int c4n = cols / 4;
            for (int v = threadIdx.x; v < nt * c4n; v += blockDim.x) {
                const int tt = v / c4n, c4 = v - tt * c4n;
                const float4 *pr =
                    reinterpret_cast<const float4 *>(a.partial + (long long)(t0 + tt) * E2) + c4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
                for (int sp = 0; sp < a.S; ++sp) {
                    const float4 q = __ldg(pr + sp * (slab / 4));
                    acc.x += q.x;
                    acc.y += q.y;
                    acc.z += q.z;
                    acc.w += q.w;
                }
                reinterpret_cast<float4 *>(&s_logit[tt][0])[c4] = acc;
                if (a.logits)
                    reinterpret_cast<float4 *>(a.logits + (long long)(t0 + tt) * E2)[c4] = acc;
            }
        } else {
            for (int v = threadIdx.x; v < nt * cols; v += blockDim.x) {
                const int tt = v / cols, c = v - tt * cols;
                const float *pr = a.partial + (long long)(t0 + tt) * E2 + c;
                float acc = 0.0f;
                for (int sp = 0; sp < a.S; ++sp) acc += __ldg(pr + sp * slab);
                s_logit[tt][c] = acc;
                if (a.logits) a.logits[(long long)(t0 + tt) * E2 + c] = acc;
            }
        }
        __syncthreads();
        // ---- phase 2: one warp per token
        if (warp < nt) {
            const long long o = (long long)(t0 + warp) * a.K;
            topk_token<EPL>(s_logit[warp], a.E, a.K, a.renorm, a.has_mask, a.thr, a.idx + o,
                            a.w + o, a.cand ? a.cand + o : nullptr, a.gk ? a.gk + o : nullptr,
                            s_counts, a.counts_all ? s_counts_all : nullptr, s_hist);
        }
        __syncthreads();  // s_logit is rewritten by the next tokens
    }
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) {
        if (s_counts[i]) atomicAdd(&a.counts[i], s_counts[i]);
        if (a.counts_all && s_counts_all[i]) atomicAdd(&a.counts_all[i], s_counts_all[i]);
    }
    if (a.hist && threadIdx.x <= a.K && s_hist[threadIdx.x]) atomicAdd(&a.hist[threadIdx.x], s_hist[threadIdx.x]);
}

// ----------------------------------------------------------------- permute --
//
// Block e lists the kept pairs of expert e in token order.  Every block
// derives the padded offsets from counts[] (exclusive sums over lower
// experts), so no separate scan kernel is needed.  Rows of expert e:
// [off_e, off_e + roundup(count_e, BN)); padding rows get pair = -1.  The
// tile list holds one entry per BN rows of a non-empty expert.
//
// With a row copy (x, xp set), R blocks share an expert: each one repeats the
// listing (identical values, so the duplicate writes agree) and then copies
// every R-th group of its rows of x into xp, one warp per row.
constexpr int kPermThreads = kGroupThreads;

__global__ void __launch_bounds__(kPermThreads) permute_kernel(const PermuteArgs a) {
    __shared__ GroupSmem sm;
    const int e = blockIdx.x / a.R, replica = blockIdx.x % a.R;
    const int tid = threadIdx.x, warp = tid >> 5;
    griddep_wait();
    griddep_launch_dependents();

    int c = 0;
    if (tid < a.E) c = a.counts[tid];
    const int padded = (c + a.BN - 1) / a.BN * a.BN;
    const int ntile = (c + a.BN - 1) / a.BN;
    const int off_e = group_block_sum(tid < e ? padded : 0, sm);
    const int toff_e = group_block_sum(tid < e ? ntile : 0, sm);
    // sub-tiles (sub_bn < BN): the same rows, in tiles of sub_bn rows
    const int nsub = a.tiles_sub ? (c + a.sub_bn - 1) / a.sub_bn : 0;
    const int soff_e = a.tiles_sub ? group_block_sum(tid < e ? nsub : 0, sm) : 0;
    if (e == 0) {
        const int tot_rows = group_block_sum(padded, sm);
        const int tot_tiles = group_block_sum(ntile, sm);
        const int tot_pairs = group_block_sum(c, sm);
        const int tot_sub = a.tiles_sub ? group_block_sum(nsub, sm) : 0;
        if (tid == 0) {
            a.meta[0] = tot_tiles;
            a.meta[1] = tot_rows;
            a.meta[2] = tot_pairs;
            if (a.tiles_sub) a.meta[3] = tot_sub;
        }
    }
    const int count_e = a.counts[e];
    const int listed = list_expert_pairs(a.idx, a.T, a.K, e, off_e, a.pair, a.pair_pos, sm);
    if (tid == 0 && listed != count_e) atomicExch(a.err, DEV_ERR_INTERNAL);

    const int padded_e = (count_e + a.BN - 1) / a.BN * a.BN;
    for (int r = count_e + tid; r < padded_e; r += kPermThreads) a.pair[off_e + r] = -1;
    const int ntile_e = padded_e / a.BN;
    for (int j = tid; j < ntile_e; j += kPermThreads) {
        const int rows = min(a.BN, count_e - j * a.BN);
        a.tiles[toff_e + j] = make_int4(e, off_e + j * a.BN, rows, 0);
        a.tile_done[toff_e + j] = 0;
    }
    if (a.tiles_sub)
        for (int j = tid; j * a.sub_bn < count_e; j += kPermThreads)
            a.tiles_sub[soff_e + j] =
                make_int4(e, off_e + j * a.sub_bn, min(a.sub_bn, count_e - j * a.sub_bn), 0);

    if (a.xp == nullptr) return;
    // Row copy.  The pair entries read back were written by this block (the
    // listing ends with a barrier); padding rows are not copied, they only
    // feed padding columns of the GEMMs, which are never stored.
    copy_listed_rows(a.x, a.xp, a.pair, off_e, count_e, replica * kGroupWarps + warp,
                     a.R * kGroupWarps, a.K, a.row_vec);
}

// ---------------------------------------------------- chunked grouping --
//
// The same grouping for large batches without a row copy, in two launches
// over chunks of CT consecutive tokens (the per-expert listing above scans
// every token once per expert).  Count: per chunk, the kept pairs of each
// expert.  Place: a chunk's pairs of expert e start at off_e plus the pairs
// of e in earlier chunks; within the chunk they follow token order (a bit per
// token and expert, ranks by popcount).  Same rows, same order, same tiles as
// the listing: every pair of expert e sits at off_e + (its token's rank among
// e's tokens).
constexpr int kChunkThreads = 256;

// Tokens per chunk: 64, 128 or 256 (the chunk's token bits fit 8 words), at
// most 256 chunks; 0 when T is too large for that.
int group_chunk_tokens(int T) {
    for (int ct = 64; ct <= 256; ct *= 2)
        if ((T + ct - 1) / ct <= 256) return ct;
    return 0;
}

__global__ void __launch_bounds__(kChunkThreads) group_count_kernel(const int *idx, int T, int K,
                                                                  int E, int CT,
                                                                  int *chunk_cnt) {
    __shared__ int s_cnt[kMaxE];
    for (int e = threadIdx.x; e < E; e += kChunkThreads) s_cnt[e] = 0;
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();
    const int t0 = blockIdx.x * CT, t1 = min(T, t0 + CT);
    for (long long i = (long long)t0 * K + threadIdx.x; i < (long long)t1 * K; i += kChunkThreads) {
        const int e = idx[i];
        if (e >= 0) atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    // expert-major: expert e's chunk counts are contiguous (pitch ncp)
    const int ncp = (gridDim.x + 3) & ~3;
    for (int e = threadIdx.x; e < E; e += kChunkThreads)
        chunk_cnt[(long long)e * ncp + blockIdx.x] = s_cnt[e];
}

// Exclusive prefixes over the threads of the block (kChunkThreads) of N
// values at once; tot[i] gets the sum of v[i].  Uses s_tmp[N][8].
template <int N>
__device__ __forceinline__ void chunk_block_scan(const int (&v)[N], int (&pre)[N], int (&tot)[N],
                                                 int (*s_tmp)[kChunkThreads / 32]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        x[i] = v[i];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, x[i], off);
            if (lane >= off) x[i] += o;
        }
    }
    __syncthreads();
    if (lane == 31)
#pragma unroll
        for (int i = 0; i < N; ++i) s_tmp[i][warp] = x[i];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) {
        int base = 0, all = 0;
#pragma unroll
        for (int w = 0; w < kChunkThreads / 32; ++w) {
            if (w < warp) base += s_tmp[i][w];
            all += s_tmp[i][w];
        }
        pre[i] = base + x[i] - v[i];
        tot[i] = all;
    }
}

__global__ void __launch_bounds__(kChunkThreads) group_place_kernel(const PermuteArgs a, int CT,
                                                                  const int *chunk_cnt) {
    __shared__ int s_base[kMaxE];   // first row of this chunk's pairs of each expert
    __shared__ int s_off[kMaxE], s_toff[kMaxE], s_soff[kMaxE];
    __shared__ unsigned s_mask[kMaxE][8];  // tokens of the chunk per expert (CT <= 256)
    __shared__ int s_tmp[4][kChunkThreads / 32];
    const int tid = threadIdx.x, c = blockIdx.x, nchunk = gridDim.x;
    griddep_wait();
    griddep_launch_dependents();
    // per-expert offsets over the padded rows, tiles and sub-tiles (E <= 256)
    const int cnt = tid < a.E ? a.counts[tid] : 0;
    const int ntile = (cnt + a.BN - 1) / a.BN;
    const int nsub = a.tiles_sub ? (cnt + a.sub_bn - 1) / a.sub_bn : 0;
    const int vals[4] = {ntile * a.BN, ntile, nsub, cnt};
    int pre[4], tot[4];
    chunk_block_scan<4>(vals, pre, tot, s_tmp);
    const int off = pre[0], toff = pre[1], soff = pre[2];
    const int tot_rows = tot[0], tot_tiles = tot[1], tot_sub = tot[2], tot_pairs = tot[3];
    if (tid < a.E) {
        s_off[tid] = off;
        s_toff[tid] = toff;
        s_soff[tid] = soff;
    }
    for (int i = tid; i < a.E * 8; i += kChunkThreads) s_mask[i / 8][i % 8] = 0u;
    const int ncp = (nchunk + 3) & ~3;
    if (tid < a.E) {
        // this expert's pairs in earlier chunks: its contiguous counts, four
        // chunks per load
        const int4 *row = reinterpret_cast<const int4 *>(chunk_cnt + (long long)tid * ncp);
        int before = 0;
#pragma unroll 8
        for (int q4 = 0; q4 < (c + 3) / 4; ++q4) {
            const int4 v = row[q4];
            const int q = 4 * q4;
            before += (q < c ? v.x : 0) + (q + 1 < c ? v.y : 0) + (q + 2 < c ? v.z : 0) +
                      (q + 3 < c ? v.w : 0);
        }
        s_base[tid] = off + before;
    }
    __syncthreads();
    if (c == 0 && tid == 0) {
        a.meta[0] = tot_tiles;
        a.meta[1] = tot_rows;
        a.meta[2] = tot_pairs;
        if (a.tiles_sub) a.meta[3] = tot_sub;
    }
    __syncthreads();
    const int t0 = c * CT, t1 = min(a.T, t0 + CT);
    for (long long i = (long long)t0 * a.K + tid; i < (long long)t1 * a.K; i += kChunkThreads) {
        const int e = a.idx[i];
        if (e >= 0) {
            const int lt = int(i / a.K) - t0;
            atomicOr(&s_mask[e][lt >> 5], 1u << (lt & 31));
        }
    }
    __syncthreads();
    for (long long i = (long long)t0 * a.K + tid; i < (long long)t1 * a.K; i += kChunkThreads) {
        const int e = a.idx[i];
        if (e >= 0) {
            const int lt = int(i / a.K) - t0, wd = lt >> 5;
            int rank = __popc(s_mask[e][wd] & ((1u << (lt & 31)) - 1u));
            for (int q = 0; q < wd; ++q) rank += __popc(s_mask[e][q]);
            const int pos = s_base[e] + rank;
            a.pair[pos] = int(i);
            a.pair_pos[i] = pos;
        }
    }
    // Experts e = c, c + nchunk, ...: padding rows, tiles, sub-tiles, and the
    // check that the chunks' counts add up to the expert's count.
    for (int e = c; e < a.E; e += nchunk) {
        const int count_e = a.counts[e];
        if (tid < 32) {  // the chunks' counts of e add up to its count
            int listed = 0;
            for (int q = tid; q < nchunk; q += 32) listed += chunk_cnt[(long long)e * ncp + q];
#pragma unroll
            for (int off2 = 16; off2 > 0; off2 >>= 1)
                listed += __shfl_xor_sync(0xffffffffu, listed, off2);
            if (tid == 0 && listed != count_e) atomicExch(a.err, DEV_ERR_INTERNAL);
        }
        const int padded = (count_e + a.BN - 1) / a.BN * a.BN;
        for (int r = count_e + tid; r < padded; r += kChunkThreads) a.pair[s_off[e] + r] = -1;
        for (int j = tid; j * a.BN < count_e; j += kChunkThreads) {
            a.tiles[s_toff[e] + j] =
                make_int4(e, s_off[e] + j * a.BN, min(a.BN, count_e - j * a.BN), 0);
            a.tile_done[s_toff[e] + j] = 0;
        }
        if (a.tiles_sub)
            for (int j = tid; j * a.sub_bn < count_e; j += kChunkThreads)
                a.tiles_sub[s_soff[e] + j] = make_int4(e, s_off[e] + j * a.sub_bn,
                                                       min(a.sub_bn, count_e - j * a.sub_bn), 0);
    }
}

// ------------------------------------------------------------------ gather --
// One warp per permuted row, 16-byte vectors; padding rows are skipped (they
// only feed padding columns of the GEMMs, which are never stored).
__global__ void __launch_bounds__(256) gather_kernel(const uint4 *x, const int *pair,
                                                     const int *meta, int K, int row_vec,
                                                     uint4 *xp) {
    griddep_wait();
    griddep_launch_dependents();
    const int rows = meta[1];
    const int lane = threadIdx.x & 31;
    for (int r = blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += gridDim.x * 8) {
        const int pr = pair[r];
        if (pr < 0) continue;
        const uint4 *src = x + (long long)(pr / K) * row_vec;
        uint4 *dst = xp + (long long)r * row_vec;
        int v = lane;
        for (; v + 96 < row_vec; v += 128) {  // four 16-byte loads in flight per lane
            const uint4 a0 = __ldg(src + v), a1 = __ldg(src + v + 32);
            const uint4 a2 = __ldg(src + v + 64), a3 = __ldg(src + v + 96);
            dst[v] = a0;
            dst[v + 32] = a1;
            dst[v + 64] = a2;
            dst[v + 96] = a3;
        }
        for (; v < row_vec; v += 32) dst[v] = __ldg(src + v);
    }
}

// ----------------------------------------------------------------- combine --
// A group of threads per token; each thread owns 8-feature chunks.  The kept
// candidates' fp32 expert outputs are added in slot order k = 0..K-1 in fp32,
// then rounded once to the output type.

// 8 floats through the read-only path (the data is not written in the kernel).
__device__ __forceinline__ void load8_ro(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p + 4));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&v)[8]) {
    uint4 raw;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4 *>(p) = raw;
}
__device__ __forceinline__ void store8(float *p, const float (&v)[8]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// G threads per token (a power of two, 32..256), 256 / G tokens per block
// and pass: the group's first warp lists the token's kept slots in slot order
// (ballot, no serial loop), then every thread of the group owns 8-feature
// chunks v = tig, tig + G, ...  Large batches take small groups, so that
// every token of the batch is in flight at once; small batches take whole
// blocks, so that a token's rows are read by many threads.
template <typename Tout, int G>
__global__ void __launch_bounds__(256) combine_kernel(const float *Y, const int *idx,
                                                      const float *w, const int *pair_pos, int T,
                                                      int K, int d, const float *Ys, int n_shared,
                                                      Tout *out, int *hdr) {
    constexpr int TPB = 256 / G;
    __shared__ int s_row[TPB][kMaxK];
    __shared__ float s_w[TPB][kMaxK];
    __shared__ int s_n[TPB];
    const int nvec = d / 8;
    const int grp = threadIdx.x / G, tig = threadIdx.x % G, lane = threadIdx.x & 31;
    griddep_wait();
    griddep_launch_dependents();
    if (hdr && blockIdx.x == 0 && threadIdx.x == 0) {
        // Every kernel of the call has finished (both streams joined before
        // this launch): fold the shared experts' timeout tag, reset the word.
        if (hdr[kHdrErrShared] == kSharedTimeoutTag) atomicExch(hdr + kHdrErr, DEV_ERR_TIMEOUT);
        hdr[kHdrErrShared] = 0;
    }
    for (int t0 = blockIdx.x * TPB; t0 < T; t0 += gridDim.x * TPB) {
        const int t = t0 + grp;
        // G == 32: each warp owns its tokens and its slot lists; nothing is
        // shared between warps, so they never wait for one another
        if (G == 32) __syncwarp();
        else __syncthreads();  // the slot lists are rewritten below
        if (tig < 32) {  // kept candidates of token t, in slot order
            int row = -1;
            float wk = 0.0f;
            if (t < T && lane < K) {
                // three independent loads; a masked slot's pair_pos and w
                // are read but not used
                const long long o = (long long)t * K + lane;
                const int e = idx[o], pp = pair_pos[o];
                const float ww = w[o];
                if (e >= 0) {
                    row = pp;
                    wk = ww;
                }
            }
            const unsigned kept = __ballot_sync(0xffffffffu, row >= 0);
            if (row >= 0) {
                const int p = __popc(kept & ((1u << lane) - 1u));
                s_row[grp][p] = row;
                s_w[grp][p] = wk;
            }
            if (lane == 0) s_n[grp] = __popc(kept);
        }
        if (G == 32) __syncwarp();
        else __syncthreads();
        if (t < T) {
            const int n = s_n[grp];
            const int *rows = s_row[grp];
            const float *ws = s_w[grp];
#pragma unroll 2
            for (int v = tig; v < nvec; v += G) {
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                int j = 0;
                for (; j + 4 <= n; j += 4) {  // four rows in flight, added in slot order
                    float y[4][8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) load8_ro(Y + (long long)rows[j + q] * d + v * 8, y[q]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float wk = ws[j + q];
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wk, y[q][i], acc[i]);
                    }
                }
                for (; j < n; ++j) {
                    float y[8];
                    load8_ro(Y + (long long)rows[j] * d + v * 8, y);
                    const float wk = ws[j];
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = fmaf(wk, y[i], acc[i]);
                }
                for (int sx = 0; sx < n_shared; ++sx) {  // shared experts, weight 1, in order
                    float y[8];
                    load8_ro(Ys + ((long long)sx * T + t) * d + v * 8, y);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] += y[i];
                }
                store8(out + (long long)t * d + v * 8, acc);
            }
        }
    }
}

// --------------------------------------------- shared experts: SwiGLU ----
// H[i] = SiLU(sum_j A[j][i]) * (sum_j B[j][i]), splits j in order, one bf16
// rounding: the shared experts' gate/up GEMM with its reduction split.  The
// same expression as the tensor-core epilogue's.
__global__ void __launch_bounds__(256) shared_swiglu_kernel(const float4 *A, const float4 *B,
                                                            int splits, long long n4,
                                                            uint2 *H) {
    griddep_wait();
    griddep_launch_dependents();
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n4; i += 256ll * gridDim.x) {
        float4 a = __ldg(A + i), b = __ldg(B + i);
        for (int j = 1; j < splits; ++j) {
            const float4 aj = __ldg(A + j * n4 + i), bj = __ldg(B + j * n4 + i);
            a.x += aj.x;
            a.y += aj.y;
            a.z += aj.z;
            a.w += aj.w;
            b.x += bj.x;
            b.y += bj.y;
            b.z += bj.z;
            b.w += bj.w;
        }
        const auto sm = [](float g, float u) { return g / (1.0f + __expf(-g)) * u; };
        const __nv_bfloat162 h0 = __floats2bfloat162_rn(sm(a.x, b.x), sm(a.y, b.y));
        const __nv_bfloat162 h1 = __floats2bfloat162_rn(sm(a.z, b.z), sm(a.w, b.w));
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t *>(&h0);
        o.y = *reinterpret_cast<const uint32_t *>(&h1);
        H[i] = o;
    }
}

// ---------------------------------------------------------- fp32 path -----
// Plain shared-memory tiled SIMT kernels for BEAM_F32 (small layers).  Each
// output is one fp32 accumulator summed over the reduction index in order.
constexpr int kT = 16;

__global__ void __launch_bounds__(256) router_f32_kernel(const float *x, const float *Wg,
                                                         const float *Wm, int T, int d, int E,
                                                         int J, float *logits, ZeroRegion z0,
                                                         ZeroRegion z1, ZeroRegion z2) {
    if (blockIdx.x == 0 && blockIdx.y == 0) {
        const int tid = threadIdx.y * kT + threadIdx.x;
        const ZeroRegion zr[3] = {z0, z1, z2};
        for (int r = 0; r < 3; ++r)
            if (zr[r].ptr)
                for (int i = tid; i < zr[r].count; i += kT * kT) zr[r].ptr[i] = 0;
    }
    __shared__ float xs[kT][kT + 1];
    __shared__ float ws[kT][kT + 1];
    const int t = blockIdx.x * kT + threadIdx.y;
    const int j = blockIdx.y * kT + threadIdx.x;
    const int jl = blockIdx.y * kT + threadIdx.y;  // weight row this thread loads
    const float *wrow = nullptr;
    if (jl < J) wrow = jl < E ? Wg + (long long)jl * d : Wm + (long long)(jl - E) * d;
    float acc = 0.0f;
    for (int k0 = 0; k0 < d; k0 += kT) {
        const int tl = blockIdx.x * kT + threadIdx.y;
        const int k = k0 + threadIdx.x;
        xs[threadIdx.y][threadIdx.x] = (tl < T && k < d) ? x[(long long)tl * d + k] : 0.0f;
        ws[threadIdx.y][threadIdx.x] = (wrow && k < d) ? wrow[k] : 0.0f;
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kT; ++kk) acc = fmaf(xs[threadIdx.y][kk], ws[threadIdx.x][kk], acc);
        __syncthreads();
    }
    if (t < T && j < J) logits[(long long)t * 2 * E + j] = acc;
}

__device__ __forceinline__ float silu_mul_f32(float g, float u) {
    return g / (1.0f + expf(-g)) * u;
}

// GEMM1 (fp32): H[row] = SiLU(xp[row] W1_e^T) * (xp[row] W3_e^T) for the rows
// of one tile; block (column block, tile).  A, B (or null): the two
// pre-activations as well, for the backward pass.
__global__ void __launch_bounds__(256) gemm1_f32_kernel(const float *xp, const float *W1,
                                                        const float *W3, const int4 *tiles,
                                                        const int *meta, int d, int I, float *H,
                                                        float *A, float *B) {
    const int ti = blockIdx.x;
    if (ti >= meta[0]) return;
    const int4 tile = tiles[ti];
    const int e = tile.x, row0 = tile.y, rows = tile.z;
    __shared__ float xs[kT][kT + 1];
    __shared__ float w1s[kT][kT + 1];
    __shared__ float w3s[kT][kT + 1];
    const int col = blockIdx.y * kT + threadIdx.x;
    const int wl = blockIdx.y * kT + threadIdx.y;  // weight row this thread loads
    for (int rr = 0; rr < rows; rr += kT) {
        float ga = 0.0f, ub = 0.0f;
        for (int k0 = 0; k0 < d; k0 += kT) {
            const int k = k0 + threadIdx.x;
            const int r = rr + threadIdx.y;
            xs[threadIdx.y][threadIdx.x] =
                (r < rows && k < d) ? xp[(long long)(row0 + r) * d + k] : 0.0f;
            const bool okw = wl < I && k < d;
            w1s[threadIdx.y][threadIdx.x] = okw ? W1[((long long)e * I + wl) * d + k] : 0.0f;
            w3s[threadIdx.y][threadIdx.x] = okw ? W3[((long long)e * I + wl) * d + k] : 0.0f;
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kT; ++kk) {
                ga = fmaf(xs[threadIdx.y][kk], w1s[threadIdx.x][kk], ga);
                ub = fmaf(xs[threadIdx.y][kk], w3s[threadIdx.x][kk], ub);
            }
            __syncthreads();
        }
        const int r = rr + threadIdx.y;
        if (r < rows && col < I) {
            H[(long long)(row0 + r) * I + col] = silu_mul_f32(ga, ub);
            if (A) {
                A[(long long)(row0 + r) * I + col] = ga;
                B[(long long)(row0 + r) * I + col] = ub;
            }
        }
    }
}

// GEMM2 (fp32): Y[row] = H[row] W2_e^T.
__global__ void __launch_bounds__(256) gemm2_f32_kernel(const float *H, const float *W2,
                                                        const int4 *tiles, const int *meta, int d,
                                                        int I, float *Y) {
    const int ti = blockIdx.x;
    if (ti >= meta[0]) return;
    const int4 tile = tiles[ti];
    const int e = tile.x, row0 = tile.y, rows = tile.z;
    __shared__ float hs[kT][kT + 1];
    __shared__ float w2s[kT][kT + 1];
    const int col = blockIdx.y * kT + threadIdx.x;
    const int wl = blockIdx.y * kT + threadIdx.y;
    for (int rr = 0; rr < rows; rr += kT) {
        float acc = 0.0f;
        for (int k0 = 0; k0 < I; k0 += kT) {
            const int k = k0 + threadIdx.x;
            const int r = rr + threadIdx.y;
            hs[threadIdx.y][threadIdx.x] =
                (r < rows && k < I) ? H[(long long)(row0 + r) * I + k] : 0.0f;
            w2s[threadIdx.y][threadIdx.x] =
                (wl < d && k < I) ? W2[((long long)e * d + wl) * I + k] : 0.0f;
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kT; ++kk) acc = fmaf(hs[threadIdx.y][kk], w2s[threadIdx.x][kk], acc);
            __syncthreads();
        }
        const int r = rr + threadIdx.y;
        if (r < rows && col < d) Y[(long long)(row0 + r) * d + col] = acc;
    }
}

}  // namespace

cudaError_t launch_topk_mask(const TopkArgs &a, int n_sm, cudaStream_t stream) {
    if (a.T <= 0) return cudaSuccess;
    // Tokens per block: one at decode sizes (more blocks, more loads in
    // flight), up to kTopkMaxTok for large batches.
    int tpb = (a.T + 127) / 128;
    if (tpb > kTopkMaxTok) tpb = kTopkMaxTok;
    int blocks = (a.T + tpb - 1) / tpb;
    if (blocks > 8 * n_sm) blocks = 8 * n_sm;
    const int epl = (a.E + 31) / 32;
    if (epl <= 1)
        return launch_pdl(topk_mask_kernel<1>, dim3(blocks), dim3(256), 0, stream, a, tpb);
    if (epl <= 2)
        return launch_pdl(topk_mask_kernel<2>, dim3(blocks), dim3(256), 0, stream, a, tpb);
    if (epl <= 4)
        return launch_pdl(topk_mask_kernel<4>, dim3(blocks), dim3(256), 0, stream, a, tpb);
    return launch_pdl(topk_mask_kernel<8>, dim3(blocks), dim3(256), 0, stream, a, tpb);
}

cudaError_t launch_permute(const PermuteArgs &a, cudaStream_t stream) {
    return launch_pdl(permute_kernel, dim3(a.E * a.R), dim3(kPermThreads), 0, stream, a);
}

bool group_chunked_fits(int T) { return group_chunk_tokens(T) > 0; }

cudaError_t launch_group_chunked(const PermuteArgs &a, int *chunk_cnt, cudaStream_t stream) {
    if (a.T <= 0) return cudaSuccess;
    const int CT = group_chunk_tokens(a.T);
    if (CT == 0) return cudaErrorInvalidValue;
    const int nchunk = (a.T + CT - 1) / CT;
    cudaError_t e = launch_pdl(group_count_kernel, dim3(nchunk), dim3(kChunkThreads), 0, stream,
                               a.idx, a.T, a.K, a.E, CT, chunk_cnt);
    if (e != cudaSuccess) return e;
    return launch_pdl(group_place_kernel, dim3(nchunk), dim3(kChunkThreads), 0, stream, a, CT,
                      static_cast<const int *>(chunk_cnt));
}

cudaError_t launch_gather(const void *x, const int *pair, const int *meta, int K,
                          long long row_bytes, int p_cap, void *xp, int n_sm,
                          cudaStream_t stream) {
    int blocks = (p_cap + 7) / 8;
    if (blocks > 8 * n_sm) blocks = 8 * n_sm;
    if (blocks <= 0) return cudaSuccess;
    return launch_pdl(gather_kernel, dim3(blocks), dim3(256), 0, stream,
                      static_cast<const uint4 *>(x), pair, meta, K, int(row_bytes / 16),
                      static_cast<uint4 *>(xp));
}

template <typename Tout>
cudaError_t launch_combine_t(const float *Y, const int *idx, const float *w, const int *pair_pos,
                             int T, int K, int d, const float *Ys, int n_shared, Tout *out,
                             int *hdr, int n_sm, cudaStream_t stream) {
    // Threads per token: the largest G that keeps every token of the batch
    // in flight at once (8 blocks of 256 threads per SM), and no more than
    // the token's 8-feature chunks need.
    const long long slots = 8LL * n_sm * 256;
    int G = 256;
    while (G > 32 && (long long)T * G > slots) G >>= 1;
    while (G > 32 && d / 8 <= G / 2) G >>= 1;
    const int tpb = 256 / G;
    long long blocks = ((long long)T + tpb - 1) / tpb;
    if (blocks > 8LL * n_sm) blocks = 8LL * n_sm;
    const dim3 grid(static_cast<unsigned>(blocks)), block(256);
    switch (G) {
        case 256: return launch_pdl(combine_kernel<Tout, 256>, grid, block, 0, stream, Y, idx, w,
                                    pair_pos, T, K, d, Ys, n_shared, out, hdr);
        case 128: return launch_pdl(combine_kernel<Tout, 128>, grid, block, 0, stream, Y, idx, w,
                                    pair_pos, T, K, d, Ys, n_shared, out, hdr);
        case 64: return launch_pdl(combine_kernel<Tout, 64>, grid, block, 0, stream, Y, idx, w,
                                   pair_pos, T, K, d, Ys, n_shared, out, hdr);
        default: return launch_pdl(combine_kernel<Tout, 32>, grid, block, 0, stream, Y, idx, w,
                                   pair_pos, T, K, d, Ys, n_shared, out, hdr);
    }
}

cudaError_t launch_combine(int dtype, const float *Y, const int *idx, const float *w,
                           const int *pair_pos, int T, int K, int d, const float *Ys,
                           int n_shared, void *out, int *hdr, int n_sm, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    if (dtype == BEAM_BF16)
        return launch_combine_t(Y, idx, w, pair_pos, T, K, d, Ys, n_shared,
                                static_cast<__nv_bfloat16 *>(out), hdr, n_sm, stream);
    return launch_combine_t(Y, idx, w, pair_pos, T, K, d, Ys, n_shared, static_cast<float *>(out),
                            hdr, n_sm, stream);
}

cudaError_t launch_shared_swiglu(const float *A, const float *B, int splits, long long n,
                                 void *H, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    const long long n4 = n / 4;  // n: a multiple of 128 (I_shared)
    long long blocks = (n4 + 255) / 256;
    if (blocks > 4 * kNominalSMs) blocks = 4 * kNominalSMs;
    return launch_pdl(shared_swiglu_kernel, dim3(unsigned(blocks)), dim3(256), 0, stream,
                      reinterpret_cast<const float4 *>(A), reinterpret_cast<const float4 *>(B),
                      splits, n4, static_cast<uint2 *>(H));
}

cudaError_t launch_router_f32(const float *x, const float *Wg, const float *Wm, int T, int d,
                              int E, float *partial, const ZeroRegion (&zero)[3],
                              cudaStream_t stream) {
    const int J = Wm ? 2 * E : E;
    dim3 grid(T > 0 ? (T + kT - 1) / kT : 1, (J + kT - 1) / kT);
    router_f32_kernel<<<grid, dim3(kT, kT), 0, stream>>>(x, Wg, Wm, T, d, E, J, partial, zero[0],
                                                         zero[1], zero[2]);
    return cudaGetLastError();
}

cudaError_t launch_gemm1_f32(const float *xp, const float *W1, const float *W3, const int4 *tiles,
                             const int *meta, int tiles_cap, int d, int I, float *H,
                             cudaStream_t stream, float *A, float *B) {
    dim3 grid(tiles_cap, (I + kT - 1) / kT);
    gemm1_f32_kernel<<<grid, dim3(kT, kT), 0, stream>>>(xp, W1, W3, tiles, meta, d, I, H, A, B);
    return cudaGetLastError();
}

cudaError_t launch_gemm2_f32(const float *H, const float *W2, const int4 *tiles, const int *meta,
                             int tiles_cap, int d, int I, float *Y, cudaStream_t stream) {
    dim3 grid(tiles_cap, (d + kT - 1) / kT);
    gemm2_f32_kernel<<<grid, dim3(kT, kT), 0, stream>>>(H, W2, tiles, meta, d, I, Y);
    return cudaGetLastError();
}

}  // namespace beam
