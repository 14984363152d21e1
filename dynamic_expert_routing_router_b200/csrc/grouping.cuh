// grouping.cuh -- listing of one expert's kept (token, slot) pairs in token
// order, by one block of kGroupThreads threads.  Shared by the grouping kernel
// of the layer (rows padded per expert for the grouped GEMMs) and the
// expert-parallel dispatch kernel (rows unpadded, grouped by destination).
// A masked pair has index -1 and matches no expert, so it is never listed
// (the news article on BEAM, §5: masked entries are left out of the count).
#pragma once

namespace beam {

constexpr int kGroupThreads = 256;
constexpr int kGroupSub = 4;  // sub-chunks of kGroupThreads tokens per pass
constexpr int kGroupWarps = kGroupThreads / 32;

struct GroupSmem {
    int red[kGroupWarps];
    int wcnt[kGroupSub * kGroupWarps];
    int wpre[kGroupSub * kGroupWarps];
    int total;
};

// Sum of v over the block (every thread gets the total).
__device__ __forceinline__ int group_block_sum(int v, GroupSmem &sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    __syncthreads();
    if (lane == 0) sm.red[warp] = v;
    __syncthreads();
    int total = 0;
#pragma unroll
    for (int i = 0; i < kGroupWarps; ++i) total += sm.red[i];
    return total;
}

// Rows off_e, off_e + 1, ... receive the pairs (t, k) with idx[t*K + k] == e,
// tokens ascending: pair[row] = t*K + k (if pair is not null) and
// pair_pos[t*K + k] = row.  Each pass covers kGroupSub * kGroupThreads tokens
// as coalesced sub-chunks; ranks follow (sub-chunk, warp, lane), i.e. token
// order.  A token matches expert e in at most one slot (the top-K candidates
// are distinct).  Returns the number of pairs listed; ends with a barrier.
__device__ __forceinline__ int list_expert_pairs(const int *idx, int T, int K, int e, int off_e,
                                                 int *pair, int *pair_pos, GroupSmem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int running = 0;
    for (int base = 0; base < T; base += kGroupThreads * kGroupSub) {
        int km[kGroupSub];
        unsigned bal[kGroupSub];
#pragma unroll
        for (int q = 0; q < kGroupSub; ++q) {
            const int t = base + q * kGroupThreads + tid;
            km[q] = -1;
            if (t < T) {
                const int *row = idx + (long long)t * K;
                for (int k = 0; k < K; ++k)
                    if (row[k] == e) km[q] = k;
            }
            bal[q] = __ballot_sync(0xffffffffu, km[q] >= 0);
            if (lane == 0) sm.wcnt[q * kGroupWarps + warp] = __popc(bal[q]);
        }
        __syncthreads();
        if (tid == 0) {
            int acc = 0;
            for (int i = 0; i < kGroupSub * kGroupWarps; ++i) {
                sm.wpre[i] = acc;
                acc += sm.wcnt[i];
            }
            sm.total = acc;
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < kGroupSub; ++q) {
            if (km[q] >= 0) {
                const int t = base + q * kGroupThreads + tid;
                const int pos = off_e + running + sm.wpre[q * kGroupWarps + warp] +
                                __popc(bal[q] & ((1u << lane) - 1u));
                if (pair) pair[pos] = t * K + km[q];
                pair_pos[(long long)t * K + km[q]] = pos;
            }
        }
        running += sm.total;
        __syncthreads();
    }
    return running;
}

// Copy token rows into listed order, one warp per row, 16-byte vectors: row
// off + r (r = first, first + step, ... < n) gets x row pair[off + r] / K.
__device__ __forceinline__ void copy_listed_rows(const uint4 *x, uint4 *dst_rows, const int *pair,
                                                 int off, int n, int first, int step, int K,
                                                 int row_vec) {
    const int lane = threadIdx.x & 31;
    for (int r = first; r < n; r += step) {
        const int pr = pair[off + r];
        const uint4 *src = x + (long long)(pr / K) * row_vec;
        uint4 *dst = dst_rows + (long long)(off + r) * row_vec;
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

}  // namespace beam
