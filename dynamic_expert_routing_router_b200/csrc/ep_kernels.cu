// ep_kernels.cu -- the device side of expert parallelism for the BEAM layer:
// G ranks each own E/G experts (rank r owns experts [r E/G, (r+1) E/G)).
//
//   ep_dispatch   lists the KEPT (token, slot) pairs in the order of the
//                 layer's grouping -- expert ascending, token ascending --
//                 which groups them by destination rank, copies each pair's
//                 token row into a send buffer and records, per pair, its send
//                 row and the local id of its expert on the destination.  A
//                 masked pair is never listed, so the mask cuts the rows that
//                 cross the interconnect as it cuts the expert work (news
//                 article on BEAM, §5: masked entries are left out of the
//                 expert-token grouping).
//   set_routing   turns received rows (one local expert id per row, -1 = none)
//                 into the routing arrays of a K = 1 layer call with weight 1,
//                 so that the layer's own grouping, expert GEMMs and combine
//                 compute Y = E_e(x) per received row.
#include "beam_internal.h"
#include "beam_ptx.cuh"
#include "grouping.cuh"

namespace beam {

namespace {

// One block per (expert, replica): every replica repeats the listing
// (identical values) and copies every R-th group of the expert's rows.
__global__ void __launch_bounds__(kGroupThreads) ep_dispatch_kernel(const EpDispatchArgs a) {
    __shared__ GroupSmem sm;
    const int e = blockIdx.x / a.R, replica = blockIdx.x % a.R;
    const int tid = threadIdx.x, warp = tid >> 5;
    griddep_wait();
    griddep_launch_dependents();
    int c = 0;
    if (tid < a.E) c = a.counts[tid];
    const int off_e = group_block_sum(tid < e ? c : 0, sm);  // unpadded rows
    const int El = a.E / a.G;
    if (e == 0 && replica == 0 && tid < a.G) {
        int n = 0;  // kept pairs bound for rank tid
        for (int j = tid * El; j < (tid + 1) * El; ++j) n += a.counts[j];
        a.send_counts[tid] = n;
    }
    const int count_e = a.counts[e];
    const int listed = list_expert_pairs(a.idx, a.T, a.K, e, off_e, a.send_pair, a.pair_pos, sm);
    if (tid == 0 && listed != count_e) atomicExch(a.err, DEV_ERR_INTERNAL);
    const int local = e - (e / El) * El;
    if (replica == 0)
        for (int r = tid; r < count_e; r += kGroupThreads) a.send_expert[off_e + r] = local;
    copy_listed_rows(a.x, a.send_rows, a.send_pair, off_e, count_e, replica * kGroupWarps + warp,
                     a.R * kGroupWarps, a.K, a.row_vec);
}

// Received rows -> routing of a K = 1 call: idx = the row's local expert (or
// -1), w = 1, per-expert counts and the kept histogram (hist[0] rows without
// an expert, hist[1] rows with one).  counts and hist start at zero.  An id
// outside [-1, E) is an error (DEV_ERR_INTERNAL) and the row is skipped.
__global__ void __launch_bounds__(256) set_routing_kernel(const int *expert_id, int N, int E,
                                                          int *idx, float *w, int *counts,
                                                          int *hist, int *err) {
    __shared__ int s_counts[kMaxE];
    __shared__ int s_hist[2];
    for (int i = threadIdx.x; i < E; i += blockDim.x) s_counts[i] = 0;
    if (threadIdx.x < 2) s_hist[threadIdx.x] = 0;
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
        int e = expert_id[i];
        if (e < -1 || e >= E) {
            atomicExch(err, DEV_ERR_INTERNAL);
            e = -1;
        }
        idx[i] = e;
        w[i] = e >= 0 ? 1.0f : 0.0f;
        if (e >= 0) atomicAdd(&s_counts[e], 1);
        atomicAdd(&s_hist[e >= 0 ? 1 : 0], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x)
        if (s_counts[i]) atomicAdd(&counts[i], s_counts[i]);
    if (threadIdx.x < 2 && s_hist[threadIdx.x]) atomicAdd(&hist[threadIdx.x], s_hist[threadIdx.x]);
}

}  // namespace

cudaError_t launch_ep_dispatch(const EpDispatchArgs &a, cudaStream_t stream) {
    if (a.T <= 0) return cudaSuccess;
    return launch_pdl(ep_dispatch_kernel, dim3(a.E * a.R), dim3(kGroupThreads), 0, stream, a);
}

cudaError_t launch_set_routing(const int *expert_id, int N, int E, int *idx, float *w, int *counts,
                               int *hist, int *err, int n_sm, cudaStream_t stream) {
    if (N <= 0) return cudaSuccess;
    int blocks = (N + 255) / 256;
    if (blocks > 4 * n_sm) blocks = 4 * n_sm;
    return launch_pdl(set_routing_kernel, dim3(blocks), dim3(256), 0, stream, expert_id, N, E, idx,
                      w, counts, hist, err);
}

}  // namespace beam
