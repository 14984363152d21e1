// backward.cu -- CUDA-core stages of the training-mode backward pass.
//
// Objective (news article on BEAM, §4, readings in the C ABI header):
//   L = sum_t <dy_t, y_t> + beta * sum_t sum_k sigmoid(z_{t,c_k}),
// trained through the straight-through estimator for the binarisation of
// Eq. (6): the forward uses the hard mask m, the backward takes dm/dm_hat = 1.
// The forward quantities needed here -- every candidate's gate/up
// pre-activations a, b and expert output E_k(x) -- come from the tensor-core
// kernels run over all candidates (grouped by expert, masked ones included).
//
//   token    per token: u_k = <dy, E_k(x)>, the mask gradient dz, the router
//            gradient dr (softmax backward, Eq. 4)
//   dh       kept rows: da, db from dh = w_k dy W2_e and a, b
//   dxp      kept rows: da W1_e + db W3_e (the expert part of dx)
//   dx       per token: dxp rows in slot order + W_gate^T dr + W_mask^T dz
//   dw13     dW1_e += sum da x, dW3_e += sum db x      (kept rows, in order)
//   dw2      dW2_e += sum w dy h                       (kept rows, in order)
//   drouter  dW_gate += dr^T x, dW_mask += dz^T x
// Every sum runs in a fixed order, so the gradients are bitwise repeatable.
#include <cuda_bf16.h>

#include <climits>

#include "beam_internal.h"
#include "beam_ptx.cuh"

namespace beam {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float load_f(const float *p, long long i) { return p[i]; }
__device__ __forceinline__ float load_f(const __nv_bfloat16 *p, long long i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ float sigm(float v) { return 1.0f / (1.0f + expf(-v)); }

// Rows of expert e in the candidate grouping: [first, first + count_all[e]).
// An expert's tiles are consecutive in the tile list and cover its rows in
// order; the first one is found by a block-wide scan.
__device__ int expert_first_row(const int4 *tiles, int ntiles, int e, int *s_first) {
    if (threadIdx.x == 0) *s_first = INT_MAX;
    __syncthreads();
    for (int i = threadIdx.x; i < ntiles; i += blockDim.x) {
        const int4 tl = tiles[i];
        if (tl.x == e) atomicMin(s_first, tl.y);
    }
    __syncthreads();
    return *s_first;
}

// ------------------------------------------------------------------- token --
template <typename TIn>
__global__ void __launch_bounds__(256) bw_token_kernel(const BwArgs a, const TIn *dy) {
    __shared__ int s_pos[kMaxK], s_cand[kMaxK];
    __shared__ float s_red[8][kMaxK];
    __shared__ float s_u[kMaxK];
    __shared__ float s_dg[kMaxE], s_gc[kMaxE];
    __shared__ float s_sdot, s_den;
    __shared__ float s_dred[8];
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.K, E = a.E, d = a.d;
    for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
        if (tid < K) {
            s_pos[tid] = a.pair_pos[(long long)t * K + tid];
            s_cand[tid] = a.cand[(long long)t * K + tid];
        }
        for (int e = tid; e < E; e += blockDim.x) s_dg[e] = s_gc[e] = 0.0f;
        __syncthreads();
        // u_k = <dy_t, Y[row of (t,k)]>: per-thread partial sums, then a fixed tree.
        float acc[kMaxK];
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) acc[k] = 0.0f;
        for (int j = tid; j < d; j += blockDim.x) {
            const float g = load_f(dy, (long long)t * d + j);
#pragma unroll
            for (int k = 0; k < kMaxK; ++k)
                if (k < K) acc[k] = fmaf(g, a.Y[(long long)s_pos[k] * d + j], acc[k]);
        }
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
            float v = acc[k];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
            if (lane == 0 && k < K) s_red[warp][k] = v;
        }
        __syncthreads();
        if (tid < K) {
            float v = 0.0f;
            for (int w8 = 0; w8 < 8; ++w8) v += s_red[w8][tid];
            s_u[tid] = v;
        }
        __syncthreads();
        // Per candidate (warp 0, lane k): mask gradient and dL/dg.
        if (warp == 0) {
            float dgk = 0.0f, gk = 0.0f;
            if (lane < K) {
                const long long o = (long long)t * K + lane;
                const float u = s_u[lane];
                gk = a.gk[o];
                const bool kept = a.idx[o] >= 0;
                dgk = kept ? u : 0.0f;
                float dzk = 0.0f;
                if (a.has_mask) {
                    const float s = sigm(a.logits[(long long)t * 2 * E + E + s_cand[lane]]);
                    dzk = (gk * u + a.beta) * s * (1.0f - s);
                }
                a.u[o] = u;
                a.dz[o] = dzk;
                s_dg[s_cand[lane]] = dgk;
                s_gc[s_cand[lane]] = gk;
            }
            float sd = gk * dgk;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sd += __shfl_xor_sync(kFull, sd, off);
            if (lane == 0) s_sdot = sd;
        }
        __syncthreads();
        const float sdot = s_sdot;
        if (a.renorm) {
            // Softmax over the candidates (Eq. 4): only they get a gradient.
            for (int e = tid; e < E; e += blockDim.x)
                a.dr[(long long)t * E + e] = s_gc[e] * (s_dg[e] - sdot);
        } else {
            // Softmax over all E logits: p_e for the others from the logits.
            const float *r = a.logits + (long long)t * 2 * E;
            const float rmax = r[s_cand[0]];
            float part = 0.0f;
            for (int e = tid; e < E; e += blockDim.x) part += expf(r[e] - rmax);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(kFull, part, off);
            if (lane == 0) s_dred[warp] = part;
            __syncthreads();
            if (tid == 0) {
                float den = 0.0f;
                for (int w8 = 0; w8 < 8; ++w8) den += s_dred[w8];
                s_den = den;
            }
            __syncthreads();
            for (int e = tid; e < E; e += blockDim.x) {
                const bool is_c = s_gc[e] != 0.0f;
                const float p = is_c ? s_gc[e] : expf(r[e] - rmax) / s_den;
                a.dr[(long long)t * E + e] = p * (s_dg[e] - sdot);
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------- kept-row tile products --
// For one tile of the candidate grouping and a 256-column slice, the kept rows
// r get C[r][n] = sum_k A[r][k] B_e[k][n] (+ A2 B2_e), where B_e is row-major
// [Kdim][N] at B + e * Kdim * N.  Threads: 4 row groups x 64 column groups,
// 4 x 4 outputs each; kept rows are compacted into groups of 16 first.
//   DH: A = dyp (dtype), B = W2 (Kdim = d, N = I); with dh = w C:
//       da = dh b SiLU'(a), db = dh SiLU(a) (a, b from the forward buffers)
//   DX: A = da, A2 = db (f32), B = W1, B2 = W3 (Kdim = I, N = d); dxp = C
enum { TG_DH = 0, TG_DX = 1 };
constexpr int kTgCols = 256, kTgKc = 16;

template <int MODE, typename TA, typename TB>
__global__ void __launch_bounds__(256) tile_product_kernel(const BwArgs a, const TA *A,
                                                           const TA *A2, const TB *B,
                                                           const TB *B2, int Kdim, int N) {
    __shared__ int s_rows[kMaxTileRows];
    __shared__ float s_w[kMaxTileRows];
    __shared__ int s_n;
    __shared__ float As[16][kTgKc + 1];
    __shared__ __align__(16) float Bs[kTgKc][kTgCols];
    griddep_wait();
    griddep_launch_dependents();
    const int ti = blockIdx.x;
    if (ti >= a.meta[0]) return;
    const int4 tile = a.tiles[ti];
    const int e = tile.x, row0 = tile.y, rows = tile.z;
    const int n0 = blockIdx.y * kTgCols;
    const int tid = threadIdx.x, tr = tid >> 6, tc = tid & 63;
    if (tid == 0) {
        int n = 0;
        for (int r = 0; r < rows; ++r) {
            const int pr = a.pair[row0 + r];
            if (pr >= 0 && a.idx[pr] >= 0) {  // kept candidate
                s_rows[n] = row0 + r;
                s_w[n] = a.w[pr];
                ++n;
            }
        }
        s_n = n;
    }
    __syncthreads();
    const int nk = s_n;
    const long long bstride = (long long)Kdim * N;
    for (int g0 = 0; g0 < nk; g0 += 16) {
        const int gn = min(16, nk - g0);
        const bool active = tr * 4 < gn;  // warp-uniform: 2 warps per row group
        float c[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) c[i][j] = 0.0f;
        for (int pass = 0; pass < (MODE == TG_DX ? 2 : 1); ++pass) {
            const TA *Ap = pass ? A2 : A;
            const TB *Bp = (pass ? B2 : B) + (long long)e * bstride;
            for (int k0 = 0; k0 < Kdim; k0 += kTgKc) {
                {   // A: 16 rows x 16 k, one element per thread
                    const int rr = tid >> 4, kk = tid & 15;
                    As[rr][kk] = (rr < gn && k0 + kk < Kdim)
                                     ? load_f(Ap, (long long)s_rows[g0 + rr] * Kdim + k0 + kk)
                                     : 0.0f;
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) {  // B: 16 k x 256 columns
                    const int idx = q * 256 + tid, kk = idx >> 8, nn = idx & 255;
                    Bs[kk][nn] = (n0 + nn < N && k0 + kk < Kdim)
                                     ? load_f(Bp, (long long)(k0 + kk) * N + n0 + nn)
                                     : 0.0f;
                }
                __syncthreads();
                if (active) {
#pragma unroll
                    for (int kk = 0; kk < kTgKc; ++kk) {
                        const float4 bv = *reinterpret_cast<const float4 *>(&Bs[kk][tc * 4]);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float av = As[tr * 4 + i][kk];
                            c[i][0] = fmaf(av, bv.x, c[i][0]);
                            c[i][1] = fmaf(av, bv.y, c[i][1]);
                            c[i][2] = fmaf(av, bv.z, c[i][2]);
                            c[i][3] = fmaf(av, bv.w, c[i][3]);
                        }
                    }
                }
                __syncthreads();
            }
        }
        if (active) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int lr = tr * 4 + i;
                if (lr >= gn) continue;
                const long long row = s_rows[g0 + lr];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = n0 + tc * 4 + j;
                    if (n >= N) continue;
                    const long long o = row * N + n;
                    if (MODE == TG_DH) {
                        const float dh = s_w[g0 + lr] * c[i][j];
                        const float av = a.A[o], bv = a.B[o], sa = sigm(av);
                        a.da[o] = dh * bv * sa * (1.0f + av * (1.0f - sa));
                        a.db[o] = dh * av * sa;
                    } else {
                        a.dxp[o] = c[i][j];
                    }
                }
            }
        }
    }
}

// ---------------------------------------------------------------------- dx --
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dx_kernel(const BwArgs a, const TIn *Wg,
                                                    const TIn *Wm) {
    __shared__ float s_dr[kMaxE];
    __shared__ int s_pos[kMaxK], s_cand[kMaxK];
    __shared__ float s_dz[kMaxK];
    __shared__ int s_kept[kMaxK];
    griddep_wait();
    griddep_launch_dependents();
    const int K = a.K, E = a.E, d = a.d;
    for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) s_dr[e] = a.dr[(long long)t * E + e];
        if (threadIdx.x < K) {
            const long long o = (long long)t * K + threadIdx.x;
            s_pos[threadIdx.x] = a.pair_pos[o];
            s_cand[threadIdx.x] = a.cand[o];
            s_dz[threadIdx.x] = a.dz[o];
            s_kept[threadIdx.x] = a.idx[o] >= 0;
        }
        __syncthreads();
        for (int j = threadIdx.x; j < d; j += blockDim.x) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k)  // expert part, kept slots in order
                if (s_kept[k]) acc += a.dxp[(long long)s_pos[k] * d + j];
            for (int e = 0; e < E; ++e) {  // W_gate^T dr
                const float c = s_dr[e];
                if (c != 0.0f) acc = fmaf(c, load_f(Wg, (long long)e * d + j), acc);
            }
            if (Wm)
                for (int k = 0; k < K; ++k)  // W_mask^T dz
                    acc = fmaf(s_dz[k], load_f(Wm, (long long)s_cand[k] * d + j), acc);
            a.dx[(long long)t * d + j] = acc;
        }
        __syncthreads();
    }
}

// -------------------------------------------------------- weight gradients --
// dW1_e[i] += sum over kept rows r of e (in order) da[r][i] x_r, likewise dW3
// with db.  Block (expert, 4 rows of I); threads over d.
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dw13_kernel(const BwArgs a, const TIn *xp, float *dW1,
                                                      float *dW3) {
    __shared__ int s_first;
    griddep_wait();
    griddep_launch_dependents();
    const int e = blockIdx.x;
    if (a.counts_kept[e] == 0) return;  // no kept pair: no gradient, rows untouched
    const int i0 = blockIdx.y * 4;
    const int first = expert_first_row(a.tiles, a.meta[0], e, &s_first);
    const int n = a.counts_all[e];
    const int d = a.d, I = a.I;
    constexpr int kCols = 8;  // d <= 2048 per pass of 256 threads
    for (int jb = 0; jb < d; jb += 256 * kCols) {
        float g1[4][kCols], g3[4][kCols];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < kCols; ++c) g1[i][c] = g3[i][c] = 0.0f;
        for (int r = first; r < first + n; ++r) {
            const int pr = a.pair[r];
            if (a.idx[pr] < 0) continue;  // masked candidate: no weight gradient
            float va[4], vb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool ok = i0 + i < I;
                va[i] = ok ? a.da[(long long)r * I + i0 + i] : 0.0f;
                vb[i] = ok ? a.db[(long long)r * I + i0 + i] : 0.0f;
            }
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                const int j = jb + c * 256 + threadIdx.x;
                const float xv = j < d ? load_f(xp, (long long)r * d + j) : 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    g1[i][c] = fmaf(va[i], xv, g1[i][c]);
                    g3[i][c] = fmaf(vb[i], xv, g3[i][c]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i0 + i >= I) continue;
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                const int j = jb + c * 256 + threadIdx.x;
                if (j >= d) continue;
                const long long o = ((long long)e * I + i0 + i) * d + j;
                dW1[o] += g1[i][c];
                dW3[o] += g3[i][c];
            }
        }
    }
}

// dW2_e[j] += sum over kept rows r of e (in order) w_r dy_r[j] h_r, with
// h = SiLU(a) b in fp32.  Block (expert, 8 rows of d); threads over I.
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dw2_kernel(const BwArgs a, const TIn *dyp, float *dW2) {
    __shared__ int s_first;
    griddep_wait();
    griddep_launch_dependents();
    const int e = blockIdx.x;
    if (a.counts_kept[e] == 0) return;
    const int j0 = blockIdx.y * 8;
    const int first = expert_first_row(a.tiles, a.meta[0], e, &s_first);
    const int n = a.counts_all[e];
    const int d = a.d, I = a.I;
    constexpr int kCols = 8;  // I <= 2048 per pass
    for (int ib = 0; ib < I; ib += 256 * kCols) {
        float g[8][kCols];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
#pragma unroll
            for (int c = 0; c < kCols; ++c) g[jj][c] = 0.0f;
        for (int r = first; r < first + n; ++r) {
            const int pr = a.pair[r];
            if (a.idx[pr] < 0) continue;
            const float wk = a.w[pr];
            float dv[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                dv[jj] = (j0 + jj < d) ? wk * load_f(dyp, (long long)r * d + j0 + jj) : 0.0f;
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                const int i = ib + c * 256 + threadIdx.x;
                float h = 0.0f;
                if (i < I) {
                    const float av = a.A[(long long)r * I + i], bv = a.B[(long long)r * I + i];
                    h = av * sigm(av) * bv;
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) g[jj][c] = fmaf(dv[jj], h, g[jj][c]);
            }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            if (j0 + jj >= d) continue;
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                const int i = ib + c * 256 + threadIdx.x;
                if (i < I) dW2[((long long)e * d + j0 + jj) * I + i] += g[jj][c];
            }
        }
    }
}

// dW_gate[e] += sum_t dr[t][e] x_t; dW_mask[e] += sum over the candidate rows
// of e (token order) dz x.  Block (expert, 256 columns of d).
template <typename TIn>
__global__ void __launch_bounds__(256) bw_drouter_kernel(const BwArgs a, const TIn *x,
                                                         const TIn *xp, float *dWg, float *dWm) {
    __shared__ int s_first;
    griddep_wait();
    griddep_launch_dependents();
    const int e = blockIdx.x;
    const int j = blockIdx.y * 256 + threadIdx.x;
    const int d = a.d, E = a.E, K = a.K;
    float gg = 0.0f;
    for (int t = 0; t < a.T; ++t) {
        const float c = a.dr[(long long)t * E + e];
        if (c != 0.0f && j < d) gg = fmaf(c, load_f(x, (long long)t * d + j), gg);
    }
    float gm = 0.0f;
    if (dWm) {
        const int first = a.counts_all[e] ? expert_first_row(a.tiles, a.meta[0], e, &s_first) : 0;
        for (int r = first; r < first + a.counts_all[e]; ++r) {
            const int pr = a.pair[r];
            const float c = a.dz[pr];
            if (j < d) gm = fmaf(c, load_f(xp, (long long)r * d + j), gm);
        }
    }
    (void)K;
    if (j < d) {
        dWg[(long long)e * d + j] += gg;
        if (dWm) dWm[(long long)e * d + j] += gm;
    }
}

}  // namespace

cudaError_t launch_backward_stages(const BwArgs &a, int dtype, const void *x, const void *xp,
                                   const void *dy, const void *dyp, const void *Wg,
                                   const void *Wm, const void *W1, const void *W3,
                                   const void *W2, float *dWg, float *dWm, float *dW1,
                                   float *dW3, float *dW2, int n_sm, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    const int tb = a.T < 8 * n_sm ? a.T : 8 * n_sm;
    const dim3 g_dh(a.tiles_cap, (a.I + kTgCols - 1) / kTgCols);
    const dim3 g_dx(a.tiles_cap, (a.d + kTgCols - 1) / kTgCols);
    const dim3 g_w13(a.E, (a.I + 3) / 4), g_w2(a.E, (a.d + 7) / 8), g_r(a.E, (a.d + 255) / 256);
    cudaError_t e;
    if (dtype == BEAM_BF16) {
        using T = __nv_bfloat16;
        const T *xb = static_cast<const T *>(x), *xpb = static_cast<const T *>(xp);
        const T *dyb = static_cast<const T *>(dy), *dypb = static_cast<const T *>(dyp);
        if ((e = launch_pdl(bw_token_kernel<T>, dim3(tb), dim3(256), 0, st, a, dyb))) return e;
        if ((e = launch_pdl(tile_product_kernel<TG_DH, T, T>, g_dh, dim3(256), 0, st, a, dypb,
                            dypb, static_cast<const T *>(W2), static_cast<const T *>(W2), a.d,
                            a.I)))
            return e;
        if ((e = launch_pdl(tile_product_kernel<TG_DX, float, T>, g_dx, dim3(256), 0, st, a,
                            static_cast<const float *>(a.da), static_cast<const float *>(a.db),
                            static_cast<const T *>(W1), static_cast<const T *>(W3), a.I, a.d)))
            return e;
        if ((e = launch_pdl(bw_dx_kernel<T>, dim3(tb), dim3(256), 0, st, a,
                            static_cast<const T *>(Wg), static_cast<const T *>(Wm))))
            return e;
        if ((e = launch_pdl(bw_dw13_kernel<T>, g_w13, dim3(256), 0, st, a, xpb, dW1, dW3)))
            return e;
        if ((e = launch_pdl(bw_dw2_kernel<T>, g_w2, dim3(256), 0, st, a, dypb, dW2))) return e;
        return launch_pdl(bw_drouter_kernel<T>, g_r, dim3(256), 0, st, a, xb, xpb, dWg, dWm);
    }
    using T = float;
    const T *xb = static_cast<const T *>(x), *xpb = static_cast<const T *>(xp);
    const T *dyb = static_cast<const T *>(dy), *dypb = static_cast<const T *>(dyp);
    if ((e = launch_pdl(bw_token_kernel<T>, dim3(tb), dim3(256), 0, st, a, dyb))) return e;
    if ((e = launch_pdl(tile_product_kernel<TG_DH, T, T>, g_dh, dim3(256), 0, st, a, dypb, dypb,
                        static_cast<const T *>(W2), static_cast<const T *>(W2), a.d, a.I)))
        return e;
    if ((e = launch_pdl(tile_product_kernel<TG_DX, float, T>, g_dx, dim3(256), 0, st, a,
                        static_cast<const float *>(a.da), static_cast<const float *>(a.db),
                        static_cast<const T *>(W1), static_cast<const T *>(W3), a.I, a.d)))
        return e;
    if ((e = launch_pdl(bw_dx_kernel<T>, dim3(tb), dim3(256), 0, st, a,
                        static_cast<const T *>(Wg), static_cast<const T *>(Wm))))
        return e;
    if ((e = launch_pdl(bw_dw13_kernel<T>, g_w13, dim3(256), 0, st, a, xpb, dW1, dW3))) return e;
    if ((e = launch_pdl(bw_dw2_kernel<T>, g_w2, dim3(256), 0, st, a, dypb, dW2))) return e;
    return launch_pdl(bw_drouter_kernel<T>, g_r, dim3(256), 0, st, a, xb, xpb, dWg, dWm);
}

}  // namespace beam
