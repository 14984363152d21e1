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

// Kept rows of one tile of the candidate grouping, compacted in order into
// s_row / s_w (row index, w = g m).  rows <= kMaxTileRows.
__device__ int stage_kept_rows(const BwArgs &a, int row0, int rows, int *s_flag, float *s_fw,
                               int *s_row, float *s_w, int *s_n) {
    for (int r = threadIdx.x; r < rows; r += blockDim.x) {
        const int pr = a.pair[row0 + r];
        const bool kept = pr >= 0 && a.idx[pr] >= 0;
        s_flag[r] = kept ? row0 + r : -1;
        s_fw[r] = kept ? a.w[pr] : 0.0f;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int n = 0;
        for (int r = 0; r < rows; ++r)
            if (s_flag[r] >= 0) {
                s_row[n] = s_flag[r];
                s_w[n] = s_fw[r];
                ++n;
            }
        *s_n = n;
    }
    __syncthreads();
    return *s_n;
}

// Eight consecutive elements as fp32 (16-byte aligned for bf16, 32 for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 raw = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    const float4 y = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}

// ------------------------------------------------- kept-row products (split) --
// For one tile and one split s of the reduction range, the kept rows r get
//   part[s][r][n] = sum_{k in split s} A[r][k] B_e[k][n]  (+ A2[r][k] B2_e[k][n])
// with B_e row-major [Kdim][N] at B + e * Kdim * N.  Each thread owns 8
// consecutive columns and streams them with one 16-byte load per k; the A rows
// (4 kept rows at a time) are staged in shared memory 512 k at a time.
//   DH: A = dyp, B = W2 (Kdim = d, N = I)
//   DX: A = da, A2 = db, B = W1, B2 = W3 (Kdim = I, N = d)
enum { TG_DH = 0, TG_DX = 1 };
constexpr int kRgKch = 512;

template <int MODE, typename TA, typename TB>
__global__ void __launch_bounds__(256) rowgemm_kernel(const BwArgs a, const TA *A, const TA *A2,
                                                      const TB *B, const TB *B2, int Kdim, int N,
                                                      int S) {
    __shared__ int s_flag[kMaxTileRows], s_row[kMaxTileRows], s_n;
    __shared__ float s_fw[kMaxTileRows], s_w[kMaxTileRows];
    __shared__ __align__(16) float As[4][kRgKch];
    __shared__ __align__(16) float A2s[MODE == TG_DX ? 4 : 1][MODE == TG_DX ? kRgKch : 4];
    griddep_wait();
    griddep_launch_dependents();
    const int ti = blockIdx.x, sp = blockIdx.y;
    if (ti >= a.meta[0]) return;
    const int4 tile = a.tiles[ti];
    const int e = tile.x;
    const int nk = stage_kept_rows(a, tile.y, tile.z, s_flag, s_fw, s_row, s_w, &s_n);
    if (nk == 0) return;
    const int kc = Kdim / S, k0 = sp * kc;
    const int NG = N / 8;
    const long long bstride = (long long)Kdim * N;
    const TB *Be = B + (long long)e * bstride;
    const TB *B2e = (MODE == TG_DX) ? B2 + (long long)e * bstride : nullptr;
    float *part = a.part + (long long)sp * a.p_cap * N;
    for (int g0 = 0; g0 < nk; g0 += 4) {
        const int gn = min(4, nk - g0);
        for (int cgb = 0; cgb < NG; cgb += blockDim.x) {
            const int cg = cgb + threadIdx.x;
            const bool active = cg < NG;
            float acc[4][8];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[r][c] = 0.0f;
            for (int kb = k0; kb < k0 + kc; kb += kRgKch) {
                const int kn = min(kRgKch, k0 + kc - kb);
                for (int q = threadIdx.x; q < 4 * kn; q += blockDim.x) {
                    const int r = q / kn, k = q - r * kn;
                    const long long ro = (r < gn) ? (long long)s_row[g0 + r] * Kdim : 0;
                    As[r][k] = (r < gn) ? load_f(A, ro + kb + k) : 0.0f;
                    if (MODE == TG_DX) A2s[r][k] = (r < gn) ? load_f(A2, ro + kb + k) : 0.0f;
                }
                __syncthreads();
                if (active) {
                    const TB *bp = Be + (long long)kb * N + cg * 8;
                    const TB *bp2 = (MODE == TG_DX) ? B2e + (long long)kb * N + cg * 8 : nullptr;
#pragma unroll 4
                    for (int k = 0; k < kn; ++k) {
                        float bv[8];
                        load8(bp + (long long)k * N, bv);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float av = As[r][k];
#pragma unroll
                            for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(av, bv[c], acc[r][c]);
                        }
                        if (MODE == TG_DX) {
                            load8(bp2 + (long long)k * N, bv);
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const float av = A2s[r][k];
#pragma unroll
                                for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(av, bv[c], acc[r][c]);
                            }
                        }
                    }
                }
                __syncthreads();
            }
            if (active) {
                for (int r = 0; r < gn; ++r) {
                    float *o = part + (long long)s_row[g0 + r] * N + cg * 8;
                    *reinterpret_cast<float4 *>(o) =
                        make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
                    *reinterpret_cast<float4 *>(o + 4) =
                        make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
                }
            }
        }
    }
}

// dh = w * (sum of the splits, in order); da = dh b SiLU'(a), db = dh SiLU(a),
// and h = SiLU(a) b in fp32, for the kept rows of a tile.
__global__ void __launch_bounds__(256) dh_finalize_kernel(const BwArgs a, int S) {
    __shared__ int s_flag[kMaxTileRows], s_row[kMaxTileRows], s_n;
    __shared__ float s_fw[kMaxTileRows], s_w[kMaxTileRows];
    griddep_wait();
    griddep_launch_dependents();
    const int ti = blockIdx.x;
    if (ti >= a.meta[0]) return;
    const int4 tile = a.tiles[ti];
    const int nk = stage_kept_rows(a, tile.y, tile.z, s_flag, s_fw, s_row, s_w, &s_n);
    const int I = a.I;
    const long long split = (long long)a.p_cap * I;
    for (int q = 0; q < nk; ++q) {
        const long long row = s_row[q];
        for (int i = threadIdx.x; i < I; i += blockDim.x) {
            const long long o = row * I + i;
            float c = 0.0f;
            for (int sp = 0; sp < S; ++sp) c += a.part[sp * split + o];
            const float dh = s_w[q] * c;
            const float av = a.A[o], bv = a.B[o], sa = sigm(av);
            a.da[o] = dh * bv * sa * (1.0f + av * (1.0f - sa));
            a.db[o] = dh * av * sa;
            a.h[o] = av * sa * bv;
        }
    }
}

// ---------------------------------------------------------------------- dx --
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dx_kernel(const BwArgs a, const TIn *Wg,
                                                    const TIn *Wm, int S) {
    __shared__ float s_dr[kMaxE];
    __shared__ int s_pos[kMaxK], s_cand[kMaxK];
    __shared__ float s_dz[kMaxK];
    __shared__ int s_kept[kMaxK];
    griddep_wait();
    griddep_launch_dependents();
    const int K = a.K, E = a.E, d = a.d;
    const long long split = (long long)a.p_cap * d;
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
            for (int k = 0; k < K; ++k)  // expert part: kept slots in order, splits in order
                if (s_kept[k]) {
                    float c = 0.0f;
                    for (int sp = 0; sp < S; ++sp) c += a.part[sp * split + (long long)s_pos[k] * d + j];
                    acc += c;
                }
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
// Kept rows of expert e (rows [first, first + n) of the candidate grouping),
// chunk [r0, r0 + cnt): compacted row indices into s_kr (returns how many).
constexpr int kWgChunk = 256;
__device__ int stage_expert_chunk(const BwArgs &a, int first, int r0, int cnt, int *s_flag,
                                  int *s_kr, int *s_n) {
    for (int q = threadIdx.x; q < cnt; q += blockDim.x) {
        const int r = first + r0 + q;
        s_flag[q] = a.idx[a.pair[r]] >= 0 ? r : -1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int n = 0;
        for (int q = 0; q < cnt; ++q)
            if (s_flag[q] >= 0) s_kr[n++] = s_flag[q];
        *s_n = n;
    }
    __syncthreads();
    return *s_n;
}

// dW1_e[i] += sum over kept rows (in order) da[r][i] x_r, dW3 likewise with db.
// Block (expert, 4 rows of I); each thread owns 8 consecutive columns of d.
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dw13_kernel(const BwArgs a, const TIn *xp, float *dW1,
                                                      float *dW3) {
    __shared__ int s_first, s_n;
    __shared__ int s_flag[kWgChunk], s_kr[kWgChunk];
    __shared__ float s_da[kWgChunk][4], s_db[kWgChunk][4];
    griddep_wait();
    griddep_launch_dependents();
    const int e = blockIdx.x;
    if (a.counts_kept[e] == 0) return;  // no kept pair: no gradient, rows untouched
    const int i0 = blockIdx.y * 4;
    const int first = expert_first_row(a.tiles, a.meta[0], e, &s_first);
    const int n = a.counts_all[e];
    const int d = a.d, I = a.I;
    for (int jb = 0; jb < d; jb += 8 * blockDim.x) {
        const int j = jb + threadIdx.x * 8;
        const bool active = j < d;
        float g1[4][8], g3[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < 8; ++c) g1[i][c] = g3[i][c] = 0.0f;
        for (int r0 = 0; r0 < n; r0 += kWgChunk) {
            const int nk = stage_expert_chunk(a, first, r0, min(kWgChunk, n - r0), s_flag, s_kr,
                                              &s_n);
            for (int q = threadIdx.x; q < 4 * nk; q += blockDim.x) {
                const int kq = q >> 2, i = q & 3;
                const bool ok = i0 + i < I;
                s_da[kq][i] = ok ? a.da[(long long)s_kr[kq] * I + i0 + i] : 0.0f;
                s_db[kq][i] = ok ? a.db[(long long)s_kr[kq] * I + i0 + i] : 0.0f;
            }
            __syncthreads();
            if (active) {
#pragma unroll 2
                for (int kq = 0; kq < nk; ++kq) {
                    float xv[8];
                    load8(xp + (long long)s_kr[kq] * d + j, xv);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float va = s_da[kq][i], vb = s_db[kq][i];
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            g1[i][c] = fmaf(va, xv[c], g1[i][c]);
                            g3[i][c] = fmaf(vb, xv[c], g3[i][c]);
                        }
                    }
                }
            }
            __syncthreads();
        }
        if (active) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (i0 + i >= I) continue;
                const long long o = ((long long)e * I + i0 + i) * d + j;
                float4 *p1 = reinterpret_cast<float4 *>(dW1 + o);
                float4 *p3 = reinterpret_cast<float4 *>(dW3 + o);
                float4 u0 = p1[0], u1 = p1[1], v0 = p3[0], v1 = p3[1];
                u0.x += g1[i][0]; u0.y += g1[i][1]; u0.z += g1[i][2]; u0.w += g1[i][3];
                u1.x += g1[i][4]; u1.y += g1[i][5]; u1.z += g1[i][6]; u1.w += g1[i][7];
                v0.x += g3[i][0]; v0.y += g3[i][1]; v0.z += g3[i][2]; v0.w += g3[i][3];
                v1.x += g3[i][4]; v1.y += g3[i][5]; v1.z += g3[i][6]; v1.w += g3[i][7];
                p1[0] = u0; p1[1] = u1; p3[0] = v0; p3[1] = v1;
            }
        }
    }
}

// dW2_e[j] += sum over kept rows (in order) w_r dy_r[j] h_r (h fp32 from the
// finalize step).  Block (expert, 8 rows of d); each thread owns 4 columns of I.
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dw2_kernel(const BwArgs a, const TIn *dyp, float *dW2) {
    __shared__ int s_first, s_n;
    __shared__ int s_flag[kWgChunk], s_kr[kWgChunk];
    __shared__ float s_dy[kWgChunk][8];
    griddep_wait();
    griddep_launch_dependents();
    const int e = blockIdx.x;
    if (a.counts_kept[e] == 0) return;
    const int j0 = blockIdx.y * 8;
    const int first = expert_first_row(a.tiles, a.meta[0], e, &s_first);
    const int n = a.counts_all[e];
    const int d = a.d, I = a.I;
    for (int ib = 0; ib < I; ib += 4 * blockDim.x) {
        const int i = ib + threadIdx.x * 4;
        const bool active = i < I;
        float g[8][4];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
#pragma unroll
            for (int c = 0; c < 4; ++c) g[jj][c] = 0.0f;
        for (int r0 = 0; r0 < n; r0 += kWgChunk) {
            const int nk = stage_expert_chunk(a, first, r0, min(kWgChunk, n - r0), s_flag, s_kr,
                                              &s_n);
            for (int q = threadIdx.x; q < 8 * nk; q += blockDim.x) {
                const int kq = q >> 3, jj = q & 7;
                const int r = s_kr[kq];
                const float wk = a.w[a.pair[r]];
                s_dy[kq][jj] = (j0 + jj < d) ? wk * load_f(dyp, (long long)r * d + j0 + jj) : 0.0f;
            }
            __syncthreads();
            if (active) {
#pragma unroll 2
                for (int kq = 0; kq < nk; ++kq) {
                    const float4 hv = *reinterpret_cast<const float4 *>(a.h + (long long)s_kr[kq] * I + i);
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        const float dv = s_dy[kq][jj];
                        g[jj][0] = fmaf(dv, hv.x, g[jj][0]);
                        g[jj][1] = fmaf(dv, hv.y, g[jj][1]);
                        g[jj][2] = fmaf(dv, hv.z, g[jj][2]);
                        g[jj][3] = fmaf(dv, hv.w, g[jj][3]);
                    }
                }
            }
            __syncthreads();
        }
        if (active) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                if (j0 + jj >= d) continue;
                float4 *p = reinterpret_cast<float4 *>(dW2 + ((long long)e * d + j0 + jj) * I + i);
                float4 v = *p;
                v.x += g[jj][0]; v.y += g[jj][1]; v.z += g[jj][2]; v.w += g[jj][3];
                *p = v;
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
    const int d = a.d, E = a.E;
    float gg = 0.0f;
    for (int t = 0; t < a.T; ++t) {
        const float c = a.dr[(long long)t * E + e];
        if (c != 0.0f && j < d) gg = fmaf(c, load_f(x, (long long)t * d + j), gg);
    }
    float gm = 0.0f;
    if (dWm) {
        const int first = a.counts_all[e] ? expert_first_row(a.tiles, a.meta[0], e, &s_first) : 0;
        for (int r = first; r < first + a.counts_all[e]; ++r) {
            const float c = a.dz[a.pair[r]];
            if (j < d) gm = fmaf(c, load_f(xp, (long long)r * d + j), gm);
        }
    }
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
    const dim3 g_dh(a.tiles_cap, a.S), g_fin(a.tiles_cap);
    const dim3 g_w13(a.E, (a.I + 3) / 4), g_w2(a.E, (a.d + 7) / 8), g_r(a.E, (a.d + 255) / 256);
    cudaError_t e;
    if (dtype == BEAM_BF16) {
        using T = __nv_bfloat16;
        const T *xb = static_cast<const T *>(x), *xpb = static_cast<const T *>(xp);
        const T *dyb = static_cast<const T *>(dy), *dypb = static_cast<const T *>(dyp);
        if ((e = launch_pdl(bw_token_kernel<T>, dim3(tb), dim3(256), 0, st, a, dyb))) return e;
        if ((e = launch_pdl(rowgemm_kernel<TG_DH, T, T>, g_dh, dim3(256), 0, st, a, dypb, dypb,
                            static_cast<const T *>(W2), static_cast<const T *>(W2), a.d, a.I, a.S)))
            return e;
        if ((e = launch_pdl(dh_finalize_kernel, g_fin, dim3(256), 0, st, a, a.S))) return e;
        if ((e = launch_pdl(rowgemm_kernel<TG_DX, float, T>, g_dh, dim3(256), 0, st, a,
                            static_cast<const float *>(a.da), static_cast<const float *>(a.db),
                            static_cast<const T *>(W1), static_cast<const T *>(W3), a.I, a.d, a.S)))
            return e;
        if ((e = launch_pdl(bw_dx_kernel<T>, dim3(tb), dim3(256), 0, st, a,
                            static_cast<const T *>(Wg), static_cast<const T *>(Wm), a.S)))
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
    if ((e = launch_pdl(rowgemm_kernel<TG_DH, T, T>, g_dh, dim3(256), 0, st, a, dypb, dypb,
                        static_cast<const T *>(W2), static_cast<const T *>(W2), a.d, a.I, a.S)))
        return e;
    if ((e = launch_pdl(dh_finalize_kernel, g_fin, dim3(256), 0, st, a, a.S))) return e;
    if ((e = launch_pdl(rowgemm_kernel<TG_DX, float, T>, g_dh, dim3(256), 0, st, a,
                        static_cast<const float *>(a.da), static_cast<const float *>(a.db),
                        static_cast<const T *>(W1), static_cast<const T *>(W3), a.I, a.d, a.S)))
        return e;
    if ((e = launch_pdl(bw_dx_kernel<T>, dim3(tb), dim3(256), 0, st, a,
                        static_cast<const T *>(Wg), static_cast<const T *>(Wm), a.S)))
        return e;
    if ((e = launch_pdl(bw_dw13_kernel<T>, g_w13, dim3(256), 0, st, a, xpb, dW1, dW3))) return e;
    if ((e = launch_pdl(bw_dw2_kernel<T>, g_w2, dim3(256), 0, st, a, dypb, dW2))) return e;
    return launch_pdl(bw_drouter_kernel<T>, g_r, dim3(256), 0, st, a, xb, xpb, dWg, dWm);
}

}  // namespace beam
