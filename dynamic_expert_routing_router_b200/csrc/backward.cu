// backward.cu -- CUDA-core stages of the training-mode backward pass (the bf16
// layer runs its two kept-row products, dh and dxp, on the tensor cores:
// MODE_GEMM2T and MODE_GEMM1T in tc_gemm.cu, over the per-expert row tiles
// listed here; the fp32 layer runs them with rowgemm_kernel below).
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

#include <type_traits>

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
#pragma unroll 4
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
// Four consecutive elements as fp32 (8-byte aligned for bf16, 16 for fp32).
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
    const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
    v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
}
__device__ __forceinline__ void load4(const float *p, float (&v)[4]) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    const float4 y = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}

// ------------------------------------------------- kept-row products (split) --
// For one tile and one split sp of the reduction range, the kept rows r get
//   part[sp][r][n] = sum_{k in split} A[r][k] B_e[k][n]  (+ A2[r][k] B2_e[k][n])
// with B_e row-major [Kdim][N] at B + e * Kdim * N.
//   DH: A = dyp, B = W2 (Kdim = d, N = I)
//   DX: A = da, A2 = db, B = W1, B2 = W3 (Kdim = I, N = d)
// The weight rows stream through a 4-stage shared-memory ring of 16-byte
// cp.async copies issued by every thread, so the copies in flight do not
// depend on how many threads compute.  A stage is 16 KB: 8 k-rows (DH) or 4
// k-rows of each matrix (DX) of one column pass of 2 KB of row (1024 bf16 /
// 512 fp32 columns, 8 per computing thread).  Kept rows go in groups of 4,
// whose A values sit in shared memory for the whole split.
enum { TG_DH = 0, TG_DX = 1 };
constexpr int kRgStages = 4;
template <int MODE>
struct RgCfg {
    static constexpr int KCH = MODE == TG_DX ? 4 : 8;  // k-rows per stage
    static constexpr int NMAT = MODE == TG_DX ? 2 : 1;
};
template <int MODE, typename TB>
__host__ __device__ constexpr int rg_cols() { return 2048 / int(sizeof(TB)); }  // columns per pass
template <int MODE, typename TB>
size_t rg_smem_bytes(int kc) {
    return size_t(kRgStages) * RgCfg<MODE>::KCH * rg_cols<MODE, TB>() * sizeof(TB) *
               RgCfg<MODE>::NMAT +
           size_t(4) * kc * sizeof(float) * RgCfg<MODE>::NMAT;
}

template <int MODE, typename TA, typename TB>
__global__ void __launch_bounds__(256, 1) rowgemm_kernel(const BwArgs a, const TA *A,
                                                         const TA *A2, const TB *B, const TB *B2,
                                                         int Kdim, int N, int S) {
    constexpr int KCH = RgCfg<MODE>::KCH, NMAT = RgCfg<MODE>::NMAT;
    constexpr int CPB = rg_cols<MODE, TB>();
    constexpr size_t MAT_BYTES = size_t(KCH) * CPB * sizeof(TB);  // one matrix, one stage
    constexpr size_t STAGE_BYTES = MAT_BYTES * NMAT;
    extern __shared__ __align__(128) unsigned char rg_smem[];
    __shared__ int s_flag[kMaxTileRows], s_row[kMaxTileRows], s_n;
    __shared__ float s_fw[kMaxTileRows], s_w[kMaxTileRows];
    griddep_wait();
    griddep_launch_dependents();
    const int ti = blockIdx.x, sp = blockIdx.y;
    if (ti >= a.meta[0]) return;
    const int4 tile = a.tiles[ti];
    const int e = tile.x;
    const int nk = stage_kept_rows(a, tile.y, tile.z, s_flag, s_fw, s_row, s_w, &s_n);
    if (nk == 0) return;
    const int kc = Kdim / S, k0 = sp * kc;
    const int nchunks = (kc + KCH - 1) / KCH;
    float *As = reinterpret_cast<float *>(rg_smem + kRgStages * STAGE_BYTES);  // [4][kc]
    float *A2s = As + 4 * kc;                                                   // DX only
    const long long bstride = (long long)Kdim * N;
    const TB *Be = B + (long long)e * bstride;
    const TB *B2e = NMAT == 2 ? B2 + (long long)e * bstride : nullptr;
    float *part = a.part + (long long)sp * a.p_cap * N;
    for (int g0 = 0; g0 < nk; g0 += 4) {
        const int gn = min(4, nk - g0);
        // A rows of the group for the whole split (batches of 8 independent loads).
        for (int q0 = threadIdx.x; q0 < 4 * kc; q0 += 8 * blockDim.x) {
            float v[8], v2[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = q0 + u * blockDim.x;
                const int r = q / kc, k = q - r * kc;
                const bool ok = q < 4 * kc && r < gn;
                const long long o = ok ? (long long)s_row[g0 + r] * Kdim + k0 + k : 0;
                v[u] = ok ? load_f(A, o) : 0.0f;
                v2[u] = (NMAT == 2 && ok) ? load_f(A2, o) : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = q0 + u * blockDim.x;
                if (q < 4 * kc) {
                    As[q] = v[u];
                    if (NMAT == 2) A2s[q] = v2[u];
                }
            }
        }
        __syncthreads();
        for (int c0 = 0; c0 < N; c0 += CPB) {
            const int ncol = min(CPB, N - c0);
            const int cg = threadIdx.x;  // 8 columns each
            const bool active = cg * 8 < ncol;
            // Copy k-rows [k0 + c*KCH, +kn) x columns [c0, c0 + ncol) into stage c.
            auto issue = [&](int c) {
                if (c < nchunks) {
                    const int kb = k0 + c * KCH, kn = min(KCH, k0 + kc - kb);
                    unsigned char *dst = rg_smem + (c % kRgStages) * STAGE_BYTES;
                    const int per_row = ncol * int(sizeof(TB)) / 16;
                    for (int q = threadIdx.x; q < kn * per_row; q += blockDim.x) {
                        const int u = q / per_row, v = q - u * per_row;
                        const long long go = (long long)(kb + u) * N + c0;
                        cp_async_16(dst + size_t(u) * CPB * sizeof(TB) + size_t(v) * 16,
                                    reinterpret_cast<const unsigned char *>(Be + go) + size_t(v) * 16);
                        if (NMAT == 2)
                            cp_async_16(dst + MAT_BYTES + size_t(u) * CPB * sizeof(TB) + size_t(v) * 16,
                                        reinterpret_cast<const unsigned char *>(B2e + go) + size_t(v) * 16);
                    }
                }
                cp_async_commit();  // every thread, every call: uniform group counts
            };
            float acc[4][8];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) acc[r][cc] = 0.0f;
#pragma unroll
            for (int c = 0; c < kRgStages - 1; ++c) issue(c);
            for (int c = 0; c < nchunks; ++c) {
                issue(c + kRgStages - 1);
                cp_async_wait<kRgStages - 1>();  // this thread's copies of chunk c landed
                __syncthreads();                   // everyone's did
                if (active) {
                    const unsigned char *st = rg_smem + (c % kRgStages) * STAGE_BYTES;
                    const int kn = min(KCH, kc - c * KCH);
                    const float *ar = As + c * KCH;
                    const float *ar2 = A2s + c * KCH;
#pragma unroll 4
                    for (int u = 0; u < kn; ++u) {
                        float bv[8];
                        load8(reinterpret_cast<const TB *>(st + size_t(u) * CPB * sizeof(TB)) + cg * 8, bv);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float av = ar[r * kc + u];
#pragma unroll
                            for (int cc = 0; cc < 8; ++cc) acc[r][cc] = fmaf(av, bv[cc], acc[r][cc]);
                        }
                        if (NMAT == 2) {
                            load8(reinterpret_cast<const TB *>(st + MAT_BYTES + size_t(u) * CPB * sizeof(TB)) + cg * 8, bv);
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const float av = ar2[r * kc + u];
#pragma unroll
                                for (int cc = 0; cc < 8; ++cc) acc[r][cc] = fmaf(av, bv[cc], acc[r][cc]);
                            }
                        }
                    }
                }
                __syncthreads();  // stage c is refilled by the next issue
            }
            cp_async_wait<0>();
            if (active) {
                for (int r = 0; r < gn; ++r) {
                    float *o = part + (long long)s_row[g0 + r] * N + c0 + cg * 8;
                    *reinterpret_cast<float4 *>(o) =
                        make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
                    *reinterpret_cast<float4 *>(o + 4) =
                        make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
                }
            }
            __syncthreads();
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
    // Every (kept row, column) of the tile in one loop, kFinBatch items per
    // thread and pass: all their loads are issued before any result is
    // stored (the stores would otherwise hold back the next item's loads).
    constexpr int kFinBatch = 4;
    const int n_items = nk * I;
    for (int qb = threadIdx.x; qb < n_items; qb += kFinBatch * blockDim.x) {
        long long o[kFinBatch];
        float c[kFinBatch], av[kFinBatch], bv[kFinBatch], wq[kFinBatch];
#pragma unroll
        for (int u = 0; u < kFinBatch; ++u) {
            const int qi = qb + u * blockDim.x;
            o[u] = -1;
            if (qi < n_items) {
                const int q = qi / I, i = qi - q * I;
                o[u] = (long long)s_row[q] * I + i;
                wq[u] = s_w[q];
                float cs = 0.0f;
                for (int sp = 0; sp < S; ++sp) cs += a.part[sp * split + o[u]];
                c[u] = cs;
                av[u] = a.A[o[u]];
                bv[u] = a.B[o[u]];
            }
        }
#pragma unroll
        for (int u = 0; u < kFinBatch; ++u) {
            if (o[u] < 0) continue;
            const float dh = wq[u] * c[u];
            const float sa = sigm(av[u]);
            const float da = dh * bv[u] * sa * (1.0f + av[u] * (1.0f - sa));
            const float db = dh * av[u] * sa;
            a.da[o[u]] = da;
            a.db[o[u]] = db;
            a.h[o[u]] = av[u] * sa * bv[u];
            if (a.da_bf) {  // operands of the tensor-core dx product
                static_cast<__nv_bfloat16 *>(a.da_bf)[o[u]] = __float2bfloat16_rn(da);
                static_cast<__nv_bfloat16 *>(a.db_bf)[o[u]] = __float2bfloat16_rn(db);
            }
        }
    }
}

// Exclusive prefix of v over the block's 256 threads (in thread order) and
// the block total; s_warp holds 8 ints and is free again on return.
__device__ __forceinline__ int block_excl_prefix(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += u;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        before += w < warp ? s_warp[w] : 0;
        tot += s_warp[w];
    }
    __syncthreads();
    *total = tot;
    return before + incl - v;
}

// ---------------------------------------------------------------------- dx --
// Block per token; each thread owns 8 consecutive columns, so every term is
// one 16-byte load and the loads of all terms are independent.  The router
// terms (nonzero dr in expert order, then the K dz in slot order) are listed
// in shared memory first.
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dx_kernel(const BwArgs a, const TIn *Wg,
                                                    const TIn *Wm, int S) {
    __shared__ float s_c[kMaxE + kMaxK];  // coefficients
    __shared__ int s_row[kMaxE + kMaxK];  // their weight rows
    __shared__ int s_pos[kMaxK];
    __shared__ int s_warp[8], s_nk;
    griddep_wait();
    griddep_launch_dependents();
    const int K = a.K, E = a.E, d = a.d;
    const long long split = (long long)a.p_cap * d;
    for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
        // Router terms: the nonzero dr[t][e] in expert order (block prefix),
        // then the K dz in slot order; kept slots' rows in slot order (warp 0).
        int ng = 0;  // block-uniform
        for (int e0 = 0; e0 < E; e0 += blockDim.x) {
            const int e = e0 + threadIdx.x;
            const float c = e < E ? a.dr[(long long)t * E + e] : 0.0f;
            int tot;
            const int pos = block_excl_prefix(c != 0.0f ? 1 : 0, s_warp, &tot);
            if (c != 0.0f) {
                s_c[ng + pos] = c;
                s_row[ng + pos] = e;
            }
            ng += tot;
        }
        if (threadIdx.x < 32) {
            const int k = threadIdx.x;
            const long long o = (long long)t * K + k;
            const bool kept = k < K && a.idx[o] >= 0;
            const unsigned bal = __ballot_sync(0xffffffffu, kept);
            if (kept) s_pos[__popc(bal & ((1u << k) - 1u))] = a.pair_pos[o];
            if (k == 0) s_nk = __popc(bal);
            if (Wm && k < K) {
                s_c[ng + k] = a.dz[o];
                s_row[ng + k] = a.cand[o];
            }
        }
        __syncthreads();
        const int nr = ng + (Wm ? K : 0), nk = s_nk;
        for (int j = threadIdx.x * 8; j < d; j += blockDim.x * 8) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int q = 0; q < nk; ++q) {  // expert part: kept slots in order, splits in order
                float c[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int sp = 0; sp < S; ++sp) {
                    float v[8];
                    load8(a.part + sp * split + (long long)s_pos[q] * d + j, v);
#pragma unroll
                    for (int i = 0; i < 8; ++i) c[i] += v[i];
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] += c[i];
            }
#pragma unroll 4
            for (int q = 0; q < nr; ++q) {  // W_gate^T dr, then W_mask^T dz
                float v[8];
                load8((q < ng ? Wg : Wm) + (long long)s_row[q] * d + j, v);
                const float cq = s_c[q];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(cq, v[i], acc[i]);
            }
            float *o = a.dx + (long long)t * d + j;
            *reinterpret_cast<float4 *>(o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            *reinterpret_cast<float4 *>(o + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        __syncthreads();
    }
}


// -------------------------------------------------------- weight gradients --
// Kept rows of expert e (rows [first, first + n) of the candidate grouping),
// chunk [r0, r0 + cnt): compacted row indices, in ascending order, into s_kr
// (returns how many).  One thread per row of the chunk: blockDim.x ==
// kWgChunk; s_wc holds the per-warp counts.
constexpr int kWgChunk = 256;
// Bring the line holding p into L2 (the gradient rows a block will read back,
// issued before its kept rows are staged so that the read overlaps them).
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ int stage_expert_chunk(const BwArgs &a, int first, int r0, int cnt, int *s_wc,
                                  int *s_kr) {
    const int q = threadIdx.x, lane = q & 31, warp = q >> 5;
    const int r = first + r0 + q;
    const bool kept = q < cnt && a.idx[a.pair[r]] >= 0;
    const unsigned bal = __ballot_sync(0xffffffffu, kept);
    if (lane == 0) s_wc[warp] = __popc(bal);
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kWgChunk / 32; ++w) {
        const int c = s_wc[w];
        base += w < warp ? c : 0;
        total += c;
    }
    if (kept) s_kr[base + __popc(bal & ((1u << lane) - 1u))] = r;
    __syncthreads();
    return total;
}

// dW1_e[i] += sum over kept rows (in order) da[r][i] x_r, dW3 likewise with db.
// Block (expert, kDw13Groups groups of 4 rows of I); each thread owns 8
// consecutive columns of d.  The expert's kept rows are listed once (when
// they fit one chunk) and serve every group; each group's gradient rows are
// prefetched into L2 while the previous group is summed, so the block's
// read-modify-writes follow one another without a fresh staging chain.
constexpr int kDw13Groups = 3;
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dw13_kernel(const BwArgs a, const TIn *xp, float *dW1,
                                                      float *dW3) {
    __shared__ int s_first;
    __shared__ int s_wc[kWgChunk / 32], s_kr[kWgChunk];
    __shared__ float s_da[kWgChunk][4], s_db[kWgChunk][4];
    griddep_wait();
    griddep_launch_dependents();
    const int e = blockIdx.x;
    if (a.counts_kept[e] == 0) return;  // no kept pair: no gradient, rows untouched
    const int d = a.d, I = a.I;
    const int ig0 = blockIdx.y * kDw13Groups * 4;  // first row of I of the block
    // gradient rows of group g, this thread's columns, into L2
    auto prefetch_group = [&](int i0, int j) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i0 + i < I) {
                const long long o = ((long long)e * I + i0 + i) * d + j;
                prefetch_l2(dW1 + o);
                prefetch_l2(dW3 + o);
            }
    };
    if (threadIdx.x * 8 < d) prefetch_group(ig0, threadIdx.x * 8);
    const int first = expert_first_row(a.tiles, a.meta[0], e, &s_first);
    const int n = a.counts_all[e];
    const bool one_chunk = n <= kWgChunk;
    int nk = one_chunk ? stage_expert_chunk(a, first, 0, n, s_wc, s_kr) : 0;
    for (int jb = 0; jb < d; jb += 8 * blockDim.x) {
        const int j = jb + threadIdx.x * 8;
        const bool active = j < d;
        for (int g = 0; g < kDw13Groups; ++g) {
            const int i0 = ig0 + 4 * g;
            if (i0 >= I) break;
            // this group's rows were prefetched one group ahead (or at the
            // start); a new column pass prefetches its first group here
            if (active && g == 0 && jb > 0) prefetch_group(i0, j);
            if (active && g + 1 < kDw13Groups && i0 + 4 < I) prefetch_group(i0 + 4, j);
            float g1[4][8], g3[4][8];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 8; ++c) g1[i][c] = g3[i][c] = 0.0f;
            for (int r0 = 0; r0 < n; r0 += kWgChunk) {
                if (!one_chunk)
                    nk = stage_expert_chunk(a, first, r0, min(kWgChunk, n - r0), s_wc, s_kr);
                for (int q = threadIdx.x; q < 4 * nk; q += blockDim.x) {
                    const int kq = q >> 2, i = q & 3;
                    const bool ok = i0 + i < I;
                    s_da[kq][i] = ok ? a.da[(long long)s_kr[kq] * I + i0 + i] : 0.0f;
                    s_db[kq][i] = ok ? a.db[(long long)s_kr[kq] * I + i0 + i] : 0.0f;
                }
                __syncthreads();
                if (active) {
#pragma unroll 4
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
}

// dW2_e[j] += sum over kept rows (in order) w_r dy_r[j] h_r (h fp32 from the
// finalize step).  Block (expert, kDw2Groups groups of 8 rows of d); each
// thread owns 4 columns of I.  As in bw_dw13_kernel, the kept rows are listed
// once and each group's gradient rows are prefetched one group ahead.
constexpr int kDw2Groups = 3;
template <typename TIn>
__global__ void __launch_bounds__(256) bw_dw2_kernel(const BwArgs a, const TIn *dyp, float *dW2) {
    __shared__ int s_first;
    __shared__ int s_wc[kWgChunk / 32], s_kr[kWgChunk];
    __shared__ float s_dy[kWgChunk][8];
    griddep_wait();
    griddep_launch_dependents();
    const int e = blockIdx.x;
    if (a.counts_kept[e] == 0) return;
    const int d = a.d, I = a.I;
    const int jg0 = blockIdx.y * kDw2Groups * 8;  // first row of d of the block
    auto prefetch_group = [&](int j0, int i) {  // one request per 32-byte sector
        if ((threadIdx.x & 1) == 0)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                if (j0 + jj < d) prefetch_l2(dW2 + ((long long)e * d + j0 + jj) * I + i);
    };
    if (threadIdx.x * 4 < I) prefetch_group(jg0, threadIdx.x * 4);
    const int first = expert_first_row(a.tiles, a.meta[0], e, &s_first);
    const int n = a.counts_all[e];
    const bool one_chunk = n <= kWgChunk;
    int nk = one_chunk ? stage_expert_chunk(a, first, 0, n, s_wc, s_kr) : 0;
    for (int ib = 0; ib < I; ib += 4 * blockDim.x) {
        const int i = ib + threadIdx.x * 4;
        const bool active = i < I;
        for (int gq = 0; gq < kDw2Groups; ++gq) {
            const int j0 = jg0 + 8 * gq;
            if (j0 >= d) break;
            // this group's rows were prefetched one group ahead (or at the
            // start); a new column pass prefetches its first group here
            if (active && gq == 0 && ib > 0) prefetch_group(j0, i);
            if (active && gq + 1 < kDw2Groups && j0 + 8 < d) prefetch_group(j0 + 8, i);
            float g[8][4];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
#pragma unroll
                for (int c = 0; c < 4; ++c) g[jj][c] = 0.0f;
            for (int r0 = 0; r0 < n; r0 += kWgChunk) {
                if (!one_chunk)
                    nk = stage_expert_chunk(a, first, r0, min(kWgChunk, n - r0), s_wc, s_kr);
                for (int q = threadIdx.x; q < 8 * nk; q += blockDim.x) {
                    const int kq = q >> 3, jj = q & 7;
                    const int r = s_kr[kq];
                    const float wk = a.w[a.pair[r]];
                    s_dy[kq][jj] =
                        (j0 + jj < d) ? wk * load_f(dyp, (long long)r * d + j0 + jj) : 0.0f;
                }
                __syncthreads();
                if (active) {
#pragma unroll 4
                    for (int kq = 0; kq < nk; ++kq) {
                        const float4 hv =
                            *reinterpret_cast<const float4 *>(a.h + (long long)s_kr[kq] * I + i);
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
}

// dW_gate[e] += sum_t dr[t][e] x_t; dW_mask[e] += sum over the candidate
// rows of e (token order) dz x.  Block (expert, 128 columns): each warp holds
// all 128 columns (4 per lane) for its own contiguous share of the terms, and
// warp 0 adds the eight partial sums in warp order before the one
// read-modify-write; a popular expert's terms are thus summed by eight warps
// at once.  Each round of 256 tokens first lists the nonzero dr[t][e] in
// token order (with renorm only the tokens that have e as a candidate), so
// the sums run without branches and load eight rows at a time.  The order is
// fixed: the same inputs give the same bits.
constexpr int kDrChunk = 256;
constexpr int kDrCols = 128;
// g[0..3] += sum over q < n (in order) c[q] * X[r[q]][j .. j+3]: the rows are
// loaded eight at a time before their terms are added.
template <typename TIn>
__device__ __forceinline__ void sum_rows(const TIn *X, int d, int j, const int *r, const float *c,
                                         int n, float (&g)[4]) {
    int q = 0;
    for (; q + 8 <= n; q += 8) {
        float v[8][4];
#pragma unroll
        for (int b = 0; b < 8; ++b) load4(X + (long long)r[q + b] * d + j, v[b]);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const float cq = c[q + b];
#pragma unroll
            for (int i = 0; i < 4; ++i) g[i] = fmaf(cq, v[b][i], g[i]);
        }
    }
    for (; q < n; ++q) {
        float v[4];
        load4(X + (long long)r[q] * d + j, v);
        const float cq = c[q];
#pragma unroll
        for (int i = 0; i < 4; ++i) g[i] = fmaf(cq, v[i], g[i]);
    }
}
template <typename TIn>
__global__ void __launch_bounds__(256) bw_drouter_kernel(const BwArgs a, const TIn *x,
                                                         const TIn *xp, float *dWg, float *dWm) {
    __shared__ int s_first, s_warp[8];
    __shared__ float s_c[kDrChunk];
    __shared__ int s_r[kDrChunk];
    __shared__ __align__(16) float s_pg[8][kDrCols], s_pm[8][kDrCols];
    griddep_wait();
    griddep_launch_dependents();
    const int e = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int j = blockIdx.y * kDrCols + lane * 4;
    const bool active = j < a.d;
    const int d = a.d, E = a.E;
    if (active && warp == 0) {
        prefetch_l2(dWg + (long long)e * d + j);
        if (dWm) prefetch_l2(dWm + (long long)e * d + j);
    }
    float gg[4] = {0.f, 0.f, 0.f, 0.f}, gm[4] = {0.f, 0.f, 0.f, 0.f};
    for (int t0 = 0; t0 < a.T; t0 += kDrChunk) {
        const int t = t0 + threadIdx.x;
        const float c = t < a.T ? a.dr[(long long)t * E + e] : 0.0f;
        int nz;
        const int pos = block_excl_prefix(c != 0.0f ? 1 : 0, s_warp, &nz);
        if (c != 0.0f) {
            s_c[pos] = c;
            s_r[pos] = t;
        }
        __syncthreads();
        const int q0 = warp * nz / 8, q1 = (warp + 1) * nz / 8;
        if (active) sum_rows(x, d, j, s_r + q0, s_c + q0, q1 - q0, gg);
        __syncthreads();
    }
    const int n = a.counts_all[e];
    if (dWm && n > 0) {
        const int first = expert_first_row(a.tiles, a.meta[0], e, &s_first);
        for (int r0 = 0; r0 < n; r0 += kDrChunk) {
            const int cnt = min(kDrChunk, n - r0);
            for (int q = threadIdx.x; q < cnt; q += blockDim.x) {
                const int r = first + r0 + q;
                s_r[q] = r;
                s_c[q] = a.dz[a.pair[r]];
            }
            __syncthreads();
            const int q0 = warp * cnt / 8, q1 = (warp + 1) * cnt / 8;
            if (active) sum_rows(xp, d, j, s_r + q0, s_c + q0, q1 - q0, gm);
            __syncthreads();
        }
    }
    if (active) {
        *reinterpret_cast<float4 *>(&s_pg[warp][lane * 4]) = make_float4(gg[0], gg[1], gg[2], gg[3]);
        *reinterpret_cast<float4 *>(&s_pm[warp][lane * 4]) = make_float4(gm[0], gm[1], gm[2], gm[3]);
    }
    __syncthreads();
    if (warp == 0 && active) {
        float4 sg = make_float4(0.f, 0.f, 0.f, 0.f), sm = sg;
#pragma unroll
        for (int w = 0; w < 8; ++w) {  // partial sums in warp order
            const float4 pg = *reinterpret_cast<const float4 *>(&s_pg[w][lane * 4]);
            const float4 pm = *reinterpret_cast<const float4 *>(&s_pm[w][lane * 4]);
            sg.x += pg.x; sg.y += pg.y; sg.z += pg.z; sg.w += pg.w;
            sm.x += pm.x; sm.y += pm.y; sm.z += pm.z; sm.w += pm.w;
        }
        float4 *pg = reinterpret_cast<float4 *>(dWg + (long long)e * d + j);
        float4 u = *pg;
        u.x += sg.x; u.y += sg.y; u.z += sg.z; u.w += sg.w;
        *pg = u;
        if (dWm) {
            float4 *pm = reinterpret_cast<float4 *>(dWm + (long long)e * d + j);
            float4 v = *pm;
            v.x += sm.x; v.y += sm.y; v.z += sm.z; v.w += sm.w;
            *pm = v;
        }
    }
}

}  // namespace

// Longest split reduction each product supports (its A rows for a whole split
// sit in shared memory): d <= 7168 for DH, I <= 4096 for DX at one split.
template <int MODE>
constexpr int rg_max_kc() { return MODE == TG_DX ? 4096 : 7168; }

template <int MODE, typename TA, typename TB>
cudaError_t launch_rowgemm(const BwArgs &a, const TA *A, const TA *A2, const TB *B, const TB *B2,
                           int Kdim, int N, cudaStream_t st) {
    const size_t smem = rg_smem_bytes<MODE, TB>(Kdim / a.S);
    if (Kdim / a.S > rg_max_kc<MODE>()) return cudaErrorInvalidValue;
    auto kern = rowgemm_kernel<MODE, TA, TB>;
    // The largest size this kernel is ever launched with; set once per device.
    static std::atomic<unsigned long long> attr_set{0};  // this instantiation only
    cudaError_t e = set_smem_once(kern, int(rg_smem_bytes<MODE, TB>(rg_max_kc<MODE>())), attr_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(a.tiles_cap, a.S), dim3(256), smem, st, a, A, A2, B, B2, Kdim, N,
                      a.S);
}

namespace {

// One block of 256 threads walks the grouping's tiles in order.  The first
// tile of each expert emits that expert's row tiles into list 0 (every
// candidate expert) and, when the expert has a kept pair, into list 1.
// Positions are exclusive prefixes over the tiles, so both lists are in
// expert order.
__global__ void __launch_bounds__(256) expert_tiles_kernel(const int4 *tiles, const int *meta,
                                                           const int *counts_kept,
                                                           const int *counts_all,
                                                           int rows_per_tile, int4 *xt_all,
                                                           int4 *xt_kept, int *xmeta) {
    __shared__ int s_warp[8];
    griddep_wait();
    griddep_launch_dependents();
    const int n = meta[0];
    int base_all = 0, base_kept = 0;  // block-uniform
    for (int b0 = 0; b0 < n; b0 += 256) {
        const int ti = b0 + threadIdx.x;
        int nt = 0, e = 0, row0 = 0, cnt = 0;
        bool kept = false;
        if (ti < n) {
            const int4 t = tiles[ti];
            e = t.x;
            row0 = t.y;
            if (ti == 0 || tiles[ti - 1].x != e) {
                cnt = counts_all[e];
                nt = (cnt + rows_per_tile - 1) / rows_per_tile;
                kept = counts_kept[e] > 0;
            }
        }
        int tot_all, tot_kept;
        const int pa = base_all + block_excl_prefix(nt, s_warp, &tot_all);
        const int pk = base_kept + block_excl_prefix(kept ? nt : 0, s_warp, &tot_kept);
        for (int j = 0; j < nt; ++j) {
            const int4 v = make_int4(e, row0 + j * rows_per_tile,
                                     min(rows_per_tile, cnt - j * rows_per_tile), 0);
            xt_all[pa + j] = v;
            if (kept) xt_kept[pk + j] = v;
        }
        base_all += tot_all;
        base_kept += tot_kept;
    }
    if (threadIdx.x == 0) {
        xmeta[0] = base_all;
        xmeta[1] = base_kept;
    }
}
}  // namespace

cudaError_t launch_expert_tiles(const int4 *tiles, const int *meta, const int *counts_kept,
                                const int *counts_all, int rows_per_tile, int4 *xt_all,
                                int4 *xt_kept, int *xmeta, cudaStream_t st) {
    return launch_pdl(expert_tiles_kernel, dim3(1), dim3(256), 0, st, tiles, meta, counts_kept,
                      counts_all, rows_per_tile, xt_all, xt_kept, xmeta);
}

namespace {
template <typename T>
cudaError_t backward_stages(const BwArgs &a, const T *x, const T *xp, const T *dy, const T *dyp,
                            const T *Wg, const T *Wm, const T *W1, const T *W3, const T *W2,
                            float *dWg, float *dWm, float *dW1, float *dW3, float *dW2, int n_sm,
                            cudaStream_t st, int phase) {
    const int tb = a.T < 8 * n_sm ? a.T : 8 * n_sm;
    cudaError_t e;
    if (phase == 0) {
        if ((e = launch_pdl(bw_token_kernel<T>, dim3(tb), dim3(256), 0, st, a, dy))) return e;
        if constexpr (std::is_same<T, float>::value) {
            if (!a.dh_tc && (e = launch_rowgemm<TG_DH, T, T>(a, dyp, dyp, W2, W2, a.d, a.I, st)))
                return e;
        } else if (!a.dh_tc) {
            return cudaErrorInvalidValue;  // bf16 runs dy W2_e on the tensor cores
        }
        return launch_pdl(dh_finalize_kernel, dim3(a.tiles_cap), dim3(256), 0, st, a,
                          a.dh_tc ? 1 : a.S);
    }
    if constexpr (std::is_same<T, float>::value) {
        if (!a.dx_tc && (e = launch_rowgemm<TG_DX, float, T>(a, a.da, a.db, W1, W3, a.I, a.d, st)))
            return e;
    } else if (!a.dx_tc) {
        return cudaErrorInvalidValue;  // bf16 runs da W1_e + db W3_e on the tensor cores
    }
    if ((e = launch_pdl(bw_dx_kernel<T>, dim3(tb), dim3(256), 0, st, a, Wg, Wm, a.dx_tc ? 1 : a.S)))
        return e;
    if ((e = launch_pdl(bw_dw13_kernel<T>, dim3(a.E, (a.I + 4 * kDw13Groups - 1) / (4 * kDw13Groups)),
                        dim3(256), 0, st, a, xp, dW1, dW3)))
        return e;
    if ((e = launch_pdl(bw_dw2_kernel<T>, dim3(a.E, (a.d + 8 * kDw2Groups - 1) / (8 * kDw2Groups)),
                        dim3(256), 0, st, a, dyp, dW2)))
        return e;
    return launch_pdl(bw_drouter_kernel<T>, dim3(a.E, (a.d + kDrCols - 1) / kDrCols), dim3(256), 0,
                      st, a, x, xp, dWg, dWm);
}
}  // namespace

cudaError_t launch_backward_stages(const BwArgs &a, int dtype, const void *x, const void *xp,
                                   const void *dy, const void *dyp, const void *Wg,
                                   const void *Wm, const void *W1, const void *W3,
                                   const void *W2, float *dWg, float *dWm, float *dW1,
                                   float *dW3, float *dW2, int n_sm, cudaStream_t st, int phase) {
    if (a.T <= 0) return cudaSuccess;
    if (dtype == BEAM_BF16) {
        using T = __nv_bfloat16;
        return backward_stages<T>(a, static_cast<const T *>(x), static_cast<const T *>(xp),
                                  static_cast<const T *>(dy), static_cast<const T *>(dyp),
                                  static_cast<const T *>(Wg), static_cast<const T *>(Wm),
                                  static_cast<const T *>(W1), static_cast<const T *>(W3),
                                  static_cast<const T *>(W2), dWg, dWm, dW1, dW3, dW2, n_sm, st,
                                  phase);
    }
    return backward_stages<float>(a, static_cast<const float *>(x), static_cast<const float *>(xp),
                                  static_cast<const float *>(dy), static_cast<const float *>(dyp),
                                  static_cast<const float *>(Wg), static_cast<const float *>(Wm),
                                  static_cast<const float *>(W1), static_cast<const float *>(W3),
                                  static_cast<const float *>(W2), dWg, dWm, dW1, dW3, dW2, n_sm, st,
                                  phase);
}

}  // namespace beam
