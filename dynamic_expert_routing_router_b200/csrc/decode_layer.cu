// decode_layer.cu -- the BEAM MoE layer of a small decode batch (T <= 16
// tokens) in ONE launch: router logits (BEAM §3.2 Eq. 5), top-K, softmax,
// binary mask and aggregation (Eq. 4, 6, 7), grouping of the kept pairs,
// SwiGLU experts for kept pairs only and the weighted combine (Eq. 8).
//
// Why: at a handful of tokens the layer's HBM floor is a few microseconds,
// while a chain of dependent launches costs several microseconds per launch
// boundary.  Here one persistent CTA per SM runs every phase; the phases hand
// off through counters in the workspace, never through a kernel boundary.
//
// Work, in a fixed global order, dealt to CTAs round-robin (CTA b takes b,
// b + G, ...) and inside a CTA to its Wc consumer warps round-robin:
//   router items   2 rows of [W_gate; W_mask] against every token -> logits;
//                  all consumer warps of the CTA share each one
//   (routing)      when every router item is counted, EVERY CTA reads all
//                  logits and takes the same top-K, mask and grouping in
//                  shared memory (identical arithmetic on identical inputs),
//                  so no second hand-off is needed; the last CTA also writes
//                  the routing and grouping arrays of the workspace
//   gate/up units  8 rows of W1 and the same 8 rows of W3 of one kept expert
//                  (one 16-row MMA tile) against the expert's tokens, over d
//                  in k-tiles -> 8 columns of H; counted per expert
//   down units     16 rows of W2 of one kept expert against its rows of H,
//                  over I in k-tiles -> 16 columns of Y; the unit completing
//                  a (token, 16-column block) of the output -- counted per
//                  pair -- sums the token's kept rows of Y in slot order (the
//                  combine kernel's arithmetic) and rounds once
// Every gate/up unit precedes every down unit in the global order, and only
// down units wait (on gate/up units), so the waits resolve whatever the
// order in which CTAs become resident.
//
// Warp roles: Wc consumer warps, a producer warp and a publisher warp.
//  * Producer lane l fills consumer warp l's M stages, in warp l's order: a
//    tile is a few 2D TMA boxes (64 columns, 128-byte swizzle: conflict-free
//    ldmatrix); before a down unit's first tile it waits for the expert's
//    gate/up units and brings the H rows in with the W2 rows.  (Row segments
//    by one bulk copy each, 16 to 32 per tile, made the producer the
//    bottleneck.)  Router rows and token rows come by plain bulk copies.
//    Every stage has one issuer and one consumer, each in order, so the
//    mbarrier parity they wait on is never ambiguous.
//  * A consumer warp runs a unit's k-tiles through mma.sync m16n8k16 (bf16
//    in, fp32 accumulate; the tokens are the N = 8 side), keeps the
//    accumulators in registers across the tiles, and writes the unit's
//    SwiGLU outputs (gate and up rows of a column sit in one lane) or rows of
//    Y.  On CUDA cores the same work took ~1800 instructions per 8 KB of
//    weights and left the kernel issue-bound.
//  * The publisher makes finished gate/up units visible: a consumer warp only
//    counts its unit in shared memory (after a CTA-scope fence), and the
//    publisher pays one GPU-scope fence for all units counted since its last
//    pass (~2 us under a full weight stream; paid per unit it stalled every
//    consumer warp).
//
// Every wait is bounded (timeout_ns of global time, or an error already
// raised); a warp that gives up records BEAM_ERR_TIMEOUT in the error word,
// the rest of the CTA stops at its next wait, and each producer lane waits
// (bounded) for its copies in flight before the CTA exits.
#include <cuda_bf16.h>

#include <climits>

#include "beam_internal.h"
#include "beam_ptx.cuh"
#include "topk_token.cuh"

namespace beam {

namespace {

constexpr int kConsumers = 14;                  // consumer warps (16 warps in all)
constexpr int kThreads = kDlThreads;            // + a producer warp and a publisher warp
constexpr int kProducer = kConsumers;           // the producer warp
constexpr int kPublisher = kConsumers + 1;      // the publisher warp
constexpr int kConsumerThreads = kConsumers * 32;
constexpr unsigned kAll = 0xffffffffu;
static_assert(kThreads == (kConsumers + 2) * 32, "a producer and a publisher warp");

// Tiles.  A gate/up tile is 8 rows of W1 and the same 8 rows of W3 x kKT1
// columns of d: boxes of 8 rows x 64 columns (1 KB), W1's at 0, 1, 2, 3 KB and
// W3's at 4, 5, 6, 7 KB.  A down tile is 16 rows of W2 and 16 rows of H x kKT2
// columns of I: boxes of 16 rows x 64 columns (2 KB), W2's at 0 and 2 KB, H's
// at 4 and 6 KB.  In a box, row r's 16-byte chunk c sits at chunk c ^ (r % 8)
// (the TMA's 128-byte swizzle; boxes and stages are 1 KB aligned).
constexpr int kKT1 = 256, kKT2 = 128;
constexpr int kStageMin = 8192;
constexpr int kSlots = 8;  // units whose k-tiles may be in flight in one CTA
constexpr int kTok = 2;  // tokens per pass of a router item (accumulators)

// ------------------------------------------------------------ primitives --

// One contiguous global range into shared memory; completion is counted on
// `bar` in bytes.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ int atom_add_acq_rel(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p), "r"(v)
                 : "memory");
    return old;
}

// Named barrier over the consumer warps only.
__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}
// Named barrier over every thread, producer and publisher warps included.
__device__ __forceinline__ void all_sync() {
    asm volatile("bar.sync 2, %0;" ::"n"(kThreads) : "memory");
}

// Bounded wait until *ctr >= need (acquire at GPU scope); gives up after
// timeout_ns or as soon as the error word or the CTA's abort flag is set.
__device__ __forceinline__ bool wait_count(const int *ctr, int need, const volatile int *err,
                                           const volatile int *abort_flag, uint64_t timeout_ns) {
    uint64_t t0 = 0;
    for (uint32_t spin = 0; spin < (1u << 26); ++spin) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= need) return true;
        if ((spin & 15u) == 0) {
            if ((err && *err) || (abort_flag && *abort_flag)) return false;
            const uint64_t t = globaltimer_ns();
            if (spin == 0) t0 = t;
            else if (t - t0 > timeout_ns) return false;
        }
        if (spin > 32) __nanosleep(32);
    }
    return false;
}

__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8]) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kAll, v, off);
    return v;
}

// The multi-kernel path's SiLU(a) * b, the same expression.
__device__ __forceinline__ float silu_mul(float g, float u) {
    return g / (1.0f + __expf(-g)) * u;
}

// Four 8x8 b16 matrices: lane i gives the row address of matrix i / 8, row
// i % 8; register m holds matrix m in the mma fragment layout.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// Two matrices: lanes 0-15 give the addresses.
__device__ __forceinline__ void ldsm_x2(uint32_t &r0, uint32_t &r1, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(addr));
}
// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col).
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory byte offset of row r, 16-byte chunk c of a swizzled box.
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return uint32_t(r * 128 + ((c ^ (r & 7)) << 4));
}

struct Routing {  // the routing and grouping of the call, in shared memory
    int cnt[kMaxE];         // kept pairs per expert
    int off[kMaxE];         // first (BN-padded) row of the expert
    int coff[kMaxE];        // first entry of the expert in tok / pl
    int toff[kMaxE];        // first tile of the expert
    int te[kMaxE];          // touched experts, ascending
    unsigned tmask[kMaxE];  // tokens of the expert (bit t)
    int idx[kDlMaxT * kMaxK];
    float w[kDlMaxT * kMaxK];
    int pos[kDlMaxT * kMaxK];  // row of a kept pair
    int tok[kDlMaxT * kMaxK];  // grouped entry -> token
    int pl[kDlMaxT * kMaxK];   // grouped entry -> t*K + k
    int nkept[kDlMaxT];
    int hist[kMaxK + 1];
    int n_touched, n_rows, n_pairs, n_tiles;
};

// A unit of the expert phase: its kind, expert, first row (of I for gate/up,
// of d for down) and number of k-tiles.
struct Unit {
    bool up;
    int e, ti, row0, nkt;  // ti: the expert's index among the touched experts
};

}  // namespace

namespace {

template <int EPL>
__global__ void __launch_bounds__(kThreads, 1)
    decode_layer_kernel(const __grid_constant__ DlMaps maps, const DecodeLayerArgs a) {
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ __align__(8) uint64_t full_bar[kDlMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kDlMaxStages];
    __shared__ __align__(8) uint64_t x_bar;
    __shared__ Routing R;
    __shared__ int s_abort;
    // gate/up units finished here per (touched expert, 128-column block of
    // H): one byte each (at most 16), four blocks to a word
    __shared__ unsigned s_done[kMaxE][4];
    __shared__ unsigned s_pub[kMaxE * 4];  // the publisher's published counts, same packing
    __shared__ int s_wtot[kMaxE / 32][4];   // expert scan: per-warp totals
    __shared__ float s_rp[kConsumers][2][kDlMaxT];  // router partial sums, per warp
    // A unit's k-tiles are items of their own, taken by any warp; their partial
    // sums meet in the unit's slot (slot j % kSlots), added in k-tile order:
    // the tile (j, kt) waits until s_next[slot] == j * NKTM + kt.
    __shared__ __align__(16) float s_acc[kSlots][32][8];
    __shared__ int s_next[kSlots];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T, d = a.d, E = a.E, I = a.I, K = a.K, NS = a.n_stages;
    const int n_rows_router = a.has_mask ? 2 * E : E;
    const int U1 = I / 8, U2 = d / 16;                      // units per expert
    const int NB = I / kKT2;  // 128-column blocks of H, 16 gate/up units each
    const int NKT1 = (d + kKT1 - 1) / kKT1, NKT2 = I / kKT2;  // k-tiles per unit
    const int XSP = d + 8;                                  // token row pitch, elements
    const size_t SB = size_t(a.stage_bytes);
    // consumer warps and stages per warp: two stages per warp (the next tile
    // loads while this one is computed) when at least 16 stages fit
    const int M = NS >= 16 ? 2 : 1, Wc = min(kConsumers, NS / M);
    uint16_t *x_s = reinterpret_cast<uint16_t *>(dsm);
    float *lg = reinterpret_cast<float *>(dsm + a.sm_off_lg);
    // the swizzle pattern follows absolute shared-memory address bits: stages
    // start on a 1 KB boundary (the launch reserves 1 KB of slack for it)
    unsigned char *stage0 = dsm + a.sm_off_stage;
    stage0 += (1024u - (smem_u32(stage0) & 1023u)) & 1023u;
    const bool forward = a.mode == DL_FORWARD;
    int *err = a.hdr + kHdrErr;
    int *router_ctr = a.hdr + kHdrDlRouter;
    const int G = gridDim.x, b = blockIdx.x;
    const int my_ri = b < a.n_ru ? (a.n_ru - 1 - b) / G + 1 : 0;
    volatile int *abort_flag = &s_abort;

    if (tid == kProducer * 32) {
        for (int s = 0; s < Wc * M; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&x_bar, 1);
        fence_barrier_init();
    }
    for (int i = tid; i < E; i += kThreads) {
        R.cnt[i] = 0;
        R.tmask[i] = 0u;
#pragma unroll
        for (int w = 0; w < 4; ++w) s_done[i][w] = s_pub[4 * i + w] = 0u;
    }
    if (tid <= K) R.hist[tid] = 0;
    if (tid == 0) s_abort = 0;
    const int NKTM = max(NKT1, NKT2);
    if (tid < kSlots) s_next[tid] = tid * NKTM;  // unit tid, k-tile 0
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();
    // CTA 0 clears this call's counters; its router publish follows the
    // barrier below, so every other CTA sees them cleared.
    if (b == 0) {
        if (forward) {
            for (int i = tid; i < E * NB; i += kThreads) a.e1_done[i] = 0;
            for (int i = tid; i < T * U2; i += kThreads) a.comb_cnt[i] = 0;
        } else {
#pragma unroll
            for (int z = 0; z < 3; ++z)
                for (int i = tid; i < a.zero[z].count; i += kThreads) a.zero[z].ptr[i] = 0;
        }
    }
    __syncthreads();

    // Any wait that gave up: record it once per warp and stop the CTA.
    auto give_up = [&]() {
        if (lane == 0) {
            if (forward) atomicExch(err, DEV_ERR_TIMEOUT);
            else atomicExch(a.hdr + kHdrErrRouter, kRouterTimeoutTag);
            *abort_flag = 1;
        }
    };
    // The expert phase's unit of global number h (after routing).
    auto unit_of = [&](int h) -> Unit {
        const int n1u = R.n_touched * U1;
        Unit u;
        u.up = h < n1u;
        if (u.up) {
            u.ti = h / U1;
            u.e = R.te[u.ti];
            u.row0 = (h % U1) * 8;
            u.nkt = NKT1;
        } else {
            const int v = h - n1u;
            u.ti = v / U2;
            u.e = R.te[u.ti];
            u.row0 = (v % U2) * 16;
            u.nkt = NKT2;
        }
        return u;
    };
    auto n_units = [&]() {
        const int n = R.n_touched * (U1 + U2);
        return b < n ? (n - 1 - b) / G + 1 : 0;
    };
    auto n_up_units = [&]() {  // this CTA's gate/up units come first
        const int n1u = R.n_touched * U1;
        return b < n1u ? (n1u - 1 - b) / G + 1 : 0;
    };
    // Expert item i of this CTA: unit j (local) and k-tile kt.
    auto item_of = [&](int i, int e1u, int &j, int &kt) {
        if (i < e1u * NKT1) {
            j = i / NKT1;
            kt = i - j * NKT1;
        } else {
            const int v = i - e1u * NKT1;
            j = e1u + v / NKT2;
            kt = v - (j - e1u) * NKT2;
        }
    };

    // -------------------------------------------------- producer warp ----
    // Lane l < Wc fills consumer warp l's stages (l * M .. l * M + M - 1)
    // with warp l's items in order: its router items, then the k-tiles of
    // its units.
    if (warp == kProducer) {
        int idx = 0, skipped = -1;
        auto acquire = [&](int i) -> bool {
            const int use = i / M;
            return use == 0 || mbar_wait_bounded(&empty_bar[lane * M + i % M],
                                                 uint32_t((use - 1) & 1), abort_flag,
                                                 a.timeout_ns);
        };
        const size_t rb = size_t(d) * 2;  // bytes of a row of W_gate / W_mask / W1 / W3
        if (lane == 0) {
            mbar_arrive_expect_tx(&x_bar, uint32_t(T) * uint32_t(rb));
            for (int t = 0; t < T; ++t)
                bulk_load(x_s + size_t(t) * XSP, static_cast<const char *>(a.x) + t * rb,
                          uint32_t(rb), &x_bar);
        }
        bool ok = true;
        if (lane < Wc)
            for (int q = lane; q < my_ri; q += Wc, ++idx) {
                if (!(ok = acquire(idx))) break;
                uint64_t *fb = &full_bar[lane * M + idx % M];
                unsigned char *st = stage0 + size_t(lane * M + idx % M) * SB;
                if (b == 0 && a.fault_skip == FAULT_ROUTER_STAGE && q == 0) {
                    skipped = idx;  // tests: this stage never fills
                    continue;
                }
                const int r0 = (b + q * G) * a.rr;
                const int rows = min(a.rr, n_rows_router - r0);
                const int ga = max(0, min(rows, E - r0));  // rows from W_gate
                mbar_arrive_expect_tx(fb, uint32_t(rows * rb));
                if (ga > 0)
                    bulk_load(st, static_cast<const char *>(a.Wg) + size_t(r0) * rb,
                              uint32_t(ga * rb), fb);
                if (rows > ga)
                    bulk_load(st + ga * rb, static_cast<const char *>(a.Wm) + size_t(r0 + ga - E) * rb,
                              uint32_t((rows - ga) * rb), fb);
            }
        if (forward) {
            __syncwarp();
            all_sync();  // the routing is in shared memory (or the CTA gave up)
            const int my_nu = n_units(), e1u = n_up_units();
            const int n_it = e1u * NKT1 + (my_nu - e1u) * NKT2;
            // A down tile's W2 rows are issued at once; its H rows only once
            // the expert's gate/up units are published, so W2 streams while
            // the gate/up phase runs.  Down tiles waiting for their H
            // (`pend`, at most M) get it before this lane waits for a stage
            // to free up (it may be one of theirs) and at the end.
            int pend_s[2], pend_e[2], pend_k[2], pend_h[2], npend = 0;
            auto flush = [&]() -> bool {
                for (int p = 0; p < npend; ++p) {
                    // this tile's 128 columns of H: complete once the 16 gate/up
                    // units that write them are published
                    if (!wait_count(a.e1_done + pend_e[p] * NB + pend_k[p] / kKT2, 16, err,
                                    abort_flag, a.timeout_ns))
                        return false;
                    asm volatile("fence.proxy.async.global;" ::: "memory");  // H: async reads
                    tma_load_3d(stage0 + size_t(pend_s[p]) * SB + 4096, &maps.h, 0, pend_h[p],
                                pend_k[p] / 64, &full_bar[pend_s[p]]);
                }
                npend = 0;
                return true;
            };
            if (lane < Wc && ok && !*abort_flag) {
                for (int g = my_ri + ((lane - my_ri) % Wc + Wc) % Wc; g < my_ri + n_it;
                     g += Wc, ++idx) {
                    int j, kt;
                    item_of(g - my_ri, e1u, j, kt);
                    const Unit u = unit_of(b + j * G);
                    if (idx / M > 0 && npend > 0 && !(ok = flush())) break;
                    if (!(ok = acquire(idx))) break;
                    const int s = lane * M + idx % M;
                    uint64_t *fb = &full_bar[s];
                    unsigned char *st = stage0 + size_t(s) * SB;
                    if (b == 0 && a.fault_skip == FAULT_EXPERT_STAGE && g == my_ri) {
                        skipped = idx;  // tests: this stage never fills
                        continue;
                    }
                    // one box of 4 (gate/up) or 2 (down) swizzled 64-column
                    // chunks per operand; chunks past d are zero-filled
                    mbar_arrive_expect_tx(fb, 8192u);
                    if (u.up) {
                        const int y = u.e * I + u.row0, z = kt * (kKT1 / 64);
                        tma_load_3d(st, &maps.w1, 0, y, z, fb);
                        tma_load_3d(st + 4096, &maps.w3, 0, y, z, fb);
                    } else {
                        tma_load_3d(st, &maps.w2, 0, u.e * d + u.row0, kt * (kKT2 / 64), fb);
                        pend_s[npend] = s;
                        pend_e[npend] = u.e;
                        pend_k[npend] = kt * kKT2;
                        pend_h[npend] = R.off[u.e];  // 16 rows from the expert's first
                        if (++npend == M && !(ok = flush())) break;
                    }
                }
                if (ok && npend > 0) ok = flush();
                if (!ok) give_up();
            }
        }
        // The token rows and this lane's latest use of each of its stages:
        // those copies may still be in flight.
        if (lane == 0) mbar_wait_bounded(&x_bar, 0, nullptr, a.timeout_ns);
        if (lane < Wc)
            for (int i = max(0, idx - M); i < idx; ++i)
                if (i != skipped)
                    mbar_wait_bounded(&full_bar[lane * M + i % M], uint32_t((i / M) & 1), nullptr,
                                      a.timeout_ns);
        return;
    }

    // ------------------------------------------------- publisher warp ----
    if (warp == kPublisher) {
        if (!forward) return;
        all_sync();
        if (*abort_flag) return;
        const int NT = R.n_touched, n1u = NT * U1, NBW = (NB + 3) / 4;
        const int my_e1u = b < n1u ? (n1u - 1 - b) / G + 1 : 0;
        // Counts already published, in shared memory beside the live ones
        // (the publisher's own; rolled loops: this warp runs beside the
        // consumers, and its code competes with theirs for the instruction
        // cache).
        int published = 0;
        uint64_t t0 = globaltimer_ns();
        while (published < my_e1u) {
            bool any = false;
#pragma unroll 1
            for (int i = lane; i < NT * NBW; i += 32)
                any |= reinterpret_cast<volatile unsigned *>(&s_done[0][0])[(i / NBW) * 4 + i % NBW] !=
                       s_pub[(i / NBW) * 4 + i % NBW];
            if (__any_sync(kAll, any)) {
                __threadfence();  // every unit counted so far, before the adds
                int mine = 0;
#pragma unroll 1
                for (int i = lane; i < NT * NBW; i += 32) {
                    const int ti = i / NBW, w = i % NBW;
                    const unsigned now =
                        reinterpret_cast<volatile unsigned *>(&s_done[0][0])[ti * 4 + w];
                    const unsigned was = s_pub[ti * 4 + w];
#pragma unroll 1
                    for (int q = 0; q < 4 && 4 * w + q < NB; ++q) {
                        const int delta = int((now >> (8 * q)) & 255u) - int((was >> (8 * q)) & 255u);
                        if (delta > 0) {
                            atomicAdd(a.e1_done + R.te[ti] * NB + 4 * w + q, delta);
                            mine += delta;
                        }
                    }
                    s_pub[ti * 4 + w] = now;
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(kAll, mine, off);
                published += mine;
                t0 = globaltimer_ns();
            } else {
                if (*abort_flag) break;
                if (globaltimer_ns() - t0 > a.timeout_ns) {
                    give_up();
                    break;
                }
                __nanosleep(64);
            }
        }
        return;
    }

    // ------------------------------------------------- consumer warps ----
    {
        const bool ok = mbar_wait_bounded(&x_bar, 0, abort_flag, a.timeout_ns);
        if (!__all_sync(kAll, ok)) give_up();
    }
    const int nch = d / 8;  // 16-byte chunks of a token row / a router row
    const uint4 *x_v4 = reinterpret_cast<const uint4 *>(x_s);
    const int xv = XSP / 8;  // token row pitch, 16-byte chunks

    // ------------------------------------------------ 1. router items ----
    // Every consumer warp takes part in each of the CTA's router items: warp w
    // owns a fixed range of the rows' 16-byte chunks (for both rows and every
    // token), and a logit is the sum of the warps' partials in warp order.
    // Router item q sits in the stages of warp q % Wc (its (q / Wc)-th item).
    const int cw = (nch + kConsumers - 1) / kConsumers;  // chunks per warp
    for (int q = 0; q < my_ri; ++q) {
        const int ow = q % Wc, oi = q / Wc, os = ow * M + oi % M;
        const bool ok =
            mbar_wait_bounded(&full_bar[os], uint32_t((oi / M) & 1), abort_flag, a.timeout_ns);
        if (!ok) give_up();
        consumers_sync();
        if (*abort_flag) break;
        const uint4 *wv = reinterpret_cast<const uint4 *>(stage0 + size_t(os) * SB);
        const int r0 = (b + q * G) * a.rr;
        const int rows = min(a.rr, n_rows_router - r0);
        const int c_end = min(nch, (warp + 1) * cw);
        for (int t0 = 0; t0 < T; t0 += kTok) {
            float acc0[kTok], acc1[kTok];
#pragma unroll
            for (int u = 0; u < kTok; ++u) acc0[u] = acc1[u] = 0.0f;
#pragma unroll 1
            for (int c = warp * cw + lane; c < c_end; c += 32) {
                float w0[8], w1[8];
                unpack8(wv[c], w0);
                unpack8(wv[rows > 1 ? nch + c : c], w1);
#pragma unroll
                for (int u = 0; u < kTok; ++u) {
                    if (t0 + u < T) {
                        float xf[8];
                        unpack8(x_v4[(t0 + u) * xv + c], xf);
#pragma unroll
                        for (int z = 0; z < 8; ++z) {
                            acc0[u] = fmaf(w0[z], xf[z], acc0[u]);
                            acc1[u] = fmaf(w1[z], xf[z], acc1[u]);
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kTok; ++u) {
                if (t0 + u < T) {
                    const float v0 = warp_sum(acc0[u]), v1 = warp_sum(acc1[u]);
                    if (lane == 0) {
                        s_rp[warp][0][t0 + u] = v0;
                        s_rp[warp][1][t0 + u] = v1;
                    }
                }
            }
        }
        consumers_sync();
        if (warp == ow && lane == 0) mbar_arrive(&empty_bar[os]);
        for (int i = tid; i < rows * T; i += kConsumerThreads) {
            const int r = i / T, t = i - r * T;
            float v = s_rp[0][r][t];
            for (int w = 1; w < kConsumers; ++w) v += s_rp[w][r][t];
            a.partial[size_t(t) * 2 * E + r0 + r] = v;
        }
        consumers_sync();  // s_rp is rewritten by the next item; stores before the publish
    }
    if (forward && tid == 0 && my_ri > 0 && !*abort_flag) {
        __threadfence();
        atomicAdd(router_ctr, my_ri);
    }
    if (!forward) return;  // router-only: the top-K kernel follows

    // ------------------------------------------------------ 2. routing ----
    if (tid == 0 && !*abort_flag &&
        !wait_count(router_ctr, a.n_ru, err, abort_flag, a.timeout_ns)) {
        atomicExch(err, DEV_ERR_TIMEOUT);
        *abort_flag = 1;
    }
    consumers_sync();
    const int cols = a.has_mask ? 2 * E : E;
    if (!*abort_flag)
        for (int i = tid; i < T * cols; i += kConsumerThreads) {
            const int t = i / cols, c = i - t * cols;
            lg[t * 2 * E + c] = __ldcg(a.partial + size_t(t) * 2 * E + c);
        }
    consumers_sync();
    if (!*abort_flag)
        for (int t = warp; t < T; t += kConsumers)
            topk_token<EPL>(lg + t * 2 * E, E, K, a.renorm, a.has_mask, a.thr, R.idx + t * K,
                            R.w + t * K, nullptr, nullptr, R.cnt, nullptr, R.hist);
    consumers_sync();
    if (!*abort_flag) {
        for (int i = tid; i < T * K; i += kConsumerThreads) {
            const int e = R.idx[i];
            if (e >= 0) atomicOr(&R.tmask[e], 1u << (i / K));
        }
        if (tid < T) {
            int c = 0;
            for (int k = 0; k < K; ++k) c += R.idx[tid * K + k] >= 0;
            R.nkept[tid] = c;
        }
    }
    consumers_sync();
    // Thread e (of the first 8 warps) takes expert e: its padded rows, pairs,
    // touched flag and tiles are scanned across the warp, then across the 8
    // warp totals (exclusive prefixes, experts ascending).
    if (warp < kMaxE / 32) {
        const int BN = a.BN, lbn = __ffs(BN) - 1;  // BN is a power of two
        const int e = tid;
        const int c = (e < E && !*abort_flag) ? R.cnt[e] : 0;
        const int nt = (c + BN - 1) >> lbn;
        int v[4] = {nt * BN, c, c > 0, nt};  // rows, pairs, touched, tiles
        int inc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int x = v[i];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(kAll, x, off);
                if (lane >= off) x += o;
            }
            inc[i] = x;
            if (lane == 31) s_wtot[warp][i] = x;
        }
        asm volatile("bar.sync 3, %0;" ::"n"(kMaxE) : "memory");  // the 8 scanning warps
        int base[4] = {0, 0, 0, 0};
        for (int w = 0; w < warp; ++w)
#pragma unroll
            for (int i = 0; i < 4; ++i) base[i] += s_wtot[w][i];
        if (e < E) {
            R.off[e] = base[0] + inc[0] - v[0];
            R.coff[e] = base[1] + inc[1] - v[1];
            R.toff[e] = base[3] + inc[3] - v[3];
            if (c > 0) R.te[base[2] + inc[2] - v[2]] = e;
        }
        if (tid == kMaxE - 1) {
            R.n_rows = base[0] + inc[0];
            R.n_pairs = base[1] + inc[1];
            R.n_touched = base[2] + inc[2];  // 0 after a failure: no expert units
            R.n_tiles = base[3] + inc[3];
        }
    }
    consumers_sync();
    if (!*abort_flag)
        for (int i = tid; i < T * K; i += kConsumerThreads) {
            const int e = R.idx[i];
            if (e >= 0) {
                const int t = i / K;
                const int rank = __popc(R.tmask[e] & ((1u << t) - 1u));
                R.pos[i] = R.off[e] + rank;
                R.pl[R.coff[e] + rank] = i;
                R.tok[R.coff[e] + rank] = t;
            }
        }
    all_sync();  // the producer may now fill expert tiles
    if (*abort_flag) return;

    // The last CTA leaves the routing and grouping arrays in the workspace,
    // as the multi-kernel path does, and zeroes the rows of tokens that keep
    // no expert (no down unit reaches them).
    if (b == G - 1) {
#pragma unroll 1
        for (int i = tid; i < T * K; i += kConsumerThreads) {
            a.idx[i] = R.idx[i];
            a.w[i] = R.w[i];
            if (R.idx[i] >= 0) a.pair_pos[i] = R.pos[i];
        }
#pragma unroll 1
        for (int i = tid; i < E; i += kConsumerThreads) a.counts[i] = R.cnt[i];
        if (tid <= K) a.hist[tid] = R.hist[tid];
        if (tid == 0) {
            a.hdr[kHdrMeta + 0] = R.n_tiles;
            a.hdr[kHdrMeta + 1] = R.n_rows;
            a.hdr[kHdrMeta + 2] = R.n_pairs;
            a.hdr[kHdrMeta + 3] = 0;
        }
#pragma unroll 1
        for (int q = warp; q < R.n_touched; q += kConsumers) {
            const int e = R.te[q], c = R.cnt[e], BN = a.BN;
            const int padded = (c + BN - 1) / BN * BN;
#pragma unroll 1
            for (int j = lane; j < padded; j += 32)
                a.pair[R.off[e] + j] = j < c ? R.pl[R.coff[e] + j] : -1;
#pragma unroll 1
            for (int j = lane; j * BN < c; j += 32)
                a.tiles[R.toff[e] + j] = make_int4(e, R.off[e] + j * BN, min(BN, c - j * BN), 0);
        }
#pragma unroll 1
        for (int t = warp; t < T; t += kConsumers)
            if (R.nkept[t] == 0)
#pragma unroll 1
                for (int v = lane; v < nch; v += 32)
                    reinterpret_cast<uint4 *>(a.out)[size_t(t) * nch + v] = make_uint4(0, 0, 0, 0);
    }

    // ------------------------------------------------- 3. expert units ----
    if (warp >= Wc) return;
    const int my_nu = n_units(), e1u = n_up_units();
    const int n_it = e1u * NKT1 + (my_nu - e1u) * NKT2;
    uint16_t *H = static_cast<uint16_t *>(a.H);
    const int gid = lane >> 2, tig = lane & 3;
    // ldmatrix addressing: A (16 x 16) lane -> row, column; B (16 x 8) lanes
    // 0-15 -> token row (lane & 7, plus 8 for the second group), k half.
    const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_col = (lane >> 4) * 8;
    const int b_n = lane & 7, b_k = ((lane >> 3) & 1) * 8;
    const uint32_t x_base = smem_u32(x_s);
    for (int g = my_ri + ((warp - my_ri) % Wc + Wc) % Wc; g < my_ri + n_it; g += Wc) {
        if (*abort_flag) break;
        int j, kt;
        item_of(g - my_ri, e1u, j, kt);
        const Unit u = unit_of(b + j * G);
        const int ne = R.cnt[u.e], coff = R.coff[u.e], hrow0 = R.off[u.e];
        const int ng = ne > 8 ? 2 : 1;  // token groups of the N = 8 side
        // B rows: token b_n of each group (the last token stands in beyond
        // the expert's tokens; those columns are never stored)
        const int nA = min(b_n, ne - 1), nB = min(8 + b_n, ne - 1);
        float acc[2][2][4];  // [token group][k-step parity][fragment]
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[q][p][i] = 0.0f;
        const int wi = g / Wc, s = warp * M + wi % M;  // this warp's item wi
        if (!__all_sync(kAll, mbar_wait_bounded(&full_bar[s], uint32_t((wi / M) & 1), abort_flag,
                                                a.timeout_ns))) {
            give_up();
            break;
        }
        const uint32_t st = smem_u32(stage0 + size_t(s) * SB);
        if (u.up) {
            const int k0 = kt * kKT1, nks = min(kKT1, d - k0) / 16;
            // A: rows 0-7 from the W1 boxes, 8-15 from the W3 boxes
            const uint32_t pa = st + (a_row < 8 ? 0u : 4096u);
            const uint32_t pb0 = x_base + uint32_t((R.tok[coff + nA] * XSP + k0 + b_k) * 2);
            const uint32_t pb1 = x_base + uint32_t((R.tok[coff + nB] * XSP + k0 + b_k) * 2);
#pragma unroll 1
            for (int ks = 0; ks < nks; ks += 2) {
                uint32_t a0[4], a1[4], b0, b1, c0, c1;
                const int jb = ks >> 2, ch = (ks & 3) * 2 + (a_col >> 3);
                ldsm_x4(a0, pa + jb * 1024 + swz(a_row & 7, ch));
                ldsm_x4(a1, pa + jb * 1024 + swz(a_row & 7, ch + 2));
                ldsm_x2(b0, b1, pb0 + ks * 32);
                ldsm_x2(c0, c1, pb0 + ks * 32 + 32);
                mma_16816(acc[0][0], a0, b0, b1);
                mma_16816(acc[0][1], a1, c0, c1);
                if (ng > 1) {
                    ldsm_x2(b0, b1, pb1 + ks * 32);
                    ldsm_x2(c0, c1, pb1 + ks * 32 + 32);
                    mma_16816(acc[1][0], a0, b0, b1);
                    mma_16816(acc[1][1], a1, c0, c1);
                }
            }
        } else {
#pragma unroll 1
            for (int ks = 0; ks < kKT2 / 16; ks += 2) {
                uint32_t a0[4], a1[4], b0, b1, c0, c1;
                const int jb = ks >> 2, ca = (ks & 3) * 2 + (a_col >> 3);
                const int cb = (ks & 3) * 2 + (b_k >> 3);
                const uint32_t pa = st + jb * 2048, ph = st + 4096 + jb * 2048;
                ldsm_x4(a0, pa + swz(a_row, ca));
                ldsm_x4(a1, pa + swz(a_row, ca + 2));
                ldsm_x2(b0, b1, ph + swz(nA, cb));
                ldsm_x2(c0, c1, ph + swz(nA, cb + 2));
                mma_16816(acc[0][0], a0, b0, b1);
                mma_16816(acc[0][1], a1, c0, c1);
                if (ng > 1) {
                    ldsm_x2(b0, b1, ph + swz(nB, cb));
                    ldsm_x2(c0, c1, ph + swz(nB, cb + 2));
                    mma_16816(acc[1][0], a0, b0, b1);
                    mma_16816(acc[1][1], a1, c0, c1);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
        // This tile's partial sums (lane: 2 groups x 4 fragment values), then
        // the unit's running sum from its slot, in k-tile order.
        float v[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[i] = acc[0][0][i] + acc[0][1][i];
            v[4 + i] = acc[1][0][i] + acc[1][1][i];
        }
        const int sl = j % kSlots, key = j * NKTM + kt;
        bool ok = true;
        if (lane == 0) {
            const volatile int *nx = &s_next[sl];
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t spin = 0; *nx != key; ++spin) {
                if (*abort_flag || globaltimer_ns() - t0 > a.timeout_ns) {
                    ok = false;
                    break;
                }
                if (spin > 16) __nanosleep(32);
            }
        }
        if (!__shfl_sync(kAll, ok, 0)) {
            give_up();
            break;
        }
        __threadfence_block();
        float4 *slot = reinterpret_cast<float4 *>(&s_acc[sl][lane][0]);
        if (kt > 0) {
            const float4 p0 = slot[0], p1 = slot[1];
            v[0] += p0.x;
            v[1] += p0.y;
            v[2] += p0.z;
            v[3] += p0.w;
            v[4] += p1.x;
            v[5] += p1.y;
            v[6] += p1.z;
            v[7] += p1.w;
        }
        if (kt + 1 < u.nkt) {  // hand the running sum to the next k-tile
            slot[0] = make_float4(v[0], v[1], v[2], v[3]);
            slot[1] = make_float4(v[4], v[5], v[6], v[7]);
            __threadfence_block();
            __syncwarp();
            if (lane == 0) *reinterpret_cast<volatile int *>(&s_next[sl]) = key + 1;
            continue;
        }
        // The unit's last k-tile: hand the slot to unit j + kSlots, then the
        // epilogue.  Lane (gid, tig) holds rows gid and gid + 8 of the tile for
        // tokens 2 tig and 2 tig + 1 of each group.
        __syncwarp();
        if (lane == 0)
            *reinterpret_cast<volatile int *>(&s_next[sl]) = (j + kSlots) * NKTM;
        for (int q = 0; q < ng; ++q) {
            const float *w4 = v + 4 * q;
            const int n0 = q * 8 + tig * 2, n1 = n0 + 1;
            if (u.up) {  // rows 0-7: gate (W1), rows 8-15: up (W3), same rows of I
                if (n0 < ne)
                    H[size_t(hrow0 + n0) * I + u.row0 + gid] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(silu_mul(w4[0], w4[2])));
                if (n1 < ne)
                    H[size_t(hrow0 + n1) * I + u.row0 + gid] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(silu_mul(w4[1], w4[3])));
            } else {
                if (n0 < ne) {
                    a.Y[size_t(hrow0 + n0) * d + u.row0 + gid] = w4[0];
                    a.Y[size_t(hrow0 + n0) * d + u.row0 + gid + 8] = w4[2];
                }
                if (n1 < ne) {
                    a.Y[size_t(hrow0 + n1) * d + u.row0 + gid] = w4[1];
                    a.Y[size_t(hrow0 + n1) * d + u.row0 + gid + 8] = w4[3];
                }
            }
        }
        __syncwarp();
        if (u.up) {
            if (lane == 0) {
                __threadfence_block();
                const int kb = u.row0 / kKT2;  // the publisher warp makes it visible
                atomicAdd(&s_done[u.ti][kb >> 2], 1u << (8 * (kb & 3)));
            }
            continue;
        }
        // 4. combine: the unit that completes (token, 16-column block) sums it.
        const int blk = u.row0 / 16;
        bool last = false;
        int t = -1;
        if (lane < ne) {
            t = R.tok[coff + lane];
            const int old = atom_add_acq_rel(a.comb_cnt + t * U2 + blk, 1);
            last = old == R.nkept[t] - 1;
        }
        unsigned lm = __ballot_sync(kAll, last);
        __syncwarp();
        while (lm) {
            const int src = __ffs(lm) - 1;
            lm &= lm - 1u;
            const int tt = __shfl_sync(kAll, t, src);
            if (lane < 16) {
                float sum = 0.0f;
                for (int k = 0; k < K; ++k) {
                    const int o = tt * K + k;
                    if (R.idx[o] >= 0)
                        sum = fmaf(R.w[o], __ldcg(a.Y + size_t(R.pos[o]) * d + u.row0 + lane), sum);
                }
                reinterpret_cast<__nv_bfloat16 *>(a.out)[size_t(tt) * d + u.row0 + lane] =
                    __float2bfloat16_rn(sum);
            }
        }
    }
}

template <int EPL>
cudaError_t launch_epl(const DlMaps &maps, const DecodeLayerArgs &a, int grid,
                       cudaStream_t stream) {
    static std::atomic<unsigned long long> done{0};
    cudaError_t e = set_smem_once(decode_layer_kernel<EPL>, kDlSmemCap, done);
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_layer_kernel<EPL>, dim3(grid), dim3(kThreads), size_t(a.smem_bytes),
                      stream, maps, a);
}

}  // namespace

bool decode_layer_config(int T, int d, int E, int I, int K, int has_mask, int n_sm,
                         DecodeLayerArgs *c) {
    if (T < 1 || T > kDlMaxT || E > kMaxE || K > kMaxK || n_sm < 1) return false;
    if (d % 128 != 0 || I % kKT2 != 0) return false;
    // A stage holds a gate/up tile, a down tile with its H rows, or the
    // rows of a router item (two rows when they fit, else one).
    const int rr = 4 * d <= kStageMin ? 2 : 1;
    const int sb = (max(kStageMin, rr * d * 2) + 1023) / 1024 * 1024;
    const int n_rows = has_mask ? 2 * E : E;
    const int x_bytes = T * (d + 8) * 2;
    const int lg_bytes = T * 2 * E * 4;
    const int off_lg = (x_bytes + 127) / 128 * 128;
    const int off_stage = (off_lg + lg_bytes + 1023) / 1024 * 1024;  // swizzled boxes: 1 KB
    const int ns = min(kDlMaxStages, (kDlSmemCap - 1024 - off_stage) / sb);
    if (ns < 4) return false;
    c->T = T;
    c->d = d;
    c->E = E;
    c->I = I;
    c->K = K;
    c->has_mask = has_mask;
    c->R1 = 8;
    c->R2 = 16;
    c->rr = rr;
    c->n_ru = (n_rows + rr - 1) / rr;
    c->n_stages = ns;
    c->stage_bytes = sb;
    c->sm_off_lg = off_lg;
    c->sm_off_stage = off_stage;
    c->smem_bytes = off_stage + ns * sb + 1024;  // + slack to align the stages
    return true;
}

cudaError_t launch_decode_layer(const DlMaps &maps, const DecodeLayerArgs &a, int grid,
                                cudaStream_t stream) {
    const int epl = (a.E + 31) / 32;
    if (epl <= 1) return launch_epl<1>(maps, a, grid, stream);
    if (epl <= 2) return launch_epl<2>(maps, a, grid, stream);
    if (epl <= 4) return launch_epl<4>(maps, a, grid, stream);
    return launch_epl<8>(maps, a, grid, stream);
}

}  // namespace beam
