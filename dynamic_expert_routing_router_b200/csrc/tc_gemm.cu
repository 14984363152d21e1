// tc_gemm.cu -- grouped GEMMs of the BEAM MoE layer on the sm_100a tensor
// cores (tcgen05.mma, fp32 accumulators in TMEM, operands staged by TMA).
//
// One persistent, warp-specialised kernel serves every role:
//   MODE_ROUTER   logits  r = x W_gate, z = x W_mask   (BEAM §3.2 steps 1-2)
//   MODE_GEMM1    H = SiLU(x W1_e^T) * (x W3_e^T)      (Eq. 3, gate/up + SwiGLU)
//                 two 128-row weight tiles (W1, W3), two accumulators
//   MODE_GEMM1_IL the same with 64 rows of W1 and the matching 64 rows of W3
//                 in one 128-row tile and one accumulator (twice the units);
//                 the epilogue warps pair gate and up rows through shared memory
//   MODE_GEMM2    Y = H W2_e^T  (fp32 out)              (Eq. 3, down projection)
//   MODE_GEMM2T   dh = dy W2_e (training): the A tile is 128 columns of W2_e
//                 over 64 of its rows, i.e. W2_e read transposed (MN-major,
//                 two 64-column TMA boxes per stage); fp32 out
//   MODE_GEMM1T   dxp = da W1_e + db W3_e (training): one reduction of 2I
//                 k-rows, W1_e with da rows then W3_e with db rows, the weights
//                 read transposed as in MODE_GEMM2T; fp32 out
//   MODE_EXPERTS  MODE_GEMM1_IL units followed by MODE_GEMM2 units in one
//                 launch: a down-projection unit of a token tile starts once
//                 every gate/up unit of that tile has published its rows of H
//                 (per-tile counter), so the second GEMM fills the first one's
//                 tail instead of waiting for a kernel boundary.
//
// Orientation: the weight rows are the MMA's M operand (128 rows per tile)
// and the tokens are its N operand (BN = 16..128 per tile), D = W * X^T.  A
// decode step touches few tokens per expert, so the weights (the bytes that
// matter) fill the 128-row side; a prefill tile uses BN = 128 tokens.
// The GEMMs run only over the tile list built from KEPT pairs: an expert
// without kept pairs has no tile, and TMA never reads its weights.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0      TMA producer (one thread): weight tile(s) + token tile per stage
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warps 2..5  epilogue: TMEM -> registers -> activation -> global memory
// Pipelines: a STAGES-deep shared-memory ring (full/empty mbarriers) and a
// 2-deep TMEM accumulator ring (tfull/tempty), so the epilogue of one unit
// overlaps the MMAs of the next.  Every wait is bounded (beam_ptx.cuh); on
// expiry the CTA records DEV_ERR_TIMEOUT, drains its own copies and MMAs,
// frees TMEM and returns.
//
// MODE_EXPERTS hands units out dynamically: CTA b starts with unit b, then
// its producer takes the next index from a global counter (all gate/up units
// first, then the smaller down units, so the tail is made of small units) and
// passes it to the MMA and epilogue warps through a 4-slot ring in shared
// memory.  It cannot deadlock: gate/up units wait on nothing outside their
// CTA; a down unit waits only for lower-numbered gate/up units, each of which
// is a CTA's first unit (that CTA owns an SM of its own: the grid is at most
// one CTA per SM) or was taken from the counter by a running CTA whose
// producer issued all of that unit's loads before taking another index.  The other modes deal units round-robin.
#include <cuda_bf16.h>

#include "beam_internal.h"
#include "beam_ptx.cuh"

namespace beam {

namespace {

constexpr int kThreads = 192;
constexpr int kUmmaK = 16;  // K of one kind::f16 MMA
constexpr int kXchLd = 17;  // padded row of the gate/up exchange buffer (floats)

template <int NUM_A, int BN, bool XCH>
struct TcCfg {
    static constexpr uint32_t A_BYTES = kBlockM * kBlockK * 2;  // 16 KB
    static constexpr uint32_t B_BYTES = BN * kBlockK * 2;
    static constexpr uint32_t STAGE_BYTES = NUM_A * A_BYTES + B_BYTES;
    static constexpr uint32_t XCH_BYTES = XCH ? kBlockM * kXchLd * 4 : 0;
    static constexpr int STAGES_FIT = int((220u * 1024u - XCH_BYTES) / STAGE_BYTES);
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr uint32_t SMEM_BYTES =
        STAGES * STAGE_BYTES + XCH_BYTES + 1024;  // + alignment slack
    static constexpr uint32_t ACC_COLS = NUM_A * BN;  // fp32 columns per accumulator
    // Two accumulator buffers (one unit's epilogue overlaps the next unit's
    // MMAs) when they fit the 512 TMEM columns, else one.
    static constexpr uint32_t ACC_BUFS = 2 * ACC_COLS <= 512 ? 2 : 1;
    static constexpr uint32_t TMEM_COLS = ACC_BUFS * ACC_COLS;
    static_assert(STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned");
    static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0,
                  "TMEM allocation must be a power of two in [32, 512]");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
    static_assert(STAGES >= 2, "pipeline too shallow");
    static_assert(SMEM_BYTES <= 227u * 1024u, "shared memory");
};

template <int MODE>
struct ModeTraits {
    static constexpr int NUM_A = MODE == MODE_GEMM1 ? 2 : 1;
    static constexpr bool XCH = MODE == MODE_GEMM1_IL || MODE == MODE_EXPERTS;
};

struct Unit {
    int phase;  // MODE_EXPERTS: 0 = gate/up unit, 1 = down unit; else 0
    int ti;     // tile index (GEMMs)
    int mb;     // weight-row block
    int a_row;  // first row of the A (weight) tile in its 2D tensor map
    int b_row;  // first row of the B (token) tile
    int kb0;    // first k-block
    int nk;     // k-blocks of this unit
    int sel;    // router: 0 = W_gate rows, 1 = W_mask rows
    int tt, s;  // router: token tile, split
    int rows;   // GEMMs: valid token rows of the tile
    int out_row;  // GEMMs: first output row (= b_row except for dense units)
};

// Named barrier of the four epilogue warps (barrier 0 is __syncthreads).
__device__ __forceinline__ void epilogue_sync() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int MODE, int BN>
__device__ __forceinline__ Unit decode_unit(int u, int n_first, const TcGemmArgs &p) {
    Unit w;
    w.phase = 0;
    w.sel = 0;
    w.tt = w.s = 0;
    w.kb0 = 0;
    w.nk = p.nk;
    if (MODE == MODE_ROUTER) {
        w.mb = u % p.n_mb;
        const int rest = u / p.n_mb;
        w.ti = 0;
        w.tt = rest % p.n_tt;
        w.s = rest / p.n_tt;
        w.sel = w.mb >= p.n_mb_gate ? 1 : 0;
        w.a_row = (w.sel ? w.mb - p.n_mb_gate : w.mb) * kBlockM;
        w.b_row = w.tt * BN;
        w.kb0 = w.s * p.nk;
        w.rows = 0;
        w.out_row = 0;
        return w;
    }
    int v = u, n_mb = p.n_mb, rows_per_mb = kBlockM, a_rows = p.a_rows_per_expert;
    if (MODE == MODE_GEMM1_IL) rows_per_mb = kBlockM / 2;
    if (MODE == MODE_GEMM2T || MODE == MODE_GEMM1T)
        rows_per_mb = 0;  // a_row: the expert's first k-row; mb picks columns
    if (MODE == MODE_EXPERTS) {
        if (u < n_first) {
            rows_per_mb = kBlockM / 2;
        } else {
            w.phase = 1;
            v = u - n_first;
            n_mb = p.n_mb2;
            a_rows = p.a_rows2;
            w.nk = p.nk2;
        }
    }
    w.mb = v % n_mb;
    w.ti = v / n_mb;
    if ((MODE == MODE_GEMM1 || MODE == MODE_GEMM2) && p.dense) {
        const int ks = p.dense_ksplit > 1 ? p.dense_ksplit : 1;
        const int js = u % ks, vv = u / ks;
        w.mb = vv % n_mb;
        w.ti = vv / n_mb;
        w.kb0 = js * p.nk / ks;
        w.nk = (js + 1) * p.nk / ks - w.kb0;
        const int sx = w.ti / p.dense_ntt, t0 = (w.ti % p.dense_ntt) * BN;
        w.a_row = sx * a_rows + w.mb * rows_per_mb;
        w.out_row = js * p.dense_slab_rows + sx * p.dense_T + t0;
        w.b_row = p.dense_gemm2 ? sx * p.dense_T + t0 : t0;
        w.rows = min(BN, p.dense_T - t0);
        return w;
    }
    const int4 t = p.tiles[w.ti];
    w.a_row = t.x * a_rows + w.mb * rows_per_mb;
    w.b_row = t.y;
    w.out_row = t.y;
    w.rows = t.z;
    return w;
}

// A bounded wait expired: record it (DEV_ERR_TIMEOUT, or the router's tag)
// and tell the CTA's other roles to stop.
// Token columns a unit computes: its valid rows rounded up to the MMA's N
// step of 16 (16 <= N <= BN for M = 128).
template <int MODE, int BN>
__device__ __forceinline__ int unit_cols(const Unit &w, const TcGemmArgs &p) {
    const int rows = MODE == MODE_ROUTER ? min(BN, p.T - w.tt * BN) : w.rows;
    const int n = (rows + 15) & ~15;
    return n < 16 ? 16 : (n > BN ? BN : n);
}

__device__ __forceinline__ void signal_abort(const TcGemmArgs &p, int *abort_flag) {
    atomicExch(p.err, p.err_code ? p.err_code : int(DEV_ERR_TIMEOUT));
    *reinterpret_cast<volatile int *>(abort_flag) = 1;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    return g / (1.0f + __expf(-g)) * u;
}

// Bounded wait until *ctr >= need (acquire at GPU scope).
__device__ __forceinline__ bool wait_counter_bounded(const int *ctr, int need,
                                                     const volatile int *abort_flag,
                                                     uint64_t timeout_ns) {
    uint64_t t0 = 0;
    for (uint32_t spin = 0; spin < (1u << 24); ++spin) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= need) return true;
        if ((spin & 31u) == 0) {
            if (*abort_flag) return false;
            const uint64_t t = globaltimer_ns();
            if (spin == 0) t0 = t;
            else if (t - t0 > timeout_ns) return false;
        }
        __nanosleep(100);
    }
    return false;
}

template <int MODE, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ TcMaps maps, const TcGemmArgs p) {
    constexpr int NUM_A = ModeTraits<MODE>::NUM_A;
    using C = TcCfg<NUM_A, BN, ModeTraits<MODE>::XCH>;
    constexpr int STAGES = C::STAGES;

    extern __shared__ uint8_t smem_raw[];
    __shared__ int xvote[4];   // epilogue warps: "accumulator arrived" votes
    __shared__ int uvote[4];   // epilogue warps: "unit received / hand-out over" votes
    __shared__ __align__(8) uint64_t full_bar[STAGES];
    __shared__ __align__(8) uint64_t empty_bar[STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    constexpr bool DYN = MODE == MODE_EXPERTS;  // dynamic unit hand-out
    constexpr int kRing = 4;
    __shared__ int unit_ring[kRing];
    __shared__ __align__(8) uint64_t unit_full[kRing];
    __shared__ __align__(8) uint64_t unit_empty[kRing];

    // 1024-byte aligned start of the stage ring (SWIZZLE_128B atoms).
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const volatile int *abort_flag = &abort_sh;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 128);
        }
        mbar_init(&drain_bar, 1);
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&unit_full[i], 1);
            mbar_init(&unit_empty[i], 1 + 4);  // MMA thread + one lane per epilogue warp
        }
        abort_sh = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&maps.a0);
        tma_prefetch_desc(&maps.a1);
        tma_prefetch_desc(&maps.b);
        if (MODE == MODE_EXPERTS) {
            tma_prefetch_desc(&maps.a2);
            tma_prefetch_desc(&maps.b2);
        }
    }
    if (warp == 1) tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = tmem_base_sh;

    // Everything above is private to the CTA; global memory only from here.
    griddep_wait();
    griddep_launch_dependents();
    if (MODE == MODE_ROUTER && blockIdx.x == 0) {
        // Per-call counters of the later kernels start at zero.
        for (int r = 0; r < 3; ++r)
            if (p.zero[r].ptr)
                for (int i = threadIdx.x; i < p.zero[r].count; i += blockDim.x) p.zero[r].ptr[i] = 0;
    }
    const bool dense = (MODE == MODE_GEMM1 || MODE == MODE_GEMM2) && p.dense;
    const int ntiles = (MODE == MODE_ROUTER) ? 0 : dense ? p.n_units / p.n_mb : p.meta[0];
    const int n_first = ntiles * p.n_mb;  // units of the first GEMM
    const int n_units = (MODE == MODE_ROUTER)    ? p.n_units
                        : (MODE == MODE_EXPERTS) ? n_first + ntiles * p.n_mb2
                                                 : n_first;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t lu = 0;; ++lu) {
                int u = blockIdx.x + int(lu) * gridDim.x;
                if (DYN) {
                    const int slot = int(lu % kRing);
                    if (!mbar_wait_bounded(&unit_empty[slot], ((lu / kRing) & 1u) ^ 1u, abort_flag,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    // The first unit of CTA b is unit b (no global round trip
                    // before the first loads); later ones come from the
                    // counter, after the gridDim.x first units.
                    u = lu == 0 ? int(blockIdx.x) : int(gridDim.x) + atomicAdd(p.work_ctr, 1);
                    if (u >= n_units) u = -1;
                    unit_ring[slot] = u;
                    mbar_arrive(&unit_full[slot]);
                    if (u < 0) break;
                } else if (u >= n_units) {
                    break;
                }
                const Unit w = decode_unit<MODE, BN>(u, n_first, p);
                const CUtensorMap *am = &maps.a0;
                const CUtensorMap *bm = &maps.b;
                if (MODE == MODE_ROUTER && w.sel) am = &maps.a1;
                if (MODE == MODE_EXPERTS && w.phase == 1) {
                    // H rows of this tile come from other CTAs' gate/up units.
                    if (!wait_counter_bounded(p.tile_done + w.ti, p.n_mb, abort_flag,
                                              p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    am = &maps.a2;
                    bm = &maps.b2;
                }
                const bool interleaved =
                    MODE == MODE_GEMM1_IL || (MODE == MODE_EXPERTS && w.phase == 0);
                for (int kb = 0; kb < w.nk; ++kb, ++it) {
                    const int s = int(it % STAGES);
                    const uint32_t ph = ((it / STAGES) & 1u) ^ 1u;
                    if (!mbar_wait_bounded(&empty_bar[s], ph, abort_flag, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (p.fault_skip && blockIdx.x == 0 && lu == 0 && kb == 0)
                        continue;  // test hook: this stage never fills (its MMA wait expires)
                    uint8_t *st = smem + size_t(s) * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full_bar[s], C::STAGE_BYTES);
                    int kx = (w.kb0 + kb) * kBlockK;
                    if (MODE == MODE_GEMM1T && 2 * kb >= w.nk) {  // second half: W3_e with db
                        am = &maps.a1;
                        bm = &maps.b2;
                        kx -= (w.nk / 2) * kBlockK;
                    }
                    if (MODE == MODE_GEMM2T || MODE == MODE_GEMM1T) {
                        // W2_e rows [kx, kx + 64) x columns [mb 128, + 128): two boxes
                        tma_load_2d(st, am, w.mb * kBlockM, w.a_row + kx, &full_bar[s]);
                        tma_load_2d(st + C::A_BYTES / 2, am, w.mb * kBlockM + kBlockM / 2,
                                    w.a_row + kx, &full_bar[s]);
                    } else if (interleaved) {
                        // rows 0..63: W1 (gate), rows 64..127: W3 (up), same I rows
                        tma_load_2d(st, &maps.a0, kx, w.a_row, &full_bar[s]);
                        tma_load_2d(st + C::A_BYTES / 2, &maps.a1, kx, w.a_row, &full_bar[s]);
                    } else {
                        tma_load_2d(st, am, kx, w.a_row, &full_bar[s]);
                    }
                    if (NUM_A == 2)
                        tma_load_2d(st + C::A_BYTES, &maps.a1, kx, w.a_row, &full_bar[s]);
                    tma_load_2d(st + NUM_A * C::A_BYTES, bm, kx, w.b_row, &full_bar[s]);
                }
                if (!ok) break;
            }
            if (!ok) {
                signal_abort(p, &abort_sh);
                // Let this CTA's own copies land before it can exit.
                for (uint32_t j = (it > uint32_t(STAGES) ? it - STAGES : 0u); j < it; ++j)
                    mbar_wait_bounded(&full_bar[j % STAGES], (j / STAGES) & 1u, nullptr,
                                      p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer --
        if (lane == 0) {
            constexpr uint32_t kAMajor =
                (MODE == MODE_GEMM2T || MODE == MODE_GEMM1T) ? kIdescAMajorMN : 0u;
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t lu = 0;; ++lu) {
                int u = blockIdx.x + int(lu) * gridDim.x;
                if (DYN) {
                    const int slot = int(lu % kRing);
                    if (!mbar_wait_bounded(&unit_full[slot], (lu / kRing) & 1u, abort_flag,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    u = unit_ring[slot];
                    mbar_arrive(&unit_empty[slot]);
                    if (u < 0) break;
                } else if (u >= n_units) {
                    break;
                }
                const Unit w = decode_unit<MODE, BN>(u, n_first, p);
                const int nk = w.nk;
                // MMA N = the unit's valid token rows rounded up to 16: the
                // padding rows of an expert's last tile cost no tensor work
                const uint32_t IDESC = umma_idesc_bf16_f32(kBlockM, unit_cols<MODE, BN>(w, p)) |
                                       kAMajor;
                const uint32_t a = lu % C::ACC_BUFS;
                if (!mbar_wait_bounded(&tempty_bar[a], ((lu / C::ACC_BUFS) & 1u) ^ 1u, abort_flag,
                                       p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d0 = tmem_base + a * C::ACC_COLS;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = int(it % STAGES);
                    if (!mbar_wait_bounded(&full_bar[s], (it / STAGES) & 1u, abort_flag,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t sa = smem_u32(smem + size_t(s) * C::STAGE_BYTES);
                    const uint32_t sb = sa + NUM_A * C::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < kBlockK / kUmmaK; ++kk) {
                        const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
                        const uint64_t bdesc = umma_desc_sw128(sb + kk * 32);
                        const uint64_t adesc =
                            (MODE == MODE_GEMM2T || MODE == MODE_GEMM1T)
                                ? umma_desc_sw128_mn(sa + kk * (kUmmaK / 8) * 1024, C::A_BYTES / 2)
                                : umma_desc_sw128(sa + kk * 32);
                        umma_bf16(d0, adesc, bdesc, IDESC, acc);
                        if (NUM_A == 2)
                            umma_bf16(d0 + BN, umma_desc_sw128(sa + C::A_BYTES + kk * 32), bdesc,
                                      IDESC, acc);
                    }
                    umma_commit(&empty_bar[s]);  // stage reusable once these MMAs finish
                }
                if (!ok) break;
                umma_commit(&tfull_bar[a]);  // accumulator complete
            }
            if (!ok) {
                signal_abort(p, &abort_sh);
                umma_commit(&drain_bar);  // wait for the MMAs already issued
                mbar_wait_bounded(&drain_bar, 0u, nullptr, p.timeout_ns);
            }
        }
    } else {
        // --------------------------------------------------- epilogue --
        const int q = warp & 3;          // TMEM lane quadrant this warp may access
        const int row = q * 32 + lane;   // row within the 128-row weight tile
        for (uint32_t lu = 0;; ++lu) {
            int u = blockIdx.x + int(lu) * gridDim.x;
            bool ok = true;
            if (DYN) {
                const int slot = int(lu % kRing);
                ok = mbar_wait_bounded(&unit_full[slot], (lu / kRing) & 1u, abort_flag,
                                       p.timeout_ns);
                ok = __all_sync(0xffffffffu, ok);
                if (ok) {
                    u = unit_ring[slot];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&unit_empty[slot]);
                }
            } else if (u >= n_units) {
                break;  // round-robin: the same u in every epilogue warp
            }
            if (DYN) {
                // The four warps must leave together (they meet at named
                // barriers): agree on "all got a unit", "hand-out finished".
                // Each vote array is written only after barriers that every
                // warp passes after its last read of it.
                if (lane == 0) uvote[warp - 2] = ok ? (u < 0 ? 2 : 1) : 0;
                epilogue_sync();
                const int v0 = uvote[0], v1 = uvote[1], v2 = uvote[2], v3 = uvote[3];
                if (!(v0 && v1 && v2 && v3)) {
                    if (lane == 0) signal_abort(p, &abort_sh);
                    break;
                }
                if (v0 == 2 || v1 == 2 || v2 == 2 || v3 == 2) break;
            }
            const Unit w = decode_unit<MODE, BN>(u, n_first, p);
            const uint32_t a = lu % C::ACC_BUFS;
            ok = mbar_wait_bounded(&tfull_bar[a], (lu / C::ACC_BUFS) & 1u, abort_flag,
                                   p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (ModeTraits<MODE>::XCH) {
                // The four warps meet at named barriers below: agree first.
                if (lane == 0) xvote[warp - 2] = ok ? 1 : 0;
                epilogue_sync();
                ok = xvote[0] && xvote[1] && xvote[2] && xvote[3];
            }
            if (!ok) {
                if (lane == 0) signal_abort(p, &abort_sh);
                break;
            }
            tc_fence_after_sync();
            const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + a * C::ACC_COLS;
            const bool gate_up_il =
                MODE == MODE_GEMM1_IL || (MODE == MODE_EXPERTS && w.phase == 0);
            const bool down = MODE == MODE_GEMM2 || MODE == MODE_GEMM2T || MODE == MODE_GEMM1T ||
                              (MODE == MODE_EXPERTS && w.phase == 1);
            const int ncol = unit_cols<MODE, BN>(w, p);  // same in the 4 epilogue warps
#pragma unroll 1
            for (int c0 = 0; c0 < ncol; c0 += 16) {
                uint32_t g[16], v[16];
                tmem_ld_16(tb + c0, g);
                if (NUM_A == 2) tmem_ld_16(tb + BN + c0, v);
                tmem_ld_wait();
                reg_fence_16(g);
                if (NUM_A == 2) reg_fence_16(v);
                if (MODE == MODE_ROUTER) {
                    const int jr = (w.sel ? w.mb - p.n_mb_gate : w.mb) * kBlockM + row;
                    if (jr < p.E) {
                        const int j = w.sel ? p.E + jr : jr;
                        float *out = static_cast<float *>(p.out) + w.s * p.out_split_stride + j;
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const int t = w.tt * BN + c0 + c;
                            if (t < p.T) out[(long long)t * p.out_ld] = __uint_as_float(g[c]);
                        }
                    }
                } else if (gate_up_il) {
                    // TMEM rows 0..63 hold gate, 64..127 up, for I rows mb*64 + r.
                    float *xch = reinterpret_cast<float *>(smem + size_t(STAGES) * C::STAGE_BYTES);
#pragma unroll
                    for (int c = 0; c < 16; ++c) xch[row * kXchLd + c] = __uint_as_float(g[c]);
                    epilogue_sync();
                    const int et = threadIdx.x - 64;  // 0..127 over the epilogue warps
                    const int r = et & 63, half = et >> 6;
                    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out) +
                                         (long long)w.out_row * p.out_ld + w.mb * (kBlockM / 2) + r;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        const int c = half * 8 + cc;
                        if (c0 + c < w.rows)
                            out[(long long)(c0 + c) * p.out_ld] = __float2bfloat16_rn(
                                silu_mul(xch[r * kXchLd + c], xch[(64 + r) * kXchLd + c]));
                    }
                    epilogue_sync();
                } else if (MODE == MODE_GEMM1) {
                    // H (bf16): the next GEMM's operand (none when the
                    // reduction is split: the partials are summed later).
                    if (p.out) {
                        __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out) +
                                             (long long)w.out_row * p.out_ld + w.mb * kBlockM + row;
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            if (c0 + c < w.rows)
                                out[(long long)(c0 + c) * p.out_ld] = __float2bfloat16_rn(
                                    silu_mul(__uint_as_float(g[c]), __uint_as_float(v[c])));
                    }
                    if (p.a_out) {  // training: both pre-activations in fp32
                        const long long o = (long long)w.out_row * p.out_ld + w.mb * kBlockM + row;
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            if (c0 + c < w.rows) {
                                p.a_out[o + (long long)(c0 + c) * p.out_ld] = __uint_as_float(g[c]);
                                p.b_out[o + (long long)(c0 + c) * p.out_ld] = __uint_as_float(v[c]);
                            }
                    }
                } else if (down) {
                    // Y (fp32): rounded once, after the weighted combine.
                    void *base = (MODE == MODE_EXPERTS) ? p.out2 : p.out;
                    const long long ld = (MODE == MODE_EXPERTS) ? p.out2_ld : p.out_ld;
                    float *out = static_cast<float *>(base) + (long long)w.out_row * ld +
                                 w.mb * kBlockM + row;
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (c0 + c < w.rows) out[(long long)(c0 + c) * ld] = __uint_as_float(g[c]);
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&tempty_bar[a]);
            if (MODE == MODE_EXPERTS && w.phase == 0) {
                // Publish this unit's rows of H to the down units of the tile.
                __threadfence();
                epilogue_sync();
                if (threadIdx.x == 64)
                    asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(p.tile_done + w.ti)
                                 : "memory");
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <int MODE, int BN>
cudaError_t launch_cfg(const TcMaps &maps, const TcGemmArgs &args, int grid,
                       cudaStream_t stream) {
    using C = TcCfg<ModeTraits<MODE>::NUM_A, BN, ModeTraits<MODE>::XCH>;
    auto kern = tc_gemm_kernel<MODE, BN>;
    static std::atomic<unsigned long long> attr_set{0};  // this instantiation only
    cudaError_t e = set_smem_once(kern, int(C::SMEM_BYTES), attr_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(grid), dim3(kThreads), C::SMEM_BYTES, stream, maps, args);
}

template <int MODE>
cudaError_t launch_bn(int bn, const TcMaps &maps, const TcGemmArgs &args, int grid,
                      cudaStream_t stream) {
    switch (bn) {
        case 16: return launch_cfg<MODE, 16>(maps, args, grid, stream);
        case 32: return launch_cfg<MODE, 32>(maps, args, grid, stream);
        case 64: return launch_cfg<MODE, 64>(maps, args, grid, stream);
        case 128: return launch_cfg<MODE, 128>(maps, args, grid, stream);
        case 256:  // prefill batches: the two expert GEMMs only
            if constexpr (MODE == MODE_GEMM1 || MODE == MODE_GEMM2)
                return launch_cfg<MODE, 256>(maps, args, grid, stream);
            else
                return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_tc_gemm(int mode, int bn, const TcMaps &maps, const TcGemmArgs &args, int grid,
                           cudaStream_t stream) {
    if (grid <= 0) return cudaSuccess;
    switch (mode) {
        case MODE_ROUTER: return launch_bn<MODE_ROUTER>(bn, maps, args, grid, stream);
        case MODE_GEMM1: return launch_bn<MODE_GEMM1>(bn, maps, args, grid, stream);
        case MODE_GEMM2: return launch_bn<MODE_GEMM2>(bn, maps, args, grid, stream);
        case MODE_GEMM1_IL: return launch_bn<MODE_GEMM1_IL>(bn, maps, args, grid, stream);
        case MODE_EXPERTS: return launch_bn<MODE_EXPERTS>(bn, maps, args, grid, stream);
        case MODE_GEMM2T: return launch_bn<MODE_GEMM2T>(bn, maps, args, grid, stream);
        case MODE_GEMM1T: return launch_bn<MODE_GEMM1T>(bn, maps, args, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace beam
