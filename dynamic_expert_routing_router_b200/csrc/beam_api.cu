// beam_api.cu -- the C entry points of libbeam_moe.so: argument checks,
// workspace layout, tensor-map encoding and the launch sequence of the BEAM
// MoE layer (router GEMM -> top-K + mask -> grouping -> gather -> gate/up GEMM
// + SwiGLU -> down GEMM -> combine).  Everything is stream-ordered; nothing
// here synchronises the host except beam_moe_check, and nothing allocates.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "beam_internal.h"
#include "beam_moe.h"

using namespace beam;

namespace {

constexpr unsigned long long kWaitTimeoutNs = 1000000000ull;  // 1 s per bounded wait
constexpr int kRouterSplitsMax = kMaxRouterSplits < 8 ? kMaxRouterSplits : 8;
constexpr int kMaxDevices = 64;

// Test hooks (beam_moe_set_fault_injection): off unless a test sets them.
std::atomic<int> g_fault{FAULT_NONE};
std::atomic<unsigned long long> g_wait_limit_ns{0};

unsigned long long wait_limit_ns() {
    const unsigned long long v = g_wait_limit_ns.load(std::memory_order_relaxed);
    return v ? v : kWaitTimeoutNs;
}
int fault_mode() { return g_fault.load(std::memory_order_relaxed); }

// Largest batch that beam_moe_forward runs as one launch
// (beam_moe_set_one_launch_tokens); the kernel itself takes up to kDlMaxT.
constexpr int kOneLaunchDefaultTokens = 4;
std::atomic<int> g_one_launch_tokens{kOneLaunchDefaultTokens};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

beam_status validate_desc(const beam_moe_desc *d) {
    if (!d) return BEAM_ERR_INVALID_ARG;
    if (d->T < 0 || d->d <= 0 || d->E <= 0 || d->I <= 0 || d->K <= 0) return BEAM_ERR_INVALID_ARG;
    if (d->K > d->E || d->K > kMaxK || d->E > kMaxE) return BEAM_ERR_INVALID_ARG;
    if (d->dtype != BEAM_BF16 && d->dtype != BEAM_F32) return BEAM_ERR_INVALID_ARG;
    if (d->renorm_topk != 0 && d->renorm_topk != 1) return BEAM_ERR_INVALID_ARG;
    if (d->mask_logit_threshold != d->mask_logit_threshold) return BEAM_ERR_INVALID_ARG;  // NaN
    if (d->dtype == BEAM_BF16) {
        if (d->d % kBlockM != 0 || d->I % kBlockM != 0) return BEAM_ERR_UNSUPPORTED_SHAPE;
    } else {
        if (d->d % 8 != 0 || d->I % 8 != 0) return BEAM_ERR_UNSUPPORTED_SHAPE;
    }
    if ((long long)d->T * d->K > INT_MAX / 2) return BEAM_ERR_UNSUPPORTED_SHAPE;
    if (d->n_shared < 0 || d->n_shared > kMaxShared) return BEAM_ERR_INVALID_ARG;
    if (d->n_shared > 0) {
        if (d->I_shared <= 0) return BEAM_ERR_INVALID_ARG;
        if (d->dtype != BEAM_BF16 || d->I_shared % kBlockM != 0) return BEAM_ERR_UNSUPPORTED_SHAPE;
        if ((long long)d->n_shared * d->T > INT_MAX / 2) return BEAM_ERR_UNSUPPORTED_SHAPE;
    }
    return BEAM_OK;
}

// Shared experts (every token, every shared expert): one token tile up to
// 128 tokens (the MMA's N follows its valid rows), so their weights are read
// once per 128 tokens, and the reductions split until about half the SMs
// have a unit (the split partials are summed in split order).  Measured
// (DeepSeekV2-Lite and Qwen1.5-MoE shapes, T = 1 and 128): half the SMs
// beat a unit per SM (whose fp32 partials cost as much as the weights),
// a quarter, and no split (T = 128, every candidate masked: 45.9 / 51.2
// against 51.2 / 59.3, 46.9 / 63.4 and 61.0 / 63.4 us).
void shared_plan(const beam_moe_desc *d, beam_moe_plan_info *P) {
    const long long T = d->T, S = d->n_shared;
    P->sh_bn = T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : 128;
    const long long ntt = T > 0 ? cdiv(T, P->sh_bn) : 1;
    const long long u1 = S * ntt * (d->I_shared / kBlockM), u2 = S * ntt * (d->d / kBlockM);
    auto split = [](long long units, long long nk) {
        long long k = cdiv(kNominalSMs / 2, units);
        if (k > 8) k = 8;
        if (k > nk) k = nk;
        return int(k < 1 ? 1 : k);
    };
    P->sh_split1 = S > 0 ? split(u1, d->d / kBlockK) : 1;
    P->sh_split2 = S > 0 ? split(u2, d->I_shared / kBlockK) : 1;
}

// Token-tile height of the expert GEMMs from the mean kept-or-not pairs per
// expert (T*K/E): decode batches use thin tiles, prefill batches 128 rows, and
// large bf16 prefill batches 256 (the gate/up GEMM then moves 64 KB of
// operands per 8.4 MFLOP stage instead of 48 KB per 4.2 MFLOP; the MMA's N
// follows each tile's valid rows, so the wider padding costs no tensor work).
int choose_bn(const beam_moe_desc *d, bool wide) {
    const long long avg = cdiv((long long)d->T * d->K, d->E);
    if (avg <= 16) return 16;
    if (avg <= 32) return 32;
    if (avg <= 64) return 64;
    if (wide && avg >= 256) return 256;
    return 128;
}

// Small bf16 batches: the router logits come from the one-launch kernel's
// router units (CUDA cores, one split) in every call -- forward, routing
// only, backward -- so that all of them take the same decisions on the same
// inputs.  `dl` receives the unit sizes for the call's mask and SM count.
bool small_batch(const beam_moe_desc *d, int has_mask, int n_sm, DecodeLayerArgs *dl) {
    return d->dtype == BEAM_BF16 &&
           decode_layer_config(d->T, d->d, d->E, d->I, d->K, has_mask, n_sm, dl);
}

// `backward`: the training call's plan (its per-expert 128-row tile lists
// need token tiles of at most 128 rows).
beam_status make_plan(const beam_moe_desc *d, beam_moe_plan_info *P, bool backward = false) {
    beam_status st = validate_desc(d);
    if (st != BEAM_OK) return st;
    std::memset(P, 0, sizeof(*P));
    const long long T = d->T, K = d->K, E = d->E;
    P->BN = choose_bn(d, d->dtype == BEAM_BF16 && !backward);
    DecodeLayerArgs dl;
    const bool small = small_batch(d, 1, kNominalSMs, &dl);
    P->one_launch = small && d->n_shared == 0 && !backward &&
                    d->T <= g_one_launch_tokens.load(std::memory_order_relaxed);
    if (small) {
        P->router_bn = 16;  // unused: the router runs on CUDA cores
        P->router_splits = 1;
    } else if (d->dtype == BEAM_BF16) {
        // Router: enough (token tile x row block x split) units to cover the
        // SMs at decode sizes, while the split partials stay smaller than the
        // router weights, and at most kRouterSplitsMax splits (T = 32 with 16
        // splits took 60.1 us per layer, with 8 57.9 us; T = 128 keeps 8);
        // prefill needs no split.
        P->router_bn = T >= 1024 ? 128 : T >= 256 ? 64 : T > 16 ? 32 : 16;
        const long long n_tt = T > 0 ? cdiv(T, P->router_bn) : 1;
        const long long base = n_tt * 2 * cdiv(E, kBlockM);
        const long long nkb = d->d / kBlockK;
        const long long cap_bytes = T > 0 ? d->d / (2 * T) : nkb;
        int S = 1;
        while (2LL * S <= kRouterSplitsMax && 2LL * S <= nkb && nkb % (2LL * S) == 0 &&
               base * 2 * S <= kNominalSMs &&
               2LL * S <= (cap_bytes > 1 ? cap_bytes : 1))
            S *= 2;
        P->router_splits = S;
    } else {
        P->router_bn = 16;
        P->router_splits = 1;
    }
    const long long p_cap = T * K + E * (P->BN - 1);
    const long long tiles_cap = cdiv(T * K, P->BN) + E;
    if (p_cap > INT_MAX / 2 || tiles_cap > INT_MAX / 2) return BEAM_ERR_UNSUPPORTED_SHAPE;
    P->p_cap = int(p_cap);
    P->tiles_cap = int(tiles_cap);
    const size_t es = d->dtype == BEAM_BF16 ? 2 : 4;
    size_t o = 0;
    P->off_err = 0;
    P->off_meta = 16;
    P->off_counts = 256;
    P->off_hist = align256(P->off_counts + 4 * size_t(E));
    P->off_partial = align256(P->off_hist + 4 * size_t(K + 1));
    P->off_idx = align256(P->off_partial + 4 * size_t(P->router_splits) * size_t(T) * 2 * size_t(E));
    P->off_w = align256(P->off_idx + 4 * size_t(T * K));
    P->off_pair = align256(P->off_w + 4 * size_t(T * K));
    P->off_pair_pos = align256(P->off_pair + 4 * size_t(p_cap));
    P->off_tiles = align256(P->off_pair_pos + 4 * size_t(T * K));
    P->off_xp = align256(P->off_tiles + 16 * size_t(tiles_cap));
    P->off_h = align256(P->off_xp + es * size_t(p_cap) * size_t(d->d));
    P->off_y = align256(P->off_h + es * size_t(p_cap) * size_t(d->I));
    P->off_tile_done = align256(P->off_y + 4 * size_t(p_cap) * size_t(d->d));  // Y is fp32
    const size_t srows = size_t(d->n_shared) * size_t(T);  // shared rows: every token
    shared_plan(d, P);
    P->off_hs = align256(P->off_tile_done + 4 * size_t(tiles_cap));
    P->off_ys = align256(P->off_hs + es * srows * size_t(d->n_shared > 0 ? d->I_shared : 0));
    // 256-row token tiles: the gate/up GEMM runs over 128-row sub-tiles of
    // them (two 128-row weight tiles and two accumulator buffers per unit).
    P->sub_bn = P->BN > kBlockM ? kBlockM : P->BN;
    P->off_tiles_sub = align256(P->off_ys + 4 * size_t(P->sh_split2) * srows * size_t(d->d));
    const size_t sub_cap = P->BN > kBlockM ? size_t(cdiv(T * K, kBlockM) + E) : 0;
    // one-launch counters: per expert, then per (token, down row block)
    P->off_ctl = align256(P->off_tiles_sub + 16 * sub_cap);
    const size_t ctl = small ? size_t(E) * size_t(d->I / 128) + size_t(T) * size_t(d->d / dl.R2)
                             : 0;
    P->off_sp = align256(P->off_ctl + 4 * ctl);
    const size_t sp = P->sh_split1 > 1 ? 2 * size_t(P->sh_split1) * srows * size_t(d->I_shared) : 0;
    o = align256(P->off_sp + 4 * sp);
    P->workspace_bytes = o;
    return BEAM_OK;
}

// Decode-sized token tiles run both expert GEMMs as one fused launch.
bool fused_experts(const beam_moe_plan_info &P) { return P.BN < 128; }

int sm_count() {
    static int cache[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return kNominalSMs;
    if (dev < 0 || dev >= kMaxDevices) return kNominalSMs;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = kNominalSMs;
        cache[dev] = n;
    }
    return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2D bf16 tensor map over a row-major [rows, inner] matrix, box = 64 x box_rows,
// 128-byte swizzle (matches the UMMA descriptors in tc_gemm.cu), zero fill.
// A tensor map holds only the address, shape, strides and box it was made
// from, so an encoded map is cached under exactly those values: repeated
// calls with the same buffers skip the driver call (host time per forward).
struct TmapKey {
    const void *base;
    unsigned long long inner, rows;
    unsigned box_rows, chunks;
    bool operator==(const TmapKey &o) const {
        return base == o.base && inner == o.inner && rows == o.rows && box_rows == o.box_rows &&
               chunks == o.chunks;
    }
};
struct TmapCache {
    static constexpr int kSets = 64, kWays = 4;
    struct Entry {
        TmapKey key;
        CUtensorMap map;
        bool valid;
    };
    std::mutex mu;
    Entry e[kSets][kWays] = {};
    int next[kSets] = {};
    static int set_of(const TmapKey &k) {
        unsigned long long h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
        h ^= k.inner * 0xC2B2AE3D27D4EB4Full ^ k.rows * 0x165667B19E3779F9ull ^ k.box_rows;
        return int((h >> 29) % kSets);
    }
};
TmapCache &tmap_cache() {
    static TmapCache c;
    return c;
}

// chunks > 0: a 3D view [inner / 64][rows][64] of the same matrix whose box
// is `chunks` consecutive 64-column chunks of box_rows rows: one copy lands
// them as `chunks` swizzled 64-column boxes, one after another.
bool make_tmap(CUtensorMap *m, const void *base, unsigned long long inner,
               unsigned long long rows, unsigned box_rows, unsigned chunks = 0) {
    const TmapKey key{base, inner, rows, box_rows, chunks};
    TmapCache &c = tmap_cache();
    const int set = TmapCache::set_of(key);
    {
        std::lock_guard<std::mutex> lk(c.mu);
        for (auto &en : c.e[set])
            if (en.valid && en.key == key) {
                *m = en.map;
                return true;
            }
    }
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn || rows == 0) return false;
    CUresult r;
    if (chunks == 0) {
        cuuint64_t dims[2] = {inner, rows};
        cuuint64_t strides[1] = {inner * 2};
        cuuint32_t box[2] = {unsigned(kBlockK), box_rows};
        cuuint32_t estr[2] = {1, 1};
        r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        if (inner % kBlockK != 0) return false;
        cuuint64_t dims[3] = {unsigned(kBlockK), rows, inner / kBlockK};
        cuuint64_t strides[2] = {inner * 2, kBlockK * 2};
        cuuint32_t box[3] = {unsigned(kBlockK), box_rows, chunks};
        cuuint32_t estr[3] = {1, 1, 1};
        r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> lk(c.mu);
    auto &slot = c.e[set][c.next[set]];
    c.next[set] = (c.next[set] + 1) % TmapCache::kWays;
    slot.key = key;
    slot.map = *m;
    slot.valid = true;
    return true;
}

// A second stream per device for the shared experts, with the events that
// fork it from the caller's stream and join it back.  Created on first use
// outside a stream capture; held under a lock from the fork to the end of
// the call's enqueue, so concurrent callers never interleave their events.
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
SideStream g_side[kMaxDevices];

// The current device's second stream, locked into *lock; null (the shared
// experts then run on the caller's stream) when it does not exist yet and
// `st` is being captured, or cannot be created.
SideStream *side_stream(cudaStream_t st, std::unique_lock<std::mutex> *lock) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::unique_lock<std::mutex> lk(g_side_mu);
    SideStream &ss = g_side[dev];
    if (!ss.s) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
            return nullptr;
        cudaStream_t s = nullptr;
        cudaEvent_t f = nullptr, j = nullptr;
        if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
            if (j) cudaEventDestroy(j);
            if (f) cudaEventDestroy(f);
            if (s) cudaStreamDestroy(s);
            cudaGetLastError();
            return nullptr;
        }
        ss.s = s;
        ss.fork = f;
        ss.join = j;
    }
    *lock = std::move(lk);
    return &ss;
}

// Records the caller's timing events between stages.  External records
// become event nodes when the call is captured into a CUDA graph, so the
// per-kernel times can also be read from graph replays.
struct Recorder {
    void *const *events;
    cudaStream_t st;
    cudaError_t rec(int i) const {
        if (!events || !events[i]) return cudaSuccess;
        return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), st,
                                        cudaEventRecordExternal);
    }
};

#define BEAM_TRY_CUDA(expr)                          \
    do {                                             \
        cudaError_t e_ = (expr);                     \
        if (e_ != cudaSuccess) return BEAM_ERR_CUDA; \
    } while (0)

struct RouteOut {
    int *idx;
    float *w;
    int *counts;
    int *hist;
    float *logits;
    int *cand = nullptr;        // training: every candidate
    float *gk = nullptr;        // training: softmax weight before the mask
    int *counts_all = nullptr;  // training: candidates per expert (caller zeroes)
};

// Stages 0-1: router GEMM into the split partials, then top-K + mask.
beam_status launch_route(const beam_moe_desc *d, const beam_moe_plan_info &P, const void *x,
                         const void *Wg, const void *Wm, const RouteOut &ro, char *ws,
                         cudaStream_t st, const Recorder &rec, int n_sm) {
    float *partial = reinterpret_cast<float *>(ws + P.off_partial);
    // The router clears meta, counts and the histogram for the later kernels,
    // never the error words (see kRouterTimeoutTag).
    int *hdr = reinterpret_cast<int *>(ws);
    ZeroRegion zero[3] = {{hdr + kHdrMeta, 4}, {ro.counts, d->E}, {ro.hist, ro.hist ? d->K + 1 : 0}};
    BEAM_TRY_CUDA(rec.rec(0));
    DecodeLayerArgs dl;
    if (small_batch(d, Wm != nullptr, n_sm, &dl)) {
        dl.mode = DL_ROUTER_ONLY;
        dl.x = x;
        dl.Wg = Wg;
        dl.Wm = Wm;
        dl.partial = partial;
        dl.hdr = hdr;
        dl.zero[0] = zero[0];
        dl.zero[1] = zero[1];
        dl.zero[2] = zero[2];
        dl.fault_skip = fault_mode() == FAULT_ROUTER_STAGE ? FAULT_ROUTER_STAGE : FAULT_NONE;
        dl.timeout_ns = wait_limit_ns();
        DlMaps none;
        std::memset(&none, 0, sizeof(none));  // the router items read no tensor map
        BEAM_TRY_CUDA(launch_decode_layer(none, dl, dl.n_ru < n_sm ? dl.n_ru : n_sm, st));
    } else if (d->dtype == BEAM_BF16) {
        TcMaps maps;
        if (!make_tmap(&maps.a0, Wg, d->d, d->E, kBlockM)) return BEAM_ERR_CUDA;
        if (!make_tmap(&maps.a1, Wm ? Wm : Wg, d->d, d->E, kBlockM)) return BEAM_ERR_CUDA;
        if (!make_tmap(&maps.b, x, d->d, d->T, P.router_bn)) return BEAM_ERR_CUDA;
        maps.a2 = maps.a0;
        maps.b2 = maps.b;
        TcGemmArgs a;
        std::memset(&a, 0, sizeof(a));
        const int mb_per = int(cdiv(d->E, kBlockM));
        a.n_mb_gate = mb_per;
        a.n_mb = Wm ? 2 * mb_per : mb_per;
        a.n_tt = int(cdiv(d->T, P.router_bn));
        a.nk = d->d / kBlockK / P.router_splits;
        a.n_units = a.n_mb * a.n_tt * P.router_splits;
        a.T = d->T;
        a.E = d->E;
        a.out = partial;
        a.out_ld = 2LL * d->E;
        a.out_split_stride = (long long)d->T * 2 * d->E;
        a.err = hdr + kHdrErrRouter;
        a.err_code = kRouterTimeoutTag;
        a.fault_skip = fault_mode() == FAULT_ROUTER_STAGE;
        a.zero[0] = zero[0];
        a.zero[1] = zero[1];
        a.zero[2] = zero[2];
        a.timeout_ns = wait_limit_ns();
        const int grid = a.n_units < n_sm ? a.n_units : n_sm;
        BEAM_TRY_CUDA(launch_tc_gemm(MODE_ROUTER, P.router_bn, maps, a, grid, st));
    } else {
        BEAM_TRY_CUDA(launch_router_f32(static_cast<const float *>(x), static_cast<const float *>(Wg),
                                        static_cast<const float *>(Wm), d->T, d->d, d->E, partial,
                                        zero, st));
    }
    BEAM_TRY_CUDA(rec.rec(1));
    TopkArgs t;
    t.partial = partial;
    t.S = P.router_splits;
    t.T = d->T;
    t.E = d->E;
    t.K = d->K;
    t.renorm = d->renorm_topk;
    t.has_mask = Wm != nullptr;
    t.thr = d->mask_logit_threshold;
    t.hdr = hdr;
    t.logits = ro.logits;
    t.idx = ro.idx;
    t.w = ro.w;
    t.counts = ro.counts;
    t.hist = ro.hist;
    t.cand = ro.cand;
    t.gk = ro.gk;
    t.counts_all = ro.counts_all;
    BEAM_TRY_CUDA(launch_topk_mask(t, n_sm, st));
    return BEAM_OK;
}

beam_status check_ws(const beam_moe_plan_info &P, const void *ws, size_t bytes) {
    if (!ws || !aligned16(ws) || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return BEAM_ERR_WORKSPACE;
    if (bytes < P.workspace_bytes) return BEAM_ERR_WORKSPACE;
    return BEAM_OK;
}

// Shared experts over every token (dense units; no grouping), Ys = the
// shared experts' outputs: on `st`, which may be a second stream beside the
// routed experts' (nothing here reads the routing).  Timeouts go to the
// header's shared-expert word (kSharedTimeoutTag), folded in by the combine.
beam_status launch_shared_experts(const beam_moe_desc *d, const beam_moe_plan_info &P,
                                  const void *x, const void *W1s, const void *W3s,
                                  const void *W2s, char *ws, cudaStream_t st, int n_sm) {
    float *ys = reinterpret_cast<float *>(ws + P.off_ys);
    {
        // Shared experts over every token (dense units; no grouping): the
        // gate/up GEMM (its reduction split sh_split1 ways: partials, then a
        // SwiGLU kernel), then the down GEMM (split sh_split2 ways: one slab
        // of Ys per split, added by the combine).
        const int bn = P.sh_bn;
        const int ntt = int(cdiv(d->T, bn));
        void *hs = ws + P.off_hs;
        const unsigned long long srows = (unsigned long long)d->n_shared * d->T;
        TcMaps m1, m2;
        if (!make_tmap(&m1.a0, W1s, d->d, (unsigned long long)d->n_shared * d->I_shared, kBlockM))
            return BEAM_ERR_CUDA;
        if (!make_tmap(&m1.a1, W3s, d->d, (unsigned long long)d->n_shared * d->I_shared, kBlockM))
            return BEAM_ERR_CUDA;
        if (!make_tmap(&m1.b, x, d->d, d->T, bn)) return BEAM_ERR_CUDA;
        m1.a2 = m1.a0;
        m1.b2 = m1.b;
        if (!make_tmap(&m2.a0, W2s, d->I_shared, (unsigned long long)d->n_shared * d->d, kBlockM))
            return BEAM_ERR_CUDA;
        if (!make_tmap(&m2.b, hs, d->I_shared, srows, bn)) return BEAM_ERR_CUDA;
        m2.a1 = m2.a0;
        m2.a2 = m2.a0;
        m2.b2 = m2.b;
        TcGemmArgs g;
        std::memset(&g, 0, sizeof(g));
        g.err = reinterpret_cast<int *>(ws) + kHdrErrShared;
        g.err_code = kSharedTimeoutTag;
        g.fault_skip = fault_mode() == FAULT_SHARED_STAGE;  // tests only
        g.timeout_ns = wait_limit_ns();
        g.dense = 1;
        g.dense_ntt = ntt;
        g.dense_T = d->T;
        g.dense_slab_rows = int(srows);
        g.n_mb = d->I_shared / kBlockM;
        g.nk = d->d / kBlockK;
        g.a_rows_per_expert = d->I_shared;
        g.dense_ksplit = P.sh_split1;
        g.n_units = d->n_shared * ntt * g.n_mb * P.sh_split1;
        g.out_ld = d->I_shared;
        float *sp = reinterpret_cast<float *>(ws + P.off_sp);
        const size_t slab1 = size_t(P.sh_split1) * srows * size_t(d->I_shared);
        if (P.sh_split1 > 1) {  // fp32 partial pre-activations only
            g.out = nullptr;
            g.a_out = sp;
            g.b_out = sp + slab1;
        } else {
            g.out = hs;
        }
        BEAM_TRY_CUDA(launch_tc_gemm(MODE_GEMM1, bn, m1, g, g.n_units < n_sm ? g.n_units : n_sm, st));
        if (P.sh_split1 > 1)
            BEAM_TRY_CUDA(launch_shared_swiglu(sp, sp + slab1, P.sh_split1,
                                               (long long)srows * d->I_shared, hs, st));
        g.a_out = g.b_out = nullptr;
        g.fault_skip = 0;
        g.dense_gemm2 = 1;
        g.n_mb = d->d / kBlockM;
        g.nk = d->I_shared / kBlockK;
        g.a_rows_per_expert = d->d;
        g.dense_ksplit = P.sh_split2;
        g.n_units = d->n_shared * ntt * g.n_mb * P.sh_split2;
        g.out = ys;
        g.out_ld = d->d;
        BEAM_TRY_CUDA(launch_tc_gemm(MODE_GEMM2, bn, m2, g, g.n_units < n_sm ? g.n_units : n_sm, st));
    }

    return BEAM_OK;
}

// Stages 2-6 of a call whose routing (idx, w, counts, hist, a clean header)
// is already in the workspace: grouping, row copy, expert GEMMs, shared
// experts, combine.  out_dtype is the combine's output type.
beam_status launch_tail(const beam_moe_desc *d, const beam_moe_plan_info &P, const void *x,
                        const void *W1, const void *W3, const void *W2, const void *W1s,
                        const void *W3s, const void *W2s, void *out, int out_dtype, char *ws,
                        cudaStream_t st, const Recorder &rec, int n_sm,
                        cudaEvent_t join = nullptr) {
    int *err = reinterpret_cast<int *>(ws + P.off_err);
    int *meta = reinterpret_cast<int *>(ws + P.off_meta);
    int *counts = reinterpret_cast<int *>(ws + P.off_counts);
    int *idx = reinterpret_cast<int *>(ws + P.off_idx);
    float *w = reinterpret_cast<float *>(ws + P.off_w);
    int *pair = reinterpret_cast<int *>(ws + P.off_pair);
    int *pair_pos = reinterpret_cast<int *>(ws + P.off_pair_pos);
    int4 *tiles = reinterpret_cast<int4 *>(ws + P.off_tiles);
    int *tile_done = reinterpret_cast<int *>(ws + P.off_tile_done);
    void *xp = ws + P.off_xp;
    void *h = ws + P.off_h;
    float *y = reinterpret_cast<float *>(ws + P.off_y);

    // Thin token tiles (decode, bf16): the grouping kernel also copies the
    // token rows (no gather launch), gate and up rows are interleaved in one
    // 128-row tile, and both expert GEMMs run in one fused launch.  128-token
    // tiles (prefill): rows gathered by their own kernel, two 128-row weight
    // tiles per unit, two GEMM launches.
    const bool fused = d->dtype == BEAM_BF16 && fused_experts(P);
    const size_t es = d->dtype == BEAM_BF16 ? 2 : 4;
    const int row_vec = int(es * size_t(d->d) / 16);
    BEAM_TRY_CUDA(rec.rec(2));
    PermuteArgs pa{idx,      counts,    d->T,
                   d->K,     d->E,      P.BN,
                   pair,     pair_pos,  tiles,
                   tile_done,
                   fused ? static_cast<const uint4 *>(x) : nullptr,
                   fused ? static_cast<uint4 *>(xp) : nullptr,
                   row_vec,  fused ? kPermCopyBlocks : 1,
                   meta,     err};
    int4 *tiles_sub = reinterpret_cast<int4 *>(ws + P.off_tiles_sub);
    if (P.sub_bn < P.BN) {  // 128-row sub-tiles for the gate/up GEMM; count in meta[3]
        pa.tiles_sub = tiles_sub;
        pa.sub_bn = P.sub_bn;
    }
    if (!fused && group_chunked_fits(d->T))  // large batches: chunked grouping (Y as scratch)
        BEAM_TRY_CUDA(launch_group_chunked(pa, reinterpret_cast<int *>(y), st));
    else
        BEAM_TRY_CUDA(launch_permute(pa, st));

    BEAM_TRY_CUDA(rec.rec(3));
    if (!fused)
        BEAM_TRY_CUDA(
            launch_gather(x, pair, meta, d->K, (long long)es * d->d, P.p_cap, xp, n_sm, st));

    if (d->dtype == BEAM_BF16) {
        const unsigned wbox = fused ? kBlockM / 2 : kBlockM;
        TcMaps maps;
        if (!make_tmap(&maps.a0, W1, d->d, (unsigned long long)d->E * d->I, wbox)) return BEAM_ERR_CUDA;
        if (!make_tmap(&maps.a1, W3, d->d, (unsigned long long)d->E * d->I, wbox)) return BEAM_ERR_CUDA;
        if (!make_tmap(&maps.b, xp, d->d, P.p_cap, P.sub_bn)) return BEAM_ERR_CUDA;
        if (!make_tmap(&maps.a2, W2, d->I, (unsigned long long)d->E * d->d, kBlockM)) return BEAM_ERR_CUDA;
        if (!make_tmap(&maps.b2, h, d->I, P.p_cap, P.BN)) return BEAM_ERR_CUDA;

        TcGemmArgs g;
        std::memset(&g, 0, sizeof(g));
        g.meta = meta;
        g.tiles = tiles;
        g.err = err;
        g.timeout_ns = wait_limit_ns();
        g.n_mb = d->I / int(wbox);
        g.nk = d->d / kBlockK;
        g.a_rows_per_expert = d->I;
        g.out = h;
        g.out_ld = d->I;

        BEAM_TRY_CUDA(rec.rec(4));
        g.fault_skip = fault_mode() == FAULT_EXPERT_STAGE;  // tests only
        if (fused) {
            g.n_mb2 = d->d / kBlockM;
            g.nk2 = d->I / kBlockK;
            g.a_rows2 = d->d;
            g.out2 = y;
            g.out2_ld = d->d;
            g.tile_done = tile_done;
            g.work_ctr = meta + 3;
            const long long units = (long long)P.tiles_cap * (g.n_mb + g.n_mb2);
            BEAM_TRY_CUDA(launch_tc_gemm(MODE_EXPERTS, P.BN, maps, g,
                                         int(units < n_sm ? units : n_sm), st));
            BEAM_TRY_CUDA(rec.rec(5));  // the down GEMM ran inside the fused launch
        } else {
            // gate/up over the 128-row sub-tiles when the tiles are 256 rows
            const bool sub = P.sub_bn < P.BN;
            long long units = (long long)(sub ? cdiv((long long)d->T * d->K, P.sub_bn) + d->E
                                              : P.tiles_cap) * g.n_mb;
            if (sub) {
                g.meta = meta + 3;
                g.tiles = tiles_sub;
            }
            BEAM_TRY_CUDA(launch_tc_gemm(MODE_GEMM1, P.sub_bn, maps, g,
                                         int(units < n_sm ? units : n_sm), st));
            BEAM_TRY_CUDA(rec.rec(5));
            g.fault_skip = 0;
            g.meta = meta;
            g.tiles = tiles;
            TcMaps m2 = maps;
            m2.a0 = maps.a2;
            m2.a1 = maps.a2;
            m2.b = maps.b2;
            g.n_mb = d->d / kBlockM;
            g.nk = d->I / kBlockK;
            g.a_rows_per_expert = d->d;
            g.out = y;
            g.out_ld = d->d;
            units = (long long)P.tiles_cap * g.n_mb;
            BEAM_TRY_CUDA(launch_tc_gemm(MODE_GEMM2, P.BN, m2, g,
                                         int(units < n_sm ? units : n_sm), st));
        }
    } else {
        BEAM_TRY_CUDA(rec.rec(4));
        BEAM_TRY_CUDA(launch_gemm1_f32(static_cast<const float *>(xp), static_cast<const float *>(W1),
                                       static_cast<const float *>(W3), tiles, meta, P.tiles_cap,
                                       d->d, d->I, static_cast<float *>(h), st));
        BEAM_TRY_CUDA(rec.rec(5));
        BEAM_TRY_CUDA(launch_gemm2_f32(static_cast<const float *>(h), static_cast<const float *>(W2),
                                       tiles, meta, P.tiles_cap, d->d, d->I, y, st));
    }

    float *ys = reinterpret_cast<float *>(ws + P.off_ys);
    if (d->n_shared > 0 && join == nullptr) {
        const beam_status ss = launch_shared_experts(d, P, x, W1s, W3s, W2s, ws, st, n_sm);
        if (ss != BEAM_OK) return ss;
    }
    // The shared experts ran on a second stream: wait for them.
    if (join) BEAM_TRY_CUDA(cudaStreamWaitEvent(st, join, 0));

    BEAM_TRY_CUDA(rec.rec(6));
    BEAM_TRY_CUDA(launch_combine(out_dtype, y, idx, w, pair_pos, d->T, d->K, d->d, ys,
                                 d->n_shared * P.sh_split2, out,
                                 d->n_shared > 0 ? reinterpret_cast<int *>(ws) : nullptr, n_sm,
                                 st));
    BEAM_TRY_CUDA(rec.rec(7));
    return BEAM_OK;
}

beam_status forward_impl(const beam_moe_desc *d, const void *x, const void *Wg, const void *Wm,
                         const void *W1, const void *W3, const void *W2, const void *W1s,
                         const void *W3s, const void *W2s, void *out, void *workspace,
                         size_t ws_bytes, void *stream, void *const *events) {
    beam_moe_plan_info P;
    beam_status s = make_plan(d, &P);
    if (s != BEAM_OK) return s;
    if (!x || !Wg || !W1 || !W3 || !W2 || !out) return BEAM_ERR_INVALID_ARG;
    for (const void *p : {x, Wg, W1, W3, W2, static_cast<const void *>(out)})
        if (!aligned16(p)) return BEAM_ERR_INVALID_ARG;
    if (d->n_shared > 0) {
        if (!W1s || !W3s || !W2s) return BEAM_ERR_INVALID_ARG;
        for (const void *p : {W1s, W3s, W2s})
            if (!aligned16(p)) return BEAM_ERR_INVALID_ARG;
    }
    if (Wm && !aligned16(Wm)) return BEAM_ERR_INVALID_ARG;
    s = check_ws(P, workspace, ws_bytes);
    if (s != BEAM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Recorder rec{events, st};
    if (d->T == 0) {  // nothing to compute; leave a clean error word and counters
        BEAM_TRY_CUDA(cudaMemsetAsync(workspace, 0, P.off_partial, st));
        for (int i = 0; i <= BEAM_MOE_FORWARD_STAGES; ++i) BEAM_TRY_CUDA(rec.rec(i));
        return BEAM_OK;
    }
    const int n_sm = sm_count();
    char *ws = static_cast<char *>(workspace);
    int *counts = reinterpret_cast<int *>(ws + P.off_counts);
    int *hist = reinterpret_cast<int *>(ws + P.off_hist);
    int *idx = reinterpret_cast<int *>(ws + P.off_idx);
    float *w = reinterpret_cast<float *>(ws + P.off_w);

    if (P.one_launch) {
        DecodeLayerArgs dl;
        if (!small_batch(d, Wm != nullptr, n_sm, &dl)) return BEAM_ERR_INTERNAL;
        dl.mode = DL_FORWARD;
        dl.renorm = d->renorm_topk;
        dl.thr = d->mask_logit_threshold;
        dl.x = x;
        dl.Wg = Wg;
        dl.Wm = Wm;
        dl.W1 = W1;
        dl.W3 = W3;
        dl.W2 = W2;
        dl.out = out;
        dl.partial = reinterpret_cast<float *>(ws + P.off_partial);
        dl.idx = idx;
        dl.w = w;
        dl.counts = counts;
        dl.hist = hist;
        dl.pair = reinterpret_cast<int *>(ws + P.off_pair);
        dl.pair_pos = reinterpret_cast<int *>(ws + P.off_pair_pos);
        dl.tiles = reinterpret_cast<int4 *>(ws + P.off_tiles);
        dl.BN = P.BN;
        dl.H = ws + P.off_h;
        dl.Y = reinterpret_cast<float *>(ws + P.off_y);
        dl.hdr = reinterpret_cast<int *>(ws);
        dl.e1_done = reinterpret_cast<int *>(ws + P.off_ctl);
        dl.comb_cnt = dl.e1_done + d->E * (d->I / 128);
        dl.fault_skip = fault_mode();
        dl.timeout_ns = wait_limit_ns();
        DlMaps maps;
        // boxes: 8 rows x 4 chunks (W1, W3), 16 rows x 2 chunks (W2, H)
        if (!make_tmap(&maps.w1, W1, d->d, (unsigned long long)d->E * d->I, 8, 4) ||
            !make_tmap(&maps.w3, W3, d->d, (unsigned long long)d->E * d->I, 8, 4) ||
            !make_tmap(&maps.w2, W2, d->I, (unsigned long long)d->E * d->d, 16, 2) ||
            !make_tmap(&maps.h, ws + P.off_h, d->I, P.p_cap, 16, 2))
            return BEAM_ERR_CUDA;
        BEAM_TRY_CUDA(rec.rec(0));
        // The kernel's counters start from zero: the header (error words,
        // meta, router count) is cleared here; CTA 0 clears the rest.
        BEAM_TRY_CUDA(cudaMemsetAsync(ws, 0, P.off_counts, st));
        BEAM_TRY_CUDA(launch_decode_layer(maps, dl, n_sm, st));
        for (int i = 1; i <= BEAM_MOE_FORWARD_STAGES; ++i) BEAM_TRY_CUDA(rec.rec(i));
        return BEAM_OK;
    }

    // Shared experts read no routing: unless the caller times the stages,
    // they run on a second stream from the start of the call, beside the
    // router, top-K, grouping and routed experts, and the combine waits for
    // both.  A captured call records the fork and the join as graph edges.
    SideStream *side = nullptr;
    std::unique_lock<std::mutex> side_lock;
    if (d->n_shared > 0 && events == nullptr) {
        side = side_stream(st, &side_lock);
        if (side && (cudaEventRecord(side->fork, st) != cudaSuccess ||
                     cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess))
            return BEAM_ERR_CUDA;
    }
    if (side) {
        s = launch_shared_experts(d, P, x, W1s, W3s, W2s, ws, side->s, n_sm);
        // The join is recorded whatever happened, so that the caller's
        // stream (or its capture) never leaves the second stream behind.
        if (cudaEventRecord(side->join, side->s) != cudaSuccess) return BEAM_ERR_CUDA;
        if (s != BEAM_OK) {
            cudaStreamWaitEvent(st, side->join, 0);
            return s;
        }
    }

    const RouteOut ro{idx, w, counts, hist, nullptr};
    s = launch_route(d, P, x, Wg, Wm, ro, ws, st, rec, n_sm);
    // launch_tail waits for the join before the combine; on an earlier exit
    // the caller's stream still joins the second stream here.
    if (s == BEAM_OK)
        s = launch_tail(d, P, x, W1, W3, W2, W1s, W3s, W2s, out, d->dtype, ws, st, rec, n_sm,
                        side ? side->join : nullptr);
    if (side && s != BEAM_OK) cudaStreamWaitEvent(st, side->join, 0);
    return s;
}


// ------------------------------------------------------------ backward --
// The backward workspace is the forward plan (its grouping now holds every
// candidate: T*K pairs fit p_cap) followed by the training-only arrays.
struct BwdPlan {
    int S;  // reduction splits of the kept-row products
    size_t off_cand, off_gk, off_counts_all, off_logits, off_dyp, off_A, off_B, off_da, off_db,
        off_h, off_part, off_u, off_dz, off_dr, off_xt_all, off_xt_kept, off_xmeta, off_dab, off_dbb,
        bytes;
};

beam_status make_bwd_plan(const beam_moe_desc *d, beam_moe_plan_info *P, BwdPlan *B) {
    beam_status s = make_plan(d, P, true);
    if (s != BEAM_OK) return s;
    if (d->n_shared != 0) return BEAM_ERR_UNSUPPORTED_SHAPE;  // shared experts: forward only
    const size_t T = size_t(d->T), K = size_t(d->K), E = size_t(d->E), I = size_t(d->I);
    const size_t dd = size_t(d->d), pc = size_t(P->p_cap);
    const size_t es = d->dtype == BEAM_BF16 ? 2 : 4;
    size_t o = P->workspace_bytes;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align256(o + bytes);
        return at;
    };
    B->off_cand = take(4 * T * K);
    B->off_gk = take(4 * T * K);
    B->off_counts_all = take(4 * E);
    B->off_logits = take(4 * T * 2 * E);
    B->off_dyp = take(es * pc * dd);
    B->off_A = take(4 * pc * I);
    B->off_B = take(4 * pc * I);
    B->off_da = take(4 * pc * I);
    B->off_db = take(4 * pc * I);
    B->off_h = take(4 * pc * I);
    // fp32 runs the kept-row products on CUDA cores, one block per tile: at
    // thin decode tiles split their reduction eight ways (d and I are
    // multiples of 8).  bf16 runs them on the tensor cores: one split.
    B->S = (d->dtype != BEAM_BF16 && P->BN < 128) ? 8 : 1;
    // fp32: the CUDA-core kept-row products hold a split's A rows in shared
    // memory (bf16 runs both products on the tensor cores).
    if (d->dtype != BEAM_BF16 && (dd / B->S > 7168 || I / B->S > 4096))
        return BEAM_ERR_UNSUPPORTED_SHAPE;
    B->off_part = take(4 * size_t(B->S) * pc * (dd > I ? dd : I));
    B->off_u = take(4 * T * K);
    B->off_dz = take(4 * T * K);
    B->off_dr = take(4 * T * E);
    // bf16: per-expert row tiles of the tensor-core GEMMs (at most one per
    // grouping tile): every candidate expert's, the kept experts', two counts
    B->off_xt_all = take(16 * size_t(P->tiles_cap));
    B->off_xt_kept = take(16 * size_t(P->tiles_cap));
    B->off_xmeta = take(8);
    // bf16: da, db rounded once more as the tensor-core dx product's operands
    B->off_dab = take(d->dtype == BEAM_BF16 ? 2 * pc * I : 0);
    B->off_dbb = take(d->dtype == BEAM_BF16 ? 2 * pc * I : 0);
    B->bytes = o;
    return BEAM_OK;
}

beam_status backward_impl(const beam_moe_desc *d, const void *x, const void *Wg, const void *Wm,
                          const void *W1, const void *W3, const void *W2, const void *dy,
                          float beta, float *dx, float *dWg, float *dWm, float *dW1, float *dW3,
                          float *dW2, void *workspace, size_t ws_bytes, void *stream) {
    beam_moe_plan_info P;
    BwdPlan B;
    beam_status s = make_bwd_plan(d, &P, &B);
    if (s != BEAM_OK) return s;
    if (!x || !Wg || !W1 || !W3 || !W2 || !dy || !dx || !dWg || !dW1 || !dW3 || !dW2)
        return BEAM_ERR_INVALID_ARG;
    if ((Wm == nullptr) != (dWm == nullptr) || !std::isfinite(beta)) return BEAM_ERR_INVALID_ARG;
    for (const void *p : {x, Wg, W1, W3, W2, dy, static_cast<const void *>(dx),
                          static_cast<const void *>(dWg), static_cast<const void *>(dW1),
                          static_cast<const void *>(dW3), static_cast<const void *>(dW2)})
        if (!aligned16(p)) return BEAM_ERR_INVALID_ARG;
    if ((Wm && !aligned16(Wm)) || (dWm && !aligned16(dWm))) return BEAM_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < B.bytes)
        return BEAM_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d->T == 0) {  // no token: no gradient; leave a clean error word
        BEAM_TRY_CUDA(cudaMemsetAsync(workspace, 0, P.off_partial, st));
        return BEAM_OK;
    }
    const int n_sm = sm_count();
    char *ws = static_cast<char *>(workspace);
    int *err = reinterpret_cast<int *>(ws + P.off_err);
    int *meta = reinterpret_cast<int *>(ws + P.off_meta);
    int *counts = reinterpret_cast<int *>(ws + P.off_counts);
    int *hist = reinterpret_cast<int *>(ws + P.off_hist);
    int *idx = reinterpret_cast<int *>(ws + P.off_idx);
    float *w = reinterpret_cast<float *>(ws + P.off_w);
    int *pair = reinterpret_cast<int *>(ws + P.off_pair);
    int *pair_pos = reinterpret_cast<int *>(ws + P.off_pair_pos);
    int4 *tiles = reinterpret_cast<int4 *>(ws + P.off_tiles);
    int *tile_done = reinterpret_cast<int *>(ws + P.off_tile_done);
    void *xp = ws + P.off_xp;
    void *h = ws + P.off_h;
    float *y = reinterpret_cast<float *>(ws + P.off_y);
    int *cand = reinterpret_cast<int *>(ws + B.off_cand);
    float *gk = reinterpret_cast<float *>(ws + B.off_gk);
    int *counts_all = reinterpret_cast<int *>(ws + B.off_counts_all);
    float *logits = reinterpret_cast<float *>(ws + B.off_logits);
    void *dyp = ws + B.off_dyp;
    float *A = reinterpret_cast<float *>(ws + B.off_A);
    float *Bv = reinterpret_cast<float *>(ws + B.off_B);

    // Routing, with every candidate and its pre-mask weight exported.
    BEAM_TRY_CUDA(cudaMemsetAsync(counts_all, 0, sizeof(int) * size_t(d->E), st));
    RouteOut ro{idx, w, counts, hist, logits};
    ro.cand = cand;
    ro.gk = gk;
    ro.counts_all = counts_all;
    s = launch_route(d, P, x, Wg, Wm, ro, ws, st, Recorder{nullptr, st}, n_sm);
    if (s != BEAM_OK) return s;

    // Every candidate grouped by expert (masked ones too: their expert
    // outputs enter the mask gradient), with x and dy rows in that order.
    const size_t es = d->dtype == BEAM_BF16 ? 2 : 4;
    PermuteArgs pa{cand,      counts_all, d->T,
                   d->K,      d->E,       P.BN,
                   pair,      pair_pos,   tiles,
                   tile_done, static_cast<const uint4 *>(x),
                   static_cast<uint4 *>(xp),
                   int(es * size_t(d->d) / 16), kPermCopyBlocks,
                   meta,      err};
    BEAM_TRY_CUDA(launch_permute(pa, st));
    BEAM_TRY_CUDA(launch_gather(dy, pair, meta, d->K, (long long)es * d->d, P.p_cap, dyp, n_sm, st));

    // Forward of every candidate: a, b (fp32), H, and Y = H W2^T.
    if (d->dtype == BEAM_BF16) {
        // Each expert's candidate rows as 128-row tiles, so that every GEMM
        // below reads an expert's weights once (not once per 16-row tile).
        int4 *xt_all = reinterpret_cast<int4 *>(ws + B.off_xt_all);
        int4 *xt_kept = reinterpret_cast<int4 *>(ws + B.off_xt_kept);
        int *xmeta = reinterpret_cast<int *>(ws + B.off_xmeta);
        BEAM_TRY_CUDA(launch_expert_tiles(tiles, meta, counts, counts_all, kBlockM, xt_all, xt_kept,
                                          xmeta, st));
        TcMaps maps;
        if (!make_tmap(&maps.a0, W1, d->d, (unsigned long long)d->E * d->I, kBlockM)) return BEAM_ERR_CUDA;
        if (!make_tmap(&maps.a1, W3, d->d, (unsigned long long)d->E * d->I, kBlockM)) return BEAM_ERR_CUDA;
        if (!make_tmap(&maps.b, xp, d->d, P.p_cap, kBlockM)) return BEAM_ERR_CUDA;
        maps.a2 = maps.a0;
        maps.b2 = maps.b;
        TcGemmArgs g;
        std::memset(&g, 0, sizeof(g));
        g.meta = xmeta;  // [0]: tiles of every candidate expert
        g.tiles = xt_all;
        g.err = err;
        g.timeout_ns = wait_limit_ns();
        g.n_mb = d->I / kBlockM;
        g.nk = d->d / kBlockK;
        g.a_rows_per_expert = d->I;
        g.out = h;
        g.out_ld = d->I;
        g.a_out = A;
        g.b_out = Bv;
        long long units = (long long)P.tiles_cap * g.n_mb;
        BEAM_TRY_CUDA(launch_tc_gemm(MODE_GEMM1, kBlockM, maps, g, int(units < n_sm ? units : n_sm), st));
        TcMaps m2;
        if (!make_tmap(&m2.a0, W2, d->I, (unsigned long long)d->E * d->d, kBlockM)) return BEAM_ERR_CUDA;
        if (!make_tmap(&m2.b, h, d->I, P.p_cap, kBlockM)) return BEAM_ERR_CUDA;
        m2.a1 = m2.a0;
        m2.a2 = m2.a0;
        m2.b2 = m2.b;
        g.a_out = g.b_out = nullptr;
        g.n_mb = d->d / kBlockM;
        g.nk = d->I / kBlockK;
        g.a_rows_per_expert = d->d;
        g.out = y;
        g.out_ld = d->d;
        units = (long long)P.tiles_cap * g.n_mb;
        BEAM_TRY_CUDA(launch_tc_gemm(MODE_GEMM2, kBlockM, m2, g, int(units < n_sm ? units : n_sm), st));
        // dh = dy W2_e for the kept experts on the tensor cores, into the
        // first split of the partials; dh_finalize then sums a single split.
        TcMaps m3;
        if (!make_tmap(&m3.a0, W2, d->I, (unsigned long long)d->E * d->d, kBlockK)) return BEAM_ERR_CUDA;
        if (!make_tmap(&m3.b, dyp, d->d, P.p_cap, kBlockM)) return BEAM_ERR_CUDA;
        m3.a1 = m3.a2 = m3.a0;
        m3.b2 = m3.b;
        g.meta = xmeta + 1;  // [1]: tiles of the kept experts
        g.tiles = xt_kept;
        g.n_mb = d->I / kBlockM;
        g.nk = d->d / kBlockK;
        g.a_rows_per_expert = d->d;
        g.out = ws + B.off_part;
        g.out_ld = d->I;
        units = (long long)P.tiles_cap * g.n_mb;
        BEAM_TRY_CUDA(launch_tc_gemm(MODE_GEMM2T, kBlockM, m3, g, int(units < n_sm ? units : n_sm), st));
    } else {
        BEAM_TRY_CUDA(launch_gemm1_f32(static_cast<const float *>(xp), static_cast<const float *>(W1),
                                       static_cast<const float *>(W3), tiles, meta, P.tiles_cap,
                                       d->d, d->I, static_cast<float *>(h), st, A, Bv));
        BEAM_TRY_CUDA(launch_gemm2_f32(static_cast<const float *>(h), static_cast<const float *>(W2),
                                       tiles, meta, P.tiles_cap, d->d, d->I, y, st));
    }

    BwArgs a;
    a.T = d->T;
    a.d = d->d;
    a.E = d->E;
    a.I = d->I;
    a.K = d->K;
    a.renorm = d->renorm_topk;
    a.has_mask = Wm != nullptr;
    a.tiles_cap = P.tiles_cap;
    a.p_cap = P.p_cap;
    a.S = B.S;
    a.beta = beta;
    a.Y = y;
    a.logits = logits;
    a.cand = cand;
    a.gk = gk;
    a.idx = idx;
    a.w = w;
    a.pair = pair;
    a.pair_pos = pair_pos;
    a.tiles = tiles;
    a.meta = meta;
    a.counts_kept = counts;
    a.counts_all = counts_all;
    a.A = A;
    a.B = Bv;
    a.da = reinterpret_cast<float *>(ws + B.off_da);
    a.db = reinterpret_cast<float *>(ws + B.off_db);
    a.h = reinterpret_cast<float *>(ws + B.off_h);
    a.part = reinterpret_cast<float *>(ws + B.off_part);
    a.dh_tc = d->dtype == BEAM_BF16 ? 1 : 0;
    a.dx_tc = a.dh_tc;
    a.da_bf = a.dx_tc ? ws + B.off_dab : nullptr;
    a.db_bf = a.dx_tc ? ws + B.off_dbb : nullptr;
    a.u = reinterpret_cast<float *>(ws + B.off_u);
    a.dz = reinterpret_cast<float *>(ws + B.off_dz);
    a.dr = reinterpret_cast<float *>(ws + B.off_dr);
    a.dx = dx;
    BEAM_TRY_CUDA(launch_backward_stages(a, d->dtype, x, xp, dy, dyp, Wg, Wm, W1, W3, W2, dWg,
                                         dWm, dW1, dW3, dW2, n_sm, st, 0));
    if (a.dx_tc) {
        // dxp = da W1_e + db W3_e on the tensor cores over the same expert
        // tiles: 2I k-rows per unit (W1_e with da, then W3_e with db).
        TcMaps m4;
        if (!make_tmap(&m4.a0, W1, d->d, (unsigned long long)d->E * d->I, kBlockK)) return BEAM_ERR_CUDA;
        if (!make_tmap(&m4.a1, W3, d->d, (unsigned long long)d->E * d->I, kBlockK)) return BEAM_ERR_CUDA;
        if (!make_tmap(&m4.b, a.da_bf, d->I, P.p_cap, kBlockM)) return BEAM_ERR_CUDA;
        if (!make_tmap(&m4.b2, a.db_bf, d->I, P.p_cap, kBlockM)) return BEAM_ERR_CUDA;
        m4.a2 = m4.a0;
        TcGemmArgs g;
        std::memset(&g, 0, sizeof(g));
        g.meta = reinterpret_cast<int *>(ws + B.off_xmeta) + 1;  // kept experts' tiles
        g.tiles = reinterpret_cast<int4 *>(ws + B.off_xt_kept);
        g.err = err;
        g.timeout_ns = wait_limit_ns();
        g.n_mb = d->d / kBlockM;
        g.nk = 2 * (d->I / kBlockK);
        g.a_rows_per_expert = d->I;
        g.out = a.part;
        g.out_ld = d->d;
        const long long units = (long long)P.tiles_cap * g.n_mb;
        BEAM_TRY_CUDA(launch_tc_gemm(MODE_GEMM1T, kBlockM, m4, g, int(units < n_sm ? units : n_sm), st));
    }
    BEAM_TRY_CUDA(launch_backward_stages(a, d->dtype, x, xp, dy, dyp, Wg, Wm, W1, W3, W2, dWg,
                                         dWm, dW1, dW3, dW2, n_sm, st, 1));
    return BEAM_OK;
}

}  // namespace

namespace beam {

size_t route_scratch_bytes(const beam_moe_desc *desc) {
    beam_moe_plan_info P;
    if (make_plan(desc, &P) != BEAM_OK) return 0;
    return P.off_idx;  // header + router partials: all the routing call uses
}

beam_status route_into_scratch(const beam_moe_desc *desc, const void *x, const void *W_gate,
                               const void *W_mask, int32_t *topk_idx, float *topk_w,
                               int32_t *expert_counts, int32_t *kept_hist, float *logits,
                               void *scratch, size_t scratch_bytes, cudaStream_t st) {
    beam_moe_plan_info P;
    beam_status s = make_plan(desc, &P);
    if (s != BEAM_OK) return s;
    if (!x || !W_gate || !topk_idx || !topk_w || !expert_counts) return BEAM_ERR_INVALID_ARG;
    for (const void *p : {x, W_gate, static_cast<const void *>(topk_idx),
                          static_cast<const void *>(topk_w), static_cast<const void *>(expert_counts)})
        if (!aligned16(p)) return BEAM_ERR_INVALID_ARG;
    if ((W_mask && !aligned16(W_mask)) || (kept_hist && !aligned16(kept_hist)) ||
        (logits && !aligned16(logits)))
        return BEAM_ERR_INVALID_ARG;
    if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & 255u) != 0 ||
        scratch_bytes < P.off_idx)
        return BEAM_ERR_WORKSPACE;
    if (desc->T == 0) {
        BEAM_TRY_CUDA(cudaMemsetAsync(scratch, 0, P.off_partial, st));
        BEAM_TRY_CUDA(cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * desc->E, st));
        if (kept_hist)
            BEAM_TRY_CUDA(cudaMemsetAsync(kept_hist, 0, sizeof(int32_t) * (desc->K + 1), st));
        return BEAM_OK;
    }
    const RouteOut ro{topk_idx, topk_w, expert_counts, kept_hist, logits};
    const Recorder rec{nullptr, st};
    return launch_route(desc, P, x, W_gate, W_mask, ro, static_cast<char *>(scratch), st, rec,
                        sm_count());
}

}  // namespace beam

namespace {

const char *const kStageNames[BEAM_MOE_FORWARD_STAGES] = {
    "router_gemm", "topk_mask", "permute", "gather", "gemm1_gate_up_swiglu", "gemm2_down",
    "combine"};

}  // namespace

extern "C" {

size_t beam_moe_backward_workspace_size(const beam_moe_desc *desc) {
    beam_moe_plan_info P;
    BwdPlan B;
    if (make_bwd_plan(desc, &P, &B) != BEAM_OK) return 0;
    return B.bytes;
}

beam_status beam_moe_backward(const beam_moe_desc *desc, const void *x, const void *W_gate,
                              const void *W_mask, const void *W1, const void *W3, const void *W2,
                              const void *dy, float beta, float *dx, float *dW_gate,
                              float *dW_mask, float *dW1, float *dW3, float *dW2,
                              void *workspace, size_t workspace_bytes, void *stream) {
    return backward_impl(desc, x, W_gate, W_mask, W1, W3, W2, dy, beta, dx, dW_gate, dW_mask,
                         dW1, dW3, dW2, workspace, workspace_bytes, stream);
}

int beam_moe_backward_kernel_count(const beam_moe_desc *desc) {
    beam_moe_plan_info P;
    BwdPlan B;
    if (make_bwd_plan(desc, &P, &B) != BEAM_OK || desc->T == 0) return 0;
    // Both: router, top-K, grouping, dy gather, gate/up, down, token, dh
    // product, dh finalize, dx product, dx, dW1/dW3, dW2, router weights (14).
    // bf16 also lists the per-expert row tiles its tensor-core GEMMs run over.
    return desc->dtype == BEAM_BF16 ? 15 : 14;
}

size_t beam_moe_workspace_size(const beam_moe_desc *desc) {
    beam_moe_plan_info P;
    if (make_plan(desc, &P) != BEAM_OK) return 0;
    return P.workspace_bytes;
}

beam_status beam_moe_plan(const beam_moe_desc *desc, beam_moe_plan_info *info) {
    if (!info) return BEAM_ERR_INVALID_ARG;
    return make_plan(desc, info);
}

beam_status beam_moe_route(const beam_moe_desc *desc, const void *x, const void *W_gate,
                           const void *W_mask, int32_t *topk_idx, float *topk_w,
                           int32_t *expert_counts, int32_t *kept_hist, float *logits,
                           void *workspace, size_t workspace_bytes, void *stream) {
    beam_moe_plan_info P;
    beam_status s = make_plan(desc, &P);
    if (s != BEAM_OK) return s;
    if (!x || !W_gate || !topk_idx || !topk_w || !expert_counts) return BEAM_ERR_INVALID_ARG;
    for (const void *p : {x, W_gate, static_cast<const void *>(topk_idx),
                          static_cast<const void *>(topk_w), static_cast<const void *>(expert_counts)})
        if (!aligned16(p)) return BEAM_ERR_INVALID_ARG;
    if ((W_mask && !aligned16(W_mask)) || (kept_hist && !aligned16(kept_hist)) ||
        (logits && !aligned16(logits)))
        return BEAM_ERR_INVALID_ARG;
    s = check_ws(P, workspace, workspace_bytes);
    if (s != BEAM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (desc->T == 0) {
        BEAM_TRY_CUDA(cudaMemsetAsync(workspace, 0, P.off_partial, st));
        BEAM_TRY_CUDA(cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * desc->E, st));
        if (kept_hist)
            BEAM_TRY_CUDA(cudaMemsetAsync(kept_hist, 0, sizeof(int32_t) * (desc->K + 1), st));
        return BEAM_OK;
    }
    const RouteOut ro{topk_idx, topk_w, expert_counts, kept_hist, logits};
    const Recorder rec{nullptr, st};
    return launch_route(desc, P, x, W_gate, W_mask, ro, static_cast<char *>(workspace), st, rec,
                        sm_count());
}

beam_status beam_moe_forward(const beam_moe_desc *desc, const void *x, const void *W_gate,
                             const void *W_mask, const void *W1, const void *W3, const void *W2,
                             void *out, void *workspace, size_t workspace_bytes, void *stream) {
    if (desc && desc->n_shared != 0) return BEAM_ERR_INVALID_ARG;  // needs the shared weights
    return forward_impl(desc, x, W_gate, W_mask, W1, W3, W2, nullptr, nullptr, nullptr, out,
                        workspace, workspace_bytes, stream, nullptr);
}

beam_status beam_moe_forward_shared(const beam_moe_desc *desc, const void *x,
                                    const void *W_gate, const void *W_mask, const void *W1,
                                    const void *W3, const void *W2, const void *W1s,
                                    const void *W3s, const void *W2s, void *out,
                                    void *workspace, size_t workspace_bytes, void *stream) {
    return forward_impl(desc, x, W_gate, W_mask, W1, W3, W2, W1s, W3s, W2s, out, workspace,
                        workspace_bytes, stream, nullptr);
}

beam_status beam_moe_forward_profiled(const beam_moe_desc *desc, const void *x,
                                      const void *W_gate, const void *W_mask, const void *W1,
                                      const void *W3, const void *W2, void *out, void *workspace,
                                      size_t workspace_bytes, void *stream,
                                      void *const *events) {
    if (!events) return BEAM_ERR_INVALID_ARG;
    if (desc && desc->n_shared != 0) return BEAM_ERR_INVALID_ARG;
    return forward_impl(desc, x, W_gate, W_mask, W1, W3, W2, nullptr, nullptr, nullptr, out,
                        workspace, workspace_bytes, stream, events);
}

beam_status beam_moe_check(const beam_moe_desc *desc, void *workspace, void *stream) {
    beam_moe_plan_info P;
    beam_status s = make_plan(desc, &P);
    if (s != BEAM_OK) return s;
    if (!workspace) return BEAM_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return BEAM_ERR_CUDA;
    int err = 0;
    if (cudaMemcpy(&err, static_cast<char *>(workspace) + P.off_err, sizeof(int),
                   cudaMemcpyDeviceToHost) != cudaSuccess)
        return BEAM_ERR_CUDA;
    if (err == DEV_ERR_TIMEOUT) return BEAM_ERR_TIMEOUT;
    if (err != 0) return BEAM_ERR_INTERNAL;
    return BEAM_OK;
}

beam_status beam_moe_ep_dispatch(const beam_moe_desc *desc, int n_ranks, const void *x,
                                 const int32_t *topk_idx, const int32_t *expert_counts,
                                 void *send_rows, int32_t *send_pair, int32_t *send_expert,
                                 int32_t *send_counts, int32_t *pair_pos, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    beam_moe_plan_info P;
    beam_status s = make_plan(desc, &P);
    if (s != BEAM_OK) return s;
    if (n_ranks < 1 || n_ranks > desc->E || desc->E % n_ranks != 0) return BEAM_ERR_INVALID_ARG;
    if (desc->n_shared != 0) return BEAM_ERR_INVALID_ARG;
    if (!x || !topk_idx || !expert_counts || !send_rows || !send_pair || !send_expert ||
        !send_counts || !pair_pos)
        return BEAM_ERR_INVALID_ARG;
    for (const void *p : {x, static_cast<const void *>(topk_idx),
                          static_cast<const void *>(expert_counts), static_cast<const void *>(send_rows),
                          static_cast<const void *>(send_pair),
                          static_cast<const void *>(send_expert),
                          static_cast<const void *>(send_counts),
                          static_cast<const void *>(pair_pos)})
        if (!aligned16(p)) return BEAM_ERR_INVALID_ARG;
    s = check_ws(P, workspace, workspace_bytes);
    if (s != BEAM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (desc->T == 0) {
        BEAM_TRY_CUDA(cudaMemsetAsync(send_counts, 0, sizeof(int32_t) * size_t(n_ranks), st));
        return BEAM_OK;
    }
    const size_t es = desc->dtype == BEAM_BF16 ? 2 : 4;
    EpDispatchArgs a;
    a.idx = topk_idx;
    a.counts = expert_counts;
    a.T = desc->T;
    a.K = desc->K;
    a.E = desc->E;
    a.G = n_ranks;
    a.x = static_cast<const uint4 *>(x);
    a.row_vec = int(es * size_t(desc->d) / 16);
    a.R = kPermCopyBlocks;
    a.send_rows = static_cast<uint4 *>(send_rows);
    a.send_pair = send_pair;
    a.send_expert = send_expert;
    a.send_counts = send_counts;
    a.pair_pos = pair_pos;
    a.err = reinterpret_cast<int *>(static_cast<char *>(workspace) + P.off_err);
    BEAM_TRY_CUDA(launch_ep_dispatch(a, st));
    return BEAM_OK;
}

beam_status beam_moe_expert_rows(const beam_moe_desc *desc, const void *x_rows,
                                 const int32_t *expert_id, const void *W1, const void *W3,
                                 const void *W2, float *y_rows, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    beam_moe_plan_info P;
    beam_status s = make_plan(desc, &P);
    if (s != BEAM_OK) return s;
    if (desc->K != 1 || desc->n_shared != 0) return BEAM_ERR_INVALID_ARG;
    if (!x_rows || !expert_id || !W1 || !W3 || !W2 || !y_rows) return BEAM_ERR_INVALID_ARG;
    for (const void *p : {x_rows, static_cast<const void *>(expert_id), W1, W3, W2,
                          static_cast<const void *>(y_rows)})
        if (!aligned16(p)) return BEAM_ERR_INVALID_ARG;
    s = check_ws(P, workspace, workspace_bytes);
    if (s != BEAM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // header (error words, meta), counts and histogram start at zero
    BEAM_TRY_CUDA(cudaMemsetAsync(workspace, 0, P.off_partial, st));
    if (desc->T == 0) return BEAM_OK;
    char *ws = static_cast<char *>(workspace);
    const int n_sm = sm_count();
    BEAM_TRY_CUDA(launch_set_routing(expert_id, desc->T, desc->E,
                                     reinterpret_cast<int *>(ws + P.off_idx),
                                     reinterpret_cast<float *>(ws + P.off_w),
                                     reinterpret_cast<int *>(ws + P.off_counts),
                                     reinterpret_cast<int *>(ws + P.off_hist),
                                     reinterpret_cast<int *>(ws + P.off_err), n_sm, st));
    return launch_tail(desc, P, x_rows, W1, W3, W2, nullptr, nullptr, nullptr, y_rows, BEAM_F32,
                       ws, st, Recorder{nullptr, st}, n_sm);
}

beam_status beam_moe_ep_combine(const beam_moe_desc *desc, const float *y_rows,
                                const int32_t *topk_idx, const float *topk_w,
                                const int32_t *pair_pos, void *out, void *stream) {
    beam_moe_plan_info P;
    beam_status s = make_plan(desc, &P);
    if (s != BEAM_OK) return s;
    if (desc->n_shared != 0) return BEAM_ERR_INVALID_ARG;
    if (desc->T == 0) return BEAM_OK;
    if (!topk_idx || !topk_w || !pair_pos || !out || !y_rows) return BEAM_ERR_INVALID_ARG;
    for (const void *p : {static_cast<const void *>(y_rows), static_cast<const void *>(topk_idx),
                          static_cast<const void *>(topk_w), static_cast<const void *>(pair_pos),
                          static_cast<const void *>(out)})
        if (!aligned16(p)) return BEAM_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    BEAM_TRY_CUDA(launch_combine(desc->dtype, y_rows, topk_idx, topk_w, pair_pos, desc->T, desc->K,
                                 desc->d, nullptr, 0, out, nullptr, sm_count(), st));
    return BEAM_OK;
}

float beam_moe_tau_to_logit(float tau) {
    if (!(tau >= 0.0f && tau <= 1.0f)) return NAN;  // NaN and values outside [0, 1]
    // ln(tau / (1 - tau)) in double, rounded once to the descriptor's float;
    // the limits tau = 0 and 1 give -inf (keep every candidate whose z is not
    // NaN) and +inf (keep none).
    const double t = double(tau);
    return float(std::log(t / (1.0 - t)));
}

beam_status beam_moe_set_fault_injection(int mode, unsigned long long wait_limit_ns) {
    if (mode != FAULT_NONE && mode != FAULT_EXPERT_STAGE && mode != FAULT_ROUTER_STAGE &&
        mode != FAULT_SHARED_STAGE)
        return BEAM_ERR_INVALID_ARG;
    g_fault.store(mode, std::memory_order_relaxed);
    g_wait_limit_ns.store(wait_limit_ns, std::memory_order_relaxed);
    return BEAM_OK;
}

const char *beam_status_str(beam_status status) {
    switch (status) {
        case BEAM_OK: return "BEAM_OK";
        case BEAM_ERR_INVALID_ARG: return "BEAM_ERR_INVALID_ARG";
        case BEAM_ERR_UNSUPPORTED_SHAPE: return "BEAM_ERR_UNSUPPORTED_SHAPE";
        case BEAM_ERR_WORKSPACE: return "BEAM_ERR_WORKSPACE";
        case BEAM_ERR_CUDA: return "BEAM_ERR_CUDA";
        case BEAM_ERR_TIMEOUT: return "BEAM_ERR_TIMEOUT";
        case BEAM_ERR_INTERNAL: return "BEAM_ERR_INTERNAL";
    }
    return "BEAM_ERR_UNKNOWN";
}

int beam_moe_set_one_launch_tokens(int max_tokens) {
    const int v = max_tokens < 0 ? 0 : max_tokens > kDlMaxT ? kDlMaxT : max_tokens;
    return g_one_launch_tokens.exchange(v, std::memory_order_relaxed);
}

int beam_moe_forward_kernel_count(const beam_moe_desc *desc) {
    beam_moe_plan_info P;
    if (make_plan(desc, &P) != BEAM_OK) return 0;
    if (desc->T == 0) return 0;
    if (P.one_launch) return 1;
    const int shared = desc->n_shared > 0 ? (P.sh_split1 > 1 ? 3 : 2) : 0;
    // Fused decode path: rows copied by the grouping kernel (no gather
    // launch) and one launch for both expert GEMMs.
    // Other batches: the grouping is two launches (chunked) up to 65536 tokens.
    if (desc->dtype == BEAM_BF16 && fused_experts(P)) return shared + BEAM_MOE_FORWARD_STAGES - 2;
    return shared + BEAM_MOE_FORWARD_STAGES + (group_chunked_fits(desc->T) ? 1 : 0);
}

const char *beam_moe_stage_name(int stage) {
    if (stage < 0 || stage >= BEAM_MOE_FORWARD_STAGES) return nullptr;
    return kStageNames[stage];
}

}  // extern "C"
