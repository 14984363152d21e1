// beam_internal.h -- launch interface between the C-ABI host code
// (beam_api.cu) and the kernels (tc_gemm.cu, simt_kernels.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "beam_moe.h"

namespace beam {

// Device error word values (workspace `err`).
enum : int { DEV_OK = 0, DEV_ERR_TIMEOUT = 1, DEV_ERR_INTERNAL = 2 };

// The router kernel never writes the error word itself: its CTAs would race
// with the clear that starts a call.  A router CTA whose bounded wait expires
// writes this tag into the header's second word instead; the top-K kernel,
// which runs after the whole router grid, folds it into the error word (and
// resets it), so the word it leaves is exactly this call's router status.  A
// tag, not a small code, so that a fresh workspace's leftover bytes are not
// taken for a timeout.
constexpr int kRouterTimeoutTag = 0x5EA71AB5;
// The shared experts' GEMMs may run on a second stream, beside the router and
// top-K kernels, so they do the same through the header's third word; the
// combine, which runs after both streams have joined, folds and resets it.
constexpr int kSharedTimeoutTag = 0x5EA75E0D;
constexpr int kHdrErr = 0, kHdrErrRouter = 1, kHdrErrShared = 2, kHdrMeta = 4;  // int offsets

// Fault injection for tests (beam_moe_set_fault_injection): which launch skips
// one stage load in CTA 0 so that its MMA issuer's bounded wait expires.
enum : int { FAULT_NONE = 0, FAULT_EXPERT_STAGE = 1, FAULT_ROUTER_STAGE = 2, FAULT_SHARED_STAGE = 3 };

// Roles of the tensor-core GEMM kernel.
enum TcMode : int {
    MODE_ROUTER = 0,  // logits: [W_gate | W_mask] rows x token rows, split over d
    MODE_GEMM1 = 1,   // SiLU(W1 x) * (W3 x) per kept pair  -> H
    MODE_GEMM2 = 2,   // W2 h per kept pair                  -> Y
    MODE_GEMM1_IL = 3, // GEMM1 with 64 rows of W1 and 64 of W3 interleaved in one tile
    MODE_EXPERTS = 4,  // MODE_GEMM1_IL units then MODE_GEMM2 units in one launch
    MODE_GEMM2T = 5,   // dy W2_e (training): W2_e read transposed (MN-major A) -> fp32 rows
    MODE_GEMM1T = 6    // da W1_e + db W3_e (training): W1_e, W3_e read transposed -> fp32 rows
};

// Tensor maps of one tensor-core launch.  a0/a1/b: the (first) GEMM's weight
// tile(s) and token tile; a2/b2: the down projection's in MODE_EXPERTS.
struct TcMaps {
    CUtensorMap a0, a1, b, a2, b2;
};

constexpr int kBlockM = 128;   // weight rows per tile (the MMA's M)
constexpr int kBlockK = 64;    // reduction elements per stage: one 128-byte bf16 row
constexpr int kNominalSMs = 148;
constexpr int kMaxE = 256;
constexpr int kMaxK = 16;
constexpr int kMaxRouterSplits = 32;  // top-K sums the split partials unrolled
constexpr int kMaxShared = 16;        // shared experts per layer
constexpr int kPermCopyBlocks = 4;    // grouping blocks per expert when they copy rows
constexpr int kMaxTileRows = 128;     // largest token tile (BN)


// Launch with programmatic stream serialization (PDL): the kernel may begin
// its prologue while the previous kernel in the stream finishes; every kernel
// of this library waits (griddep_wait) before touching global memory.
// cudaFuncSetAttribute(kern, MaxDynamicSharedMemorySize, bytes) once per
// kernel and device (the attribute persists; repeating it costs host time on
// every launch).  `done` is the caller's flag word for this one kernel (one
// bit per device); `bytes` must be the same on every call for that kernel.
template <typename... KArgs>
cudaError_t set_smem_once(void (*kern)(KArgs...), int bytes,
                          std::atomic<unsigned long long> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

struct ZeroRegion {
    int *ptr;
    int count;
};

// Arguments of the tensor-core GEMM (all three modes).
struct TcGemmArgs {
    int n_mb;            // weight-row blocks per token tile
    int nk;              // k-blocks per unit
    int n_tt;            // router: token tiles
    int n_mb_gate;       // router: m-blocks read from W_gate; the rest from W_mask
    int n_units;         // router: number of units (GEMMs take it from meta[0])
    int T, E;            // router: tokens and experts (logit columns 2E)
    int a_rows_per_expert;  // GEMM1: I, GEMM2: d
    const int *meta;     // GEMMs: meta[0] = tiles in the tile list
    const int4 *tiles;   // GEMMs: (expert, first row, valid rows, 0)
    void *out;           // router: f32 partial [S][T][2E]; GEMM1: H (bf16); GEMM2: Y (f32)
    long long out_ld;    // elements per output row
    long long out_split_stride;  // router: elements per split slab
    int *err;            // device error word (router: the header's router word)
    int err_code;        // value written on a wait expiry (0 = DEV_ERR_TIMEOUT)
    int fault_skip;      // 1: CTA 0 skips the first stage load of its first unit (tests)
    ZeroRegion zero[3];  // router: regions CTA 0 clears for the later kernels
    unsigned long long timeout_ns;
    // MODE_EXPERTS: the down projection that follows the gate/up units
    int n_mb2, nk2, a_rows2;  // d/128 row blocks, I/64 k-blocks, d rows per expert
    void *out2;               // Y (f32)
    long long out2_ld;
    float *a_out, *b_out;     // MODE_GEMM1 (or null): fp32 pre-activations, like H
    int *tile_done;           // per tile: gate/up units whose H rows are published
    int *work_ctr;            // next unit to hand out (zeroed by the router kernel)

    // MODE_GEMM1 / MODE_GEMM2 over every token (shared experts): tile ti of
    // n_units / n_mb is (shared expert ti / dense_ntt, token tile ti % dense_ntt);
    // GEMM1 reads x rows, GEMM2 reads and both write rows s * T + token.
    int dense, dense_ntt, dense_T, dense_gemm2;
    // Split reduction of dense units: unit u is (tile, m-block, split u % ksplit)
    // over k-blocks [split * nk / ksplit, (split + 1) * nk / ksplit); its output
    // rows move by split * dense_slab_rows (one slab per split).  GEMM1 with a
    // null `out` writes only the fp32 pre-activations (a_out, b_out).
    int dense_ksplit;
    int dense_slab_rows;
};

cudaError_t launch_tc_gemm(int mode, int bn, const TcMaps &maps, const TcGemmArgs &args, int grid,
                           cudaStream_t stream);

// Top-K + softmax + mask + aggregation (one warp per token).
struct TopkArgs {
    const float *partial;  // [S][T][2E]
    int S, T, E, K, renorm, has_mask;
    float thr;             // keep iff z >= thr (logit of the threshold tau)
    int *hdr;              // workspace header: block 0 sets err from the router word
    float *logits;         // [T][2E] or NULL
    int *idx;              // [T][K]
    float *w;              // [T][K]
    int *counts;           // [E]
    int *hist;             // [K+1] or NULL
    // Training (backward) extras, each NULL-able: every candidate (masked or
    // not) in slot order, its softmax weight before the mask, and candidate
    // counts per expert (zeroed by the caller).
    int *cand;             // [T][K]
    float *gk;             // [T][K]
    int *counts_all;       // [E]
};
cudaError_t launch_topk_mask(const TopkArgs &a, int n_sm, cudaStream_t stream);

// Expert grouping: one block per expert.
struct PermuteArgs {
    const int *idx;
    const int *counts;
    int T, K, E, BN;
    int *pair, *pair_pos;
    int4 *tiles;
    int *tile_done;  // cleared for every tile written (MODE_EXPERTS counters)
    // Optional row copy (fused decode path): x rows into grouped order, done by
    // R blocks per expert instead of a separate gather launch.  x, xp null: none.
    const uint4 *x;
    uint4 *xp;
    int row_vec;  // 16-byte vectors per row
    int R;        // blocks per expert (>= 1)
    int *meta;
    int *err;
    int4 *tiles_sub;  // or null: the same rows as tiles of sub_bn rows (count -> meta[3])
    int sub_bn;
};
cudaError_t launch_permute(const PermuteArgs &a, cudaStream_t stream);

// The same grouping (R = 1, no row copy) as two launches over token chunks:
// per-chunk counts into chunk_cnt (at most 256 * E ints of scratch, 16-byte
// aligned), then the placement.  Identical pair, pair_pos, tiles, tiles_sub and meta.
// Only for T <= 65536 (group_chunked_fits).
bool group_chunked_fits(int T);
cudaError_t launch_group_chunked(const PermuteArgs &a, int *chunk_cnt, cudaStream_t stream);

// Expert-parallel dispatch (ep_kernels.cu): kept pairs listed by expert
// (ascending) then token, which groups them by destination rank r = e / (E/G).
struct EpDispatchArgs {
    const int *idx;      // [T][K] candidate or -1
    const int *counts;   // [E] kept pairs per expert
    int T, K, E, G;
    const uint4 *x;      // token rows
    int row_vec;         // 16-byte vectors per row
    int R;               // blocks per expert (row copy)
    uint4 *send_rows;    // [P][row_vec] kept pairs' token rows, in listed order
    int *send_pair;      // [P] t*K + k of each send row
    int *send_expert;    // [P] local expert id of each send row on its destination
    int *send_counts;    // [G] send rows per destination rank
    int *pair_pos;       // [T][K] send row of a kept pair
    int *err;
};
cudaError_t launch_ep_dispatch(const EpDispatchArgs &a, cudaStream_t stream);
// Received rows -> routing of a K = 1 layer call with weight 1 (counts, hist
// zeroed by the caller).
cudaError_t launch_set_routing(const int *expert_id, int N, int E, int *idx, float *w, int *counts,
                               int *hist, int *err, int n_sm, cudaStream_t stream);

// ---------------------------------------------------------------------------
// The whole layer of a small decode batch in one launch (decode_layer.cu).
// One persistent CTA per SM (15 consumer warps and one producer warp); the
// phases hand off through counters in the workspace, never through a kernel
// boundary:
//   router items   2 rows of [W_gate; W_mask] against every token -> logits
//   routing        every CTA reads all logits and takes the same top-K, mask
//                  and grouping in shared memory (no second hand-off)
//   gate/up items  one row of W1 and of W3 of one kept expert -> H[., i]
//   down items     R2 rows of W2 of one kept expert -> columns of Y; the item
//                  that completes a (token, row block) of the output sums the
//                  token's kept rows of Y in slot order (the combine)
// The producer streams each item's rows (bulk copies) into a ring of
// shared-memory stages ahead of the consumer warps.
constexpr int kDlThreads = 512;        // 15 consumer warps + 1 producer warp
constexpr int kDlMaxT = 16;             // tokens per call on this path
constexpr int kDlMaxStages = 32;
constexpr int kDlSmemCap = 196 * 1024;  // dynamic shared memory budget
constexpr int kHdrDlRouter = 8;         // header int: router units published

enum : int { DL_FORWARD = 0, DL_ROUTER_ONLY = 1 };

struct DecodeLayerArgs {
    int mode;                    // DL_FORWARD, or DL_ROUTER_ONLY (logits only)
    int T, d, E, I, K, renorm, has_mask;
    float thr;                   // keep iff z >= thr
    const void *x, *Wg, *Wm, *W1, *W3, *W2;  // bf16
    void *out;                   // bf16 [T][d]
    float *partial;              // [T][2E] logits (one split)
    int *idx;                    // [T][K]
    float *w;                    // [T][K]
    int *counts, *hist;          // [E], [K+1]
    int *pair, *pair_pos;        // grouping rows (BN-padded per expert)
    int4 *tiles;
    int BN;
    void *H;                     // bf16 [rows][I]
    float *Y;                    // [rows][d]
    int *hdr;                    // workspace header (error words, meta, router counter)
    int *e1_done;                // [E][I / 128] gate/up units finished per block of H
    int *comb_cnt;               // [T][d / R2] down items finished per (token, row block)
    ZeroRegion zero[3];          // router-only mode: regions CTA 0 clears
    int rr, n_ru;                // rows per router item, router items
    int R1, R2;                  // rows per gate/up item (of I), per down item (of d)
    int n_stages, stage_bytes;
    int sm_off_lg, sm_off_stage, smem_bytes;  // dynamic shared memory layout
    int fault_skip;              // tests: FAULT_* of this call
    unsigned long long timeout_ns;
};

// Shape limits and unit sizes of the one-launch path; false if the shape does
// not fit it (the caller then takes the multi-kernel path).
bool decode_layer_config(int T, int d, int E, int I, int K, int has_mask, int n_sm,
                         DecodeLayerArgs *cfg);
// Tensor maps of the expert weights and of H for the one-launch path's tiles
// (128-byte swizzle, boxes of 64 columns): W1 and W3 [E*I, d] with boxes of
// 8 rows, W2 [E*d, I] and H [rows, I] with boxes of 16 rows.  Router-only
// launches do not read them.
struct DlMaps {
    CUtensorMap w1, w3, w2, h;
};
cudaError_t launch_decode_layer(const DlMaps &maps, const DecodeLayerArgs &a, int grid,
                                cudaStream_t stream);

// Shared experts with a split gate/up reduction: H = SiLU(sum of the gate
// partials) * (sum of the up partials), summed in split order, rounded to bf16.
cudaError_t launch_shared_swiglu(const float *A, const float *B, int splits, long long n,
                                 void *H, cudaStream_t stream);

// Gather token rows into expert order (row_bytes multiple of 16).
cudaError_t launch_gather(const void *x, const int *pair, const int *meta, int K,
                          long long row_bytes, int p_cap, void *xp, int n_sm,
                          cudaStream_t stream);

// out[t] = sum_k w[t,k] * Y[pair_pos[t,k]] over kept k; Y fp32, fp32 sums,
// one rounding to the output dtype.  hdr (or null): the call's header, whose
// shared-expert timeout tag is folded into its error word.
cudaError_t launch_combine(int dtype, const float *Y, const int *idx, const float *w,
                           const int *pair_pos, int T, int K, int d, const float *Ys,
                           int n_shared, void *out, int *hdr, int n_sm, cudaStream_t stream);

// Training-mode backward (backward.cu).  Rows are those of the grouping of all
// candidates (masked ones included); every array lives in the workspace.
struct BwArgs {
    int T, d, E, I, K, renorm, has_mask, tiles_cap, p_cap;
    int S;                   // splits of the reduction in the kept-row products
    float beta;
    const float *Y;          // [p_cap][d] every candidate's expert output
    const float *logits;     // [T][2E] router logits (r, then z)
    const int *cand;         // [T][K] candidates
    const float *gk;         // [T][K] softmax weights before the mask
    const int *idx;          // [T][K] candidate or -1 (masked)
    const float *w;          // [T][K] g * m
    const int *pair;         // [p_cap] row -> t*K + k (-1 on padding)
    const int *pair_pos;     // [T][K] row of a candidate
    const int4 *tiles;       // tile list of the grouping
    const int *meta;         // [0] tiles
    const int *counts_kept;  // [E] kept pairs per expert
    const int *counts_all;   // [E] candidates per expert
    const float *A, *B;      // [p_cap][I] gate / up pre-activations
    float *da, *db;          // [p_cap][I]
    float *h;                // [p_cap][I] SiLU(a) b in fp32 (kept rows)
    float *part;             // [S][p_cap][max(d, I)] split partial products
    int dh_tc;               // 1: dy W2_e is already in part (one split, tensor cores)
    int dx_tc;               // 1: da W1_e + db W3_e runs on the tensor cores between the
                             //    two stage phases, into part (one split)
    void *da_bf, *db_bf;     // [p_cap][I] bf16 copies of da, db (kept rows) or null
    float *u, *dz;           // [T][K]
    float *dr;               // [T][E]
    float *dx;               // [T][d]
};
// Each expert's candidate rows as tiles of at most rows_per_tile rows (one
// block): from the grouping's tile list, an expert gives
// ceil(candidates / rows_per_tile) tiles starting at its first row.  xt_all
// lists every candidate expert's (count in xmeta[0]); xt_kept only those of
// experts with a kept pair (xmeta[1]).  Neither is longer than the grouping's
// tile list when rows_per_tile >= BN.
cudaError_t launch_expert_tiles(const int4 *tiles, const int *meta, const int *counts_kept,
                                const int *counts_all, int rows_per_tile, int4 *xt_all,
                                int4 *xt_kept, int *xmeta, cudaStream_t st);
// phase 0: token stage, dh product (unless dh_tc), dh finalize; phase 1: dx
// product (unless dx_tc), dx, dW1/dW3, dW2, router weights.
cudaError_t launch_backward_stages(const BwArgs &a, int dtype, const void *x, const void *xp,
                                   const void *dy, const void *dyp, const void *Wg,
                                   const void *Wm, const void *W1, const void *W3,
                                   const void *W2, float *dWg, float *dWm, float *dW1,
                                   float *dW3, float *dW2, int n_sm, cudaStream_t st, int phase);

// fp32 SIMT path (BEAM_F32).
cudaError_t launch_router_f32(const float *x, const float *Wg, const float *Wm, int T, int d,
                              int E, float *partial, const ZeroRegion (&zero)[3],
                              cudaStream_t stream);
cudaError_t launch_gemm1_f32(const float *xp, const float *W1, const float *W3, const int4 *tiles,
                             const int *meta, int tiles_cap, int d, int I, float *H,
                             cudaStream_t stream, float *A = nullptr, float *B = nullptr);
cudaError_t launch_gemm2_f32(const float *H, const float *W2, const int4 *tiles, const int *meta,
                             int tiles_cap, int d, int I, float *Y, cudaStream_t stream);

// Routing (the two kernels of beam_moe_route) into caller-provided scratch
// of at least route_scratch_bytes(desc) bytes, 256-byte aligned.
size_t route_scratch_bytes(const beam_moe_desc *desc);  // 0 on a bad descriptor
beam_status route_into_scratch(const beam_moe_desc *desc, const void *x, const void *W_gate,
                               const void *W_mask, int32_t *topk_idx, float *topk_w,
                               int32_t *expert_counts, int32_t *kept_hist, float *logits,
                               void *scratch, size_t scratch_bytes, cudaStream_t stream);

}  // namespace beam
