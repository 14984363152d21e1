/*
 * beam_moe.h -- C ABI of the BEAM-masked MoE layer forward pass (B200, sm_100a).
 *
 * The operation is the MoE layer of "BEAM: Binary Expert Activation Masking
 * for Dynamic Routing in MoE" (arXiv 2605.14438), §3.2, for one batch of T
 * tokens x [T, d]:
 *
 *   r = x W_gate                 main-router logits                (step 1)
 *   g = Softmax(Top-K(r))        candidate weights                 (Eq. 1/4)
 *   m = [sigmoid(x W_mask) >= 0.5] on the K candidates             (Eq. 5-6)
 *   w = g * m                    no renormalisation after the mask (Eq. 7)
 *   y = sum_k w_k E_{c_k}(x)     only kept (token, expert) pairs   (Eq. 8)
 *   E_e(x) = (SiLU(x W1_e^T) * (x W3_e^T)) W2_e^T                  (Eq. 3)
 *
 * A token whose candidates are all masked gets y = 0 (it passes the layer
 * through the residual, which stays the caller's).  A masked pair is never
 * scheduled, so an expert without kept pairs has none of its weights read.
 *
 * Conventions (all entry points):
 *  - Layouts are row-major and contiguous: x [T,d]; W_gate, W_mask [E,d]
 *    (row e = column e of the paper's d x N matrices); W1 (gate), W3 (up)
 *    [E,I,d]; W2 (down) [E,d,I]; out [T,d].
 *  - dtype BEAM_BF16: x, weights and out are bfloat16; accumulation is fp32;
 *    the SwiGLU activations H (the second GEMM's operand) are rounded to bf16
 *    once; the per-pair expert outputs stay fp32 and the weighted sum is
 *    rounded to bf16 once.  dtype BEAM_F32: everything fp32.  Logits, softmax
 *    weights and the combine are fp32 in both.
 *  - Every pointer except the host descriptor is a DEVICE pointer, 16-byte
 *    aligned.  The caller owns every buffer, including the workspace; the
 *    library allocates nothing and keeps no state between calls.
 *  - Every launch is ordered on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and the calls never synchronise the host, except
 *    beam_moe_check.  Argument and shape errors are returned before anything
 *    is launched; a failed launch returns BEAM_ERR_CUDA.
 *  - Constraints: 1 <= K <= min(E, 16), E <= 256, T >= 0.  BEAM_BF16 needs
 *    d % 128 == 0 and I % 128 == 0; BEAM_F32 needs d % 8 == 0 and I % 8 == 0
 *    (else BEAM_ERR_UNSUPPORTED_SHAPE).  T*K and the workspace rows must fit
 *    in int32.
 *  - Top-K ties go to the lower expert index; candidates are listed by
 *    descending logit (the paper does not fix either).  The mask test is taken
 *    on the pre-sigmoid value, z >= 0 <=> sigmoid(z) >= 0.5 (Eq. 6); NaN is
 *    not kept.  Non-finite inputs are the caller's responsibility.
 */
#ifndef BEAM_MOE_H
#define BEAM_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BEAM_OK = 0,
    BEAM_ERR_INVALID_ARG = 1,       /* NULL / misaligned pointer, bad K, E, dtype, ... */
    BEAM_ERR_UNSUPPORTED_SHAPE = 2, /* d or I not a multiple of the tile width */
    BEAM_ERR_WORKSPACE = 3,         /* workspace NULL, misaligned or too small */
    BEAM_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
    BEAM_ERR_TIMEOUT = 5,           /* a bounded device-side wait gave up */
    BEAM_ERR_INTERNAL = 6           /* a device-side consistency check failed */
} beam_status;

typedef enum { BEAM_BF16 = 0, BEAM_F32 = 1 } beam_dtype;

/* One MoE layer call: T tokens of width d, E experts, top-K, SwiGLU width I.
 * renorm_topk = 1: softmax over the K largest logits (Eq. 4, sums to 1).
 * renorm_topk = 0: softmax over all E logits, restricted to the K largest.
 * mask_logit_threshold: the binarisation threshold tau of Eq. (6) given as
 *   its logit, ln(tau / (1 - tau)); a candidate is kept iff its mask
 *   pre-activation z >= mask_logit_threshold (i.e. sigmoid(z) >= tau).
 *   0 is the paper's tau = 0.5, so a zero-initialised descriptor keeps the
 *   method's default; other values reproduce the threshold ablation (news
 *   article on BEAM, §8); beam_moe_tau_to_logit converts a tau.  Must not
 *   be NaN.
 * n_shared, I_shared: always-on shared experts (news article on BEAM, §5:
 *   models such as Qwen1.5-MoE and DeepSeek-V2-Lite keep running them for
 *   every token, all-masked tokens included), n_shared SwiGLU experts of
 *   width I_shared, each added with weight 1 after the routed sum.  0 = none
 *   (beam_moe_forward); > 0 needs beam_moe_forward_shared, BEAM_BF16,
 *   n_shared <= 16 and I_shared % 128 == 0. */
typedef struct {
    int T, d, E, I, K;
    int dtype;       /* beam_dtype */
    int renorm_topk; /* 0 or 1 */
    float mask_logit_threshold;
    int n_shared, I_shared;
} beam_moe_desc;

/* Workspace layout chosen for a descriptor (byte offsets from the workspace
 * base).  Exposed so that tests and tools can read the intermediate arrays
 * after beam_moe_forward; none of it is needed to call the layer.
 *   err       int32      device error word (0 = ok), read by beam_moe_check
 *   meta      int32[4]   [0] tiles in the tile list, [1] padded rows,
 *                        [2] kept pairs P, [3] work counter of the fused
 *                        expert kernel (units handed out so far), or with
 *                        256-row tiles the number of 128-row sub-tiles
 *   counts    int32[E]   kept pairs per expert
 *   hist      int32[K+1] tokens by number of kept candidates
 *   partial   f32[S][T][2E] router partial logits (S = router_splits)
 *   idx       int32[T][K] candidate expert, -1 where masked
 *   w         f32[T][K]   g * m
 *   pair      int32[p_cap] permuted row -> t*K + k (-1 on padding rows);
 *             expert e owns rows [off_e, off_e + roundup(counts[e], BN)),
 *             experts in ascending order, tokens ascending inside
 *   pair_pos  int32[T][K] permuted row of a kept pair (undefined if masked)
 *   tiles     int32[tiles_cap][4] (expert, first row, valid rows, 0)
 *   tile_done int32[tiles_cap] gate/up units finished per tile (fused path)
 *   xp        [p_cap][d]  gathered token rows (dtype)
 *   h         [p_cap][I]  SiLU(x W1^T) * (x W3^T) per pair (dtype)
 *   y         f32[p_cap][d] expert output per pair
 *   hs        [n_shared*T][I_shared] shared experts' SwiGLU activations (dtype)
 *   ys        f32[sh_split2][n_shared*T][d] shared experts' outputs, one slab per
 *             split of their down reduction (the combine adds every slab)
 *   sp        f32[2][sh_split1][n_shared*T][I_shared] partial gate and up
 *             pre-activations of the shared experts' split reduction
 *   tiles_sub int32[][4] with 256-row tiles: the same rows as 128-row tiles,
 *             the gate/up GEMM's units (their count in meta[3])
 *   ctl       int32[]     one-launch path: gate/up units finished per expert,
 *                         down units finished per (token, output row block)
 * With one_launch the layer runs as one kernel that writes err, meta,
 * counts, hist, partial (one split), idx, w, pair, pair_pos, tiles, h and y
 * as above; xp, tile_done, hs, ys and tiles_sub are not used.             */
typedef struct {
    int BN;            /* token rows per expert tile; the padding unit */
    int router_bn;     /* token rows per router tile */
    int router_splits; /* router split-K factor S */
    int p_cap;         /* rows of xp / h / y / pair */
    int tiles_cap;     /* entries of the tile list */
    int sub_bn;        /* token rows of the gate/up GEMM's tiles (BN, or 128 when BN = 256) */
    int one_launch;    /* 1: beam_moe_forward runs the whole layer as one kernel */
    int sh_bn;         /* shared experts: token rows per tile */
    int sh_split1;     /* shared experts: splits of the gate/up reduction (over d) */
    int sh_split2;     /* shared experts: splits of the down reduction (over I_shared) */
    size_t off_err, off_meta, off_counts, off_hist, off_partial, off_idx, off_w,
        off_pair, off_pair_pos, off_tiles, off_xp, off_h, off_y, off_tile_done, off_hs,
        off_ys, off_tiles_sub, off_ctl, off_sp;
    size_t workspace_bytes;
} beam_moe_plan_info;

/* Stage slots of one beam_moe_forward call (router GEMM, top-K + mask,
 * grouping, gather, gate/up GEMM, down GEMM, combine).  With token tiles
 * thinner than 128 rows (decode batches, bf16) the grouping kernel copies the
 * token rows itself, so the gather slot is empty, and the two expert GEMMs run
 * as one fused launch in the gate/up slot, so the down slot is empty too; see
 * beam_moe_forward_kernel_count. */
#define BEAM_MOE_FORWARD_STAGES 7

/* Bytes of device workspace beam_moe_forward needs for `desc` (0 on a bad
 * descriptor).  Grows with T: O(T*K*(2d + I)) for the permuted activations. */
size_t beam_moe_workspace_size(const beam_moe_desc *desc);

/* Fill `info` with the workspace layout for `desc`.  Host only. */
beam_status beam_moe_plan(const beam_moe_desc *desc, beam_moe_plan_info *info);

/* Routing alone: §3.2 steps 1-3 and Eq. (7).
 *   x, W_gate [E,d], W_mask [E,d] or NULL (mask disabled: all candidates kept)
 *   topk_idx  int32 [T,K]  candidate expert id, -1 where masked      (written)
 *   topk_w    f32   [T,K]  g * m                                     (written)
 *   expert_counts int32 [E] kept pairs per expert                    (written)
 *   kept_hist int32 [K+1] tokens by kept count, or NULL              (written)
 *   logits    f32 [T,2E] or NULL: r in columns [0,E), the mask pre-activation
 *             z in [E,2E) (not written when W_mask is NULL)          (written)
 *   workspace of beam_moe_workspace_size(desc) bytes (partial logits).
 * Uses the same kernels, tiling and summation order as beam_moe_forward, so
 * both take bitwise identical routing decisions for the same inputs. */
beam_status beam_moe_route(const beam_moe_desc *desc, const void *x, const void *W_gate,
                           const void *W_mask, int32_t *topk_idx, float *topk_w,
                           int32_t *expert_counts, int32_t *kept_hist, float *logits,
                           void *workspace, size_t workspace_bytes, void *stream);

/* The whole layer, Eq. (4)-(8): out [T,d] = sum of kept experts' outputs
 * weighted by g * m.  W_mask NULL runs the same kernels with the mask test
 * off (vanilla Top-K MoE).  Launches beam_moe_forward_kernel_count(desc)
 * kernels: with 128-row token tiles (bf16 prefill batches, and BEAM_F32) all
 * seven stages -- router GEMM, top-K + mask, grouping, row gather, gate/up
 * GEMM + SwiGLU, down GEMM, weighted combine; with thinner tiles (bf16 decode
 * batches) five, because the grouping copies the token rows and both expert
 * GEMMs run as one launch.  No host synchronisation; capturable into a CUDA
 * graph. */
beam_status beam_moe_forward(const beam_moe_desc *desc, const void *x, const void *W_gate,
                             const void *W_mask, const void *W1, const void *W3,
                             const void *W2, void *out, void *workspace,
                             size_t workspace_bytes, void *stream);

/* beam_moe_forward with shared experts (desc->n_shared > 0): out = routed sum
 * (Eq. 8) + sum over the shared experts of E_s(x), the shared experts run for
 * every token.  W1s (gate), W3s (up) [n_shared, I_shared, d], W2s (down)
 * [n_shared, d, I_shared], bf16.  Two or three more launches than
 * beam_moe_forward (a gate/up GEMM, when its reduction is split a SwiGLU
 * kernel, and a down GEMM over all tokens; see beam_moe_forward_kernel_count).
 * They read no routing, so they run on a second stream that the library owns
 * (one per device, created by the first such call made outside a stream
 * capture): the call records an event on `stream` at its start, the second
 * stream waits for it, and `stream` waits for the second stream's event
 * before the combine.  Work issued on `stream` after the call therefore
 * follows all of it, as with any other call; a captured call records the
 * fork and the join as graph edges.  A first call made inside a capture runs
 * the shared experts on `stream` itself.  Calls are serialised on the host
 * from the fork to the end of their enqueue (a lock), so concurrent callers
 * never interleave their events.  With n_shared == 0 it is beam_moe_forward
 * (the shared pointers may be NULL). */
beam_status beam_moe_forward_shared(const beam_moe_desc *desc, const void *x,
                                    const void *W_gate, const void *W_mask, const void *W1,
                                    const void *W3, const void *W2, const void *W1s,
                                    const void *W3s, const void *W2s, void *out,
                                    void *workspace, size_t workspace_bytes, void *stream);

/* beam_moe_forward that also records `events[i]` (cudaEvent_t, created by the
 * caller) on `stream` before stage i and events[BEAM_MOE_FORWARD_STAGES]
 * after the last one, so the caller can time each kernel with
 * cudaEventElapsedTime.  The records are "external" (cudaEventRecordExternal):
 * captured into a CUDA graph they become event nodes that every replay
 * re-records.  A NULL entry records nothing at that point (each record costs
 * a few microseconds of device time, so time one kernel with just the two
 * events around it).  Same launches and results as beam_moe_forward. */
beam_status beam_moe_forward_profiled(const beam_moe_desc *desc, const void *x,
                                      const void *W_gate, const void *W_mask,
                                      const void *W1, const void *W3, const void *W2,
                                      void *out, void *workspace, size_t workspace_bytes,
                                      void *stream, void *const *events);

/* Bytes of the fixed device array behind beam_moe_route_noalloc (16 MiB). */
#define BEAM_MOE_ROUTE_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* beam_moe_route for callers that cannot allocate device memory.  The paper
 * has no counterpart: this is a service of this library.
 *
 * Who needs it: plugins inside a host runtime whose memory pool owns all of
 * the device memory and lets its extensions allocate none (a serving engine
 * that reserves the GPU when it starts, for example), and callers inside a
 * fixed memory budget, where a new allocation may fail or fragment the pool.
 * The caller still passes every input and output exactly as for
 * beam_moe_route; the scratch (router partial logits, error words, counters)
 * lives in a file-scope device array of BEAM_MOE_ROUTE_NOALLOC_SCRATCH_BYTES
 * that every GPU loading the library holds until the process exits.  Nothing
 * here calls cudaMalloc, cudaFree or any allocating routine.
 *  - Size limit: the call needs beam_moe_plan(desc)->off_idx bytes of
 *    scratch; larger batches return BEAM_ERR_WORKSPACE before any launch (for
 *    d=2048, E=128 every T up to 8192 fits).
 *  - The first call on a device looks the array's address up on that device
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - All calls share the one array, which keeps the last call's contents:
 *    calls whose kernels may overlap on the GPU (different streams, or
 *    concurrent host threads) race on it and must be ordered by the caller.
 *    Each call clears what must start at zero.
 *  - Same kernels and results as beam_moe_route.  Its device error word is in
 *    the array: read it with beam_moe_route_noalloc_check. */
beam_status beam_moe_route_noalloc(const beam_moe_desc *desc, const void *x,
                                   const void *W_gate, const void *W_mask, int32_t *topk_idx,
                                   float *topk_w, int32_t *expert_counts, int32_t *kept_hist,
                                   float *logits, void *stream);

/* Synchronise `stream`, then read the error word of the last
 * beam_moe_route_noalloc call on the current device: BEAM_OK, or
 * BEAM_ERR_TIMEOUT when a bounded device wait of the router expired (its
 * outputs are then not valid).  Allocates nothing. */
beam_status beam_moe_route_noalloc_check(void *stream);

/* Kernel launches one forward call makes for `desc`: 5 (bf16 with
 * decode-sized token tiles) or 7, plus 2 with shared experts; 0 for T = 0 or
 * a bad descriptor. */
int beam_moe_forward_kernel_count(const beam_moe_desc *desc);

/* Tuning switch of the one-launch path (plan field one_launch): bf16 calls
 * without shared experts and with at most max_tokens tokens (and at most 16,
 * whose token rows, logits and weight stages fit one CTA's shared memory)
 * run router, top-K + mask, grouping, both expert projections and the
 * combine as ONE kernel whose phases hand off through counters in the
 * workspace.  Larger batches take the multi-kernel path.  0 turns it off.
 * Default 4: the batch sizes where it was measured faster.  Returns the
 * previous value; process-wide, not per call.  Routing at those sizes (and
 * only the routing) is the same in both paths: the router logits of every
 * bf16 call with T <= 16 come from the same router code. */
int beam_moe_set_one_launch_tokens(int max_tokens);

/* ------------------------------------------------------------ training --
 * Backward pass of the layer for training the mask router (techwalker news
 * article on BEAM, §4: the binary decision is trained through a
 * straight-through estimator, and a penalty weighted by beta on the
 * candidates' mask scores pushes towards fewer active experts).  The pages
 * give both in words; the readings taken here:
 *   objective  L = sum_t <dy_t, y_t> + beta * sum_t sum_{k<K} sigmoid(z_{t,c_k})
 *              (the penalty adds up the K candidates' scores of every token;
 *              divide beta by the token count for a mean)
 *   estimator  the forward keeps the hard mask of Eq. (6); the backward
 *              passes the gradient straight through the threshold
 *              (dm/dsigmoid = 1) and keeps the sigmoid's slope
 *   candidates every candidate's expert is evaluated, masked or not: candidate
 *              k's mask gets g_k <dy, E_k(x)> through the estimator either way
 *   weights    only kept candidates get expert-weight gradients (their
 *              weight in Eq. 7 is g_k; a masked candidate's is 0)
 * Arguments: the forward's inputs (same layouts, dtype of desc) and dy [T,d]
 * in that dtype; beta finite.  desc->n_shared must be 0.
 * Outputs, fp32, row-major like their weights:
 *   dx [T,d]                       overwritten
 *   dW_gate, dW_mask [E,d]         accumulated (+=); dW_mask NULL iff W_mask NULL
 *   dW1, dW3 [E,I,d], dW2 [E,d,I]  accumulated (+=) for experts with at least
 *                                  one kept pair; other experts' rows are not
 *                                  touched (zero them once per step)
 * Every sum runs in a fixed order: the gradients are bitwise repeatable.
 * Workspace: beam_moe_backward_workspace_size bytes, 256-byte aligned; the
 * caller owns it and every output.  Errors as for beam_moe_forward; also
 * BEAM_ERR_UNSUPPORTED_SHAPE for shared experts, and for fp32 layers with
 * d > 7168 or I > 4096 at 128-token tiles (8x larger at decode tile sizes),
 * beyond which a split of the CUDA-core kept-row products no longer fits in
 * shared memory.
 * Precision (bf16): both kept-row products (dh = dy W2_e and
 * dxp = da W1_e + db W3_e) run on the tensor cores with bf16 operands and fp32
 * accumulation; their da, db operands are da, db rounded once to bf16, while
 * dW1, dW3 use da, db in fp32. */
size_t beam_moe_backward_workspace_size(const beam_moe_desc *desc);
beam_status beam_moe_backward(const beam_moe_desc *desc, const void *x, const void *W_gate,
                              const void *W_mask, const void *W1, const void *W3, const void *W2,
                              const void *dy, float beta, float *dx, float *dW_gate,
                              float *dW_mask, float *dW1, float *dW3, float *dW2,
                              void *workspace, size_t workspace_bytes, void *stream);
/* Kernel launches of one beam_moe_backward call: 15 for bf16 (its dh = dy W2_e
 * product runs on the tensor cores, after a launch that lists each kept
 * expert's candidate rows), 14 for fp32; 0 for T = 0 or a bad descriptor. */
int beam_moe_backward_kernel_count(const beam_moe_desc *desc);

/* ------------------------------------------------- expert parallelism --
 * G ranks (one process per GPU), rank r owning experts [r E/G, (r+1) E/G).
 * The pages describe the exchange only in general terms (the MoE tutorial
 * page on "Beam", §4.2: tokens travel to the GPU that holds their expert by
 * an all-to-all) and BEAM's own contribution to it in the news article on
 * BEAM, §5: masked entries are left out of the expert-token grouping.  Here
 * only KEPT pairs are dispatched, so the mask cuts the rows that cross the
 * interconnect by the kept fraction.  A step, per rank:
 *   beam_moe_route (own tokens) -> beam_moe_ep_dispatch -> all-to-all of the
 *   send counts, rows and local expert ids -> beam_moe_expert_rows on the
 *   received rows -> all-to-all of the fp32 rows back -> beam_moe_ep_combine.
 * The exchanges are the caller's (NCCL through torch.distributed in the
 * Python binding); these calls never touch another GPU's memory. */

/* Dispatch of the kept pairs of one routed batch (desc, topk_idx and
 * expert_counts as written by beam_moe_route on `workspace`).  Pairs are
 * listed by expert (ascending) then token (ascending) -- the order of the
 * layer's own grouping -- so the rows bound for rank r are contiguous and
 * ranks appear in order.  Writes, with P = the number of kept pairs:
 *   send_rows   [P, d] (desc dtype)  the pairs' token rows, in that order
 *   send_pair   int32 [P]    t*K + k of each row
 *   send_expert int32 [P]    the row's expert id local to its destination
 *   send_counts int32 [n_ranks]  rows per destination rank
 *   pair_pos    int32 [T,K]  send row of each kept pair (masked: unwritten)
 * Capacity: send_rows/send_pair/send_expert hold T*K entries.  Needs
 * E % n_ranks == 0, 1 <= n_ranks <= E and n_shared == 0.  A consistency
 * failure sets the workspace error word (BEAM_ERR_INTERNAL through
 * beam_moe_check), which this call never clears: check once after the step. */
beam_status beam_moe_ep_dispatch(const beam_moe_desc *desc, int n_ranks, const void *x,
                                 const int32_t *topk_idx, const int32_t *expert_counts,
                                 void *send_rows, int32_t *send_pair, int32_t *send_expert,
                                 int32_t *send_counts, int32_t *pair_pos, void *workspace,
                                 size_t workspace_bytes, void *stream);

/* Expert outputs of pre-routed rows: y_rows[i] = E_{expert_id[i]}(x_rows[i])
 * (Eq. 3), fp32, computed by the layer's own grouping and expert GEMMs, so a
 * row's value is the per-pair output the one-GPU layer combines.  desc: T =
 * number of rows, E = the experts in W1/W3/W2, K = 1, n_shared = 0; the
 * router fields are unused.  expert_id int32 [T]: an id in [0, E) or -1 (the
 * row gets zeros); any other value sets BEAM_ERR_INTERNAL and is treated as
 * -1.  Workspace: beam_moe_workspace_size(desc) bytes; errors through
 * beam_moe_check on it. */
beam_status beam_moe_expert_rows(const beam_moe_desc *desc, const void *x_rows,
                                 const int32_t *expert_id, const void *W1, const void *W3,
                                 const void *W2, float *y_rows, void *workspace,
                                 size_t workspace_bytes, void *stream);

/* Eq. (8) at the source rank: out_t = sum over kept k, in slot order, of
 * topk_w[t,k] * y_rows[pair_pos[t,k]] (fp32 sums, one rounding to the desc
 * dtype); 0 for a token with no kept candidate.  y_rows: the returned fp32
 * rows in send order (non-NULL even when no pair is kept; nothing is then
 * read).  T = 0 does nothing. */
beam_status beam_moe_ep_combine(const beam_moe_desc *desc, const float *y_rows,
                                const int32_t *topk_idx, const float *topk_w,
                                const int32_t *pair_pos, void *out, void *stream);

/* Synchronise `stream`, then read the workspace error word written by the last
 * call: BEAM_OK, BEAM_ERR_TIMEOUT (a bounded device wait expired, the kernel
 * returned early; that call's outputs are not valid) or BEAM_ERR_INTERNAL (a
 * device consistency check failed).  Every call resets the word, so it
 * describes the last call made on the workspace.  After a timeout the
 * workspace and the context stay usable: the next call starts clean. */
beam_status beam_moe_check(const beam_moe_desc *desc, void *workspace, void *stream);

/* The descriptor's mask_logit_threshold for a threshold tau of Eq. (6):
 * ln(tau / (1 - tau)) evaluated in double and rounded once to float, so that
 * a candidate is kept iff sigmoid(z) >= tau <=> z >= the returned value.
 * tau = 0.5 gives 0 exactly; tau = 0 gives -inf, tau = 1 gives +inf; NaN for
 * tau outside [0, 1] (which beam_moe_plan rejects). */
float beam_moe_tau_to_logit(float tau);

/* Testing aid, off by default; the paper has no counterpart.  It lets a test
 * observe the bounded-wait path without faulting or hanging the GPU:
 *   mode 0  off;
 *   mode 1  in every later forward call, CTA 0 of the expert GEMM launch (the
 *           fused expert kernel at decode tile sizes, the gate/up GEMM
 *           otherwise; bf16 only) skips the first shared-memory stage of its
 *           first unit: it issues neither the copy nor the transaction count,
 *           so the MMA issuer's bounded wait on that stage expires;
 *   mode 2  the same in CTA 0 of the router GEMM of every later route or
 *           forward call (bf16 only);
 *   mode 3  the same in CTA 0 of the shared experts' gate/up GEMM of every
 *           later forward call with shared experts (bf16 only).
 * The kernels then record the timeout, let their own copies and MMAs land,
 * free their tensor memory and return: beam_moe_check reports
 * BEAM_ERR_TIMEOUT and the context stays usable.  wait_limit_ns replaces the
 * 1 s limit of every bounded device wait (0 restores it).  Process-wide; set
 * it while no other thread is calling the library.  BEAM_ERR_INVALID_ARG for
 * an unknown mode. */
beam_status beam_moe_set_fault_injection(int mode, unsigned long long wait_limit_ns);

/* Static, NUL-terminated name of a status code. */
const char *beam_status_str(beam_status status);

/* Name of forward stage i (0 <= i < BEAM_MOE_FORWARD_STAGES), else NULL. */
const char *beam_moe_stage_name(int stage);

#ifdef __cplusplus
}
#endif
#endif
