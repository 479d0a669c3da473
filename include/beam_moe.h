/*
 * beam_moe.h -- C ABI of the Beam sparse mixture-of-experts block (forward
 * pass) on NVIDIA B200 (sm_100a).
 *
 * The block, as the Beam pages define it:
 *   - router: sigmoid scores over all experts, computed in FP32 from FP32
 *     router weights; a learned per-expert bias is added for selection; the
 *     experts form n_group groups, a group's score is the sum of its two best
 *     biased scores, the topk_group best groups are kept and the top_k best
 *     experts inside them are chosen (launch blog "Introducing Beam", section
 *     "Mixture of Experts"; transformers page "Beam", section "Overview",
 *     "Sparse MoE" bullet and the paragraph on FP32 router weights and bias);
 *   - each chosen expert is a SwiGLU MLP, down(silu(gate x) * up x), with the
 *     SwiGLU product in FP32 (launch blog, sections "Mixture of Experts" and
 *     "Residual Stream");
 *   - the expert outputs are combined with the normalised router weights and
 *     scaled by routed_scaling (2.5 for Beam);
 *   - optionally, the post-sub-layer RMSNorm ("sandwich" norm) and the
 *     depth-scaled residual update of step k:
 *         stream <- sqrt((k-1)/k) * stream + norm(out) / sqrt(k)
 *     (launch blog, section "Residual Stream"; transformers page, "Overview",
 *     depth-scaled residual bullet).
 * Conventions the pages leave open, fixed here: the bias steers selection
 * only; a group's score uses the biased scores; the combine weights are the
 * unbiased sigmoid scores of the chosen experts divided by their sum; ties go
 * to the lower group / expert index.
 *
 * Memory.  Every tensor argument is a DEVICE pointer unless its name ends in
 * _host.  The caller owns all of them.  Weights are borrowed by the handle and
 * must stay valid and unchanged until beam_moe_destroy.  The handle owns only
 * its workspace (sized by max_tokens at create time) and its TMA descriptors
 * (an NVFP4 handle also owns its tiled copy of the expert weights, whose
 * inputs are read at create only).
 * Device pointers must be 16-byte aligned.  Layouts are row-major, C order.
 *
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL: the legacy
 * default stream).  Calls are stream-ordered and asynchronous unless stated:
 * the host does not wait.  A handle's workspace is shared by its calls, so a
 * handle must not be used on two streams concurrently.
 *
 * Errors.  Every call validates its arguments on the host first and returns a
 * negative beam_status without launching anything when they are invalid.
 * Device-side failures (a bounded wait inside a kernel that ran out) set a
 * sticky status word in the handle; beam_moe_get_status reads and clears it.
 * beam_moe_last_error returns a text for the last host-side error.
 */
#ifndef BEAM_MOE_H
#define BEAM_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct beam_moe *beam_moe_t;

typedef enum {
    BEAM_OK = 0,
    BEAM_ERR_INVALID_ARG = -1, /* bad shape, pointer, size or alignment       */
    BEAM_ERR_UNSUPPORTED = -2, /* valid for the method, not for these kernels */
    BEAM_ERR_CUDA = -3,        /* a CUDA runtime / driver call failed          */
    BEAM_ERR_OOM = -4,         /* workspace allocation failed                  */
    BEAM_ERR_TIMEOUT = -5,     /* a bounded device-side wait ran out           */
    BEAM_ERR_CHECK = -6,       /* a checked-mode validation failed             */
    BEAM_ERR_RANGE = -7        /* an NVFP4 forward met an activation above
                                  65504 x 256 in magnitude (its f16 operands)  */
} beam_status;

/*
 * Create a handle for one MoE block: the router (sigmoid scores, per-expert
 * bias, n_group groups scored by their two best biased scores, topk_group
 * groups kept, top_k experts chosen) and E SwiGLU experts, as the launch blog
 * "Introducing Beam", section "Mixture of Experts", and the transformers
 * page "Beam", section "Overview", "Sparse MoE" bullet, define them; the
 * optional post-norm as in the blog's section "Residual Stream".
 *
 * hidden        H, hidden size (Beam: 5120).  Must be a multiple of 128.
 * n_experts     E (Beam: 256).  Must be a multiple of 32 and at most 1024.
 * inter         I, expert intermediate size (Beam: 2560).  Multiple of 128.
 * n_group       number of expert groups (Beam: 8); E % n_group == 0, the
 *               group size E/n_group must be >= 2.
 * topk_group    groups kept per token (Beam: 4); 1 <= topk_group <= n_group.
 * top_k         experts chosen per token (Beam: 8);
 *               1 <= top_k <= min(32, topk_group * E / n_group).
 * routed_scaling  scale applied to the combined output (Beam: 2.5).
 * router_w      fp32 [E, H]: logit_e = x . router_w[e].
 * expert_bias   fp32 [E]: added to the sigmoid scores for selection only.
 * w_gate        bf16 [E, I, H]: gate projection of every expert.
 * w_up          bf16 [E, I, H]: up projection.
 * w_down        bf16 [E, H, I]: down projection.
 * post_norm_w   fp32 [H] RMSNorm weight applied to the block output before
 *               the residual update, or NULL for no norm.
 * norm_eps      RMSNorm epsilon (Beam: 1e-6); ignored without post_norm_w.
 * max_tokens    largest T any call on this handle will pass (>= 1); sizes
 *               the workspace (about T*top_k*(4H + 2I) + T*(4H) bytes).
 * Kernel-side shape limits (else BEAM_ERR_UNSUPPORTED): E/32 experts per
 * lane in {1, 2, 4, 8, 16, 32}, group size a multiple of E/32 with
 * (group size)/(E/32) a power of two, n_group <= 32.
 * On success *out receives the handle.  Allocates device memory and launches
 * one kernel on the legacy default stream (splitting router_w into the bf16
 * pieces the tensor-core router uses), waiting for it: the handle's one
 * derived weight is then complete before create returns, so the first call
 * may come on any stream, or inside a stream capture, with no ordering
 * against create.  The current CUDA device at create time is the handle's
 * device.
 */
int beam_moe_create(beam_moe_t *out, int hidden, int n_experts, int inter, int n_group,
                    int topk_group, int top_k, float routed_scaling, const float *router_w,
                    const float *expert_bias, const void *w_gate, const void *w_up,
                    const void *w_down, const float *post_norm_w, float norm_eps,
                    int max_tokens);

/*
 * Create a handle for one dense SwiGLU MLP layer (Beam's first three layers;
 * launch blog "Introducing Beam", section "Mixture of Experts"):
 *   out = W_down . bf16(silu(W_gate . x) * (W_up . x))   (SwiGLU product in FP32)
 * with the same optional post-norm and depth-scaled residual update as the
 * sparse block, and no routing or routed scaling.
 *
 * hidden        H (Beam: 5120).  Multiple of 128, at most 8192.
 * inter         intermediate size of the layer.  Multiple of 128.
 * w_gate, w_up  bf16 [inter, H];  w_down  bf16 [H, inter].
 * post_norm_w, norm_eps, max_tokens: as beam_moe_create.
 * The handle takes beam_moe_forward, beam_moe_forward_host,
 * beam_moe_launch_plan, beam_moe_set_gemm_tuning (tile_rows, ctas,
 * cta_pairs and down_pair apply), the status, wait-limit and profiling
 * calls, and beam_moe_destroy; the routing calls return
 * BEAM_ERR_UNSUPPORTED.  With token tiles of up to 64 rows (decode-sized
 * batches) both GEMMs run stream-K: each SM takes an equal share of the
 * (weight tile, K step) units, and a tile split between SMs is finished by
 * the last of them, which adds the FP32 pieces in K order.
 * Allocates device memory; launches nothing.
 */
int beam_moe_create_dense(beam_moe_t *out, int hidden, int inter, const void *w_gate,
                          const void *w_up, const void *w_down, const float *post_norm_w,
                          float norm_eps, int max_tokens);

/*
 * Create a handle for one MoE block whose expert weights are NVFP4, the
 * 4-bit format the Beam launch blog recommends for Blackwell GPUs (launch
 * blog "Introducing Beam", section "Mixture of Experts"): each weight is an
 * E2M1 element times the FP8 E4M3 scale of its block of 16 consecutive
 * elements along the row, times one FP32 scale per tensor.
 *
 * Arguments as beam_moe_create, with each expert tensor given as
 *   *_codes   uint8 [E, R, K/2]: element 2j of a row in the low nibble of
 *             byte j, 2j + 1 in the high nibble (a nibble: sign bit 3,
 *             exponent bits 2..1 with bias 1, mantissa bit 0);
 *   *_scales  uint8 [E, R, K/16]: E4M3 scale of elements 16b .. 16b + 15;
 *   *_global  the tensor's FP32 scale (finite);
 * with R = inter, K = hidden for gate and up, R = hidden, K = inter for
 * down.  Device pointers, 16-byte aligned, read during this call only: the
 * handle allocates and keeps its own tiled copy (0.5625 bytes per weight)
 * made by kernels on the legacy default stream, which this call waits for.
 * The grouped GEMMs decode the weights to f16 (exact: an E2M1 x E4M3
 * product has at most 6 significant bits and lies between 2^-10 and 2688 in
 * magnitude) for the tensor cores, take the bf16 activations as f16 times
 * 2^-8 (exact for magnitudes from 2^-9 up to 65504 x 2^8, within 2^-17
 * below that) and apply the per-tensor scales and 2^8 to the FP32
 * accumulators.  An activation above 65504 x 2^8 in magnitude records
 * BEAM_ERR_RANGE in the status word (beam_moe_get_status).
 * The handle takes the same calls as a bf16 handle.  Differences: token
 * tiles of at most 128 rows (tile_rows 256 acts as 128); the cta_pairs,
 * gather_rows, token_stages and down_pair tunings are ignored (single-CTA
 * kernels over the sorted activations).  Errors as beam_moe_create, and
 * BEAM_ERR_OOM if the tiled copy cannot be allocated.
 */
int beam_moe_create_nvfp4(beam_moe_t *out, int hidden, int n_experts, int inter, int n_group,
                          int topk_group, int top_k, float routed_scaling, const float *router_w,
                          const float *expert_bias, const uint8_t *gate_codes,
                          const uint8_t *gate_scales, float gate_global, const uint8_t *up_codes,
                          const uint8_t *up_scales, float up_global, const uint8_t *down_codes,
                          const uint8_t *down_scales, float down_global, const float *post_norm_w,
                          float norm_eps, int max_tokens);

/*
 * Decode rows x K NVFP4 elements (codes uint8 [rows, K/2], scales uint8
 * [rows, K/16], laid out as for beam_moe_create_nvfp4) to bf16 [rows, K]:
 * each element times its block scale, exact; no per-tensor scale.  The
 * same products the NVFP4 grouped GEMMs give the tensor cores (as f16 there;
 * both formats hold them exactly).  Device pointers; codes and out
 * 16-byte aligned.  K a positive multiple of 16, rows >= 0 (0: nothing to
 * do).  Needs no handle.  Asynchronous on `stream`.  Returns
 * BEAM_ERR_INVALID_ARG for bad arguments, BEAM_ERR_CUDA if the launch fails.
 */
int beam_nvfp4_dequant(void *stream, const uint8_t *codes, const uint8_t *scales, long long rows,
                       int K, void *out);

/*
 * Route T tokens: the router step alone (launch blog "Introducing Beam",
 * section "Mixture of Experts": sigmoid scores plus the expert bias, groups
 * scored by the sum of their two best scores, the best groups kept, the top
 * experts chosen inside them, their weights normalised; transformers page
 * "Beam", "Sparse MoE" bullet and the FP32 router paragraph).
 * x         bf16 [T, H].
 * topk_idx  int32 [T, top_k] (out): chosen experts, in descending biased
 *           score, ties to the lower index.
 * topk_w    fp32 [T, top_k] (out): the chosen experts' unbiased sigmoid
 *           scores divided by their sum (sum to 1; routed_scaling not
 *           applied).
 * 0 <= T <= max_tokens; T == 0 returns BEAM_OK and launches nothing.
 */
int beam_moe_route(beam_moe_t h, void *stream, const void *x, int T, int32_t *topk_idx,
                   float *topk_w);

/*
 * Routing without any device allocation (the Beam pages have no counterpart:
 * this entry point exists for callers, not for the method).  Callers that
 * cannot call cudaMalloc -- an inference engine that reserves nearly all GPU
 * memory for its own pools at start-up, or a latency-critical path that must
 * not enter the CUDA allocator, whose cudaMalloc / cudaFree can synchronise
 * the device -- and so cannot create a handle, get the same routing as
 * beam_moe_route here, with no handle.
 * Scratch: a fixed 8 MiB device array inside the library (2,097,152 fp32
 * partial logits), held by every GPU that loads the library until the
 * process exits.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  All calls on a device share the array, so
 * calls that overlap on the GPU (different streams, no ordering between them)
 * race and give undefined results; calls ordered on one stream are safe.
 * Nothing in the array needs clearing: each call writes every element it
 * reads.  No cudaMalloc, cudaFree or allocating library call is made.
 * The array's device address is looked up once per device and kept for the
 * life of the process, so this entry point does not support cudaDeviceReset:
 * after a reset the kept address belongs to the destroyed context.
 * Arguments as beam_moe_create / beam_moe_route: x bf16 [T, H], router_w fp32
 * [E, H], expert_bias fp32 [E] (16-byte aligned device pointers), topk_idx
 * int32 [T, top_k] and topk_w fp32 [T, top_k] (device, out).  hidden must be
 * a multiple of 32; n_experts, n_group, topk_group, top_k follow the rules of
 * beam_moe_create.  Returns BEAM_ERR_INVALID_ARG for bad arguments and when
 * T * n_experts > 2,097,152 (the scratch capacity), BEAM_ERR_UNSUPPORTED for
 * shapes the kernels do not cover, BEAM_ERR_CUDA if the set-up or the launch
 * fails.  T == 0 returns BEAM_OK.  Asynchronous on `stream`.
 */
int beam_moe_route_static(void *stream, const void *x, int T, int hidden, int n_experts,
                          int n_group, int topk_group, int top_k, const float *router_w,
                          const float *expert_bias, int32_t *topk_idx, float *topk_w);

/*
 * Router logits for T tokens, x . router_w^T in FP32 (the quantity the
 * transformers page returns with output_router_logits=True).
 * logits    fp32 [T, E] (out).
 */
int beam_moe_router_logits(beam_moe_t h, void *stream, const void *x, int T, float *logits);

/*
 * Routing of T tokens from given FP32 logits [T, E] (device, 16-byte
 * aligned; e.g. from beam_moe_router_logits), with `expert_bias` (fp32 [E],
 * device, 16-byte aligned) in place of the handle's bias, or the handle's
 * bias when NULL.  The expert bias steers selection only (launch blog
 * "Introducing Beam", section "Mixture of Experts"; transformers page
 * "Beam", "Sparse MoE" bullet), so the effect of a new bias on the routing
 * and the expert loads needs no new logits.  Outputs as beam_moe_route.
 * Reads nothing of x or the router matrix; T <= max_tokens; T == 0 returns
 * BEAM_OK.  Asynchronous on `stream`.
 */
int beam_moe_route_logits(beam_moe_t h, void *stream, const float *logits, int T,
                          const float *expert_bias, int32_t *topk_idx, float *topk_w);

/*
 * Forward pass of the block for T tokens: routing, the chosen experts'
 * SwiGLU MLPs and their weighted sum scaled by routed_scaling (launch blog
 * "Introducing Beam", section "Mixture of Experts"), and optionally the
 * post-norm and the depth-scaled residual update (same blog, section
 * "Residual Stream"; transformers page "Beam", "Overview").
 * x         bf16 [T, H].
 * out       bf16 [T, H] (out): routed_scaling * sum_j w_j * expert_j(x),
 *           rounded to nearest even; may be NULL when residual is given.
 * residual  fp32 [T, H] (in/out) or NULL.  When given, the block output o
 *           (fp32, before rounding) is normalised with post_norm_w if the
 *           handle has one, n = o / sqrt(mean(o^2) + eps) * post_norm_w,
 *           else n = o; then residual <- sqrt((k-1)/k) * residual + n/sqrt(k).
 * k         residual step (>= 1); ignored without residual.
 * out and residual must not both be NULL.  0 <= T <= max_tokens.
 */
int beam_moe_forward(beam_moe_t h, void *stream, const void *x, int T, void *out,
                     float *residual, int k);

/*
 * beam_moe_forward with HOST buffers: copies x_host (and residual_host) to
 * one of the handle's two device staging slots, runs the forward pass on
 * `stream` and copies the results back, then waits until they landed.
 * x_host bf16 [T, H]; out_host bf16 [T, H] or NULL; residual_host fp32
 * [T, H] (in/out) or NULL.  Pinned host memory gives asynchronous copies;
 * pageable memory works too.  Synchronous.
 */
int beam_moe_forward_host(beam_moe_t h, void *stream, const void *x_host, int T,
                          void *out_host, float *residual_host, int k);

/*
 * The same pass without waiting: a pipeline for a stream of host batches.
 * The copy to the device runs on the handle's copy-in stream, the pass on
 * `stream`, the copy back on its copy-out stream, ordered by events.  Calls
 * alternate between two staging slots, so the copy-in of one call overlaps
 * the compute of the previous call and the copy-out overlaps the next.  The
 * host buffers must stay untouched until the results landed; call
 * beam_moe_host_join (then synchronise `stream`) before reading out_host /
 * residual_host.  Passes run in call order on `stream`; use one stream per
 * handle.
 */
int beam_moe_forward_host_async(beam_moe_t h, void *stream, const void *x_host, int T,
                                void *out_host, float *residual_host, int k);

/*
 * Make `stream` wait (without blocking the host) until every copy back of
 * earlier beam_moe_forward_host_async calls has landed in host memory.
 */
int beam_moe_host_join(beam_moe_t h, void *stream);

/*
 * Make the copies of later beam_moe_forward_host_async calls start only
 * after the work enqueued on `stream` so far (for instance a timing event).
 */
int beam_moe_host_fence(beam_moe_t h, void *stream);

/*
 * Dispatch bookkeeping of the last forward pass on this handle (for checks):
 * copies to HOST buffers, after synchronising `stream`.
 * counts_host   int32 [E]: tokens routed to each expert.
 * offsets_host  int32 [E+1]: exclusive prefix sum of counts.
 * pair_row_host int32 [T*top_k]: row of (token t, slot j) = pair t*top_k+j in
 *               the expert-sorted activation buffer; rows of one expert are
 *               contiguous and ordered by pair index.
 * T must equal the T of that forward pass.  Any pointer may be NULL.
 */
int beam_moe_dispatch_info(beam_moe_t h, void *stream, int T, int32_t *counts_host,
                           int32_t *offsets_host, int32_t *pair_row_host);

/*
 * Routing statistics of the last route / forward call on this handle:
 * *rederived_host (host) receives how many tokens had their decision
 * re-derived from FP32 CUDA-core logits because their margin on the
 * tensor-core logits was too thin (0 when the CUDA-core path ran).
 * Synchronises `stream`.
 */
int beam_moe_router_stats(beam_moe_t h, void *stream, int32_t *rederived_host);

/*
 * The launch configuration a forward pass of T tokens (0 <= T <= max_tokens)
 * uses under the handle's current tuning, written to plan_host (int32 [11],
 * host): {largest token tile of the grouped GEMMs (rows), 1 if
 * they run on CTA pairs (cta_group::2), CTAs per grouped GEMM, 1 if the down
 * projection takes two weight blocks per work item, 1 if the router logits
 * run on the tensor cores (with exact re-derivation of thin-margin tokens),
 * K slices of the router logits (0 for a dense layer), 1 if the gate|up GEMM
 * gathers token rows from x, 1 if the gate|up GEMM and 1 if the down GEMM
 * run stream-K (dense layers at decode-sized token tiles: every SM takes an
 * equal share of the weight tiles' K steps, and the last CTA to finish a
 * tile's share adds the pieces in K order), 1 if the down GEMM stores the expert
 * outputs in FP32 (else bf16), 1 if the gate|up GEMM runs on interleaved
 * gate and up tiles (see beam_moe_set_gate_up_layout)}.  A function of T and
 * the tuning only; launches nothing.
 * Returns BEAM_ERR_INVALID_ARG for a NULL pointer or T out of range.
 */
int beam_moe_launch_plan(beam_moe_t h, int T, int32_t *plan_host);

/*
 * Synchronise `stream`, then return and clear the device status word:
 * BEAM_OK, BEAM_ERR_TIMEOUT when a bounded in-kernel wait ran out, or
 * BEAM_ERR_CHECK when a checked-mode validation failed, since the last call.
 * While the word is set, kernels of this handle skip their work (or stop at
 * their next wait), so results of calls made meanwhile are not valid.
 */
int beam_moe_get_status(beam_moe_t h, void *stream);

/*
 * Checked mode (off by default), the stand-in for a memory checker.  With
 * on = 1 every forward pass of this handle also validates, on the device:
 * each token's experts (in [0, E), none twice, weights in (0, 1]); the
 * dispatch tables (offsets from 0 growing by the counts to T*top_k, token
 * tiles per expert = ceil(count / tile)); every pair's row inside its
 * expert's range, with the two row maps inverse.  A failure records
 * BEAM_ERR_CHECK in the status word (no trap); every later kernel of the
 * pass then skips its work, so none indexes memory with a bad expert or row.
 * beam_moe_get_status returns it, with the first failing index (a token for
 * the routing check, a pair, or T*top_k for the tables) in
 * beam_moe_last_error.  Costs two small kernels per forward pass.
 */
int beam_moe_set_checks(beam_moe_t h, int on);

/*
 * Test hook for checked mode: the next `passes` forward passes overwrite
 * slot 0 of token 0's routing with the expert index n_experts (out of range)
 * before the checks run.  BEAM_ERR_INVALID_ARG unless checked mode is on;
 * BEAM_ERR_UNSUPPORTED on a dense layer.
 */
int beam_moe_debug_corrupt_routing(beam_moe_t h, int passes);

/*
 * Set the limit of every in-kernel wait of this handle, in nanoseconds
 * (default 2e9).  Values < 1000 are rejected.
 */
int beam_moe_set_wait_limit(beam_moe_t h, int64_t limit_ns);

/*
 * Tuning of the grouped GEMMs; results do not depend on any of it.
 * ctas            CTAs of the persistent kernels, 0 = one per SM (default);
 *                 fewer CTAs put more work items on each.  0..65535.
 * tile_rows       largest token tile: 16, 32, 64, 128 or 256 rows, or 0 to
 *                 choose from the mean number of tokens per expert (default).
 * down_pair       -1: choose (default); 0: the down projection takes one
 *                 weight block per work item; 1: two consecutive blocks that
 *                 share the token tile (needs hidden to be a multiple of two
 *                 blocks, else ignored).
 * cta_pairs       1 (default): token tiles of 64 rows or more run on pairs of
 *                 SMs that share each MMA (needs inter and hidden to be
 *                 multiples of 256); 0: one CTA per SM always.
 * router_mode     -1 (default): FP32 CUDA-core logits below 512 tokens,
 *                 tensor-core logits from 512 on; 0: always CUDA cores;
 *                 1: always tensor cores; 2: tensor cores with every token's
 *                 routing re-derived on the CUDA-core path (a check of that
 *                 path).  The tensor-core logits use the router weight split
 *                 into three bf16 pieces (every product with a bf16 token
 *                 value is exact in FP32, the sum is accumulated in FP32 by
 *                 the tensor cores); a token whose decision margin -- the
 *                 smallest gap between neighbours in the ranking of its top
 *                 k+1 candidates (it fixes the chosen set and their order),
 *                 or weakest kept vs strongest dropped group score -- is
 *                 below 4e-5 has its logits recomputed with FP32 CUDA-core
 *                 dot products and is selected again, so decisions keep
 *                 CUDA-core accuracy.  beam_moe_router_logits always uses
 *                 the CUDA-core path.
 * gather_rows     1: the gate|up GEMM loads its token rows straight from x,
 *                 four rows per TMA gather4 copy, so dispatch makes no
 *                 expert-sorted copy of x; 0: dispatch copies x into the
 *                 sorted buffer and the GEMM loads boxes of it; -1
 *                 (default): gather when token tiles are at most 32 rows
 *                 (the gathers of a large tile outlast its MMAs).
 * token_stages    CTA-pair kernels: depth of the token-row ring, 2..8, or 0
 *                 for the default (3); the weight ring takes the rest of
 *                 shared memory.
 */
int beam_moe_set_gemm_tuning(beam_moe_t h, int ctas, int tile_rows, int down_pair,
                             int cta_pairs, int router_mode, int gather_rows, int token_stages);

/*
 * Layout of the gate|up GEMM's weight tiles on CTA pairs (results do not
 * depend on it; a layout choice, not a change of the method):
 *   0   separate tiles: each CTA holds 128 gate rows and the same 128 up
 *       rows, in two accumulators of N columns each;
 *   1   interleaved tiles: each CTA's 128-row tile holds 64 gate rows and
 *       the same 64 up rows in 16-row groups, one accumulator of N columns,
 *       so two accumulators fit tensor memory even at 256-token tiles and
 *       one work item's epilogue overlaps the next item's MMAs; needs inter
 *       a multiple of 128;
 *  -1   (default) separate: the interleaved tiles load each token tile for
 *       half as many weight rows, and at the Beam prefill shape that extra
 *       token traffic outweighs the overlap (measured 37% slower).
 * Ignored where the gate|up GEMM does not run on CTA pairs.  Returns
 * BEAM_ERR_INVALID_ARG for a layout outside [-1, 1].
 */
int beam_moe_set_gate_up_layout(beam_moe_t h, int layout);

/*
 * Per-stage timing of forward passes, for measurement.  After
 * beam_moe_profile_begin(h, max_calls), each of the next max_calls forward
 * passes records CUDA events on its stream around its five stages: router,
 * dispatch, gate|up GEMM, down GEMM, combine.  beam_moe_profile_end waits for
 * the last recorded event, writes the summed milliseconds of each stage to
 * stage_ms (fp32 [5], host) and the number of timed passes to *calls (host),
 * and stops recording.  Synchronous; allocates no device memory.
 */
int beam_moe_profile_begin(beam_moe_t h, int max_calls);
int beam_moe_profile_end(beam_moe_t h, float *stage_ms, int *calls);

/*
 * Failure-detection check of the two kinds of in-kernel wait, each with the
 * handle's wait limit: one kernel waits on a shared-memory barrier that
 * nothing completes, a second polls a global counter that nothing
 * increments (the wait of the dense stream-K GEMMs).  Each must give up,
 * record BEAM_ERR_TIMEOUT in the status word and return; the status word is
 * read and cleared after each.  Returns BEAM_ERR_TIMEOUT if both did, else
 * the first other status.  Synchronous.
 */
int beam_moe_check_wait_timeout(beam_moe_t h, void *stream);

/* Text of the last host-side error on this handle ("" if none). */
const char *beam_moe_last_error(beam_moe_t h);

/* Text of the last error of a beam_moe_create / beam_moe_create_dense call
 * that returned no handle, on the calling thread. */
const char *beam_moe_create_error(void);

/* Free the workspace and the handle.  Synchronises the handle's device. */
int beam_moe_destroy(beam_moe_t h);

#ifdef __cplusplus
}
#endif

#endif /* BEAM_MOE_H */
