/*
 * moe.h -- C ABI of the B200 (sm_100a) routed Mixture-of-Experts FFN forward.
 *
 * The layer, for a batch of T tokens x_t (hidden size H):
 *   logits   optionally the router projection logits_t = W_r x_t, else given;
 *   route    softmax over the E router logits of each token, the k largest
 *            logits kept, their probabilities renormalised to sum 1 when
 *            norm_topk is set;
 *   top-p    optional per-token trim: each token keeps the shortest prefix
 *            of its k slots whose weights reach topp (renormalised);
 *   budget   optional cap N on the number of distinct experts the whole
 *            batch uses: when the batch union holds more than N experts,
 *            only the N with the highest aggregate gate weight survive and
 *            each token's remaining weights are renormalised;
 *   dispatch the kept (token, slot) pairs grouped by expert;
 *   FFN      per expert e: y = W_down[e] (silu(W_gate[e] x) * (W_up[e] x));
 *   combine  out_t = sum_j w_tj y_tj + sigmoid(g . x_t) FFN_shared(x_t).
 *
 * Passages that define the operation (web pages, by title and section):
 *   SpecForge PR #943, "Qwen3.8-27B DSpark MoE drafter with 16 x 1024 top-2
 *     experts", section "Modifications": the config keys hidden,
 *     n_routed_experts, moe_intermediate_size, num_experts_per_tok, the
 *     2048-wide sigmoid-gated shared expert, the softmax router with
 *     renormalised top-k ("qwen3_5_moe preset") and grouped_mm dispatch;
 *     its FFN parameter table (3*H*I parameters per expert).
 *   colibri issue_budget.md, "EXPERT_BUDGET", section "How it works", steps
 *     1-5 (the budget) and section "Safety" (off by default, dropped experts
 *     omitted and the rest renormalised); section "Relationship to existing
 *     features" (TOPP trims each position's top-K to its top-p mass, and
 *     composes with the budget, TOPP first).
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, row-major and densely packed.  bf16 values are passed as
 *     their 16-bit patterns (moe_bf16_t).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  All
 *     work is enqueued on it; no entry point synchronises, allocates device
 *     or host memory, or keeps state between calls, so calls on different
 *     streams with different buffers may run concurrently.
 *   - T = 0 is a no-op returning MOE_OK.
 *   - Return codes: MOE_OK, or a negative MOE_ERR_* below; nothing is
 *     launched when an argument check fails.
 *   - Limits: 1 <= E <= 1024; 1 <= k <= min(E, 32); H % 128 == 0;
 *     I % 64 == 0; Is % 64 == 0 (Is = 0: no shared expert); budget >= 0;
 *     topp finite and >= 0; 0 <= T and T * (k + 1) * H < 2^31.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t; /* bf16 bit pattern */

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)   /* null/misaligned pointer, bad size or flag */
#define MOE_ERR_UNSUPPORTED (-2)   /* shape outside the limits above, or no sm_100 device */
#define MOE_ERR_WORKSPACE (-3)     /* ws_bytes < moe_workspace_bytes(cfg, T) */
#define MOE_ERR_CUDA (-4)          /* a CUDA launch or driver call failed */
#define MOE_ERR_DEVICE (-5)        /* a kernel reported an error in the status word */

/* Bits of the device status word (see moe_status_read). */
#define MOE_STATUS_TIMEOUT 1       /* a pipeline wait ran past its limit; results invalid */
#define MOE_STATUS_BOUNDS 2        /* checked library only (libmoe_checked.so, built with
                                      MOE_DEBUG_BOUNDS): an input index was out of range --
                                      an expert id outside [-1, E) in a kept slot, dispatch
                                      offsets not a prefix sum within T*k, a perm entry outside
                                      [0, T*k); the access was skipped, results invalid */
#define MOE_STATUS_NONFINITE 4     /* checked library only: moe_forward's router logits (given
                                      or projected) held a NaN or an infinity, outside the
                                      contract (a softmax over them is undefined); results
                                      invalid.  moe_route alone has no status word to report it */

typedef struct {
    int32_t hidden;                   /* H */
    int32_t n_routed_experts;         /* E */
    int32_t moe_intermediate_size;    /* I */
    int32_t num_experts_per_tok;      /* k */
    int32_t shared_intermediate_size; /* Is; 0 = no shared expert */
    int32_t norm_topk;                /* 1: renormalise the kept weights to sum 1 */
    int32_t budget;                   /* N (EXPERT_BUDGET); 0 = off */
    float topp;                       /* per-token top-p mass (TOPP); 0 (or >= 1) = off */
} moe_config_t;

typedef struct {
    const moe_bf16_t *w_gate;      /* [E, I, H] routed gate projections */
    const moe_bf16_t *w_up;        /* [E, I, H] routed up projections */
    const moe_bf16_t *w_down;      /* [E, H, I] routed down projections */
    const moe_bf16_t *ws_gate;     /* [Is, H] shared gate projection, NULL if Is = 0 */
    const moe_bf16_t *ws_up;       /* [Is, H] shared up projection, NULL if Is = 0 */
    const moe_bf16_t *ws_down;     /* [H, Is] shared down projection, NULL if Is = 0 */
    const moe_bf16_t *ws_gate_vec; /* [H] shared-expert gate vector g, NULL if Is = 0 */
    const moe_bf16_t *w_router;    /* [E, H] router projection; read by moe_forward only when its logits are NULL */
} moe_weights_t;

/* Optional device outputs of moe_forward; any NULL member is kept inside
 * the workspace instead. */
typedef struct {
    int32_t *topk_idx;     /* [T, k] */
    float *topk_w;         /* [T, k] */
    float *sgate;          /* [T]    (Is > 0 only) */
    int32_t *keff;         /* [T]    */
    uint8_t *expert_kept;  /* [E]    (written only when budget > 0) */
    int32_t *n_dropped;    /* [1]    (written only when budget > 0) */
    int32_t *counts;       /* [E]    */
    int32_t *offsets;      /* [E+1]  */
    int32_t *perm;         /* [T*k]  first offsets[E] entries valid */
    int32_t *slot_pos;     /* [T*k]  */
    float *logits;         /* [T, E] the router projection's logits (when moe_forward computed them) */
} moe_aux_t;

/* Bytes of device workspace the calls below need for a batch of T tokens
 * (0 for an invalid config).  The workspace is caller-allocated scratch;
 * its first 8 KB hold the status word and the expert FFN's scheduling
 * counters.  Zero that block once after allocating (moe_status_clear);
 * every kernel leaves the counters at zero, and moe_dispatch re-zeroes them.
 * One workspace serves one stream at a time. */
size_t moe_workspace_bytes(const moe_config_t *cfg, int32_t T);

/* Router projection: logits[t, e] = sum_h x[t, h] * w_router[e, h], bf16
 * operands on the tensor cores with fp32 accumulation, fp32 out (SpecForge
 * PR #943, "Modifications": the softmax router's logits; a bias-free linear
 * map).  Small batches split the H sum over CTAs and add the fp32 partials in
 * a fixed order, so the result is the same bits on every run.
 *   x [T, H]; w_router [E, H]; logits [T, E] f32.  Uses the workspace (its
 *   head must be zeroed once, as for every call below). */
int moe_router_logits(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *w_router,
                      float *logits, void *ws, size_t ws_bytes, void *stream);

/* Route: for each token t, topk_idx[t, 0..k) = the k experts with the
 * largest logits (descending; equal logits: lower expert id first),
 * topk_w[t, j] = softmax(logits[t])[topk_idx[t, j]], divided by the sum of
 * the k kept probabilities when cfg->norm_topk.  With 0 < cfg->topp < 1 the
 * top-p trim follows: slot 0 stays, slot j > 0 stays while the weights of
 * slots 0..j-1 (added in slot order, fp32) are below topp; the rest become
 * (idx -1, w 0), and with norm_topk the kept weights are divided by their
 * sum (slot order).  When sgate != NULL (needs Is > 0, x and ws_gate_vec),
 * sgate[t] = sigmoid(ws_gate_vec . x_t).  keff[t] = the kept slots (k
 * without the trim); keff may be NULL only when the trim is off.
 *   logits [T, E] f32; x [T, H]; ws_gate_vec [H]; topk_idx [T, k] i32;
 *   topk_w [T, k] f32; sgate [T] f32; keff [T] i32. */
int moe_route(const moe_config_t *cfg, int32_t T, const float *logits, const moe_bf16_t *x,
              const moe_bf16_t *ws_gate_vec, int32_t *topk_idx, float *topk_w, float *sgate,
              int32_t *keff, void *stream);

/* Budget (EXPERT_BUDGET, colibri issue_budget.md "How it works"): works in
 * place on the router output topk_idx/topk_w [T, k]; slots with idx -1 (a
 * top-p trim's tail) take no part.  Let U be the set of experts any token
 * routes to.  When cfg->budget > 0 and |U| > budget: agg[e] = sum of the
 * weights routed to e (tokens, then slots, ascending); the budget experts
 * first in (agg descending, id ascending) are kept; every token's kept slots
 * move to the front in their original order, the tail becomes (idx -1, w 0),
 * keff[t] = kept slots, and a token that lost a slot has its kept weights
 * divided by their sum when cfg->norm_topk.  Otherwise topk_idx/topk_w are
 * unchanged and keff[t] = the token's valid slots (k without a trim).
 * expert_kept[e] = 1 for experts of the final union; *n_dropped = |U| -
 * budget or 0.  keff [T] i32; expert_kept [E] u8; n_dropped [1] i32 (all
 * device).  Uses the workspace. */
int moe_budget(const moe_config_t *cfg, int32_t T, int32_t *topk_idx, float *topk_w, int32_t *keff,
               uint8_t *expert_kept, int32_t *n_dropped, void *ws, size_t ws_bytes, void *stream);

/* Dispatch: groups the kept slots s = t*k + j (j < keff[t]; keff == NULL
 * means every slot) by expert, bit-exactly:
 *   counts[e] = kept slots routed to e; offsets[0] = 0,
 *   offsets[e+1] = offsets[e] + counts[e];
 *   perm[offsets[e] ..] = those slot ids in ascending order;
 *   slot_pos[s] = position of slot s in perm, -1 for a dropped slot;
 *   x_perm[p, :] = x[perm[p] / k, :] when x_perm != NULL.
 * topk_idx [T, k]; keff [T]; x [T, H]; counts [E]; offsets [E+1];
 * perm [T*k]; slot_pos [T*k]; x_perm [T*k, H].  Uses the workspace. */
int moe_dispatch(const moe_config_t *cfg, int32_t T, const int32_t *topk_idx, const int32_t *keff,
                 const moe_bf16_t *x, int32_t *counts, int32_t *offsets, int32_t *perm,
                 int32_t *slot_pos, moe_bf16_t *x_perm, void *ws, size_t ws_bytes, void *stream);

/* Expert FFN over the dispatched tokens (tcgen05 grouped GEMMs; both phases
 * in one launch while the mean expert group is under 128 tokens, two
 * launches above), writing the weighted per-slot outputs in token order:
 *   ybuf[t, j, :] = topk_w[t, j] * FFN_{topk_idx[t, j]}(x_t)   for each kept slot,
 *   ybuf[t, k, :] = sgate[t] * FFN_shared(x_t)                  when Is > 0,
 * rounded to bf16; other rows of ybuf are left untouched.
 * x [T, H] (read for the shared expert); x_perm [T*k, H] and offsets, perm
 * from moe_dispatch; topk_w [T, k]; sgate [T] (Is > 0); ybuf [T, k+1, H].
 * Uses the workspace (intermediate activations, status word). */
int moe_expert_ffn(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                   const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                   const moe_weights_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, void *stream);

/* The two phases of moe_expert_ffn, for callers that time or overlap them:
 * gate_up computes h = silu(W_gate x) * (W_up x) for every dispatched row
 * (and the shared expert's rows) into the workspace; down reads h from the
 * same workspace and writes ybuf as moe_expert_ffn does.  Arguments as in
 * moe_expert_ffn. */
int moe_expert_gate_up(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                       const int32_t *offsets, const moe_weights_t *w, void *ws, size_t ws_bytes, void *stream);
int moe_expert_down(const moe_config_t *cfg, int32_t T, const int32_t *offsets, const int32_t *perm,
                    const float *topk_w, const float *sgate, const moe_weights_t *w, moe_bf16_t *ybuf, void *ws,
                    size_t ws_bytes, void *stream);

/* Expert FFN for callers that cannot allocate device memory.  The pages
 * have no counterpart of this entry point; it exists for integration.
 *
 * Same computation, arguments and results as moe_expert_ffn, but with no
 * workspace: the scratch it needs (the gate/up activations and the
 * scheduling counters) lives in a fixed device array inside the library.
 * Use it when the caller cannot allocate -- e.g. a plugin that its host
 * framework hands only input and output buffers, or a serving loop that
 * must not allocate (an allocation can synchronise the device) once it runs.
 *   - Limit: 2 * (T*k*I + T*Is) bytes of activations must fit in
 *     MOE_NOALLOC_SCRATCH_BYTES; larger batches return MOE_ERR_WORKSPACE
 *     before anything is launched (use moe_expert_ffn for them).
 *   - The array (MOE_NOALLOC_SCRATCH_BYTES + 8 KB) is held on every device
 *     that loads the library until the process exits.
 *   - The first call on a device looks the array's address up (a CUDA
 *     runtime query); make that first call before capturing a stream into a
 *     CUDA graph.  The address is kept for the life of the process: after a
 *     cudaDeviceReset (or any teardown of the device's primary context) the
 *     library's device array is reloaded elsewhere and this entry point must
 *     not be used on that device again in the same process.
 *   - All calls share the one array: calls whose work overlaps on the GPU
 *     (e.g. on two streams at once) race and corrupt each other.  Each call
 *     re-zeroes the counters it needs (an async memset on `stream`); nothing
 *     else of the previous call's contents is relied on.
 *   - The call allocates nothing: no cudaMalloc, cudaFree or allocating
 *     library routine.
 *   - device_status (device pointer, may be NULL) receives the kernel's
 *     MOE_STATUS_* bits of this call.
 * Arguments otherwise as in moe_expert_ffn (no ws/ws_bytes). */
#define MOE_NOALLOC_SCRATCH_BYTES (8u << 20)
int moe_expert_ffn_noalloc(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                           const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                           const moe_weights_t *w, moe_bf16_t *ybuf, int32_t *device_status, void *stream);

/* ---------------------------------------------------------------------
 * The expert FFN with MXFP8 expert weights (block-scaled FP8: E4M3 codes,
 * one UE8M0 power-of-two scale per 32 consecutive weights along the
 * reduction axis), the FP8 expert weights that DeepGEMM fork PR #5 "big M
 * opt: splitT1 + L2 scatter + 2 stream" names against its W8A8 reference.
 * Weights only: activations stay bf16.  Each weight tile is turned into bf16
 * in tensor memory on its way to the tensor cores; every E4M3 code times its
 * block's power of two is a bf16 value (for scales 2^-117 .. 2^119), so the
 * layer computes exactly what moe_expert_ffn computes on the dequantised
 * weights, while half the weight bytes cross HBM.
 *   Codes: moe_quantize_mxfp8 of each matrix, in the bf16 weights' shapes.
 *   Scales: moe_quantize_mxfp8's [rows, K / 32] scales repacked once by
 *   moe_mxfp8_pack_scales (below) -- rows is E * I for w_gate / w_up and
 *   E * H for w_down, K the matrix's reduction size.
 * Limits on top of the general ones: H, I and Is multiples of 128.
 * --------------------------------------------------------------------- */
typedef struct {
    const uint8_t *w_gate;          /* [E, I, H] E4M3 codes */
    const uint8_t *w_up;            /* [E, I, H] E4M3 codes */
    const uint8_t *w_down;          /* [E, H, I] E4M3 codes */
    const uint8_t *w_gate_scale;    /* packed UE8M0 scales of w_gate (E * I rows, K = H) */
    const uint8_t *w_up_scale;      /* packed scales of w_up */
    const uint8_t *w_down_scale;    /* packed scales of w_down (E * H rows, K = I) */
    const uint8_t *ws_gate;         /* [Is, H] shared-expert codes, NULL if Is = 0 */
    const uint8_t *ws_up;           /* [Is, H], NULL if Is = 0 */
    const uint8_t *ws_down;         /* [H, Is], NULL if Is = 0 */
    const uint8_t *ws_gate_scale;   /* packed scales of ws_gate (Is rows, K = H), NULL if Is = 0 */
    const uint8_t *ws_up_scale;     /* packed scales of ws_up, NULL if Is = 0 */
    const uint8_t *ws_down_scale;   /* packed scales of ws_down (H rows, K = Is), NULL if Is = 0 */
    const moe_bf16_t *ws_gate_vec;  /* [H] bf16 shared-expert gate vector, NULL if Is = 0 */
    const moe_bf16_t *w_router;     /* [E, H] bf16 router projection (moe_forward_mxfp8 without logits) */
} moe_weights_mxfp8_t;

/* Repack MXFP8 scales [rows, K / 32] (as moe_quantize_mxfp8 writes them) into
 * the layout the FFN reads: [rows / 64][K / 128][64][4] -- for every group of
 * 64 rows and every 128 weights along K, the group's 64 x 4 scales as one
 * 256-byte run.  rows % 64 == 0, K % 128 == 0; both pointers device,
 * 16-byte aligned; same byte count in and out.  Run once per weight load. */
int moe_mxfp8_pack_scales(int64_t rows, int32_t K, const uint8_t *scales, uint8_t *packed, void *stream);

/* moe_expert_ffn with MXFP8 expert weights; arguments and results as
 * moe_expert_ffn (the same workspace size). */
int moe_expert_ffn_mxfp8(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                         const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                         const moe_weights_mxfp8_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, void *stream);

/* moe_forward with MXFP8 expert weights: routing, budget, dispatch and
 * combine as moe_forward, the expert FFN as moe_expert_ffn_mxfp8. */
int moe_forward_mxfp8(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const float *logits,
                      const moe_weights_mxfp8_t *w, moe_bf16_t *out, const moe_aux_t *aux, void *ws,
                      size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------
 * The expert FFN with NVFP4 expert weights (E2M1 codes, an E4M3 scale per 16
 * consecutive weights along the reduction axis, an fp32 scale per matrix):
 * the FP4 expert weights of DeepGEMM fork PR #5 "big M opt: splitT1 + L2
 * scatter + 2 stream" (megamoe_nvfp4) and of DeepGEMM PR #381's B200 FP8 x
 * FP4 policy, here with bf16 activations.  Each weight tile is turned into
 * bf16 in tensor memory on its way to the tensor cores: an E2M1 code times
 * its E4M3 block scale is always a bf16 value, so the MMAs see exactly the
 * weights the format stands for, and the matrix scale multiplies each
 * projection's fp32 output (gate and up before the SwiGLU, down before the
 * gate weight).  A quarter of the bf16 weight bytes cross HBM.
 *   Codes: moe_quantize_nvfp4 of each weight array (nmat = E for the routed
 *   experts, 1 for each shared matrix), [rows, K / 2] bytes per matrix.
 *   Scales: moe_quantize_nvfp4's [rows, K / 16] block scales repacked once
 *   by moe_nvfp4_pack_scales (below) -- rows is E * I for w_gate / w_up and
 *   E * H for w_down, K the matrix's reduction size.
 *   Matrix scales: moe_quantize_nvfp4's tensor_scale output.
 * Limits on top of the general ones: H, I and Is multiples of 128.
 * --------------------------------------------------------------------- */
typedef struct {
    const uint8_t *w_gate;          /* [E, I, H / 2] E2M1 codes, two per byte (lower K in the low nibble) */
    const uint8_t *w_up;            /* [E, I, H / 2] */
    const uint8_t *w_down;          /* [E, H, I / 2] */
    const uint8_t *w_gate_scale;    /* packed E4M3 block scales of w_gate (E * I rows, K = H) */
    const uint8_t *w_up_scale;      /* packed block scales of w_up */
    const uint8_t *w_down_scale;    /* packed block scales of w_down (E * H rows, K = I) */
    const float *w_gate_tscale;     /* [E] fp32 matrix scales of w_gate (4-byte aligned) */
    const float *w_up_tscale;       /* [E] of w_up */
    const float *w_down_tscale;     /* [E] of w_down */
    const uint8_t *ws_gate;         /* [Is, H / 2] shared-expert codes, NULL if Is = 0 */
    const uint8_t *ws_up;           /* [Is, H / 2], NULL if Is = 0 */
    const uint8_t *ws_down;         /* [H, Is / 2], NULL if Is = 0 */
    const uint8_t *ws_gate_scale;   /* packed block scales of ws_gate (Is rows, K = H), NULL if Is = 0 */
    const uint8_t *ws_up_scale;     /* packed block scales of ws_up, NULL if Is = 0 */
    const uint8_t *ws_down_scale;   /* packed block scales of ws_down (H rows, K = Is), NULL if Is = 0 */
    const float *ws_tscale;         /* [3] fp32 matrix scales of ws_gate, ws_up, ws_down; NULL if Is = 0 */
    const moe_bf16_t *ws_gate_vec;  /* [H] bf16 shared-expert gate vector, NULL if Is = 0 */
    const moe_bf16_t *w_router;     /* [E, H] bf16 router projection (moe_forward_nvfp4 without logits) */
} moe_weights_nvfp4_t;

/* Repack NVFP4 block scales [rows, K / 16] (as moe_quantize_nvfp4 writes
 * them) into the layout the FFN reads: [rows / 64][K / 128][64][8] -- for
 * every group of 64 rows and every 128 weights along K, the group's 64 x 8
 * scales as one 512-byte run.  rows % 64 == 0, K % 128 == 0; both pointers
 * device, 16-byte aligned; same byte count in and out.  Run once per weight
 * load. */
int moe_nvfp4_pack_scales(int64_t rows, int32_t K, const uint8_t *scales, uint8_t *packed, void *stream);

/* moe_expert_ffn with NVFP4 expert weights; arguments and results as
 * moe_expert_ffn (the same workspace size). */
int moe_expert_ffn_nvfp4(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                         const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                         const moe_weights_nvfp4_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, void *stream);

/* moe_forward with NVFP4 expert weights: routing, budget, dispatch and
 * combine as moe_forward, the expert FFN as moe_expert_ffn_nvfp4. */
int moe_forward_nvfp4(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const float *logits,
                      const moe_weights_nvfp4_t *w, moe_bf16_t *out, const moe_aux_t *aux, void *ws,
                      size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------
 * Expert parallelism: the E experts split over W ranks (one GPU each), rank
 * r holding experts [r * epr, (r + 1) * epr), epr = E / W -- the layout of
 * the multi-rank MegaMoE of DeepGEMM PR #381 ("B200 performance", EP8) and
 * DeepGEMM fork PR #5, whose dispatch sends each token's routed rows to the
 * ranks holding its experts and whose combine brings the weighted expert
 * outputs back.  The exchange is the caller's collective (NCCL all-to-all);
 * these three calls are the per-rank steps around it (see the package's
 * ep.py for the whole layer):
 *   1. moe_route, then moe_ep_rank_ids, then moe_dispatch with W "experts"
 *      on the rank ids: slots grouped by destination rank (perm, counts) and
 *      the rows to send (x_perm, in that order);
 *   2. moe_ep_pack: for each row to send, the expert id local to its rank
 *      and the routing weight;
 *   3. (exchange; at the destination moe_dispatch + moe_expert_ffn with k = 1
 *      on the received rows and their local ids and weights, moe_combine to
 *      make the weighted outputs contiguous; exchange back)
 *   4. moe_ep_unpack: the returned rows, in send order, to the token-ordered
 *      ybuf rows; the shared expert on the home rank; moe_combine.
 * --------------------------------------------------------------------- */

/* rank_idx[s] = topk_idx[s] / experts_per_rank for s < T*k (-1 stays -1).
 * topk_idx, rank_idx [T, k] i32 (device). */
int moe_ep_rank_ids(int32_t T, int32_t k, int32_t experts_per_rank, const int32_t *topk_idx, int32_t *rank_idx,
                    void *stream);

/* For p < *n_sent (device int: the dispatch's offsets[W]), with s = perm[p]:
 * local_idx[p] = topk_idx[s] % experts_per_rank, local_w[p] = topk_w[s].
 * n_max >= *n_sent bounds the launch (T*k).  perm from moe_dispatch on the
 * rank ids; local_idx, local_w [n_max] (device). */
int moe_ep_pack(int32_t n_max, const int32_t *n_sent, int32_t experts_per_rank, const int32_t *perm,
                const int32_t *topk_idx, const float *topk_w, int32_t *local_idx, float *local_w, void *stream);

/* ybuf[s + s / k, :] = rows[p, :] for p < *n_returned (device int), s =
 * perm[p]: the weighted expert outputs, returned in send order, to the
 * token-ordered rows moe_combine adds.  rows [n_max, H]; ybuf [T, k+1, H];
 * n_max <= T*k. */
int moe_ep_unpack(const moe_config_t *cfg, int32_t T, int32_t n_max, const int32_t *n_returned, const int32_t *perm,
                  const moe_bf16_t *rows, moe_bf16_t *ybuf, void *stream);

/* Combine: out[t, :] = bf16( sum_{j < keff[t]} ybuf[t, j, :] + [Is > 0] ybuf[t, k, :] ),
 * summed in fp32 in slot order and rounded once (a token with no kept slot
 * and no shared expert gets 0).  keff == NULL means k; a keff entry outside
 * [0, k] counts as the nearest end (a token's own rows are all it reads).
 * ybuf [T, k+1, H]; keff [T]; out [T, H]. */
int moe_combine(const moe_config_t *cfg, int32_t T, const moe_bf16_t *ybuf, const int32_t *keff,
                moe_bf16_t *out, void *stream);

/* The whole layer: [router projection] -> route -> [top-p] -> [budget] ->
 * dispatch -> expert FFN -> combine, enqueued on one stream with no host
 * sync.  x [T, H]; logits [T, E] f32, or NULL to compute them from
 * w->w_router (moe_router_logits; then aux->logits, if set, receives them);
 * out [T, H]; aux may be NULL. */
int moe_forward(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const float *logits,
                const moe_weights_t *w, moe_bf16_t *out, const moe_aux_t *aux, void *ws,
                size_t ws_bytes, void *stream);

/* Status word: MOE_STATUS_* bits set by kernels (sticky until cleared).
 * moe_status_read enqueues a copy on `stream`, waits for the stream, and
 * returns MOE_OK with *status_out filled (host pointer).  moe_status_clear
 * enqueues a zeroing of the workspace's first 8 KB (status word and
 * scheduling counters) on `stream`. */
int moe_status_read(const void *ws, int32_t *status_out, void *stream);
int moe_status_clear(void *ws, void *stream);

/* Static text for a return code. */
const char *moe_error_string(int code);

/* ---------------------------------------------------------------------
 * Block-scaled expert weights: the pack step (run once when the weights are
 * loaded).  The formats are the FP8 and NVFP4 expert weights of DeepGEMM
 * fork PR #5 "big M opt: splitT1 + L2 scatter + 2 stream" (its megamoe_nvfp4
 * kernels, its B200 FP8 x FP4 policy), with the published definitions:
 * E4M3 without infinities (largest finite 448), E2M1 (magnitudes 0, 0.5, 1,
 * 1.5, 2, 3, 4, 6), UE8M0 (2^(c - 127)).  Rounding is to nearest, ties to
 * the even code, saturating; the sign bit copies the input's.  Inputs must
 * be finite: a NaN or infinite weight has no defined code (a NaN counts as
 * the largest magnitude, so in NVFP4 it spoils its whole matrix's scale);
 * the quantisers do not check for them.  The blocks
 * run along the last (reduction) axis of a row-major matrix: rows of
 * W_gate / W_up [I, H] and of W_down [H, I].  The layer consumes both
 * (moe_expert_ffn_mxfp8 / moe_forward_mxfp8, moe_expert_ffn_nvfp4 /
 * moe_forward_nvfp4 above).
 * --------------------------------------------------------------------- */

/* MXFP8: blocks of 32 consecutive elements share a UE8M0 scale
 * X = 2^(floor(log2(amax)) - 8) (clamped to [2^-127, 2^127]; an all-zero
 * block takes 2^-127), each element is x / X rounded to E4M3.
 * w      [rows, K] bf16, K a multiple of 32 (device, 16-byte aligned);
 * codes  [rows, K] uint8 E4M3 (device, 16-byte aligned, written);
 * scales [rows, K / 32] uint8 UE8M0 (device, written).
 * Enqueued on `stream`; MOE_ERR_INVALID_ARG for a bad size or pointer. */
int moe_quantize_mxfp8(int64_t rows, int32_t K, const moe_bf16_t *w, uint8_t *codes, uint8_t *scales,
                       void *stream);

/* NVFP4: nmat matrices of [rows, K], stored one after another.  Each matrix
 * has an fp32 scale s_t = amax / (6 * 448) (1 when all zero); blocks of 16
 * consecutive elements share an E4M3 scale s_b = E4M3(amax_b / (6 * s_t));
 * each element is E2M1(x / (s_b * s_t)), all in IEEE fp32 in that order.
 * w            [nmat, rows, K] bf16, K a multiple of 16 (device, 16-byte aligned);
 * codes        [nmat, rows, K / 2] uint8, two E2M1 codes per byte, element 2i
 *              in the low nibble (device, 16-byte aligned, written);
 * scales       [nmat, rows, K / 16] uint8 E4M3 (device, written);
 * tensor_scale [nmat] fp32 (device, 4-byte aligned, written; also the
 *              reduction's scratch while the call runs).
 * 1 <= nmat <= 65535.  Enqueued on `stream`; MOE_ERR_INVALID_ARG for a bad
 * size or pointer. */
int moe_quantize_nvfp4(int32_t nmat, int64_t rows, int32_t K, const moe_bf16_t *w, uint8_t *codes, uint8_t *scales,
                       float *tensor_scale, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H */
