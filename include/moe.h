/*
 * moe.h -- C ABI of the B200 (sm_100a) top-k Mixture-of-Experts FFN layer forward.
 *
 * The layer (inference, one GPU):
 *
 *   xn      = RMSNorm(x) * gamma                       (rounded to the activation dtype)
 *   logits  = xn . W_r                                 (FP32 accumulation)
 *   idx, g  = top-k of the FP32 logits (+ per-expert bias), softmax gates in FP32,
 *             optionally renormalised over the selected k
 *   counts, offsets, perm = per-expert histogram + prefix scan + stable permutation,
 *             with an optional capacity C*T*k/E per expert (overflow dropped)
 *   y_a     = g_a * SwiGLU_e(xn_t)                     (grouped GEMM over experts)
 *   out     = x + sum_shared SwiGLU_s(xn) + sum_{kept a of t} y_a
 *
 * Sources (page title, section):
 *   "MoE: dynamism the compiler cannot remove" -- the natural implementation
 *     (router -> top-k -> per-expert dispatch), the capacity section (buffers of
 *     C*T*k/E rows, overflow tokens pass through on the residual) and the grouped
 *     GEMM section (one launch over the total work T*k; each block finds its group
 *     from a small descriptor array).
 *   picx.dev summary of the moe-ceilings study, Sub-study 1 -- gate probabilities
 *     accumulated in FP32 before the top-k; the router is kept un-quantised.
 *   "MoE Research", section 2 -- shared (always-on) experts; per-expert bias terms
 *     for auxiliary-loss-free balancing.  Section 3 -- grouped GEMM and sorting.
 *   "MoE at the inference level ...", Workarounds -- gather -> grouped GEMM ->
 *     scatter; int4 / fp8 expert weights.
 *
 * Conventions common to every entry point:
 *   - Every tensor pointer is DEVICE memory owned by the caller; shapes are
 *     row-major with the last index contiguous.  The library allocates no device
 *     memory.  Its only state shared between calls is the built-in scratch
 *     array of moe_permute_static (1 MiB per device, see there for the rule on
 *     overlapping calls); every other entry point works in the caller's
 *     workspace only.
 *   - Alignment: tensors need only the alignment of their element type, except
 *     that with tensor-core experts (bf16 / int8 / int4) xn, the expert weights
 *     and their scales must be 16-byte aligned (TMA operands; MOE_ERR_INVALID
 *     otherwise).  16-byte aligned tensors take vectorised kernels elsewhere.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream and never synchronise the host,
 *     except moe_get_device_status.
 *   - Argument errors are returned synchronously (MOE_ERR_INVALID /
 *     MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE) and nothing is launched.  A failed
 *     launch returns MOE_ERR_CUDA.
 *   - Errors found on the device (an expert id outside [0,E) in topk_idx, a
 *     pipeline wait that ran out) set an int32 error word at the start of the
 *     workspace; read it with moe_get_device_status.  Kernels never trap.
 *   - No C++ exception crosses this boundary.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,      /* bad argument (NULL pointer, k > E, size out of range) */
  MOE_ERR_UNSUPPORTED = 2,  /* legal but not implemented (dtype/shape combination)   */
  MOE_ERR_WORKSPACE = 3,    /* workspace missing or smaller than moe_workspace_size */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call failed                             */
  MOE_ERR_DEVICE = 5        /* the device error word is set (moe_get_device_status)  */
} moe_status;

/* MOE_FP8: FP8 E4M3 expert weights (weight-only, like MOE_INT8) -- "MoE at the
 * inference level ...", Workarounds: int4 / fp8 expert weights to halve the bytes. */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_INT8 = 2, MOE_INT4 = 3, MOE_FP8 = 4 } moe_dtype;

/* Per-expert router bias ("MoE Research", section 2):
 *   NONE   : no bias.
 *   LOGIT  : the bias is part of the router logits; it moves both the selection
 *            and the gate probabilities.
 *   SELECT : auxiliary-loss-free style; the bias moves the selection only and the
 *            gates are the softmax of the unbiased logits. */
typedef enum { MOE_BIAS_NONE = 0, MOE_BIAS_LOGIT = 1, MOE_BIAS_SELECT = 2 } moe_bias_mode;

/* Routing ("MoE: dynamism the compiler cannot remove", capacity section):
 *   TOPK           : each token picks its top-k experts (the layer of the pages);
 *   EXPERT_CHOICE  : each expert picks the C = ceil(C_f * T*k/E) tokens (C_f = the
 *                    capacity factor, 1 when <= 0; at most T) with the largest gate
 *                    probability -- the softmax over the experts of the token's FP32
 *                    logits (plus the bias in LOGIT mode); that probability is the
 *                    assignment's gate.  Every expert holds exactly C rows; a token
 *                    may get several experts or none.  Ties at an expert's C-th
 *                    score go to the lower token.  Not with SELECT bias or FP32
 *                    experts. */
typedef enum { MOE_ROUTE_TOPK = 0, MOE_ROUTE_EXPERT_CHOICE = 1 } moe_routing;

/* Layer configuration.  All fields are 32-bit so that the layout is the same
 * from every language. */
typedef struct moe_config {
  int32_t T;               /* tokens in the batch, >= 1                                 */
  int32_t d;               /* model dim, multiple of 8 (of 128 for bf16/int experts)    */
  int32_t E;               /* routed experts, 1..512, multiple of 8 for a bf16 router   */
  int32_t k;               /* experts per token, 1..min(E, 32)                          */
  int32_t f;               /* expert hidden dim (multiple of 128 for bf16/int experts)  */
  int32_t n_shared;        /* always-on shared experts, 0..8; each has hidden f         */
  float capacity_factor;   /* <= 0: uncapped; else cap = ceil(C*T*k/E) rows per expert,
                              computed in double; assignments ranked in flat order
                              a = t*k + j and kept iff their rank < cap                */
  int32_t renormalize;     /* nonzero: gates divided by their sum over the k selected  */
  int32_t bias_mode;       /* moe_bias_mode                                             */
  float rms_eps;           /* RMSNorm epsilon                                           */
  int32_t act_dtype;       /* x (and the residual): MOE_BF16 or MOE_F32                 */
  int32_t out_dtype;       /* out: MOE_BF16 or MOE_F32 (MOE_F32 when act_dtype is F32);
                              the combine sums in FP32 and rounds once to this type    */
  int32_t router_dtype;    /* W_r: MOE_BF16 or MOE_F32 (must equal act_dtype)           */
  int32_t expert_dtype;    /* MOE_F32 (requires act F32) | MOE_BF16 | MOE_INT8 | MOE_INT4
                              | MOE_FP8                                                 */
  int32_t group_size;      /* int4: scale group along K; must be 128                    */
  int32_t wait_kcycles;    /* limit of every pipeline wait inside the kernels, in units of
                              1024 SM clock cycles; 0 = the default, 10^9 cycles (about
                              half a second).  A wait that runs out sets device error 2
                              and the kernel returns early (moe_get_device_status)      */
  int32_t routing;         /* moe_routing (0 = top-k)                                    */
  int32_t prefill_tiles;   /* tensor-core experts at prefill (more than 64 rows per expert on
                              average): 1 = tiles of 128 tokens on single CTAs, 2 = tiles
                              of 256 tokens on pairs of CTAs (one cta_group::2 MMA per
                              k-step), 0 = automatic: pairs for bf16 experts when the
                              batch averages at least 512 rows per routed expert (a pair
                              tile half empty costs twice a single one), else single
                              CTAs.  All give the same bits; other values are rejected  */
} moe_config;

/* Layer weights (device pointers, caller-owned).
 *   rms_gamma   [d] float32
 *   w_router    [d, E]            router dtype
 *   router_bias [E] float32, or NULL (required unless bias_mode == NONE)
 *   w_gate/w_up F32/BF16: [E, d, f] of that type (W[k][n], n contiguous).
 *               INT8: int8 [E, f, d]; FP8: uint8 E4M3 codes [E, f, d]; INT4: uint8
 *               [E, f, d/2] -- quantised codes are stored transposed, the reduction
 *               dim d contiguous (code q[n][k] is weight W[k][n])
 *   w_down      F32/BF16: [E, f, d]; INT8 / FP8: [E, d, f]; INT4: uint8 [E, d, f/2]
 *   s_gate/s_up INT8, FP8: bf16 [E, f]; INT4: bf16 [E, d/128, f]; otherwise NULL
 *   s_down      INT8, FP8: bf16 [E, d]; INT4: bf16 [E, f/128, d]; otherwise NULL
 *   sh_*        the same for the n_shared shared experts ([S, ...]); NULL if S == 0
 * int8 weights are symmetric with one scale per output column; int4 weights are
 * symmetric signed 4-bit (two's complement), two per byte along the contiguous
 * (reduction) dim, eight per 4-byte word: nibble j of the little-endian word holds
 * k = 8w + (0, 2, 4, 6, 1, 3, 5, 7)[j] (even k in the low nibbles of the word's bytes,
 * odd k in the high ones), with one scale per 128 rows of K and output column; fp8
 * weights are E4M3 codes (no infinities, largest finite 448) with one scale per
 * output column.  In every case the weight the layer uses is bf16(q * s): the
 * exact product rounded once, formed inside the expert GEMM's main loop. */
typedef struct moe_weights {
  const void* rms_gamma;
  const void* w_router;
  const void* router_bias;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
  const void* s_gate;
  const void* s_up;
  const void* s_down;
  const void* sh_gate;
  const void* sh_up;
  const void* sh_down;
  const void* sh_s_gate;
  const void* sh_s_up;
  const void* sh_s_down;
} moe_weights;

/* Bytes of device workspace the calls below need for this configuration (worst
 * case over routings: T*k kept slots).  0 on an invalid configuration.  The
 * workspace needs 256-byte alignment; its first 4 bytes are the device error
 * word.
 * Source: "MoE: dynamism the compiler cannot remove", grouped GEMM section --
 * the per-expert row counts are data dependent, so the grouped kernels read
 * them from descriptor buffers kept at fixed addresses and sized for the worst
 * case (every one of the T*k assignments kept); a fixed size and fixed
 * addresses are also what lets the calls be captured in a CUDA graph. */
size_t moe_workspace_size(const moe_config* cfg);

/* Zero the device error word (asynchronous).  The pages have no counterpart:
 * it resets the failure report that moe_get_device_status reads, and the state
 * the single-launch decode layer keeps in the workspace's first 256 bytes (its
 * grid-barrier words).  Call it after a device error before the workspace is used
 * again. */
moe_status moe_clear_device_status(void* ws, size_t ws_bytes, void* stream);

/* Steps a1 + a2: RMSNorm and the router GEMM.
 *   x       [T, d] act dtype          xn_out [T, d] act dtype (bf16 or fp32), or NULL
 *   logits  [T, E] float32 (no bias)  ws: workspace (xn is kept there when xn_out is NULL)
 * RMSNorm is computed in double per token, xn = (x * (mean(x^2) + eps)^-1/2) * gamma,
 * and rounded once (round-to-nearest-even) to the activation dtype.  The router
 * multiplies that rounded xn by W_r with FP32 accumulation (picx.dev summary,
 * Sub-study 1: router kept un-quantised, gates in FP32). */
moe_status moe_rmsnorm_router(const moe_config* cfg, const moe_weights* w, const void* x,
                              void* xn_out, float* logits, void* ws, size_t ws_bytes,
                              void* stream);

/* Step a3: softmax + top-k + bias + renormalisation, one warp per token.
 * Sources: picx.dev summary of the moe-ceilings study, Sub-study 1
 * (FusedSoftmax: the gate probabilities are accumulated in FP32 before the
 * top-k); "MoE: dynamism the compiler cannot remove", natural implementation
 * (router logits -> top-k indices and weights); "MoE Research", section 2
 * (per-expert bias terms that move the selection to even out the load).
 *   logits    [T, E] float32 router logits (bias not included)
 *   bias      [E] float32 or NULL (see moe_bias_mode)
 *   topk_idx  [T, k] int32: selected experts by descending key (logit, plus the
 *             bias in LOGIT/SELECT mode), ties to the lower expert index; NaN keys
 *             order below every number
 *   topk_gate [T, k] float32: softmax over all E (FP32), of the biased logits in
 *             LOGIT mode and of the plain logits otherwise; renormalised over the
 *             k selected when cfg->renormalize
 * Deterministic; given identical logits the indices are bit-exact to any correct
 * implementation of the rule above. */
moe_status moe_route(const moe_config* cfg, const float* logits, const float* bias,
                     int32_t* topk_idx, float* topk_gate, void* stream);

/* Expert-choice routing (cfg->routing == MOE_ROUTE_EXPERT_CHOICE): the routing
 * and permutation steps of that mode.
 * Source: "MoE: dynamism the compiler cannot remove", capacity section -- each
 * expert picks its top T*k/E tokens, which balances the load by construction.
 *   logits     [T, E] float32 router logits (bias not included)
 *   bias       [E] float32 or NULL (LOGIT mode adds it before the softmax)
 *   scores_out [T, E] float32 or NULL: the FP32 softmax over the experts, on which
 *              the picks are taken
 *   tok        [E*C] int32: slot e*C + c holds the c-th token expert e picked, in
 *              ascending token order (C = moe_expert_choice_capacity(cfg))
 *   gate       [E*C] float32: that token's score for expert e
 *   slot_te    [T, E] int32: the slot of (token, expert), or -1 if not picked
 *   ws         workspace (the scores are kept there expert-major)
 * The picks are deterministic and, given identical FP32 scores, bit-exact to any
 * correct implementation of the rule above. */
moe_status moe_route_expert_choice(const moe_config* cfg, const float* logits, const float* bias,
                                   float* scores_out, int32_t* tok, float* gate,
                                   int32_t* slot_te, void* ws, size_t ws_bytes, void* stream);

/* Tokens each expert picks under expert-choice routing (0 for a top-k or an
 * invalid configuration).  Source: as moe_route_expert_choice. */
int32_t moe_expert_choice_capacity(const moe_config* cfg);

/* Steps a4 + a5: per-expert histogram, prefix scan, capacity and the stable
 * permutation ("MoE Research", section 3: grouped GEMM and sorting).  No global
 * atomics; deterministic.
 *   topk_idx    [T*k] int32 (flat assignment a = t*k + j)
 *   counts      [E]   int32: assignments per expert before capacity
 *   offsets     [E+1] int32: exclusive scan of kept[e] = min(counts[e], cap)
 *   perm_assign [T*k] int32: slot s (< offsets[E]) holds assignment a; token = a / k
 *   slot_of     [T*k] int32: slot of assignment a, or -1 when dropped by capacity
 *   n_dropped   [1]   int32: sum_e max(0, counts[e] - cap)
 *   ws          workspace (only its error word is used; an id outside [0,E) sets
 *               it, and that assignment is dropped) */
moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, int32_t* counts,
                       int32_t* offsets, int32_t* perm_assign, int32_t* slot_of,
                       int32_t* n_dropped, void* ws, size_t ws_bytes, void* stream);

/* moe_permute without a workspace.  The pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- for example a
 * plugin slot in another inference engine that hands an operator its input and
 * output tensors but no allocator, or a serving process that reserves all of its
 * device memory at start-up so that any later allocation would fail.
 *
 * Same outputs as moe_permute, bit for bit.  The per-CTA counts of the
 * multi-CTA path live in a 1 MiB array built into the library (a static device
 * array that every GPU using the library holds until the process exits), so
 * E * ceil(T*k / 2048) must be at most 262144; larger batches return
 * MOE_ERR_WORKSPACE and launch nothing.  Nothing is allocated or freed.
 *
 * The first call on each device looks up that array's device address (under a
 * lock); make that first call before any stream capture.  Every call on a device
 * shares the one array, so calls whose kernels overlap on the GPU (other
 * streams, other host threads) race and give wrong results: serialise them.
 * Expert ids outside [0, E) are dropped (slot -1) without a report, since there
 * is no workspace to carry the device error word. */
moe_status moe_permute_static(const moe_config* cfg, const int32_t* topk_idx, int32_t* counts,
                              int32_t* offsets, int32_t* perm_assign, int32_t* slot_of,
                              int32_t* n_dropped, void* stream);

/* Steps a6 + a7: grouped SwiGLU expert GEMMs over the permuted tokens
 * ("MoE: dynamism the compiler cannot remove", grouped GEMM section), plus the
 * shared experts on every token.
 *   xn          [T, d] act dtype (normalised activations)
 *   offsets     [E+1], perm_assign [T*k]: as written by moe_permute
 *   topk_gate   [T*k] float32
 *   y_assign    [T*k, d] float32: row a = g_a * SwiGLU_{e(a)}(xn_{a/k}) for every kept
 *               assignment a; rows of dropped assignments are left untouched
 *   y_shared    [S, T, d] float32: SwiGLU_s(xn_t), or NULL when S == 0
 * bf16 / int experts run on the tcgen05 tensor cores (bf16 operands, FP32
 * accumulation; the intermediate h is rounded to bf16); fp32 experts run in FP32
 * on the CUDA cores. */
moe_status moe_grouped_ffn(const moe_config* cfg, const moe_weights* w, const void* xn,
                           const int32_t* offsets, const int32_t* perm_assign,
                           const float* topk_gate, float* y_assign, float* y_shared,
                           void* ws, size_t ws_bytes, void* stream);

/* Step a8: combine.
 * Sources: "MoE: dynamism the compiler cannot remove", natural implementation
 * (each expert's output, weighted by its gate, is added into the token's output
 * row) and capacity section (a token slot dropped by capacity contributes
 * nothing: the token passes through on the residual); "MoE Research", section 2
 * (the shared experts' outputs are added for every token).
 * out[t] = residual[t] + sum_s y_shared[s, t] +
 * sum_{j : slot_of[t*k+j] >= 0} y_assign[t*k+j], summed in FP32 in that fixed order
 * (deterministic), rounded to the activation dtype.
 *   residual [T, d] act dtype or NULL (then out is the MoE delta only)
 *   out      [T, d] out dtype */
moe_status moe_combine(const moe_config* cfg, const float* y_assign, const int32_t* slot_of,
                       const float* y_shared, const void* residual, void* out,
                       void* stream);

/* The whole layer: a1..a8 on one stream, no host synchronisation.
 * Decode batches (T <= 32) of bf16 experts with a bf16 router of at most 256
 * experts and 16-byte aligned tensors run as ONE cooperative launch of one CTA per
 * SM ("MoE: dynamism the compiler cannot remove", batch-1 section: the layer is
 * launch bound at small batches), its steps separated by bounded grid-wide
 * barriers in the workspace; every other configuration runs as a chain of
 * kernels (moe_layer_launch_count).
 * Source: the whole chain of "MoE: dynamism the compiler cannot remove",
 * natural implementation (pre-norm, router, top-k, dispatch to the experts,
 * gated sum) with its capacity section, in the grouped form of that page's
 * grouped GEMM section (one launch over all experts' rows) and the
 * gather -> grouped GEMM -> scatter structure of "MoE at the inference level",
 * Workarounds.
 *   x [T, d] act dtype, out [T, d] out dtype.  Optional outputs (NULL to skip):
 *   logits_out [T, E] float32, topk_idx_out [T, k] int32, counts_out [E] int32.
 * With expert-choice routing the chain is RMSNorm, router, scores, the experts'
 * picks, the grouped GEMMs over the E*C picks and a combine that adds, per token,
 * the rows of the experts that picked it in ascending expert order; topk_idx_out
 * must then be NULL and counts_out receives C for every expert.
 * Between the down GEMM and the combine the gated routed rows of tensor-core
 * experts are kept in bf16 (the round-to-nearest-even of the FP32 rows that
 * moe_grouped_ffn returns), so the result equals moe_combine applied to those
 * rounded rows, bit for bit. */
moe_status moe_layer_forward(const moe_config* cfg, const moe_weights* w, const void* x,
                             void* out, void* ws, size_t ws_bytes, float* logits_out,
                             int32_t* topk_idx_out, int32_t* counts_out, void* stream);

/* moe_layer_forward with per-step timing marks, for profiling.
 * Source: picx.dev summary of the moe-ceilings study, Summary and Sub-study 1
 * (the forward is profiled module by module to find where the time goes before
 * anything is fused).  It always runs the layer as a chain of kernels, also
 * for the decode batches that moe_layer_forward runs as a single launch.
 * events[0] is recorded on `stream` before the first kernel and events[i] right
 * after step i (i = 1 .. moe_layer_step_count(cfg)).  The steps are RMSNorm,
 * router, route, permute, [gather], gate/up GEMM, down GEMM, combine (expert
 * choice: route = the scores, permute = the experts' picks):
 *   - up to 32 tokens the route launch also builds the permutation, and the
 *     permute step is empty;
 *   - the bracketed step exists for tensor-core experts: it gathers the routed
 *     token rows, except on bf16 decode tiles, where the gate/up GEMM gathers
 *     them itself and the step is empty.
 * `events` holds caller-created cudaEvent_t handles (as void*); n_events must be
 * at least moe_layer_step_count(cfg) + 1.  No optional outputs. */
moe_status moe_layer_forward_profiled(const moe_config* cfg, const moe_weights* w,
                                      const void* x, void* out, void* ws, size_t ws_bytes,
                                      void* const* events, int32_t n_events, void* stream);

/* Synchronise `stream`, then read the device error word into *code (0 = none;
 * 1 = expert id out of range; 2 = a pipeline wait ran out).  Returns MOE_ERR_DEVICE
 * when the word is nonzero.
 * The pages have no counterpart: this is the failure-detection side of the
 * boundary.  The grouped GEMMs' pipelines wait on barriers inside the kernel
 * (the persistent, descriptor-driven form of "MoE: dynamism the compiler cannot
 * remove", grouped GEMM section); every such wait is bounded, and a wait that
 * runs out, or a routed expert id outside [0, E), is reported here instead of
 * trapping the device. */
moe_status moe_get_device_status(const void* ws, int32_t* code, void* stream);

/* Static, human-readable name of a status (no counterpart in the pages). */
const char* moe_status_string(moe_status s);

/* Number of kernels moe_layer_forward launches for this configuration (for
 * launch accounting); 0 on an invalid configuration.
 * Source: "MoE: dynamism the compiler cannot remove", batch-1 section, and the
 * picx.dev summary of the moe-ceilings study, Practical Implications: the MoE
 * layer is launch bound at small batches (about a thousand launches per forward
 * with a per-expert loop), so the number of launches is a figure to report. */
int32_t moe_layer_launch_count(const moe_config* cfg);

/* Number of steps moe_layer_forward_profiled marks (see there, and its source);
 * 0 if invalid. */
int32_t moe_layer_step_count(const moe_config* cfg);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
