/*
 * moe.h - C ABI of the B200 (sm_100a) sparse top-k Mixture-of-Experts layer forward.
 *
 * One layer forward, as defined by the pages it is built from:
 *   router logits h = W_g x (+ router bias)       "Appendix C - Acronyms & Symbols",
 *   P = softmax(h), top-k set T_k(x), gates g_i      table "Core MoE symbols";
 *   capacity C = ceil(C_f k T / E), dispatch into    same page, "Capacity &
 *   per-expert buffers, overflow dropped             communication"; "Code Walkthrough -
 *                                                    SER", "Load balancing";
 *   expert MLP w1/b1 -> ReLU|GELU|Swish -> w2/b2,    "Code Walkthrough - SER", "The
 *   gate-weighted combine, shared experts            gating / routing path";
 *                                                    Appendix C "Parameter accounting";
 *   f_i, P_i, L_aux = alpha E sum f_i P_i,           Appendix C, "Balancing";
 *   z-loss beta mean (log sum e^h)^2
 *   credit c = g ||o_i(x)||_2 and the expert-        "Sparse MoE Expert-Credit Loss
 *   attributed loss l_i                              Reweighting Diagram", panel (b).
 *
 * Conventions for every entry point:
 *   - Array arguments are DEVICE pointers (CUDA global memory) owned by the caller,
 *     row-major, densely packed, and at least 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). All device work is enqueued asynchronously on it; no entry point
 *     synchronises the device.
 *   - Every call that can fail returns an int status (MOE_OK = 0, negative on
 *     error). Argument errors are detected on the host BEFORE anything is
 *     enqueued; moe_last_error() then returns a message naming the bad argument.
 *   - The library never allocates device memory at run time: scratch comes
 *     from the caller's workspace or, for moe_forward_noalloc only, from the
 *     fixed built-in device array documented at that declaration.
 *   - NaN or Inf inputs are not supported: outputs are then unspecified, but no
 *     kernel faults or waits forever.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,  /* a NULL or inconsistent argument             */
    MOE_ERR_UNSUPPORTED = -2,  /* a valid configuration this library does not support */
    MOE_ERR_CUDA = -3,         /* a CUDA runtime or driver call failed         */
    MOE_ERR_WORKSPACE = -4,    /* workspace NULL, misaligned or too small      */
    MOE_ERR_TIMEOUT = -5,      /* a bounded device-side wait gave up           */
    MOE_ERR_STATE = -6,        /* call out of order (stats before a forward)   */
    MOE_ERR_INTERNAL = -7      /* a self-check found the library misbehaving   */
};

/* Activations ("Code Walkthrough - SER", gating / routing path: ReLU, GELU, Swish).
 * GELU is the exact form 0.5 z (1 + erf(z / sqrt 2)); Swish is z * sigmoid(z). */
enum { MOE_ACT_RELU = 0, MOE_ACT_GELU = 1, MOE_ACT_SWISH = 2 };

/* Top-k methods (same page, "Configuration"): GREEDY selects the highest logits;
 * NOISY adds caller-supplied noise to the logits before selection. */
enum { MOE_TOPK_GREEDY = 0, MOE_TOPK_NOISY = 1 };

/* Storage type of x, w1, w2 and y. Router weights and biases are always fp32.
 * BF16 runs the expert FFNs on the tcgen05 tensor cores (fp32 accumulation);
 * FP32 runs them on fp32 CUDA cores. */
enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_FP32 = 1 };

/* Which vector's norm the expert credit c = g ||h||_2 uses ("Sparse MoE
 * Expert-Credit Loss Reweighting Diagram", panel (b)): the expert's output
 * (default) or its hidden activation act(w1 x + b1). */
enum { MOE_CREDIT_OUTPUT = 0, MOE_CREDIT_HIDDEN = 1 };

/* Order in which assignments fill an expert's capacity ("Appendix C",
 * "Capacity & communication"; the pages fix none): TOKEN = ascending token
 * index, each token's choices together; RANK = every token's first choice (in
 * token order), then every second choice, and so on (GShard's order). */
enum { MOE_PRIORITY_TOKEN = 0, MOE_PRIORITY_RANK = 1 };

/* Layer configuration. Field names follow the SER walkthrough's configuration
 * (num_experts, num_active, input_dim, expert_dim, output_dim, top_k_method,
 * load_balance_coef); the remaining fields carry Appendix C's symbols. */
typedef struct {
    int32_t num_experts;      /* E, routed experts, 1..256                          */
    int32_t num_active;       /* k, experts per token, 1..min(E, 16)                */
    int32_t input_dim;        /* d; multiple of 64 for BF16                         */
    int32_t expert_dim;       /* F = d_ff; multiple of 64 for BF16                  */
    int32_t output_dim;       /* O; multiple of 64 for BF16                         */
    int32_t num_shared;       /* S always-on shared experts (weight 1), 0..4        */
    float capacity_factor;    /* C_f; C = ceil(C_f k T / E). <= 0: no limit (C = T) */
    int32_t activation;       /* MOE_ACT_*                                          */
    int32_t top_k_method;     /* MOE_TOPK_*                                         */
    int32_t use_selection_bias; /* 1: add weights->sel_bias b_i to the selection key */
    int32_t dtype;            /* MOE_DTYPE_*                                        */
    int32_t max_tokens;       /* largest T a forward may pass; 0 = no limit        */
    float load_balance_coef;  /* alpha of L_aux                                     */
    float z_loss_coef;        /* beta of the z-loss                                 */
    float temperature;        /* router softmax temperature; only 1 is supported   */
    int32_t credit_norm;      /* MOE_CREDIT_*                                       */
    int32_t capacity_priority; /* MOE_PRIORITY_*                                    */
    int32_t use_mlp_gater;    /* 1: logits from the MLP gate (SER "Configuration") */
    int32_t gater_hidden_dim; /* H of the MLP gate, 1..256 (default 128)           */
    int32_t ep_size;          /* expert-parallel group size G (1 = all experts here) */
    int32_t ep_rank;          /* this rank's place in it, 0..G-1                    */
} moe_config_t;

/* Defaults of the SER walkthrough's configuration: E=8, k=2, 512/1024/512,
 * GREEDY, alpha=0.01; plus no shared experts, C_f=1.25, GELU, beta=1e-3, BF16,
 * temperature 1. */
MOE_API moe_config_t moe_config_default(void);

/* Layer weights, BORROWED: the layer keeps the pointers (and TMA descriptors
 * built over them), so they must stay valid and at the same address until
 * moe_destroy. Their contents may change between forwards (e.g. an optimizer
 * step); each forward reads the current values. Shared experts are the last S
 * entries of the expert stacks (G = E + S groups).
 *   w_gate   [E][d]    fp32, router matrix W_g                     (required)
 *            [E][H]    with use_mlp_gater: the gate's output layer W_2
 *   b_gate   [E]       fp32, router bias (the gate's b_2)          (NULL = none)
 *   gater_w1 [H][d]    fp32, the MLP gate's hidden layer W_1        (required iff use_mlp_gater)
 *   gater_b1 [H]       fp32, its bias b_1                          (NULL = zero)
 * The MLP gate ("Code Walkthrough - SER": "via the router/router_bias linear
 * layer, or the optional MLP gate") is h = W_2 relu(W_1 x + b_1) + b_2.
 * With ep_size = G > 1 the expert stacks hold only this rank's E/G routed
 * experts (global ids ep_rank*E/G ..), then the S shared experts; the router
 * (w_gate, b_gate, sel_bias) covers all E experts.
 *   sel_bias [E]       fp32, selection bias b_i                    (required iff use_selection_bias)
 *   w1       [G][F][d] dtype, first expert layer (row f, column j) (required)
 *   b1       [G][F]    fp32                                        (NULL = zero)
 *   w2       [G][O][F] dtype, second expert layer                  (required)
 *   b2       [G][O]    fp32                                        (NULL = zero) */
typedef struct {
    const float *w_gate;
    const float *b_gate;
    const float *sel_bias;
    const void *w1;
    const void *w2;
    const float *b1;
    const float *b2;
    const float *gater_w1;
    const float *gater_b1;
} moe_weights_t;

/* Optional routing outputs of a forward (any pointer may be NULL; the struct
 * itself may be NULL). Written by moe_forward and read again by the
 * moe_aux_stats that follows, so they must not change in between.
 *   logits     [T][E] fp32  router logits h (clean: no noise, no selection bias)
 *   gates      [T][k] fp32  renormalised gates g, in top-k order
 *   topk_idx   [T][k] int32 selected experts, by descending selection key;
 *                           equal keys go to the lower expert index
 *   slot       [T][k] int32 rank in the expert's buffer (ascending token order),
 *                           or -1 if the assignment was dropped by the capacity cap
 *   count_pre  [E]    int32 selections per expert before the cap
 *   count_kept [E]    int32 assignments kept per expert (min(count_pre, C)) */
typedef struct {
    float *logits;
    float *gates;
    int32_t *topk_idx;
    int32_t *slot;
    int32_t *count_pre;
    int32_t *count_kept;
} moe_routing_t;

/* Statistics written by moe_aux_stats (device pointers; any may be NULL).
 * "Appendix C - Acronyms & Symbols", table "Balancing"; "Code Walkthrough -
 * SER", "Load balancing"; "Sparse MoE Expert-Credit Loss Reweighting Diagram",
 * panel (b).
 *   f           [E] fp32  f_i = count_pre_i / (k T)  (selections before the cap)
 *   p_mean      [E] fp32  P_i = mean over tokens of softmax(h)_i
 *   l_aux       [1] fp32  alpha E sum_i f_i P_i
 *   l_z         [1] fp32  beta mean_t (log sum_i e^{h_ti})^2
 *   n_dropped   [1] int32 assignments dropped by the capacity cap
 *   credit      [T][k] fp32 c = g ||o_e(x_t)||_2 for kept assignments, 0 if dropped
 *               (o_e = the expert's output before gate weighting, as stored)
 *   expert_loss [E] fp32  l_i = (1/T) sum_t credit_{t,i} token_loss_t over kept
 *               assignments; needs token_loss
 *   importance  [E] fp32  sum over the batch of the renormalised gates routed to
 *               expert i (every selection, before the cap)
 *   cv_load     [1] fp32  squared coefficient of variation of count_pre
 *               (population variance / mean^2; 0 for a zero mean)
 *   cv_importance [1] fp32 the same for importance
 *   l_total     [1] fp32  the walkthrough's weighted aux_loss: load_balance_coef
 *               * cv_load + l_z ("Load balancing": load_balance_coef * load_balance
 *               + z_loss_coef * z_loss, load_balance being the coefficient-of-
 *               variation style balance loss; l_z already carries z_loss_coef) */
typedef struct {
    float *f;
    float *p_mean;
    float *l_aux;
    float *l_z;
    int32_t *n_dropped;
    float *credit;
    float *expert_loss;
    float *importance;
    float *cv_load;
    float *cv_importance;
    float *l_total;
} moe_stats_t;

typedef struct moe_layer moe_layer_t; /* opaque; host state only */

/* Validate `cfg`, borrow `w` and build the layer's host state (tile plans and TMA
 * descriptors over the weights). No device memory is allocated and nothing is
 * enqueued. On success *out owns a layer to release with moe_destroy; on error
 * *out is set to NULL. Errors: INVALID_ARG (NULL pointer, dims out of range,
 * k > E, missing sel_bias), UNSUPPORTED (temperature != 1, a dim not a multiple
 * the BF16 path needs, E > 256), CUDA (no device or no sm_100 device). */
MOE_API int moe_layer_create(const moe_config_t *cfg, const moe_weights_t *w, moe_layer_t **out);

/* Bytes of device workspace a forward over T tokens needs (0 if T < 0 or the
 * layer is NULL). The workspace holds the permuted activations, the hidden
 * activations, the per-assignment expert outputs and the routing scratch. */
MOE_API size_t moe_workspace_bytes(const moe_layer_t *layer, int32_t T);

/* Capacity C = ceil(C_f k T / E) (T when C_f <= 0) that a forward over T tokens uses. */
MOE_API int64_t moe_capacity(const moe_layer_t *layer, int32_t T);

/* One layer forward over T >= 0 tokens.
 *   x           [T][d] dtype   input tokens                           (required if T > 0)
 *   logit_noise [T][E] fp32    noise added to the logits before selection;
 *                              required for NOISY, ignored for GREEDY
 *   workspace   >= moe_workspace_bytes(layer, T) bytes, 256-byte aligned, caller-owned;
 *               it must stay untouched until the moe_aux_stats that follows
 *   y           [T][O] dtype   output: sum of shared experts plus gate-weighted
 *                              kept routed experts                    (required if T > 0)
 *   routing     optional routing outputs (see moe_routing_t)
 * T = 0 is valid and enqueues nothing. Errors: INVALID_ARG, WORKSPACE, CUDA
 * (launch failure), INVALID_ARG if T > max_tokens. */
MOE_API int moe_forward(moe_layer_t *layer, const void *x, int32_t T, const float *logit_noise,
                void *workspace, size_t ws_bytes, void *y, const moe_routing_t *routing,
                void *stream);

/* Forward without a caller workspace. The source pages have no counterpart to
 * this call; it exists for callers that cannot allocate device memory
 * themselves, such as a plugin whose host application owns all device memory
 * through its own pool, or a latency-critical loop that must not call
 * cudaMalloc/cudaFree (they can synchronise the device).
 * Same arguments, outputs and errors as moe_forward, minus the workspace: the
 * scratch is a built-in device array of MOE_NOALLOC_SCRATCH_BYTES (64 MiB) that
 * every GPU loading this library holds until process exit. Nothing is allocated.
 *   - A T whose moe_workspace_bytes exceeds that size is rejected on the host
 *     with MOE_ERR_WORKSPACE and nothing is enqueued (at the default SER shape,
 *     512/1024/512 with 8 experts and 2 active, T = 4096 fits).
 *   - The first call on a device looks up the array's device address (with that
 *     device current); make that first call before any stream capture. The
 *     address is cached for the life of the process: after cudaDeviceReset (or
 *     anything else that destroys and re-creates the device's primary context)
 *     the cache is stale and this call must not be used on that device again.
 *   - All calls, on every layer and stream, share the one array and it keeps
 *     the previous call's contents. The forward re-initialises everything it
 *     reads (its control words are cleared at the start), but two calls whose
 *     work overlaps on the GPU race on the array: serialise them (one stream,
 *     or events). moe_aux_stats after this call reads the array too, so it must
 *     run before the next moe_forward_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
MOE_API int moe_forward_noalloc(moe_layer_t *layer, const void *x, int32_t T, const float *logit_noise, void *y,
                                const moe_routing_t *routing, void *stream);

/* Router planes kept across forwards (bf16 layers; no counterpart on the pages).
 * The tensor-core router reads the fp32 router matrix (w_gate, or the MLP gate's
 * gater_w1) as three bf16 planes hi + mid + lo, [E_pad][3 d] bf16, and by default
 * every forward splits it again into its workspace, one extra launch.
 * moe_prepare_router splits it once, enqueued on `stream`, into `planes`
 * (device, caller-owned, >= moe_router_planes_bytes(layer) bytes, 256-byte
 * aligned, valid until it is replaced or the layer is destroyed), and every later
 * forward of this layer reads the planes from there and does not split. The
 * planes hold the matrix as it was when this call ran: after changing the router
 * weights call it again. planes = NULL returns to splitting every forward.
 * Errors: INVALID_ARG, UNSUPPORTED (fp32 layers), WORKSPACE (too small or
 * misaligned), CUDA. moe_router_planes_bytes is 0 for fp32 layers or NULL. */
MOE_API size_t moe_router_planes_bytes(const moe_layer_t *layer);
MOE_API int moe_prepare_router(moe_layer_t *layer, void *planes, size_t bytes, void *stream);

/* Balancing and credit statistics of the most recent moe_forward on this layer,
 * computed from what that forward left in its workspace (and routing buffers).
 *   token_loss [T] fp32 per-token losses l_t (NULL: expert_loss is not written)
 * Errors: STATE if no forward has run, INVALID_ARG if out is NULL. */
MOE_API int moe_aux_stats(moe_layer_t *layer, const float *token_loss, const moe_stats_t *out,
                  void *stream);

/* Data-parallel statistics. The statistics are functions of sums that add over
 * token shards ("Appendix C", "Balancing": f_i and P_i are batch fractions and
 * means; the z-loss is a batch mean), so ranks that each run moe_forward on
 * their own tokens get the statistics of the whole batch from:
 *   1. moe_stat_partials: this rank's sums into `partials` (device, fp32,
 *      MOE_STAT_PARTIALS(E) floats):
 *        [0, E)  sum_t P[t][e]       [E, 2E)  selections per expert before the cap
 *        [2E]    sum_t lse_t^2       [2E+1]   T        [2E+2] dropped assignments
 *        [2E+3, 3E+3) sum over kept assignments of credit * token_loss
 *                     (zero when token_loss is NULL)
 *        [3E+3, 4E+3) importance: sum of the selections' gates per expert
 *      Counts travel as fp32 and are exact up to 2^24 per expert;
 *   2. a sum all-reduce of `partials` across the ranks (NCCL, by the caller);
 *   3. moe_stats_from_partials: every statistic of moe_stats_t except credit
 *      (per token; moe_aux_stats writes the local one) for the summed batch,
 *      expert_loss only when has_token_loss.
 * moe_aux_stats is steps 1 and 3 on this rank alone. Errors: STATE before any
 * forward, INVALID_ARG for NULL pointers. */
#define MOE_STAT_PARTIALS(E) (4 * (E) + 3)
MOE_API int moe_stat_partials(moe_layer_t *layer, const float *token_loss, float *partials, void *stream);
MOE_API int moe_stats_from_partials(moe_layer_t *layer, const float *partials, int32_t has_token_loss,
                                    const moe_stats_t *out, void *stream);

/* Aux-loss-free balancing ("Appendix C - Acronyms & Symbols", table
 * "Balancing": per-expert selection bias b_i, update rate gamma). Enqueues on
 * `stream`, for every expert e:
 *     sel_bias[e] += gamma * sign(k T / E - load_e)
 * where load_e is the expert's selection count before the cap: taken from
 * `partials` (MOE_STAT_PARTIALS(E) floats, e.g. summed across data-parallel
 * ranks, T from the same sums) or, when partials is NULL, from the most recent
 * moe_forward of this layer. The sign is decided on integers; the one fp32 add
 * is the only rounding. sel_bias: device [E] fp32, updated in place (pass the
 * layer's own weights->sel_bias to make the next forward use it). Errors:
 * INVALID_ARG (NULL sel_bias, NaN gamma), STATE (no partials and no forward). */
MOE_API int moe_update_selection_bias(moe_layer_t *layer, const float *partials, float gamma, float *sel_bias,
                                      void *stream);

/* Layer-wise reweighting bookkeeping ("Sparse MoE Expert-Credit Loss
 * Reweighting Diagram", panel (c)), enqueued on `stream` for one layer:
 *     lhat_e <- ema * lhat_e + (1 - ema) * expert_loss_e
 *     mu     <- softmax(mu + eta * lhat)          (mu as printed, not its log)
 *     *objective = sum_e mu_e * expert_loss_e     (updated mu; NULL to skip)
 * expert_loss: device [E] fp32 (e.g. moe_stats_t.expert_loss); lhat, mu: device
 * [E] fp32, updated in place; objective: device [1] fp32 or NULL. fp32, fixed
 * reduction order. Errors: INVALID_ARG for NULL arrays or non-finite ema/eta. */
MOE_API int moe_dro_update(moe_layer_t *layer, const float *expert_loss, float ema, float eta, float *lhat,
                           float *mu, float *objective, void *stream);

/* Expert parallelism ("Appendix C - Acronyms & Symbols", "Capacity &
 * communication": with expert-parallel degree G each device holds E/G experts
 * and tokens reach them by an all-to-all dispatch and come back by an
 * all-to-all combine). For layers created with ep_size = G > 1 (bf16 only);
 * moe_forward returns MOE_ERR_STATE for them. One forward on every rank:
 *   1. moe_ep_dispatch: router, top-k, dispatch with this rank's capacity
 *      C = ceil(C_f k T / E) over all E experts, and the rows of the kept
 *      assignments scattered into the row space (expert-major, each expert's
 *      rows padded to 32). Arguments as moe_forward without y.
 *   2. moe_ep_layout (synchronises `stream`): expert_rows (host [E]) = rows of
 *      each expert's padded segment; rows_in / rows_out = device pointers to the
 *      row space's input rows [sum expert_rows][d] (send buffer) and output rows
 *      [..][O] (receive buffer of step 5), valid until the next dispatch. The
 *      rows for rank q are the contiguous segments of experts q E/G ..
 *      (q+1) E/G - 1.
 *   3. the caller's all-to-all (e.g. NCCL): send each rank its segments and
 *      its E/G expert_rows entries; receive R rows, source-major.
 *   4. moe_ep_experts: the expert MLPs of this rank's experts on the received
 *      rows: recv_x [R][d] bf16, recv_rows device [G][E/G] int32 (padded rows
 *      per source and local expert, summing to R), recv_out [R][O] bf16 out;
 *      workspace of moe_ep_experts_workspace_bytes(R) bytes, 256-byte aligned.
 *      R must be a multiple of 32.
 *   5. the caller's all-to-all back: recv_out rows to their sources, into
 *      rows_out at the positions their inputs left from.
 *   6. moe_ep_combine: the shared experts on this rank's tokens and the
 *      gate-weighted combine into y [T][O]; moe_aux_stats may follow.
 * x and the workspace of step 1 must stay valid and unchanged until step 6 (the
 * shared experts read x there).
 * Errors: STATE for layers with ep_size 1 or calls out of order, INVALID_ARG,
 * WORKSPACE, CUDA as elsewhere. */
MOE_API int moe_ep_dispatch(moe_layer_t *layer, const void *x, int32_t T, const float *logit_noise, void *workspace,
                            size_t ws_bytes, const moe_routing_t *routing, void *stream);
MOE_API int moe_ep_layout(moe_layer_t *layer, int32_t *expert_rows, void **rows_in, void **rows_out, void *stream);
MOE_API size_t moe_ep_experts_workspace_bytes(const moe_layer_t *layer, int32_t R);
MOE_API int moe_ep_experts(moe_layer_t *layer, const void *recv_x, const int32_t *recv_rows, int32_t R,
                           void *recv_out, void *workspace, size_t ws_bytes, void *stream);
MOE_API int moe_ep_combine(moe_layer_t *layer, void *y, void *stream);

/* Self-check of the bounded waits the tcgen05 kernels rely on (no counterpart
 * on the pages): one GPU thread waits on an mbarrier that nothing arrives on;
 * after the wait limit (2 s) it records the timeout and returns, as every role
 * of the expert GEMM and router kernels does when a wait runs out. Synchronises
 * `stream`. Returns MOE_OK when the timeout was detected and reported as
 * designed (the context stays usable), MOE_ERR_INTERNAL if it was not,
 * MOE_ERR_CUDA on a CUDA error. Takes about two seconds. */
MOE_API int moe_selftest_bounded_wait(void *stream);

/* Self-check of the bounded waits inside the real expert GEMM (no counterpart on
 * the pages): one moe_forward of this layer over x [T][d] (GREEDY top-k, bf16,
 * ep_size 1, d >= 192) with workspace and y as for moe_forward, in which the
 * expert-GEMM launch's leader CTAs announce the bytes of their third pipeline
 * stage but load none of them, and every wait of that launch gives up after
 * 20 ms. The MMA role's wait runs out, the kernel's roles stop (those waiting
 * for a token tile's GEMM 1 rows too), drain their copies and MMAs and free
 * TMEM, the rest of the forward runs on the unfinished outputs (y is
 * unspecified), and moe_device_status then reports MOE_ERR_TIMEOUT. Synchronises
 * `stream`. Returns MOE_OK when the timeout was detected and reported, MOE_ERR_
 * INTERNAL if it was not, the errors of moe_forward otherwise. The layer and
 * context stay usable: the next moe_forward runs normally. */
MOE_API int moe_selftest_gemm_timeout(moe_layer_t *layer, const void *x, int32_t T, void *workspace, size_t ws_bytes,
                                      void *y, void *stream);

/* Self-check of the bounded waits inside the fused router (no counterpart on
 * the pages; failure detection): runs the router of a forward alone (no
 * dispatch, expert GEMMs or combine), with a test-only launch argument that
 * makes every CTA pair's leader skip its loads of the third pipeline stage and
 * every wait of the launch give up after 20 ms. The MMA role's wait runs out,
 * every role stops, copies in flight land, the CTAs pass the grid barrier
 * without routing, both CTAs of each pair meet at the cluster barrier and TMEM
 * is freed. Synchronises `stream`; returns MOE_OK if the status word reports
 * the timeout, MOE_ERR_INTERNAL if it does not, the argument errors of
 * moe_forward otherwise (GREEDY bf16 layers with a linear router and
 * input_dim >= 192 only). The routing outputs are left incomplete, so the
 * layer then has no forward for moe_aux_stats; the next moe_forward runs
 * normally on the same layer and context. */
MOE_API int moe_selftest_router_timeout(moe_layer_t *layer, const void *x, int32_t T, void *workspace,
                                        size_t ws_bytes, void *stream);

/* Device status word of the most recent forward: synchronises `stream`, then
 * returns MOE_OK, or MOE_ERR_TIMEOUT if a bounded device-side wait gave up. */
MOE_API int moe_device_status(moe_layer_t *layer, void *stream);

/* Optional stage timing with caller-owned CUDA events (cudaEvent_t passed as
 * void*, created with timing enabled). After this call every moe_forward records
 *   events[0] before the router,        events[1] after the router,
 *   events[2] after the dispatch,       events[3] after the row scatter that
 *                                       feeds expert GEMM 1 (fp32 layers have
 *                                       none: events[3] follows events[2]),
 *   events[4] after expert GEMM 1,      events[5] after expert GEMM 2,
 *   events[6] after the combine,
 * (moe_forward of a bf16 layer runs both expert GEMMs in one launch, so that
 * GEMM 2 starts on a token tile as soon as GEMM 1 has stored its hidden rows:
 * events[4] and events[5] then both follow that launch, and events[3]..
 * events[5] time the two GEMMs together)
 * and every moe_aux_stats records events[7] after its kernels, all on the
 * call's stream. The array is copied; events == NULL turns timing off. Nothing
 * is allocated and nothing synchronises. */
#define MOE_TIMING_EVENTS 8
MOE_API int moe_set_timing_events(moe_layer_t *layer, void *const *events);

/* Number of kernels the most recent moe_forward plus moe_aux_stats enqueued. */
MOE_API int32_t moe_launch_count(const moe_layer_t *layer);

/* Release the layer's host state (NULL is a no-op). Borrowed weights are untouched. */
MOE_API void moe_destroy(moe_layer_t *layer);

/* Static name of a status code ("MOE_OK", "MOE_ERR_INVALID_ARG", ...). */
MOE_API const char *moe_status_string(int status);

/* Message of the last error on the calling thread ("" if none). */
MOE_API const char *moe_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
