/*
 * moe_oracle.h - CPU reference ("oracle") for the sparse top-k MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY. This is the plain, slow, fp64 definition of what the
 * layer computes. The tests, the smoke check and the benchmark's CPU-baseline leg
 * call it to check and to time the CUDA path; the product path never calls,
 * links or includes it, and it shares no code, header or table with the CUDA
 * sources.
 *
 * Sources, by page and section:
 *   [C]  "Appendix C - Acronyms & Symbols" (MoE course): tables "Core MoE symbols",
 *        "Parameter accounting", "Balancing", "Capacity & communication".
 *   [D]  "Sparse MoE Expert-Credit Loss Reweighting Diagram": "What the diagram
 *        shows", panel (b) (expert credit and expert-attributed loss).
 *   [W]  "Code Walkthrough - SER (Sparse Expert Routing)": sections
 *        "Configuration", "The gating / routing path", "Load balancing".
 *
 * Readings taken where the pages leave a step open (each is also listed with its
 * reason in the design notes):
 *   - noise and the selection bias change only which experts are selected; gates,
 *     P_i and the z-loss use the clean logits h;
 *   - the selection key is formed in fp32 with one round-to-nearest add, the same
 *     precision the GPU takes that integer decision in;
 *   - top-k ties go to the lower expert index; indices are listed by descending key;
 *   - capacity priority is ascending token index; f_i counts selections before
 *     capacity drops; gates are not renormalised after a drop;
 *   - shared experts have weight 1; N in the attributed loss is T; the credit's
 *     ||h|| is the norm of the expert's output before gate weighting, and p is the
 *     renormalised gate g.
 *
 * Every array is row-major and caller-owned. Floating-point work is in double;
 * bf16 operands are passed as their raw 16-bit patterns and widened exactly.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_ACT_RELU = 0, ORC_ACT_GELU = 1, ORC_ACT_SWISH = 2 };
enum { ORC_BF16 = 0, ORC_F32 = 1 };

/* Exact widening of one stored element (bf16 bit pattern or fp32) to double. */
double orc_load(const void *base, int64_t i, int dtype);

/* [C] "Core MoE symbols": router logits h = W_g x, one score per expert; [W]
 * "The gating / routing path": the linear router has a bias (router_bias).
 * x [T][d] (dtype x_dtype), w_gate [E][d] fp32, b_gate [E] fp32 or NULL -> h [T][E]. */
void orc_router_logits(int T, int d, int E, const void *x, int x_dtype,
                       const float *w_gate, const float *b_gate, double *h);

/* [C] "Core MoE symbols": P = softmax(h); [C] "Balancing": log sum_i e^{h_i}
 * (the z-loss argument). h [T][E] -> P [T][E], lse [T]. */
void orc_softmax_lse(int T, int E, const double *h, double *P, double *lse);

/* [W] "The gating / routing path" (noisy top-k adds noise to the logits before
 * selection) and [C] "Balancing" (per-expert selection bias b_i): the key is
 * fl32(h32 + noise32) or fl32(h32 + b32), or h32 itself when both are NULL.
 * h32 [T][E], noise [T][E] or NULL, sel_bias [E] or NULL -> key [T][E]. */
void orc_selection_keys(int T, int E, const float *h32, const float *noise,
                        const float *sel_bias, float *key);

/* [C] "Core MoE symbols" T_k(x) and "Acronyms" top-k: the indices of the k
 * largest keys, largest first; equal keys go to the lower expert index.
 * key [T][E] -> idx [T][k]. */
void orc_topk(int T, int E, int k, const float *key, int32_t *idx);

/* [C] "Core MoE symbols": g_i is the renormalised probability of selected
 * expert i: g_r = P[idx_r] / sum_r' P[idx_r']. P [T][E], idx [T][k] -> g [T][k]. */
void orc_gates(int T, int E, int k, const double *P, const int32_t *idx, double *g);

/* [C] "Capacity & communication": C = ceil(C_f k T / E); C_f <= 0 means no
 * limit, and C = T then (no expert can receive more than T assignments). */
int64_t orc_capacity(double capacity_factor, int k, int T, int E);

/* [C] "Capacity & communication" (dispatch tensor D, fixed buffer of C per
 * expert) and [W] "Load balancing" (hard capacity cap that drops overflow).
 * Each expert's assignments are ranked in ascending token order; an assignment
 * is kept iff its rank < C. slot [T][k] = rank or -1 if dropped;
 * count_pre [E] = selections before the cap; count_kept [E]; *n_dropped. */
void orc_dispatch(int T, int E, int k, int64_t C, const int32_t *idx, int32_t *slot,
                  int32_t *count_pre, int32_t *count_kept, int32_t *n_dropped);

/* The same capacity cap with GShard's rank-major priority (the reading of
 * "Capacity & communication" taken for capacity_priority = rank): every token's
 * first choice joins the queues in token order, then every token's second
 * choice, and so on. Outputs as orc_dispatch. */
void orc_dispatch_rank_major(int T, int E, int k, int64_t C, const int32_t *idx, int32_t *slot,
                             int32_t *count_pre, int32_t *count_kept, int32_t *n_dropped);

/* [W] "Configuration" (use_mlp_gater, gater_hidden_dim) and "The gating /
 * routing path" (gate logits "via the router/router_bias linear layer, or the
 * optional MLP gate"): h = W_2 relu(W_1 x + b_1) + b_2 with hidden width H.
 * x [T][d] (x_dtype), w1 [H][d], b1 [H] or NULL, w2 [E][H], b2 [E] or NULL (fp32)
 * -> h [T][E]. */
void orc_router_mlp(int T, int d, int H, int E, const void *x, int x_dtype, const float *w1,
                    const float *b1, const float *w2, const float *b2, double *h);

/* One expert's weights ([C] "Core MoE symbols": expert i is an FFN with its own
 * weights; [W]: w1/b1 -> activation -> w2/b2). w1 [F][d], w2 [O][F] in w_dtype;
 * b1 [F], b2 [O] fp32 or NULL. */
typedef struct {
    const void *w1;
    const float *b1;
    const void *w2;
    const float *b2;
} orc_expert;

/* [W] "The gating / routing path": o = w2 act(w1 x + b1) + b2 with act one of
 * ReLU, GELU (exact erf form) and Swish (z * sigmoid(z)). x [d] -> o [O]. */
void orc_expert_ffn(int d, int F, int O, int act, int w_dtype, const orc_expert *ex,
                    const double *x, double *o);

/* [W] "The gating / routing path" (expert outputs combined, weighted by the
 * gates), [C] "Capacity & communication" (combine tensor: gate-weighted
 * un-scatter) and [C] "Parameter accounting" (shared always-on experts), with
 * the credit of [D] panel (b).
 * For each listed token t = tokens[j]:
 *   y[j] = sum_{s<S} o_{E+s}(x_t) + sum_{r<k, slot[t][r] >= 0} g[t][r] o_{idx[t][r]}(x_t)
 *   credit[j][r] = g[t][r] * ||o_{idx[t][r]}(x_t)||_2 if kept, else 0.
 * experts has E+S entries (shared last); entries no listed token uses may hold
 * NULL pointers. x [T][d] (x_dtype); idx, slot [T][k]; g [T][k] double ->
 * y [n_tokens][O], credit [n_tokens][k] (NULL to skip). Tokens are processed
 * independently, optionally in parallel. */
void orc_experts_combine(int n_tokens, const int32_t *tokens, int T, int d, int F, int O,
                         int E, int S, int k, int act, int x_dtype, int w_dtype,
                         const void *x, const orc_expert *experts, const int32_t *idx,
                         const int32_t *slot, const double *g, double *y, double *credit);

/* [D] panel (b), second reading of ||h_{l,i}||: the norm of expert i's hidden
 * activation a = act(w1 x + b1) (length F) instead of its output. For each listed
 * token t = tokens[j]: credit[j][r] = g[t][r] * ||a_{idx[t][r]}(x_t)||_2 if kept,
 * else 0. Arguments as orc_experts_combine. */
void orc_experts_credit_hidden(int n_tokens, const int32_t *tokens, int d, int F, int E, int k,
                               int act, int x_dtype, int w_dtype, const void *x,
                               const orc_expert *experts, const int32_t *idx, const int32_t *slot,
                               const double *g, double *credit);

/* [D] panel (c), the layer-wise bookkeeping: the EMA tracker
 *   lhat_i <- ema * lhat_i + (1 - ema) * l_i,
 * the expert weights mu <- softmax(mu + eta * lhat) (mu as printed, not its log),
 * and the objective term of this layer sum_i mu_i l_i with the updated mu.
 * l [E]; lhat, mu [E] updated in place; returns the objective term. */
double orc_dro_update(int E, double ema, double eta, const double *l, double *lhat, double *mu);

/* [C] "Balancing": f_i = fraction of the batch's selections dispatched to expert
 * i (count_pre_i / (k T)), P_i = mean_t P[t][i], L_aux = alpha E sum_i f_i P_i,
 * L_z = beta mean_t lse_t^2. */
void orc_balance_stats(int T, int E, int k, const double *P, const double *lse,
                       const int32_t *count_pre, double alpha, double beta,
                       double *f, double *p_mean, double *l_aux, double *l_z);

/* [D] panel (b): expert-attributed loss
 * l_i = (1/T) sum_t sum_r [idx[t][r] = i and kept] credit[t][r] * token_loss[t].
 * credit [T][k] double, token_loss [T] fp32 -> expert_loss [E]. */
void orc_expert_loss(int T, int E, int k, const int32_t *idx, const int32_t *slot,
                     const double *credit, const float *token_loss, double *expert_loss);

/* Threads the oracle's parallel loops use (1 when built without OpenMP). */
/* [W] "Load balancing": an importance loss "balances total importance per
 * expert". Importance of expert i = the sum over the batch of the gate weights
 * routed to it (renormalised gates g, every selection, before capacity drops).
 * idx, g [T][k] -> imp [E]. */
void orc_importance(int T, int E, int k, const int32_t *idx, const double *g, double *imp);

/* [W] "Load balancing": a "coefficient-of-variation style balance across
 * experts". Squared coefficient of variation of v[0..n): population variance
 * over the squared mean (0 when the mean is 0). */
double orc_cv_squared(int n, const double *v);

/* [W] "Load balancing": the weighted combination the walkthrough's aux_loss
 * returns, load_balance_coef * load_balance + z_loss_coef * z_loss. Its
 * load_balance term is the walkthrough's coefficient-of-variation style balance
 * loss (the squared coefficient of variation of the per-expert selection counts
 * before capacity, as orc_cv_squared), its z_loss term the mean over tokens of
 * the squared log-partition. count_pre [E], lse [T]. */
double orc_aux_loss(int T, int E, const int32_t *count_pre, const double *lse, double load_balance_coef,
                    double z_loss_coef);

/* [C] "Balancing": per-expert selection bias b_i (aux-loss-free balancing) with
 * update rate gamma: b_i <- b_i + gamma * sign(mean load - load_i), load_i =
 * selections of expert i before capacity, mean load = k T / E (the sign is
 * decided exactly, on k T - E load_i). The sum is rounded once to the bias's
 * fp32 storage. load [E]; b [E] updated in place. */
void orc_selection_bias_update(int E, int k, int64_t T, const int64_t *load, float gamma, float *b);

int orc_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif
