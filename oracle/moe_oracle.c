/*
 * moe_oracle.c - CPU reference for the sparse top-k MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY (see moe_oracle.h): plain loops in double, written to
 * be read against the pages, not to be fast. Build with -O2 -ffp-contract=off and
 * without fast-math, so that every expression rounds as written.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

double orc_load(const void *base, int64_t i, int dtype)
{
    if (dtype == ORC_F32)
        return (double)((const float *)base)[i];
    /* bf16 is the top half of an IEEE fp32 word: widening is a 16-bit shift. */
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Appendix C, "Core MoE symbols": h = W_g x (one score per expert); the linear
 * router of the SER walkthrough adds router_bias. */
void orc_router_logits(int T, int d, int E, const void *x, int x_dtype,
                       const float *w_gate, const float *b_gate, double *h)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < E; ++i) {
            double s = 0.0;
            for (int j = 0; j < d; ++j)
                s += (double)w_gate[(int64_t)i * d + j] * orc_load(x, (int64_t)t * d + j, x_dtype);
            if (b_gate)
                s += (double)b_gate[i];
            h[(int64_t)t * E + i] = s;
        }
    }
}

/* Appendix C: P = softmax(h) and the log-partition log sum_i e^{h_i}. The max is
 * subtracted first so that exp never overflows; the result is the same function. */
void orc_softmax_lse(int T, int E, const double *h, double *P, double *lse)
{
    for (int t = 0; t < T; ++t) {
        const double *ht = h + (int64_t)t * E;
        double m = ht[0];
        for (int i = 1; i < E; ++i)
            if (ht[i] > m)
                m = ht[i];
        double z = 0.0;
        for (int i = 0; i < E; ++i)
            z += exp(ht[i] - m);
        for (int i = 0; i < E; ++i)
            P[(int64_t)t * E + i] = exp(ht[i] - m) / z;
        lse[t] = m + log(z);
    }
}

/* SER walkthrough, gating path (noise added to the logits before selection) and
 * Appendix C, "Balancing" (selection bias b_i): one fp32 add, rounded to nearest. */
void orc_selection_keys(int T, int E, const float *h32, const float *noise,
                        const float *sel_bias, float *key)
{
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < E; ++i) {
            int64_t a = (int64_t)t * E + i;
            volatile float v = h32[a];
            if (noise)
                v = h32[a] + noise[a];
            else if (sel_bias)
                v = h32[a] + sel_bias[i];
            key[a] = v;
        }
    }
}

/* Appendix C, T_k(x): the k highest-scoring experts. Selection by k passes of an
 * arg-max over the experts not yet taken; scanning in ascending index with a
 * strict ">" gives equal keys to the lower index. */
void orc_topk(int T, int E, int k, const float *key, int32_t *idx)
{
    char *taken = (char *)malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        const float *kt = key + (int64_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int r = 0; r < k; ++r) {
            int best = -1;
            for (int i = 0; i < E; ++i) {
                if (taken[i])
                    continue;
                if (best < 0 || kt[i] > kt[best])
                    best = i;
            }
            taken[best] = 1;
            idx[(int64_t)t * k + r] = best;
        }
    }
    free(taken);
}

/* Appendix C: g_i, the renormalised probability of a selected expert. */
void orc_gates(int T, int E, int k, const double *P, const int32_t *idx, double *g)
{
    for (int t = 0; t < T; ++t) {
        double s = 0.0;
        for (int r = 0; r < k; ++r)
            s += P[(int64_t)t * E + idx[(int64_t)t * k + r]];
        for (int r = 0; r < k; ++r)
            g[(int64_t)t * k + r] = P[(int64_t)t * E + idx[(int64_t)t * k + r]] / s;
    }
}

/* Appendix C, "Capacity & communication": C = ceil(C_f k T / E). */
int64_t orc_capacity(double capacity_factor, int k, int T, int E)
{
    if (capacity_factor <= 0.0)
        return (int64_t)T;
    return (int64_t)ceil(capacity_factor * (double)k * (double)T / (double)E);
}

/* Appendix C (dispatch into fixed buffers of C) and the SER walkthrough's hard
 * capacity cap: every expert keeps a queue; tokens join it in ascending order. */
void orc_dispatch(int T, int E, int k, int64_t C, const int32_t *idx, int32_t *slot,
                  int32_t *count_pre, int32_t *count_kept, int32_t *n_dropped)
{
    for (int e = 0; e < E; ++e)
        count_pre[e] = 0;
    for (int t = 0; t < T; ++t) {
        for (int r = 0; r < k; ++r) {
            int e = idx[(int64_t)t * k + r];
            int32_t rank = count_pre[e];
            count_pre[e] = rank + 1;
            slot[(int64_t)t * k + r] = (rank < C) ? rank : -1;
        }
    }
    int32_t dropped = 0;
    for (int e = 0; e < E; ++e) {
        count_kept[e] = (count_pre[e] < C) ? count_pre[e] : (int32_t)C;
        dropped += count_pre[e] - count_kept[e];
    }
    *n_dropped = dropped;
}

/* Capacity cap with rank-major priority: queues filled choice by choice. */
void orc_dispatch_rank_major(int T, int E, int k, int64_t C, const int32_t *idx, int32_t *slot,
                             int32_t *count_pre, int32_t *count_kept, int32_t *n_dropped)
{
    for (int e = 0; e < E; ++e)
        count_pre[e] = 0;
    for (int r = 0; r < k; ++r) {
        for (int t = 0; t < T; ++t) {
            int e = idx[(int64_t)t * k + r];
            int32_t rank = count_pre[e];
            count_pre[e] = rank + 1;
            slot[(int64_t)t * k + r] = (rank < C) ? rank : -1;
        }
    }
    int32_t dropped = 0;
    for (int e = 0; e < E; ++e) {
        count_kept[e] = (count_pre[e] < C) ? count_pre[e] : (int32_t)C;
        dropped += count_pre[e] - count_kept[e];
    }
    *n_dropped = dropped;
}

/* SER walkthrough: the optional MLP gate, h = W_2 relu(W_1 x + b_1) + b_2. */
void orc_router_mlp(int T, int d, int H, int E, const void *x, int x_dtype, const float *w1,
                    const float *b1, const float *w2, const float *b2, double *h)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        double *z = (double *)malloc(sizeof(double) * (size_t)H);
        for (int u = 0; u < H; ++u) {
            double s = 0.0;
            for (int j = 0; j < d; ++j)
                s += (double)w1[(int64_t)u * d + j] * orc_load(x, (int64_t)t * d + j, x_dtype);
            if (b1)
                s += (double)b1[u];
            z[u] = s > 0.0 ? s : 0.0;
        }
        for (int i = 0; i < E; ++i) {
            double s = 0.0;
            for (int u = 0; u < H; ++u)
                s += (double)w2[(int64_t)i * H + u] * z[u];
            if (b2)
                s += (double)b2[i];
            h[(int64_t)t * E + i] = s;
        }
        free(z);
    }
}

static double activation(int act, double z)
{
    switch (act) {
    case ORC_ACT_RELU:
        return z > 0.0 ? z : 0.0;
    case ORC_ACT_GELU:
        return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));
    default: /* Swish: z * sigmoid(z) */
        return z / (1.0 + exp(-z));
    }
}

/* SER walkthrough: the first half of an expert's MLP, a = act(w1 x + b1). */
static void expert_hidden(int d, int F, int act, int w_dtype, const orc_expert *ex, const double *x,
                          double *a)
{
    for (int f = 0; f < F; ++f) {
        double z = 0.0;
        for (int j = 0; j < d; ++j)
            z += orc_load(ex->w1, (int64_t)f * d + j, w_dtype) * x[j];
        if (ex->b1)
            z += (double)ex->b1[f];
        a[f] = activation(act, z);
    }
}

/* SER walkthrough: an expert's two-layer MLP, w1/b1 -> activation -> w2/b2. */
void orc_expert_ffn(int d, int F, int O, int act, int w_dtype, const orc_expert *ex,
                    const double *x, double *o)
{
    double *a = (double *)malloc(sizeof(double) * (size_t)F);
    expert_hidden(d, F, act, w_dtype, ex, x, a);
    for (int n = 0; n < O; ++n) {
        double s = 0.0;
        for (int f = 0; f < F; ++f)
            s += orc_load(ex->w2, (int64_t)n * F + f, w_dtype) * a[f];
        if (ex->b2)
            s += (double)ex->b2[n];
        o[n] = s;
    }
    free(a);
}

/* SER walkthrough (gate-weighted combine of the expert outputs), Appendix C
 * (combine tensor; shared always-on experts) and the credit diagram, panel (b):
 * c = g * ||o||_2 for each kept assignment. */
void orc_experts_combine(int n_tokens, const int32_t *tokens, int T, int d, int F, int O,
                         int E, int S, int k, int act, int x_dtype, int w_dtype,
                         const void *x, const orc_expert *experts, const int32_t *idx,
                         const int32_t *slot, const double *g, double *y, double *credit)
{
    (void)T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int j = 0; j < n_tokens; ++j) {
        int t = tokens[j];
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *o = (double *)malloc(sizeof(double) * (size_t)O);
        double *yj = y + (int64_t)j * O;
        for (int c = 0; c < d; ++c)
            xt[c] = orc_load(x, (int64_t)t * d + c, x_dtype);
        for (int n = 0; n < O; ++n)
            yj[n] = 0.0;
        for (int s = 0; s < S; ++s) {
            orc_expert_ffn(d, F, O, act, w_dtype, &experts[E + s], xt, o);
            for (int n = 0; n < O; ++n)
                yj[n] += o[n];
        }
        for (int r = 0; r < k; ++r) {
            int64_t a = (int64_t)t * k + r;
            double c = 0.0;
            if (slot[a] >= 0) {
                orc_expert_ffn(d, F, O, act, w_dtype, &experts[idx[a]], xt, o);
                double ss = 0.0;
                for (int n = 0; n < O; ++n) {
                    yj[n] += g[a] * o[n];
                    ss += o[n] * o[n];
                }
                c = g[a] * sqrt(ss);
            }
            if (credit)
                credit[(int64_t)j * k + r] = c;
        }
        free(o);
        free(xt);
    }
}

/* Credit diagram, panel (b), with ||h|| read as the hidden activation's norm. */
void orc_experts_credit_hidden(int n_tokens, const int32_t *tokens, int d, int F, int E, int k,
                               int act, int x_dtype, int w_dtype, const void *x,
                               const orc_expert *experts, const int32_t *idx, const int32_t *slot,
                               const double *g, double *credit)
{
    (void)E;
#pragma omp parallel for schedule(dynamic, 1)
    for (int j = 0; j < n_tokens; ++j) {
        int t = tokens[j];
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *a = (double *)malloc(sizeof(double) * (size_t)F);
        for (int c = 0; c < d; ++c)
            xt[c] = orc_load(x, (int64_t)t * d + c, x_dtype);
        for (int r = 0; r < k; ++r) {
            int64_t as = (int64_t)t * k + r;
            double c = 0.0;
            if (slot[as] >= 0) {
                expert_hidden(d, F, act, w_dtype, &experts[idx[as]], xt, a);
                double ss = 0.0;
                for (int f = 0; f < F; ++f)
                    ss += a[f] * a[f];
                c = g[as] * sqrt(ss);
            }
            credit[(int64_t)j * k + r] = c;
        }
        free(a);
        free(xt);
    }
}

/* Credit diagram, panel (c): EMA of the expert losses, mu <- softmax(mu + eta lhat),
 * and sum_i mu_i l_i. */
double orc_dro_update(int E, double ema, double eta, const double *l, double *lhat, double *mu)
{
    double m = -INFINITY;
    for (int i = 0; i < E; ++i) {
        lhat[i] = ema * lhat[i] + (1.0 - ema) * l[i];
        const double z = mu[i] + eta * lhat[i];
        if (z > m)
            m = z;
    }
    double s = 0.0;
    for (int i = 0; i < E; ++i)
        s += exp(mu[i] + eta * lhat[i] - m);
    double obj = 0.0;
    for (int i = 0; i < E; ++i) {
        mu[i] = exp(mu[i] + eta * lhat[i] - m) / s;
        obj += mu[i] * l[i];
    }
    return obj;
}

/* Appendix C, "Balancing": f_i, P_i, L_aux = alpha E sum_i f_i P_i and the router
 * z-loss beta * mean_t (log sum_i e^{h_i})^2. */
void orc_balance_stats(int T, int E, int k, const double *P, const double *lse,
                       const int32_t *count_pre, double alpha, double beta,
                       double *f, double *p_mean, double *l_aux, double *l_z)
{
    double aux = 0.0;
    for (int i = 0; i < E; ++i) {
        double s = 0.0;
        for (int t = 0; t < T; ++t)
            s += P[(int64_t)t * E + i];
        p_mean[i] = s / (double)T;
        f[i] = (double)count_pre[i] / ((double)k * (double)T);
        aux += f[i] * p_mean[i];
    }
    *l_aux = alpha * (double)E * aux;
    double z = 0.0;
    for (int t = 0; t < T; ++t)
        z += lse[t] * lse[t];
    *l_z = beta * z / (double)T;
}

/* Credit diagram, panel (b): l_i = (1/N) sum_j c_i(x_j) l_j 1[i in T_j], N = T. */
void orc_expert_loss(int T, int E, int k, const int32_t *idx, const int32_t *slot,
                     const double *credit, const float *token_loss, double *expert_loss)
{
    for (int i = 0; i < E; ++i)
        expert_loss[i] = 0.0;
    for (int t = 0; t < T; ++t)
        for (int r = 0; r < k; ++r) {
            int64_t a = (int64_t)t * k + r;
            if (slot[a] >= 0)
                expert_loss[idx[a]] += credit[a] * (double)token_loss[t];
        }
    for (int i = 0; i < E; ++i)
        expert_loss[i] /= (double)T;
}

/* Load balancing: importance = sum of routed gate weights per expert. */
void orc_importance(int T, int E, int k, const int32_t *idx, const double *g, double *imp)
{
    for (int i = 0; i < E; ++i)
        imp[i] = 0.0;
    for (int t = 0; t < T; ++t)
        for (int r = 0; r < k; ++r)
            imp[idx[(int64_t)t * k + r]] += g[(int64_t)t * k + r];
}

/* Load balancing: squared coefficient of variation (population variance). */
double orc_cv_squared(int n, const double *v)
{
    double mean = 0.0;
    for (int i = 0; i < n; ++i)
        mean += v[i];
    mean /= (double)n;
    if (mean == 0.0)
        return 0.0;
    double var = 0.0;
    for (int i = 0; i < n; ++i)
        var += (v[i] - mean) * (v[i] - mean);
    var /= (double)n;
    return var / (mean * mean);
}

/* Load balancing: aux_loss = load_balance_coef * (CV^2 of the selection counts)
 * + z_loss_coef * mean_t lse_t^2. */
double orc_aux_loss(int T, int E, const int32_t *count_pre, const double *lse, double load_balance_coef,
                    double z_loss_coef)
{
    double *load = (double *)malloc(sizeof(double) * (size_t)E);
    for (int i = 0; i < E; ++i)
        load[i] = (double)count_pre[i];
    const double balance = orc_cv_squared(E, load);
    free(load);
    double z = 0.0;
    for (int t = 0; t < T; ++t) {
        const double v = lse[t];
        z += v * v;
    }
    return load_balance_coef * balance + z_loss_coef * (z / (double)T);
}

/* Balancing: b_i <- b_i + gamma sign(kT/E - load_i), rounded to fp32. */
void orc_selection_bias_update(int E, int k, int64_t T, const int64_t *load, float gamma, float *b)
{
    for (int i = 0; i < E; ++i) {
        const int64_t diff = (int64_t)k * T - (int64_t)E * load[i];
        const double s = diff > 0 ? 1.0 : (diff < 0 ? -1.0 : 0.0);
        b[i] = (float)((double)b[i] + (double)gamma * s);
    }
}

#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the parallel loops above will use (1 without OpenMP). */
int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
