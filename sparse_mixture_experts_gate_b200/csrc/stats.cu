// stats.cu - balancing and credit statistics of one layer forward.
//
// "Appendix C - Acronyms & Symbols", table "Balancing": f_i (fraction of the
// batch's selections dispatched to expert i, counted before capacity drops),
// P_i (mean router mass on expert i), L_aux = alpha E sum_i f_i P_i and the
// router z-loss beta * mean_t (log sum_i e^{h_ti})^2. "Sparse MoE Expert-Credit
// Loss Reweighting Diagram", panel (b): the expert-attributed loss
// l_i = (1/N) sum_j c_i(x_j) l_j 1[i in T_j], N = T, over kept assignments.
//
// The statistics are a function of sums that add over token shards, so they are
// computed in two steps: partial sums over this forward's tokens, then the
// statistics from (local, or all-reduced across data-parallel ranks) sums.
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Partial sums (additive over token shards), layout of moe_stat_partials:
//   [0, E)       sum_t P[t][e]          [E, 2E)      selections before the cap
//   [2E]         sum_t lse_t^2          [2E+1]       T
//   [2E+2]       dropped assignments    [2E+3, 3E+3) sum over kept assignments
//                                                    of credit * token_loss
//   [3E+3, 4E+3) importance: sum of the selections' gates per expert
// Sum over the 256 threads of one CTA in a fixed order (shuffle tree, then the
// eight warp sums in order); every thread gets the result.
__device__ __forceinline__ float block_sum_256(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    __syncthreads();  // `red` may still be read from a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w];
    return t;
}

__device__ __forceinline__ void finalize_body(const FinalizeArgs &a, float *red);

// One CTA per expert (CTA E does the per-token scalars); every sum has a fixed
// order (thread-strided, then a fixed shuffle tree and warp order), so repeated
// runs give bit-identical results. With `fin` set, the CTA that writes the last
// partial words (counted on done_counter) also forms the statistics from them,
// so that moe_aux_stats is one launch; it leaves the counter at zero again.
__global__ void __launch_bounds__(256) stat_partials_kernel(StatsArgs a, FinalizeArgs fin, int fuse) {
    __shared__ float red[8];
    __shared__ int last;
    const int tid = threadIdx.x;
    if (blockIdx.x == a.E) {  // sum_t lse_t^2, T, drops
        float z = 0.f;
        for (int t = tid; t < a.T; t += 256) z = fmaf(a.lse[t], a.lse[t], z);
        z = block_sum_256(z, red);
        if (tid == 0) {
            a.partials[2 * a.E] = z;
            a.partials[2 * a.E + 1] = (float)a.T;
            a.partials[2 * a.E + 2] = (float)a.ctrl[kCtrlDropped];
        }
    } else {
        const int e = blockIdx.x;
        float ps = 0.f;
        for (int i = tid; i < a.n_chunks; i += 256) ps += a.psum_part[(int64_t)i * a.E + e];
        ps = block_sum_256(ps, red);
        float el = 0.f;
        if (a.token_loss) {
            const int r0 = a.group_start[e], r1 = r0 + a.group_rows[e];
            for (int row = r0 + tid; row < r1; row += 256) {
                const int ai = a.row_assign[row];
                el += a.credit[ai] * a.token_loss[ai / a.k];
            }
            el = block_sum_256(el, red);
        }
        // Importance: this expert's selection gates, in priority order.
        float imp = 0.f;
        {
            const int g0 = a.pre_start[e], n = a.count_pre[e];
            for (int j = tid; j < n; j += 256) imp += a.gate_sorted[g0 + j];
            imp = block_sum_256(imp, red);
        }
        if (tid == 0) {
            a.partials[e] = ps;
            a.partials[a.E + e] = (float)a.count_pre[e];
            a.partials[2 * a.E + 3 + e] = el;
            a.partials[3 * a.E + 3 + e] = imp;
        }
    }
    if (!fuse) return;
    if (tid == 0) {
        __threadfence();  // this CTA's partial words are visible before it is counted
        const int old = atomicAdd(a.done_counter, 1);
        last = old == (int)gridDim.x - 1;
        if (last) {
            __threadfence();
            *a.done_counter = 0;  // ready for the next call
        }
    }
    __syncthreads();
    if (last) finalize_body(fin, red);
}

// Squared coefficient of variation of one value per thread (threads >= n hold
// nothing): population variance over the squared mean, 0 when the mean is 0.
__device__ __forceinline__ float block_cv_squared(float v, bool valid, int n, float *red) {
    const float mean = block_sum_256(valid ? v : 0.f, red) / (float)n;
    const float d = valid ? v - mean : 0.f;
    const float var = block_sum_256(d * d, red) / (float)n;
    return mean != 0.f ? var / (mean * mean) : 0.f;
}

// Statistics from (possibly all-reduced) partial sums: f_i = count_i / (k T),
// P_i = sum_t P / T, L_aux = alpha E sum_i f_i P_i, L_z = beta sum lse^2 / T,
// l_i = sum credit * loss / T, importance_i, the squared coefficients of
// variation of the loads and of the importances, and the weighted aux loss
// alpha CV^2(loads) + L_z ("Code Walkthrough - SER", "Load balancing": aux_loss
// = load_balance_coef * load_balance + z_loss_coef * z_loss, load_balance
// being the coefficient-of-variation style loss of the loads). One CTA of
// 256 threads (E <= 256), thread e owns expert e; every sum is a fixed tree.
// The partial sums may have been written by other CTAs of the same launch, so
// they are read from L2.
__device__ __forceinline__ void finalize_body(const FinalizeArgs &a, float *red) {
    const int e = threadIdx.x;
    const bool own = e < a.E;
    const float T = __ldcg(a.partials + 2 * a.E + 1);
    const float inv_t = T > 0.f ? 1.f / T : 0.f;
    const float inv_kt = T > 0.f ? 1.f / ((float)a.k * T) : 0.f;
    float pm = 0.f, f = 0.f, load = 0.f, imp = 0.f;
    if (own) {
        pm = __ldcg(a.partials + e) * inv_t;
        load = __ldcg(a.partials + a.E + e);
        f = load * inv_kt;
        imp = __ldcg(a.partials + 3 * a.E + 3 + e);
        if (a.p_mean) a.p_mean[e] = pm;
        if (a.f) a.f[e] = f;
        if (a.expert_loss) a.expert_loss[e] = __ldcg(a.partials + 2 * a.E + 3 + e) * inv_t;
        if (a.importance) a.importance[e] = imp;
    }
    const float fp = block_sum_256(own ? f * pm : 0.f, red);
    const float cv_load = block_cv_squared(load, own, a.E, red);
    const float cv_imp = block_cv_squared(imp, own, a.E, red);
    if (e == 0) {
        const float l_aux = a.alpha * (float)a.E * fp;
        const float l_z = a.beta * __ldcg(a.partials + 2 * a.E) * inv_t;
        if (a.l_aux) *a.l_aux = l_aux;
        if (a.l_z) *a.l_z = l_z;
        if (a.l_total) *a.l_total = a.alpha * cv_load + l_z;
        if (a.n_dropped) *a.n_dropped = (int32_t)__ldcg(a.partials + 2 * a.E + 2);
        if (a.cv_load) *a.cv_load = cv_load;
        if (a.cv_importance) *a.cv_importance = cv_imp;
    }
}

__global__ void __launch_bounds__(256) stats_finalize_kernel(FinalizeArgs a) {
    __shared__ float red[8];
    finalize_body(a, red);
}

// Aux-loss-free balancing ("Balancing": per-expert selection bias b_i, update
// rate gamma): b_e += gamma * sign(k T / E - load_e). The sign is decided on
// integers (k T - E load_e); gamma * sign is exact, so the one fp32 add is the
// only rounding. One CTA, thread e owns expert e.
__global__ void __launch_bounds__(256) bias_update_kernel(BiasUpdateArgs a) {
    const int e = threadIdx.x;
    if (e >= a.E) return;
    int64_t load, T;
    if (a.partials) {
        load = (int64_t)a.partials[a.E + e];
        T = (int64_t)a.partials[2 * a.E + 1];
    } else {
        load = a.count_pre[e];
        T = a.T;
    }
    const int64_t diff = (int64_t)a.k * T - (int64_t)a.E * load;
    const float sgn = diff > 0 ? 1.f : (diff < 0 ? -1.f : 0.f);
    a.sel_bias[e] = __fadd_rn(a.sel_bias[e], a.gamma * sgn);
}

// Squared norm of every routed row (warp per row, 16-byte loads, fp32 sums in
// lane-strided then shuffle-tree order). The credit's hidden-activation reading
// ("Sparse MoE Expert-Credit Loss Reweighting Diagram", panel (b)) uses the
// rows of H as stored.
__global__ void __launch_bounds__(256) row_norms_kernel(RowNormArgs a) {
    const int lane = threadIdx.x & 31;
    const int rows = min(a.ctrl[kCtrlRoutedRows], a.max_rows);
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < rows; row += nwarps) {
        if (a.row_assign[row] < 0) continue;
        float ss = 0.f;
        if (a.bf16) {
            const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.m) + (int64_t)row * a.n);
            for (int v = lane; v < a.n / 8; v += 32) {
                const uint4 u = __ldg(p + v);
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __bfloat1622float2(h[j]);
                    ss = fmaf(f.x, f.x, ss);
                    ss = fmaf(f.y, f.y, ss);
                }
            }
        } else {
            const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(a.m) + (int64_t)row * a.n);
            for (int v = lane; v < a.n / 4; v += 32) {
                const float4 f = __ldg(p + v);
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
                ss = fmaf(f.z, f.z, ss);
                ss = fmaf(f.w, f.w, ss);
            }
        }
        ss = warp_sum(ss);
        if (lane == 0) a.norm2[row] = ss;
    }
}

// Panel (c) of the reweighting diagram, one layer: lhat <- ema lhat + (1-ema) l,
// mu <- softmax(mu + eta lhat), objective = sum mu l. One CTA, thread e owns
// expert e; max and sums are fixed trees.
__global__ void __launch_bounds__(256) dro_update_kernel(DroArgs a) {
    __shared__ float red[8];
    const int e = threadIdx.x;
    const bool own = e < a.E;
    float l = 0.f, z = -INFINITY;
    if (own) {
        l = a.l[e];
        const float lh = fmaf(a.ema, a.lhat[e], (1.f - a.ema) * l);
        a.lhat[e] = lh;
        z = fmaf(a.eta, lh, a.mu[e]);
    }
    // block max
    float m = z;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((e & 31) == 0) red[e >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
    const float ex = own ? expf(z - m) : 0.f;
    const float sum = block_sum_256(ex, red);
    const float mu = ex / sum;
    if (own) a.mu[e] = mu;
    const float obj = block_sum_256(own ? mu * l : 0.f, red);
    if (e == 0 && a.objective) *a.objective = obj;
}

}  // namespace

cudaError_t launch_stat_partials(const StatsArgs &a, const FinalizeArgs *fin, cudaStream_t s, int *launches) {
    FinalizeArgs none = {};
    stat_partials_kernel<<<a.E + 1, 256, 0, s>>>(a, fin ? *fin : none, fin ? 1 : 0);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_stats_finalize(const FinalizeArgs &a, cudaStream_t s, int *launches) {
    stats_finalize_kernel<<<1, 256, 0, s>>>(a);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_row_norms(const RowNormArgs &a, int num_sms, cudaStream_t s, int *launches) {
    int blocks = (a.max_rows + 7) / 8;
    if (blocks > num_sms * 8) blocks = num_sms * 8;
    if (blocks < 1) return cudaSuccess;
    row_norms_kernel<<<blocks, 256, 0, s>>>(a);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_dro_update(const DroArgs &a, cudaStream_t s, int *launches) {
    dro_update_kernel<<<1, 256, 0, s>>>(a);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_bias_update(const BiasUpdateArgs &a, cudaStream_t s, int *launches) {
    bias_update_kernel<<<1, 256, 0, s>>>(a);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace moe
