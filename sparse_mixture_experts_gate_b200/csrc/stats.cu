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
// One warp per expert; every sum has a fixed order (lane-strided, then a fixed
// shuffle tree), so repeated runs give bit-identical results.
__global__ void __launch_bounds__(256) stat_partials_expert_kernel(StatsArgs a) {
    const int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (e >= a.E) return;
    float ps = 0.f;
    for (int i = lane; i < a.n_chunks; i += 32) ps += a.psum_part[(int64_t)i * a.E + e];
    ps = warp_sum(ps);
    float el = 0.f;
    if (a.token_loss) {
        const int r0 = a.group_start[e], r1 = r0 + a.group_rows[e];
        for (int row = r0 + lane; row < r1; row += 32) {
            const int ai = a.row_assign[row];
            el += a.credit[ai] * a.token_loss[ai / a.k];
        }
        el = warp_sum(el);
    }
    if (lane == 0) {
        a.partials[e] = ps;
        a.partials[a.E + e] = (float)a.count_pre[e];
        a.partials[2 * a.E + 3 + e] = el;
    }
}

__global__ void __launch_bounds__(256) stat_partials_scalar_kernel(StatsArgs a) {
    __shared__ float red[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float z = 0.f;
    for (int t = tid; t < a.T; t += 256) z = fmaf(a.lse[t], a.lse[t], z);
    z = warp_sum(z);
    if (lane == 0) red[warp] = z;
    __syncthreads();
    if (tid == 0) {
        float zt = 0.f;
        for (int w = 0; w < 8; ++w) zt += red[w];
        a.partials[2 * a.E] = zt;
        a.partials[2 * a.E + 1] = (float)a.T;
        a.partials[2 * a.E + 2] = (float)a.ctrl[kCtrlDropped];
    }
}

// Statistics from (possibly all-reduced) partial sums: f_i = count_i / (k T),
// P_i = sum_t P / T, L_aux = alpha E sum_i f_i P_i, L_z = beta sum lse^2 / T,
// l_i = sum credit * loss / T. One CTA; the L_aux sum is a fixed tree.
__global__ void __launch_bounds__(256) stats_finalize_kernel(FinalizeArgs a) {
    __shared__ float red[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float T = a.partials[2 * a.E + 1];
    const float inv_t = T > 0.f ? 1.f / T : 0.f;
    const float inv_kt = T > 0.f ? 1.f / ((float)a.k * T) : 0.f;
    float fp = 0.f;
    for (int e = tid; e < a.E; e += 256) {
        const float pm = a.partials[e] * inv_t;
        const float f = a.partials[a.E + e] * inv_kt;
        if (a.p_mean) a.p_mean[e] = pm;
        if (a.f) a.f[e] = f;
        if (a.expert_loss) a.expert_loss[e] = a.partials[2 * a.E + 3 + e] * inv_t;
        fp = fmaf(f, pm, fp);
    }
    fp = warp_sum(fp);
    if (lane == 0) red[warp] = fp;
    __syncthreads();
    if (tid == 0) {
        float ft = 0.f;
        for (int w = 0; w < 8; ++w) ft += red[w];
        if (a.l_aux) *a.l_aux = a.alpha * (float)a.E * ft;
        if (a.l_z) *a.l_z = a.beta * a.partials[2 * a.E] * inv_t;
        if (a.n_dropped) *a.n_dropped = (int32_t)a.partials[2 * a.E + 2];
    }
}

}  // namespace

cudaError_t launch_stat_partials(const StatsArgs &a, cudaStream_t s, int *launches) {
    stat_partials_expert_kernel<<<(a.E * 32 + 255) / 256, 256, 0, s>>>(a);
    stat_partials_scalar_kernel<<<1, 256, 0, s>>>(a);
    *launches += 2;
    return cudaGetLastError();
}

cudaError_t launch_stats_finalize(const FinalizeArgs &a, cudaStream_t s, int *launches) {
    stats_finalize_kernel<<<1, 256, 0, s>>>(a);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace moe
