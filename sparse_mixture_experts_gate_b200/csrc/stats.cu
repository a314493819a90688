// stats.cu - balancing and credit statistics of one layer forward.
//
// "Appendix C - Acronyms & Symbols", table "Balancing": f_i (fraction of the
// batch's selections dispatched to expert i, counted before capacity drops),
// P_i (mean router mass on expert i), L_aux = alpha E sum_i f_i P_i and the
// router z-loss beta * mean_t (log sum_i e^{h_ti})^2. "Sparse MoE Expert-Credit
// Loss Reweighting Diagram", panel (b): the expert-attributed loss
// l_i = (1/N) sum_j c_i(x_j) l_j 1[i in T_j], N = T, over kept assignments.
//
// Every reduction has a fixed order (per-lane strided sums, then a fixed
// shuffle tree), so repeated runs give bit-identical statistics.
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// One warp per expert: P_i from the per-chunk partial sums, f_i, and the
// attributed loss over the expert's kept rows (ascending row = ascending token).
__global__ void __launch_bounds__(256) stats_expert_kernel(StatsArgs a) {
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
        const float pm = ps / (float)a.T;
        const float f = (float)((double)a.count_pre[e] / ((double)a.k * (double)a.T));
        a.p_mean_ws[e] = pm;
        a.f_ws[e] = f;
        if (a.p_mean) a.p_mean[e] = pm;
        if (a.f) a.f[e] = f;
        if (a.expert_loss && a.token_loss) a.expert_loss[e] = el / (float)a.T;
    }
}

// Single CTA: z-loss over tokens, L_aux over experts, dropped count.
__global__ void __launch_bounds__(256) stats_scalar_kernel(StatsArgs a) {
    __shared__ float red[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float z = 0.f;
    for (int t = tid; t < a.T; t += 256) z = fmaf(a.lse[t], a.lse[t], z);
    z = warp_sum(z);
    if (lane == 0) red[warp] = z;
    __syncthreads();
    float zt = 0.f;
    if (tid == 0)
        for (int w = 0; w < 8; ++w) zt += red[w];
    __syncthreads();
    float fp = 0.f;
    for (int e = tid; e < a.E; e += 256) fp = fmaf(a.f_ws[e], a.p_mean_ws[e], fp);
    fp = warp_sum(fp);
    if (lane == 0) red[warp] = fp;
    __syncthreads();
    if (tid == 0) {
        float ft = 0.f;
        for (int w = 0; w < 8; ++w) ft += red[w];
        if (a.l_aux) *a.l_aux = a.alpha * (float)a.E * ft;
        if (a.l_z) *a.l_z = a.beta * zt / (float)a.T;
        if (a.n_dropped) *a.n_dropped = a.ctrl[kCtrlDropped];
    }
}

}  // namespace

cudaError_t launch_stats(const StatsArgs &a, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    stats_expert_kernel<<<(a.E * 32 + 255) / 256, 256, 0, s>>>(a);
    stats_scalar_kernel<<<1, 256, 0, s>>>(a);
    *launches += 2;
    return cudaGetLastError();
}

}  // namespace moe
