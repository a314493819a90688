// router.cu - the gating step of the MoE layer forward.
//
// "Appendix C - Acronyms & Symbols", table "Core MoE symbols": router logits
// h = W_g x (one score per expert), P = softmax(h), the top-k set T_k(x) and the
// gates g_i (renormalised probabilities of the selected experts). "Code
// Walkthrough - SER", gating / routing path: a linear router with a bias; noisy
// top-k adds noise to the logits before selection. Appendix C, "Balancing": the
// per-expert selection bias b_i and the log-partition that the z-loss squares.
//
// router_simt_kernel: logits on fp32 CUDA cores (K tiled through shared
// memory), then the per-token routing step of route_common.cuh (a warp per
// token). It routes fp32 layers; bf16 layers route in router_fused.cu. The
// optional MLP gate (same page, "Configuration": use_mlp_gater,
// gater_hidden_dim) is h = W_g relu(W_1 x + b_1) + b: its hidden layer is a
// router pass with W_1 and logits_only (or the tensor-core kernel in
// logits-only mode for bf16 x), its output layer router_simt_kernel over the
// hidden pre-activations with x_relu set.
#include "moe_common.cuh"
#include "moe_kernels.cuh"
#include "route_common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kKC = 32;  // K chunk staged in shared memory

// Sums the warps' per-lane P sums in warp order and writes this block's row of
// psum_part [blocks][E] (a fixed order, so the statistics are reproducible).
template <int RE>
__device__ __forceinline__ void write_block_psum(const float (&pacc)[RE], const RouterArgs &a) {
    __shared__ float red[kWarps][32 * RE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < RE; ++q) red[warp][lane + 32 * q] = pacc[q];
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += kThreads) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w][e];
        a.psum_part[(int64_t)blockIdx.x * a.E + e] = s;
    }
}

template <typename XT, int RE, int RT>
__global__ void __launch_bounds__(kThreads) router_simt_kernel(RouterArgs a) {
    constexpr int TM = kWarps * RT;   // tokens per CTA
    constexpr int EP = 32 * RE;       // padded expert count
    __shared__ float xs[kKC][TM + 1];
    __shared__ float ws[kKC][EP + 1];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t_base = blockIdx.x * TM;
    const XT *x = static_cast<const XT *>(a.x);

    float acc[RT][RE];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int q = 0; q < RE; ++q) acc[i][q] = 0.f;

    for (int k0 = 0; k0 < a.d; k0 += kKC) {
        // Stage x[t_base .. +TM][k0 .. +KC] transposed into xs[kk][t].
        for (int i = tid; i < TM * kKC; i += kThreads) {
            const int t = i / kKC, kk = i % kKC;
            const int gt = t_base + t, gk = k0 + kk;
            float v = (gt < a.T && gk < a.d) ? to_f32(x[(int64_t)gt * a.d + gk]) : 0.f;
            if (a.x_relu) v = fmaxf(v, 0.f);
            xs[kk][t] = v;
        }
        // Stage W_g[0 .. EP][k0 .. +KC] transposed into ws[kk][e].
        for (int i = tid; i < EP * kKC; i += kThreads) {
            const int e = i / kKC, kk = i % kKC;
            const int gk = k0 + kk;
            ws[kk][e] = (e < a.E && gk < a.d) ? a.w_gate[(int64_t)e * a.d + gk] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kKC; ++kk) {
            float xv[RT], wv[RE];
#pragma unroll
            for (int i = 0; i < RT; ++i) xv[i] = xs[kk][warp * RT + i];
#pragma unroll
            for (int q = 0; q < RE; ++q) wv[q] = ws[kk][lane + 32 * q];
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int q = 0; q < RE; ++q) acc[i][q] = fmaf(xv[i], wv[q], acc[i][q]);
        }
        __syncthreads();
    }

    if (a.logits_only) {  // a hidden layer: pre-activations only, no routing
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const int t = t_base + warp * RT + i;
            if (t >= a.T) break;
#pragma unroll
            for (int q = 0; q < RE; ++q) {
                const int e = lane + 32 * q;
                if (e < a.E) a.logits[(int64_t)t * a.E + e] = acc[i][q] + (a.b_gate ? a.b_gate[e] : 0.f);
            }
        }
        return;
    }
    float pacc[RE];
#pragma unroll
    for (int q = 0; q < RE; ++q) pacc[q] = 0.f;
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int t = t_base + warp * RT + i;
        if (t >= a.T) break;  // warp-uniform
        float kadd[RE];
        const bool has_add = key_addend<RE>(t, lane, a, kadd);
        float h[RE];
#pragma unroll
        for (int q = 0; q < RE; ++q) {
            const int e = lane + 32 * q;
            h[q] = -INFINITY;
            if (e < a.E) {
                h[q] = acc[i][q] + (a.b_gate ? a.b_gate[e] : 0.f);
                a.logits[(int64_t)t * a.E + e] = h[q];
            }
        }
        route_warp<RE>(h, has_add, kadd, t, lane, a, pacc);
    }
    write_block_psum<RE>(pacc, a);
}

template <typename XT, int RE>
cudaError_t launch_re(const RouterArgs &a, cudaStream_t s, int rt) {
    if (rt == 4) {
        constexpr int TM = kWarps * 4;
        router_simt_kernel<XT, RE, 4><<<(a.T + TM - 1) / TM, kThreads, 0, s>>>(a);
    } else {
        constexpr int TM = kWarps * 1;
        router_simt_kernel<XT, RE, 1><<<(a.T + TM - 1) / TM, kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

template <typename XT>
cudaError_t launch_x(const RouterArgs &a, cudaStream_t s, int rt) {
    if (a.E <= 32) return launch_re<XT, 1>(a, s, rt);
    if (a.E <= 64) return launch_re<XT, 2>(a, s, rt);
    if (a.E <= 128) return launch_re<XT, 4>(a, s, rt);
    return launch_re<XT, 8>(a, s, rt);
}

int router_rt(int T) { return T >= 4096 ? 4 : 1; }

}  // namespace

// Blocks of the router kernel = rows of psum_part it writes.
int router_psum_blocks(int T) {
    if (T <= 0) return 0;
    const int tm = kWarps * router_rt(T);
    return (T + tm - 1) / tm;
}

cudaError_t launch_router(const RouterArgs &a, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    ++*launches;
    const int rt = router_rt(a.T);
    return a.x_bf16 ? launch_x<__nv_bfloat16>(a, s, rt) : launch_x<float>(a, s, rt);
}

}  // namespace moe
