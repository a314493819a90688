// router.cu - the gating step of the MoE layer forward.
//
// "Appendix C - Acronyms & Symbols", table "Core MoE symbols": router logits
// h = W_g x (one score per expert), P = softmax(h), the top-k set T_k(x) and the
// gates g_i (renormalised probabilities of the selected experts). "Code
// Walkthrough - SER", gating / routing path: a linear router with a bias; noisy
// top-k adds noise to the logits before selection. Appendix C, "Balancing": the
// per-expert selection bias b_i and the log-partition that the z-loss squares.
//
// route_warp() is the per-token step shared by both kernels below: one warp owns
// one token, lane l holds experts l, l+32, ..., and max, log-partition, top-k
// and gates are warp-shuffle reductions. Selection keys are formed with one
// fp32 round-to-nearest add; equal keys go to the lower expert index.
//   router_simt_kernel      - fp32 layers: logits on fp32 CUDA cores (K tiled
//                             through shared memory), then route_warp;
//   route_from_logits_kernel - bf16 layers: route_warp over the logits the
//                             tensor-core kernel (router_tc.cu) wrote.
// The optional MLP gate (same page, "Configuration": use_mlp_gater,
// gater_hidden_dim) is h = W_g relu(W_1 x + b_1) + b: its hidden layer is a
// router pass with W_1 and logits_only (or the tensor-core kernel for bf16 x),
// its output layer router_simt_kernel over the hidden pre-activations with
// x_relu set.
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kKC = 32;  // K chunk staged in shared memory

// The selection key's addend for expert lane + 32 q of token t: the logit
// noise, else the per-expert selection bias; returns false (no addend) for
// plain routing. Callers load it before their own stores so that the loads
// are in flight together.
template <int RE>
__device__ __forceinline__ bool key_addend(int t, int lane, const RouterArgs &a, float (&kadd)[RE]) {
    const float *src = a.noise ? a.noise + (int64_t)t * a.E : a.sel_bias;
#pragma unroll
    for (int q = 0; q < RE; ++q) {
        const int e = lane + 32 * q;
        kadd[q] = (src && e < a.E) ? src[e] : 0.f;
    }
    return src != nullptr;
}

// h[q] = clean logit of expert lane + 32 q (-inf for e >= E). Writes lse[t],
// idx[t][0..k), gates[t][0..k) and adds the token's probabilities P[t][e] to
// pacc[q] (the caller's per-lane running sums over its tokens).
template <int RE>
__device__ __forceinline__ void route_warp(const float (&h)[RE], bool has_add, const float (&kadd)[RE], int t,
                                           int lane, const RouterArgs &a, float (&pacc)[RE]) {
    float key[RE];
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < RE; ++q) {
        const int e = lane + 32 * q;
        key[q] = -INFINITY;
        if (e < a.E) {
            float kv = h[q];
            if (has_add) kv = __fadd_rn(h[q], kadd[q]);
            // A NaN key (NaN input) selects like -inf: every pick is still a
            // valid, distinct expert index (the lowest free one).
            key[q] = kv != kv ? -INFINITY : kv;
            m = fmaxf(m, h[q]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float ex[RE], z = 0.f;
#pragma unroll
    for (int q = 0; q < RE; ++q) {
        ex[q] = (lane + 32 * q < a.E) ? expf(h[q] - m) : 0.f;
        z += ex[q];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane == 0) a.lse[t] = m + logf(z);
    const float inv_z = 1.f / z;
#pragma unroll
    for (int q = 0; q < RE; ++q) pacc[q] += ex[q] * inv_z;

    // Top-k by (key desc, expert index asc); the winner's clean exp(h - m)
    // feeds its gate.
    uint32_t taken = 0u;
    float gsel_sum = 0.f, my_gate_num = 0.f;
    int my_idx = -1;
    for (int r = 0; r < a.k; ++r) {
        float bk = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < RE; ++q) {
            const int e = lane + 32 * q;
            if (e < a.E && !(taken & (1u << q))) {
                if (key[q] > bk || (key[q] == bk && e < be)) {
                    bk = key[q];
                    be = e;
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ok > bk || (ok == bk && oe < be)) {
                bk = ok;
                be = oe;
            }
        }
        // The owner lane of expert `be` marks it taken and broadcasts exp(h - m).
        const int owner = be & 31, oq = be >> 5;
        float num = 0.f;
        if (lane == owner) {
#pragma unroll
            for (int q = 0; q < RE; ++q)
                if (q == oq) {
                    taken |= (1u << q);
                    num = ex[q];
                }
        }
        num = __shfl_sync(0xffffffffu, num, owner);
        gsel_sum += num;
        if (lane == r) {
            my_gate_num = num;
            my_idx = be;
        }
    }
    if (lane < a.k) {
        a.idx[(int64_t)t * a.k + lane] = my_idx;
        a.gates[(int64_t)t * a.k + lane] = my_gate_num / gsel_sum;
    }
}

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

// One warp per token over logits already in memory (bias included).
template <int RE>
__global__ void __launch_bounds__(kThreads) route_from_logits_kernel(RouterArgs a) {
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * kThreads) >> 5;
    float pacc[RE];
#pragma unroll
    for (int q = 0; q < RE; ++q) pacc[q] = 0.f;
    for (int t = warp; t < a.T; t += nwarps) {
        float kadd[RE];
        const bool has_add = key_addend<RE>(t, lane, a, kadd);
        float h[RE];
        if (a.logit_part) {
            // Split-K partials added in split order, then the bias; the loads
            // of four splits are issued together.
            const int64_t plane = (int64_t)a.T * a.E;
            const float *part = a.logit_part + (int64_t)t * a.E;
#pragma unroll
            for (int q = 0; q < RE; ++q) {
                const int e = lane + 32 * q;
                h[q] = e < a.E ? part[e] : -INFINITY;
            }
            int sp = 1;
            for (; sp + 3 < a.ksplit; sp += 4) {
                float p[4][RE];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int q = 0; q < RE; ++q) {
                        const int e = lane + 32 * q;
                        p[i][q] = e < a.E ? part[(sp + i) * plane + e] : 0.f;
                    }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int q = 0; q < RE; ++q) h[q] = __fadd_rn(h[q], p[i][q]);
            }
            for (; sp < a.ksplit; ++sp)
#pragma unroll
                for (int q = 0; q < RE; ++q) {
                    const int e = lane + 32 * q;
                    if (e < a.E) h[q] = __fadd_rn(h[q], part[sp * plane + e]);
                }
#pragma unroll
            for (int q = 0; q < RE; ++q) {
                const int e = lane + 32 * q;
                if (e < a.E) {
                    if (a.b_gate) h[q] += a.b_gate[e];
                    a.logits[(int64_t)t * a.E + e] = h[q];
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < RE; ++q) {
                const int e = lane + 32 * q;
                h[q] = e < a.E ? a.logits[(int64_t)t * a.E + e] : -INFINITY;
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

template <int RE>
cudaError_t launch_route(const RouterArgs &a, cudaStream_t s, int num_sms) {
    route_from_logits_kernel<RE><<<router_psum_blocks(a.T, num_sms, true), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

int router_rt(int T) { return T >= 4096 ? 4 : 1; }

}  // namespace

// Blocks of the routing kernel = rows of psum_part it writes.
int router_psum_blocks(int T, int num_sms, bool from_logits) {
    if (T <= 0) return 0;
    if (!from_logits) {
        const int tm = kWarps * router_rt(T);
        return (T + tm - 1) / tm;
    }
    int blocks = (T + kWarps - 1) / kWarps;
    return blocks < num_sms * 8 ? blocks : num_sms * 8;
}

cudaError_t launch_router(const RouterArgs &a, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    ++*launches;
    const int rt = router_rt(a.T);
    return a.x_bf16 ? launch_x<__nv_bfloat16>(a, s, rt) : launch_x<float>(a, s, rt);
}

cudaError_t launch_route_from_logits(const RouterArgs &a, int num_sms, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    ++*launches;
    if (a.E <= 32) return launch_route<1>(a, s, num_sms);
    if (a.E <= 64) return launch_route<2>(a, s, num_sms);
    if (a.E <= 128) return launch_route<4>(a, s, num_sms);
    return launch_route<8>(a, s, num_sms);
}

}  // namespace moe
