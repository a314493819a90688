// route_common.cuh - the per-token routing step of the router kernels.
//
// "Appendix C - Acronyms & Symbols", table "Core MoE symbols": P = softmax(h),
// the top-k set T_k(x) and the gates g_i (the selected experts' probabilities
// renormalised over the set); table "Balancing": the per-expert selection bias
// b_i and the log-partition the z-loss squares. "Code Walkthrough - SER",
// gating / routing path: noisy top-k adds noise to the logits before selection.
//
// One warp owns one token: lane l holds experts l, l + 32, ..., and max,
// log-partition, top-k and gates are warp-shuffle reductions. Selection keys are
// formed with one fp32 round-to-nearest add; equal keys go to the lower expert
// index. The argument block `a` of either router kernel provides noise,
// sel_bias, E, k and the outputs lse, idx, gates.
#pragma once

#include "moe_common.cuh"

namespace moe {

// The selection key's addend for expert lane + 32 q of token t: the logit
// noise, else the per-expert selection bias; returns false (no addend) for
// plain routing. Callers load it before their own stores so that the loads
// are in flight together.
template <int RE, class A>
__device__ __forceinline__ bool key_addend(int t, int lane, const A &a, float (&kadd)[RE]) {
    const float *src = a.noise ? a.noise + (int64_t)t * a.E : a.sel_bias;
#pragma unroll
    for (int q = 0; q < RE; ++q) {
        const int e = lane + 32 * q;
        kadd[q] = (src && e < a.E) ? src[e] : 0.f;
    }
    return src != nullptr;
}

// Order-preserving code of a selection key (never NaN here): a larger key has
// a larger code, and -0 and +0, which compare equal, have the same code.
__device__ __forceinline__ uint32_t key_code(float k) {
    const uint32_t u = __float_as_uint(k == 0.f ? 0.f : k);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// h[q] = clean logit of expert lane + 32 q (-inf for e >= E). Writes lse[t],
// idx[t][0..k), gates[t][0..k) and adds the token's probabilities P[t][e] to
// pacc[q] (the caller's per-lane running sums over its tokens).
template <int RE, class A>
__device__ __forceinline__ void route_warp(const float (&h)[RE], bool has_add, const float (&kadd)[RE], int t,
                                           int lane, const A &a, float (&pacc)[RE]) {
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
        // The warp's winner: the largest key, then the lowest expert index
        // among the lanes that hold it (two warp reductions).
        const uint32_t code = key_code(bk);
        const uint32_t top = __reduce_max_sync(0xffffffffu, code);
        be = static_cast<int>(__reduce_min_sync(0xffffffffu, code == top ? static_cast<uint32_t>(be) : 0xffffffffu));
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

}  // namespace moe
