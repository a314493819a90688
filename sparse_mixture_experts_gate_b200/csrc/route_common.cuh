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

// The float whose key_code is c (the inverse on every code key_code makes).
__device__ __forceinline__ float code_key(uint32_t c) {
    return __uint_as_float((c & 0x80000000u) ? (c & 0x7fffffffu) : ~c);
}

// A lane's selection entry packed for one unsigned compare: the key's code
// above, 7 - q below (q = the entry's slot, expert lane + 32 q), so that a
// larger value is the larger key and, between equal keys, the lower expert.
// 0 marks no entry (padding experts, or an entry already taken): it is below
// every real entry, whose code is at least key_code(-inf) > 0.
__device__ __forceinline__ uint64_t pack_entry(uint32_t code, int q) {
    return (static_cast<uint64_t>(code) << 8) | static_cast<uint64_t>(7 - q);
}

__device__ __forceinline__ void cas_desc(uint64_t &x, uint64_t &y) {
    const uint64_t hi = x > y ? x : y, lo = x > y ? y : x;
    x = hi;
    y = lo;
}

// Sorts a lane's RE (<= 8) entries in descending order (a fixed network of
// compare-exchanges: Batcher's odd-even merge sort for 8, smaller ones below).
template <int RE>
__device__ __forceinline__ void sort_entries(uint64_t (&v)[RE]) {
    if constexpr (RE == 2) {
        cas_desc(v[0], v[1]);
    } else if constexpr (RE == 4) {
        cas_desc(v[0], v[1]); cas_desc(v[2], v[3]);
        cas_desc(v[0], v[2]); cas_desc(v[1], v[3]);
        cas_desc(v[1], v[2]);
    } else if constexpr (RE == 8) {
        cas_desc(v[0], v[1]); cas_desc(v[2], v[3]); cas_desc(v[4], v[5]); cas_desc(v[6], v[7]);
        cas_desc(v[0], v[2]); cas_desc(v[1], v[3]); cas_desc(v[4], v[6]); cas_desc(v[5], v[7]);
        cas_desc(v[1], v[2]); cas_desc(v[5], v[6]);
        cas_desc(v[0], v[4]); cas_desc(v[1], v[5]); cas_desc(v[2], v[6]); cas_desc(v[3], v[7]);
        cas_desc(v[2], v[4]); cas_desc(v[3], v[5]);
        cas_desc(v[1], v[2]); cas_desc(v[3], v[4]); cas_desc(v[5], v[6]);
    } else {
        static_assert(RE == 1, "RE is 1, 2, 4 or 8");
    }
}

// Routes NT tokens with one warp, their steps interleaved so that the
// dependency chains of the reductions overlap. For token i (valid[i]):
// h[i][q] = clean logit of expert lane + 32 q (-inf for e >= E), kadd[i][q]
// its key addend (with has_add). Writes lse[t], idx[t][0..k), gates[t][0..k)
// and adds the token's probabilities P[t][e] to pacc[q] (the caller's per-lane
// running sums over its tokens).
//
// Softmax: m = max of the logits (a NaN logit is skipped, as fmaxf does):
// fmaxf within the lane, then one warp reduction over order-preserving codes.
// Top-k by (key desc, expert index asc): each lane sorts its entries once;
// every round the warp takes the largest head key, then the lowest expert
// index among the lanes holding it, and the winning lane drops its head. Lane
// r keeps round r's winner and afterwards fetches the winner's clean
// exp(h - m) from the owning lane; the gates are those numerators over their
// sum.
template <int RE, int NT, class A>
__device__ __forceinline__ void route_warp_n(const float (&h)[NT][RE], bool has_add, const float (&kadd)[NT][RE],
                                             const int (&t)[NT], const bool (&valid)[NT], int lane, const A &a,
                                             float (&pacc)[RE]) {
    uint64_t ent[NT][RE];
    float ex[NT][RE], m[NT], z[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        float lm = -INFINITY;
#pragma unroll
        for (int q = 0; q < RE; ++q) {
            const int e = lane + 32 * q;
            ent[i][q] = 0ull;
            if (e < a.E) {
                float kv = h[i][q];
                if (has_add) kv = __fadd_rn(h[i][q], kadd[i][q]);
                // A NaN key (NaN input) selects like -inf: every pick is still a
                // valid, distinct expert index (the lowest free one).
                ent[i][q] = pack_entry(key_code(kv != kv ? -INFINITY : kv), q);
                lm = fmaxf(lm, h[i][q]);
            }
        }
        m[i] = code_key(__reduce_max_sync(0xffffffffu, key_code(lm)));
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        z[i] = 0.f;
#pragma unroll
        for (int q = 0; q < RE; ++q) {
            ex[i][q] = (lane + 32 * q < a.E) ? expf(h[i][q] - m[i]) : 0.f;
            z[i] += ex[i][q];
        }
        sort_entries<RE>(ent[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int i = 0; i < NT; ++i) z[i] += __shfl_xor_sync(0xffffffffu, z[i], off);
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        if (!valid[i]) continue;
        if (lane == 0) a.lse[t[i]] = m[i] + logf(z[i]);
        const float inv_z = 1.f / z[i];
#pragma unroll
        for (int q = 0; q < RE; ++q) pacc[q] += ex[i][q] * inv_z;
    }

    uint32_t my_w[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) my_w[i] = 0u;
    for (int r = 0; r < a.k; ++r) {
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            const uint64_t head = ent[i][0];
            const uint32_t code = static_cast<uint32_t>(head >> 8);
            const uint32_t hidx = static_cast<uint32_t>(lane + 32 * (7 - static_cast<int>(head & 0xffu)));
            const uint32_t top = __reduce_max_sync(0xffffffffu, code);
            const uint32_t w = __reduce_min_sync(0xffffffffu, code == top ? hidx : 0xffffffffu);
            if (hidx == w) {  // the winning lane drops its head
#pragma unroll
                for (int q = 0; q + 1 < RE; ++q) ent[i][q] = ent[i][q + 1];
                ent[i][RE - 1] = 0ull;
            }
            if (lane == r) my_w[i] = w;
        }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        const int src = static_cast<int>(my_w[i] & 31u), wq = static_cast<int>(my_w[i] >> 5);
        float num = 0.f;
#pragma unroll
        for (int q = 0; q < RE; ++q) {
            const float v = __shfl_sync(0xffffffffu, ex[i][q], src);
            if (q == wq) num = v;
        }
        float gsum = lane < a.k ? num : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) gsum += __shfl_xor_sync(0xffffffffu, gsum, off);
        if (valid[i] && lane < a.k) {
            a.idx[(int64_t)t[i] * a.k + lane] = static_cast<int>(my_w[i]);
            a.gates[(int64_t)t[i] * a.k + lane] = num / gsum;
        }
    }
}

// One token per warp (see route_warp_n).
template <int RE, class A>
__device__ __forceinline__ void route_warp(const float (&h)[RE], bool has_add, const float (&kadd)[RE], int t,
                                           int lane, const A &a, float (&pacc)[RE]) {
    const float(&h1)[1][RE] = reinterpret_cast<const float(&)[1][RE]>(h);
    const float(&k1)[1][RE] = reinterpret_cast<const float(&)[1][RE]>(kadd);
    const int t1[1] = {t};
    const bool v1[1] = {true};
    route_warp_n<RE, 1>(h1, has_add, k1, t1, v1, lane, a, pacc);
}

}  // namespace moe
