// combine.cu - gate-weighted combine of the expert outputs, with the credit.
//
// "Code Walkthrough - SER", gating / routing path: the expert outputs are
// combined, weighted by the gates. "Appendix C - Acronyms & Symbols": the
// combine tensor is the gate-weighted un-scatter ("Capacity & communication"),
// and shared experts are always on ("Parameter accounting"; weight 1 here).
// "Sparse MoE Expert-Credit Loss Reweighting Diagram", panel (b): the credit
// c = p ||h||_2, here the applied gate times the norm of the expert's output
// row as the layer stores it (the same values the combine reads).
//
//   y[t] = sum_{s < S} O[shared row of t] + sum_{r < k, kept} g[t][r] O[row(t, r)]
//
// in fp32, in exactly that order (shared experts first, then r ascending), so
// the result does not depend on scheduling. One warp per token, or for short
// batches a block of eight warps per token, each taking every eighth 256-column
// stretch; 16-byte vector loads of the expert-output rows; dropped assignments
// contribute nothing. The squared norms are summed from the same loads (per
// lane in column order, then a fixed shuffle tree, then the warps of a block in
// order).
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;  // warps per block
constexpr int kMaxS = 4;
constexpr int kBatch = 8;  // routed-term loads issued together

// 16-byte vectors of expert-output elements: raw load, then unpack to fp32.
template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;  // 8 bf16 per 16 bytes
    __device__ static void unpack(const uint4 &u, float (&v)[8]) {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(h[j]);
            v[2 * j] = f.x;
            v[2 * j + 1] = f.y;
        }
    }
    __device__ static void store(__nv_bfloat16 *p, const float (&v)[8]) {
        uint4 u;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j] = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        *reinterpret_cast<uint4 *>(p) = u;
    }
};
template <>
struct Vec<float> {
    static constexpr int N = 4;
    __device__ static void unpack(const uint4 &u, float (&v)[4]) {
        v[0] = __uint_as_float(u.x);
        v[1] = __uint_as_float(u.y);
        v[2] = __uint_as_float(u.z);
        v[3] = __uint_as_float(u.w);
    }
    __device__ static void store(float *p, const float (&v)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};

template <typename T>
__device__ __forceinline__ uint4 load_raw(const T *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// NB: batches of eight routed terms the kernel is built for (k <= 8 NB).
// SL: warps per token, 1 or kWarps (then a block holds one token).
template <typename T, int NB, int SL>
__global__ void __launch_bounds__(kWarps * 32, 2) combine_kernel(CombineArgs a) {
    static_assert(SL == 1 || SL == kWarps, "one token per warp or per block");
    constexpr int V = Vec<T>::N;
    constexpr int kMaxK = NB * kBatch;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t = SL == 1 ? blockIdx.x * kWarps + warp : blockIdx.x;
    const int slice = SL == 1 ? 0 : warp;
    if (t >= a.T) return;  // uniform over the block when SL > 1
    const int nsh = a.S, k = a.k;
    int my_row = -1;
    float my_g = 0.f;
    if (lane < k) {
        my_row = a.row_of[(int64_t)t * k + lane];
        my_g = a.gates[(int64_t)t * k + lane];
    }
    int srow[kMaxS], rrow[kMaxK];
    float rg[kMaxK];
#pragma unroll
    for (int i = 0; i < kMaxS; ++i) srow[i] = i < nsh ? a.group_start[a.E + i] + t : -1;
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {  // lanes >= k hold row -1
        rrow[r] = __shfl_sync(0xffffffffu, my_row, r);
        rg[r] = __shfl_sync(0xffffffffu, my_g, r);
    }
    const T *o = static_cast<const T *>(a.o);
    T *y = static_cast<T *>(a.y) + (int64_t)t * a.O;
    // Per routed term, this lane's part of ||o||^2.
    float ss[kMaxK];
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) ss[r] = 0.f;
    for (int c = (slice * 32 + lane) * V; c < a.O; c += SL * 32 * V) {
        // Every term's vector (shared terms and the first eight routed terms)
        // is requested before any is used, so a lane has them all in flight.
        uint4 us[kMaxS], ur[kBatch];
#pragma unroll
        for (int i = 0; i < kMaxS; ++i)
            if (srow[i] >= 0) us[i] = load_raw(o + (int64_t)srow[i] * a.O + c);
#pragma unroll
        for (int i = 0; i < kBatch; ++i)
            if (rrow[i] >= 0) ur[i] = load_raw(o + (int64_t)rrow[i] * a.O + c);
        float acc[V];
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxS; ++i) {
            if (srow[i] < 0) continue;
            float v[V];
            Vec<T>::unpack(us[i], v);
#pragma unroll
            for (int j = 0; j < V; ++j) acc[j] += v[j];
        }
#pragma unroll
        for (int r0 = 0; r0 < kMaxK; r0 += kBatch) {
            if (r0 >= k) break;
            if (r0 > 0) {  // further batches (k > 8)
#pragma unroll
                for (int i = 0; i < kBatch; ++i)
                    if (rrow[r0 + i] >= 0) ur[i] = load_raw(o + (int64_t)rrow[r0 + i] * a.O + c);
            }
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                const int r = r0 + i;
                if (rrow[r] < 0) continue;
                float v[V];
                Vec<T>::unpack(ur[i], v);
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    acc[j] = fmaf(rg[r], v[j], acc[j]);
                    ss[r] = fmaf(v[j], v[j], ss[r]);
                }
            }
        }
        Vec<T>::store(y + c, acc);
    }
    // Credit of each routed assignment: gate times the norm of the expert
    // output row as stored (fixed shuffle tree, then the slices in order).
    __shared__ float part[SL > 1 ? SL : 1][kMaxK];
    float credit = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {
        if (r >= k) break;
        float v = ss[r];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (SL > 1) {
            if (lane == 0) part[slice][r] = v;
        } else if (lane == r && rrow[r] >= 0) {
            credit = rg[r] * sqrtf(a.row_norm2 ? a.row_norm2[rrow[r]] : v);
        }
    }
    if (SL > 1) {
        __syncthreads();
        if (slice != 0) return;
        if (lane < k && my_row >= 0) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < SL; ++w) v += part[w][lane];
            credit = my_g * sqrtf(a.row_norm2 ? a.row_norm2[my_row] : v);
        }
    }
    if (lane < k) a.credit[(int64_t)t * k + lane] = credit;
}

// The common case of bf16 layers (at most one shared expert, k <= 8) with one
// warp per token, software-pipelined over the 256-column stretches: the loads
// of stretch c + 256 are issued before stretch c is summed, so a lane keeps two
// stretches of every term in flight (the general kernel keeps one and waits
// out the memory latency once per stretch). Same arithmetic in the same order
// as combine_kernel, so the results are bit-identical.
template <bool SHARED>
__global__ void __launch_bounds__(kWarps * 32, 2) combine_pipe_kernel(CombineArgs a) {
    constexpr int V = 8;            // bf16 per 16-byte vector
    constexpr int kStep = 32 * V;   // columns per stretch
    constexpr int kTerms = kBatch + 1;  // routed terms, then the shared one
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t = blockIdx.x * kWarps + warp;
    if (t >= a.T) return;
    const int k = a.k;
    int my_row = -1;
    float my_g = 0.f;
    if (lane < k) {
        my_row = a.row_of[(int64_t)t * k + lane];
        my_g = a.gates[(int64_t)t * k + lane];
    }
    int rrow[kBatch];
    float rg[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {  // lanes >= k hold row -1
        rrow[r] = __shfl_sync(0xffffffffu, my_row, r);
        rg[r] = __shfl_sync(0xffffffffu, my_g, r);
    }
    const int srow = SHARED ? a.group_start[a.E] + t : -1;
    const __nv_bfloat16 *o = static_cast<const __nv_bfloat16 *>(a.o);
    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(a.y) + (int64_t)t * a.O;
    float ss[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) ss[r] = 0.f;
    auto load = [&](uint4 (&u)[kTerms], int c) {
#pragma unroll
        for (int i = 0; i < kBatch; ++i)
            if (rrow[i] >= 0) u[i] = load_raw(o + (int64_t)rrow[i] * a.O + c);
        if (SHARED) u[kBatch] = load_raw(o + (int64_t)srow * a.O + c);
    };
    auto consume = [&](const uint4 (&u)[kTerms], int c) {
        float acc[V];
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] = 0.f;
        if (SHARED) {
            float v[V];
            Vec<__nv_bfloat16>::unpack(u[kBatch], v);
#pragma unroll
            for (int j = 0; j < V; ++j) acc[j] += v[j];
        }
#pragma unroll
        for (int r = 0; r < kBatch; ++r) {
            if (rrow[r] < 0) continue;
            float v[V];
            Vec<__nv_bfloat16>::unpack(u[r], v);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                acc[j] = fmaf(rg[r], v[j], acc[j]);
                ss[r] = fmaf(v[j], v[j], ss[r]);
            }
        }
        Vec<__nv_bfloat16>::store(y + c, acc);
    };
    uint4 u0[kTerms], u1[kTerms];
    int c = lane * V;
    if (c < a.O) load(u0, c);
    for (; c < a.O; c += 2 * kStep) {
        const int c1 = c + kStep;
        if (c1 < a.O) load(u1, c1);
        consume(u0, c);
        if (c1 >= a.O) break;
        if (c1 + kStep < a.O) load(u0, c1 + kStep);
        consume(u1, c1);
    }
    // Credit of each routed assignment (fixed shuffle tree).
    float credit = 0.f;
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
        if (r >= k) break;
        float v = ss[r];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == r && rrow[r] >= 0) credit = rg[r] * sqrtf(a.row_norm2 ? a.row_norm2[rrow[r]] : v);
    }
    if (lane < k) a.credit[(int64_t)t * k + lane] = credit;
}

template <typename T, int NB>
void launch_t(const CombineArgs &a, int num_sms, cudaStream_t s) {
    // A block per token while one warp per token would leave fewer than eight
    // warps per SM.
    const int blocks = (a.T + kWarps - 1) / kWarps;
    if (a.T < kWarps * num_sms)
        combine_kernel<T, NB, kWarps><<<a.T, kWarps * 32, 0, s>>>(a);
    else if (a.bf16 && NB == 1 && a.S == 1)
        combine_pipe_kernel<true><<<blocks, kWarps * 32, 0, s>>>(a);
    else if (a.bf16 && NB == 1 && a.S == 0)
        combine_pipe_kernel<false><<<blocks, kWarps * 32, 0, s>>>(a);
    else
        combine_kernel<T, NB, 1><<<blocks, kWarps * 32, 0, s>>>(a);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs &a, int num_sms, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    if (a.k > 2 * kBatch) return cudaErrorInvalidValue;
    if (a.bf16) {
        if (a.k <= kBatch)
            launch_t<__nv_bfloat16, 1>(a, num_sms, s);
        else
            launch_t<__nv_bfloat16, 2>(a, num_sms, s);
    } else {
        if (a.k <= kBatch)
            launch_t<float, 1>(a, num_sms, s);
        else
            launch_t<float, 2>(a, num_sms, s);
    }
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
