// combine.cu - gate-weighted combine of the expert outputs, with the credit.
//
// "Code Walkthrough - SER", gating / routing path: the expert outputs are
// combined, weighted by the gates. "Appendix C - Acronyms & Symbols": the
// combine tensor is the gate-weighted un-scatter ("Capacity & communication"),
// and shared experts are always on ("Parameter accounting"; weight 1 here).
// "Sparse MoE Expert-Credit Loss Reweighting Diagram", panel (b): the credit
// c = p ||h||_2, here the applied gate times the norm of the expert's output.
//
//   y[t] = sum_{s < S} O[shared row of t] + sum_{r < k, kept} g[t][r] O[row(t, r)]
//
// in fp32, in exactly that order (shared experts first, then r ascending), so
// the result does not depend on scheduling. One CTA per token; 16-byte vector
// loads of the expert-output rows; dropped assignments contribute nothing.
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxK = 16;
constexpr int kMaxS = 4;

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;  // 8 bf16 per 16 bytes
    __device__ static void load(const __nv_bfloat16 *p, float (&v)[8]) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
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
    __device__ static void load(const float *p, float (&v)[4]) {
        const float4 u = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = u.x;
        v[1] = u.y;
        v[2] = u.z;
        v[3] = u.w;
    }
    __device__ static void store(float *p, const float (&v)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};

template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a) {
    constexpr int V = Vec<T>::N;
    __shared__ int s_row[kMaxK + kMaxS];
    __shared__ float s_g[kMaxK + kMaxS];
    const int t = blockIdx.x;
    const int nsh = a.S;
    const int tid = threadIdx.x;
    if (tid < nsh) {
        s_row[tid] = a.group_start[a.E + tid] + t;
        s_g[tid] = 1.f;
    } else if (tid < nsh + a.k) {
        const int r = tid - nsh;
        const int64_t ai = (int64_t)t * a.k + r;
        const int row = a.row_of[ai];
        const float g = a.gates[ai];
        s_row[tid] = row;
        s_g[tid] = g;
        // Credit of this assignment: gate times the norm of the expert output.
        float c = 0.f;
        if (row >= 0) {
            float ss = 0.f;
            for (int j = 0; j < a.n_parts; ++j) ss += a.norm_part[(int64_t)row * a.n_parts + j];
            c = g * sqrtf(ss);
        }
        a.credit[ai] = c;
    }
    __syncthreads();
    const T *o = static_cast<const T *>(a.o);
    T *y = static_cast<T *>(a.y) + (int64_t)t * a.O;
    const int nterm = nsh + a.k;
    for (int c = tid * V; c < a.O; c += kThreads * V) {
        float acc[V];
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] = 0.f;
        for (int i = 0; i < nterm; ++i) {
            const int row = s_row[i];
            if (row < 0) continue;
            const float g = s_g[i];
            float v[V];
            Vec<T>::load(o + (int64_t)row * a.O + c, v);
            if (i < nsh) {
#pragma unroll
                for (int j = 0; j < V; ++j) acc[j] += v[j];
            } else {
#pragma unroll
                for (int j = 0; j < V; ++j) acc[j] = fmaf(g, v[j], acc[j]);
            }
        }
        Vec<T>::store(y + c, acc);
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    if (a.bf16)
        combine_kernel<__nv_bfloat16><<<a.T, kThreads, 0, s>>>(a);
    else
        combine_kernel<float><<<a.T, kThreads, 0, s>>>(a);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
