// router_tc.cu - router logits on the sm_100a tensor cores, at fp32 accuracy.
//
// "Appendix C - Acronyms & Symbols", table "Core MoE symbols": router logits
// h = W_g x, one score per expert; "Code Walkthrough - SER", gating / routing
// path: the linear router carries a bias. The routing decisions that follow
// (softmax, selection key, top-k, gates) are integer decisions taken on these
// fp32 logits, so the logits must be as accurate as an fp32 dot product.
//
// Two things make a bf16 tensor-core GEMM fp32-accurate here:
//  * operands: every forward splits the fp32 router matrix into three bf16
//    planes, W = hi + mid + lo (each the bf16 rounding of what the earlier
//    planes leave; the sum matches W to ~2^-27 relative), and x is exactly
//    bf16, so h = sum_p x . W_p is one GEMM with K = 3d whose products are
//    exact: A is x read three times (the K coordinate wraps), B = [hi|mid|lo];
//  * accumulation: the tensor core's fp32 accumulator does not round to
//    nearest, and its error grows with the number of MMA steps and with the
//    accumulator's magnitude. So the MMA starts a fresh partial every kDrain K
//    blocks (kDrain * 4 MMA steps) and the epilogue adds each partial into a
//    running fp32 sum held in registers, with ordinary round-to-nearest adds.
// Eight epilogue warps, two per TMEM lane quarter, each own 64 of the N <= 128
// columns of 32 tokens; TMEM holds two partial buffers so the MMA runs ahead.
// Output: logits [T][E] (bias included). Softmax, keys, top-k and gates are
// taken from them by the routing kernel in router.cu. With few tiles (small T)
// the drain groups of a tile are split over ksplit CTAs (split-K); each writes
// its fp32 partial sums and the routing kernel adds them in split order.
#include "moe_common.cuh"
#include "moe_kernels.cuh"
#include "tc_pipeline.cuh"

namespace moe {
namespace {

constexpr int kDrain = 2;          // K blocks per partial accumulator
constexpr int kRouterThreads = 320;  // producer, MMA, 8 epilogue warps

// W_g [E][d] fp32 -> [E_pad][3d] bf16 planes (rows >= E are zero).
__global__ void __launch_bounds__(256) router_split_kernel(const float *__restrict__ w, int E, int E_pad, int d,
                                                           __nv_bfloat16 *__restrict__ out) {
    const int64_t n = (int64_t)E_pad * d;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(i / d), j = (int)(i - (int64_t)e * d);
        const float v = e < E ? w[i] : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(hi);  // exact: hi is v rounded to 8 mantissa bits
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);  // exact for the same reason
        const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
        __nv_bfloat16 *row = out + (int64_t)e * 3 * d;
        row[j] = hi;
        row[d + j] = mid;
        row[2 * d + j] = lo;
    }
}

template <int BN>
__global__ void __launch_bounds__(kRouterThreads, 1)
    router_logits_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                            const RouterTcArgs a) {
    static_assert(BN <= 128, "each epilogue thread holds BN / 2 <= 64 running sums");
    constexpr int HALF = BN / 2;  // columns per epilogue thread
    using L = TcLayout<BN>;
    extern __shared__ uint8_t smem_raw[];
    const TcShared<BN> s = tc_carve<BN>(smem_raw);
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
    }
    const uint32_t tmem_base = tc_setup<BN>(s, 256);
    const int n_tiles = a.E_pad / BN;
    const int ks = a.ksplit;
    const int total = ((a.T + kBM - 1) / kBM) * n_tiles * ks;  // tile = (m * n_tiles + n) * ks + split
    const int dblocks = a.d / kBK;
    const int kblocks = 3 * dblocks;
    const int groups = (kblocks + kDrain - 1) / kDrain;
    const int gps = (groups + ks - 1) / ks;  // drain groups per split
    auto grange = [&](int tile) {
        const int sp = tile % ks;
        const int g0 = min(sp * gps, groups), g1 = min(g0 + gps, groups);
        return make_int2(g0, g1);
    };
    const int warp = threadIdx.x >> 5;

    if (warp == 0) {
        int arow = 0, brow = 0;
        auto tile_begin = [&](int tile, int) {
            const int mn = tile / ks;
            const int m = mn / n_tiles, n = mn - m * n_tiles;
            arow = m * kBM;
            brow = n * BN;
        };
        auto load = [&](int, int kb, uint8_t *sA, uint8_t *sB, uint64_t *bar, int lane) {
            if (lane == 0) {
                tma_load_2d(&map_x, bar, sA, (kb % dblocks) * kBK, arow);
                tma_load_2d(&map_w, bar, sB, kb * kBK, brow);
            }
        };
        tc_producer_range<BN>(s, total, a.status, tile_begin, load, [&](int tile) {
            const int2 gr = grange(tile);
            return make_int2(gr.x * kDrain, min(gr.y * kDrain, kblocks));
        });
    } else if (warp == 1) {
        if ((threadIdx.x & 31) == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
            uint32_t it = 0, gcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const int2 gr = grange(tile);
                for (int g = gr.x; g < gr.y && ok; ++g, ++gcount) {
                    const uint32_t buf = gcount & 1u, use = gcount >> 1;
                    if (!mbar_wait(&s.tempty[buf], (use & 1u) ^ 1u, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t d_tmem = tmem_base + buf * kTcAccCols / 2;
                    const int kb0 = g * kDrain, kb1 = min(kb0 + kDrain, kblocks);
                    for (int kb = kb0; kb < kb1; ++kb, ++it) {
                        const int st = it % L::NS;
                        const uint32_t ph = (it / L::NS) & 1u;
                        if (!mbar_wait(&s.full[st], ph, a.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint64_t ad = sw128_kmajor_desc(smem_u32(s.sA + st * L::A_BYTES));
                        const uint64_t bd = sw128_kmajor_desc(smem_u32(s.sB + st * L::B_BYTES));
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk)
                            tc_mma_bf16(d_tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
                        tc_commit(&s.empty[st]);
                    }
                    if (ok) tc_commit(&s.tfull[buf]);
                }
            }
            tc_commit(s.mma_done);
            mbar_wait_drain(s.mma_done, 0u);
        }
    } else {
        const int q = warp & 3, lane = threadIdx.x & 31;
        const int col0 = ((warp - 2) >> 2) * HALF;  // this warp's half of the N tile
        uint32_t gcount = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            const int mn = tile / ks, sp = tile % ks;
            const int m = mn / n_tiles, n = mn - m * n_tiles;
            const int t = m * kBM + q * 32 + lane;
            const int2 gr = grange(tile);
            float sum[HALF];
#pragma unroll
            for (int j = 0; j < HALF; ++j) sum[j] = 0.f;
            for (int g = gr.x; g < gr.y; ++g, ++gcount) {
                const uint32_t buf = gcount & 1u, use = gcount >> 1;
                int got = 1;
                if (lane == 0) got = mbar_wait(&s.tfull[buf], use & 1u, a.status) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t acc_addr =
                    tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kTcAccCols / 2 + col0;
#pragma unroll
                for (int c = 0; c < HALF; c += 32) {
                    uint32_t r[32];
                    if (HALF - c >= 32) {
                        tmem_ld_32x32b_x32(acc_addr + c, r);
                    } else {
                        tmem_ld_32x32b_x16(acc_addr + c, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c + j < HALF)
                            sum[c + j] = g == gr.x ? __uint_as_float(r[j]) : __fadd_rn(sum[c + j], __uint_as_float(r[j]));
                }
                tc_fence_before_sync();
                mbar_arrive(&s.tempty[buf]);
            }
            if (!ok || t >= a.T) continue;
            const int e0 = n * BN + col0;
            // ksplit > 1: raw partial sums (the routing kernel adds splits and bias).
            const float *bias = ks > 1 ? nullptr : a.b_gate;
            float *lrow = (ks > 1 ? a.partial + (int64_t)sp * a.T * a.E : a.logits) + (int64_t)t * a.E + e0;
            if ((a.E & 3) == 0 && e0 + HALF <= a.E) {
#pragma unroll
                for (int j = 0; j < HALF; j += 4) {
                    float4 v = make_float4(sum[j], sum[j + 1], sum[j + 2], sum[j + 3]);
                    if (bias) {
                        const float4 b = __ldg(reinterpret_cast<const float4 *>(bias + e0 + j));
                        v.x += b.x;
                        v.y += b.y;
                        v.z += b.z;
                        v.w += b.w;
                    }
                    *reinterpret_cast<float4 *>(lrow + j) = v;
                }
            } else {
#pragma unroll
                for (int j = 0; j < HALF; ++j)
                    if (e0 + j < a.E) lrow[j] = sum[j] + (bias ? __ldg(bias + e0 + j) : 0.f);
            }
        }
    }
    tc_teardown<BN>(s, tmem_base);
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap &mx, const CUtensorMap &mw, const RouterTcArgs &a, cudaStream_t s) {
    constexpr int smem = TcLayout<BN>::SMEM;
    cudaError_t e = set_smem_limit_once<router_logits_tc_kernel<BN>>(smem);
    if (e != cudaSuccess) return e;
    const int tiles = ((a.T + kBM - 1) / kBM) * (a.E_pad / BN) * a.ksplit;
    router_logits_tc_kernel<BN><<<tiles < a.num_sms ? tiles : a.num_sms, kRouterThreads, smem, s>>>(mx, mw, a);
    return cudaGetLastError();
}

}  // namespace

int router_tc_epad(int E) {
    int p = 16;
    while (p < E && p < 128) p <<= 1;
    return p < E ? (E + 127) / 128 * 128 : p;
}

int router_tc_bn(int E) { return router_tc_epad(E) < 128 ? router_tc_epad(E) : 128; }

// K splits. With fewer tiles than half the SMs, enough splits to fill them
// (at least 8 drain groups per split). Otherwise 1 or 2, whichever needs fewer
// waves of tiles per unit of work (ceil(tiles ks / SMs) / ks): two splits turn
// 3.46 waves (E=256, T=32768: 512 tiles on 148 SMs) into 7 half-length ones,
// for one extra [T][E] fp32 partial written and read.
int router_tc_ksplit(int T, int E, int d, int num_sms) {
    const int tiles = ((T + kBM - 1) / kBM) * (router_tc_epad(E) / router_tc_bn(E));
    const int groups = (3 * (d / kBK) + kDrain - 1) / kDrain;
    if (tiles <= 0 || num_sms <= 0) return 1;
    if (2 * tiles > num_sms) {
        const int w1 = (tiles + num_sms - 1) / num_sms, w2 = (2 * tiles + num_sms - 1) / num_sms;
        return (w2 < 2 * w1 && groups >= 16) ? 2 : 1;
    }
    int ks = num_sms / tiles;
    if (ks > groups / 8) ks = groups / 8;  // keep at least 8 drain groups per split
    return ks < 1 ? 1 : ks;
}

cudaError_t launch_router_logits_tc(const CUtensorMap &map_x, const CUtensorMap &map_w, const RouterTcArgs &a,
                                    __nv_bfloat16 *w_split, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    const int64_t n = (int64_t)a.E_pad * a.d;
    int blocks = (int)((n + 255) / 256);
    if (blocks > a.num_sms * 16) blocks = a.num_sms * 16;
    router_split_kernel<<<blocks, 256, 0, s>>>(a.w_gate, a.E, a.E_pad, a.d, w_split);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    *launches += 2;
    switch (router_tc_bn(a.E)) {
        case 16: return launch_bn<16>(map_x, map_w, a, s);
        case 32: return launch_bn<32>(map_x, map_w, a, s);
        case 64: return launch_bn<64>(map_x, map_w, a, s);
        case 128: return launch_bn<128>(map_x, map_w, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
