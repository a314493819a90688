// router_fused.cu - the router of bf16 layers in one kernel: fp32-accurate
// logits on the sm_100a tensor cores, then softmax, log-partition, selection
// key, top-k and gates for every token.
//
// "Appendix C - Acronyms & Symbols", table "Core MoE symbols": router logits
// h = W_g x, one score per expert, P = softmax(h), the top-k set T_k(x) and the
// renormalised gates g_i; "Code Walkthrough - SER", gating / routing path: the
// linear router carries a bias, and gate_forward takes the input to logits,
// softmax and the top-k selection in one call.
//
// Accuracy. The routing decisions are integer decisions on fp32 logits, so the
// logits must be as accurate as an fp32 dot product. x is exactly bf16 and the
// fp32 router matrix is split into three bf16 planes W = hi + mid + lo (each the
// bf16 rounding of what the earlier planes leave), so every product the tensor
// core forms is exact. Its fp32 accumulator does not round to nearest and its
// error grows with the accumulator's magnitude and the number of MMA steps, so
// the MMAs of one K block are issued smallest plane first (lo, mid, hi) and the
// accumulator is drained every kDrain K blocks into fp32 running sums in
// registers, with ordinary round-to-nearest adds.
//
// Work. A unit is (token tile of 256, expert tile of BN <= 128, K split). A CTA
// pair (cta_group::2) computes it: each CTA stages its 128 token rows of x once
// per K block of 64 and its BN/2 rows of each of the three planes, and the
// leader issues 12 MMAs of M = 256 (tokens) x N = BN (experts) x K = 16 on it,
// so x is read once for all three planes. Each CTA's TMEM holds its 128 tokens x
// BN experts in two partial buffers so that the MMAs run ahead of the drains.
//
// Routing. Two phases in the one launch. Phase A: every unit's CTA pair
// writes its result (the logits themselves when a token tile is one unit,
// otherwise fp32 partial sums). A grid-wide barrier follows (the launch is
// cooperative, so every CTA is resident; the wait is bounded). Phase B: every
// warp of every CTA takes tokens of its CTA's contiguous share, adds each
// token's partials in a fixed order (K split), adds the bias, writes the
// logits and routes the token (route_common.cuh), so the routing is spread over
// all SMs; each CTA writes one row of per-expert P sums (its warps' sums added
// in warp order).
//
// Roles (384 threads per CTA): warp 0 loads (TMA), warp 1 owns TMEM and, in
// the leader, issues the MMAs; warps 2..9 drain the accumulators (two warps per
// TMEM lane quarter, BN/2 columns each); warps 10 and 11 have no phase-A role
// (the registers the others need leave room for them). In phase B all twelve
// warps route. Every
// wait is bounded; on a timeout the roles stop, in-flight copies and MMAs are
// drained, phase B is skipped, both CTAs meet at the cluster barrier and TMEM is
// freed.
#include "moe_common.cuh"
#include "moe_kernels.cuh"
#include "route_common.cuh"

namespace moe {
namespace {

constexpr int kTokCta = 128;      // token rows per CTA; the pair's M is 256
constexpr int kTokTileR = 256;    // tokens per unit
// K blocks of 64 per partial accumulator: 48 MMA steps of K = 16 before the
// running sums take it over (logit error 3.7e-6 against the fp64 oracle on the
// smoke shape; 1.5e-6 with 2, at 8% more router time at E = 256).
constexpr int kDrain = 4;

// Epilogue warps: two per TMEM lane quarter (BN / 2 columns of running sums
// per thread).
template <int BN>
struct RCfg {
    static constexpr int kEpiWarps = 8;
    static constexpr int kRouteWarps = 2;  // warps with no phase-A role that route in phase B
    static constexpr int kThreads = 64 + 32 * (kEpiWarps + kRouteWarps);
    static constexpr int kA = kTokCta * kBK * 2;          // x rows of this CTA, one K block
    static constexpr int kBHalf = (BN / 2) * kBK * 2;     // one plane, this CTA's BN/2 expert rows
    static constexpr int kStage = kA + 3 * kBHalf;
    static constexpr int kStages = (200 * 1024) / kStage < 8 ? (200 * 1024) / kStage : 8;
    static constexpr int kTmemCols = 2 * BN;              // two partial buffers
    static constexpr int kWarps = kThreads / 32;
    static constexpr int kRedBytes = kWarps * 256 * 4;     // per-warp P sums of phase B
    static constexpr int kCols = BN / (kEpiWarps / 4);     // accumulator columns per epilogue thread
    static constexpr int kSmem = 1024 + kStages * kStage + kRedBytes + 512;
    static_assert(BN == 32 || BN == 64 || BN == 128, "expert tile");
    static_assert(kBHalf % 1024 == 0, "plane tiles keep the 1024-byte swizzle alignment");
    static_assert(kSmem <= 232448, "exceeds the shared memory a CTA may use");
};

struct RSmem {
    uint8_t *stages;
    float *red;
    uint64_t *full, *empty, *tfull, *tempty, *drained, *mma_done;
    uint32_t *tmem_slot;
};

template <int BN>
__device__ __forceinline__ RSmem rcarve(uint8_t *raw) {
    using C = RCfg<BN>;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    RSmem s;
    s.stages = base;
    s.red = reinterpret_cast<float *>(base + C::kStages * C::kStage);
    s.full = reinterpret_cast<uint64_t *>(base + C::kStages * C::kStage + C::kRedBytes);
    s.empty = s.full + C::kStages;
    s.tfull = s.empty + C::kStages;
    s.tempty = s.tfull + 2;
    s.drained = s.tempty + 2;
    s.mma_done = s.drained + 2;
    s.tmem_slot = reinterpret_cast<uint32_t *>(s.mma_done + 1);
    return s;
}

// Unit u = (token tile m, expert tile n, split sp), u = (m * n_tiles + n) * ks + sp.
struct Unit {
    int m, n, sp, kb0, kb1;
};

__device__ __forceinline__ Unit unit_of(const RouterFusedArgs &a, int u) {
    Unit r;
    r.sp = u % a.ksplit;
    const int mn = u / a.ksplit;
    r.n = mn % a.n_tiles;
    r.m = mn / a.n_tiles;
    const int dblocks = a.d / kBK;
    const int per = (dblocks + a.ksplit - 1) / a.ksplit;
    r.kb0 = min(r.sp * per, dblocks);
    r.kb1 = min(r.kb0 + per, dblocks);
    return r;
}

// Phase B for tokens [t_begin, t_end): a warp routes two tokens at a time
// (t and t + nwarps, interleaved by route_warp_n). A token's logits are read
// (one unit per tile) or formed from the partials of its K splits, added in
// split order two splits' loads at a time, plus the bias, and written. A
// selection bias, the same for every token, is loaded once. Leaves this
// warp's per-expert P sums in red[warp][.].
template <int BN, int RE>
__device__ __forceinline__ void route_tokens(const RouterFusedArgs &a, float *red, int warp, int nwarps, int lane,
                                             int t_begin, int t_end) {
    constexpr int NT = 2;  // tokens a warp routes at once
    float pacc[RE];
#pragma unroll
    for (int q = 0; q < RE; ++q) pacc[q] = 0.f;
    const int ks = a.ksplit;
    const bool merged = a.n_tiles * ks == 1;
    const bool has_add = a.noise != nullptr || a.sel_bias != nullptr;
    float kadd[NT][RE];
    if (!a.noise) {  // the selection bias (or nothing), the same for every token
        key_addend<RE>(0, lane, a, kadd[0]);
#pragma unroll
        for (int i = 1; i < NT; ++i)
#pragma unroll
            for (int q = 0; q < RE; ++q) kadd[i][q] = kadd[0][q];
    }
    const int64_t split_stride = (int64_t)kTokTileR * BN;
    for (int t0 = t_begin + warp; t0 < t_end; t0 += NT * nwarps) {
        int t[NT];
        bool valid[NT];
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            t[i] = t0 + i * nwarps;
            valid[i] = t[i] < t_end;
        }
        float h[NT][RE];
        if (merged) {
#pragma unroll
            for (int i = 0; i < NT; ++i)
#pragma unroll
                for (int q = 0; q < RE; ++q) {
                    const int e = lane + 32 * q;
                    h[i][q] = valid[i] ? (e < a.E ? __ldcg(a.logits + (int64_t)t[i] * a.E + e) : -INFINITY) : 0.f;
                }
        } else {
            // Every split's partial of both tokens is loaded before any is
            // summed (in split order), so the loads are in flight together.
            int64_t off[NT][RE];
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                const int m = t[i] / kTokTileR, tl = t[i] - m * kTokTileR;
#pragma unroll
                for (int q = 0; q < RE; ++q) {
                    const int e = lane + 32 * q;
                    const int n = e / BN, c = e - n * BN;
                    off[i][q] = ((int64_t)((m * a.n_tiles + n) * ks) * kTokTileR + tl) * BN + c;
                }
            }
            for (int sp = 0; sp < ks; sp += 2) {
                float v0[NT][RE], v1[NT][RE];
#pragma unroll
                for (int i = 0; i < NT; ++i)
#pragma unroll
                    for (int q = 0; q < RE; ++q) {
                        const bool in = valid[i] && lane + 32 * q < a.E;
                        v0[i][q] = in ? __ldcg(a.part + off[i][q] + sp * split_stride) : 0.f;
                        v1[i][q] = in && sp + 1 < ks ? __ldcg(a.part + off[i][q] + (sp + 1) * split_stride) : 0.f;
                    }
#pragma unroll
                for (int i = 0; i < NT; ++i)
#pragma unroll
                    for (int q = 0; q < RE; ++q) {
                        h[i][q] = sp == 0 ? v0[i][q] : __fadd_rn(h[i][q], v0[i][q]);
                        if (sp + 1 < ks) h[i][q] = __fadd_rn(h[i][q], v1[i][q]);
                    }
            }
#pragma unroll
            for (int i = 0; i < NT; ++i)
#pragma unroll
                for (int q = 0; q < RE; ++q) {
                    const int e = lane + 32 * q;
                    if (e < a.E) {
                        if (a.b_gate) h[i][q] = __fadd_rn(h[i][q], __ldg(a.b_gate + e));
                        if (valid[i]) a.logits[(int64_t)t[i] * a.E + e] = h[i][q];
                    } else {
                        h[i][q] = -INFINITY;
                    }
                }
        }
        if (!a.route) continue;
        if (a.noise) {
#pragma unroll
            for (int i = 0; i < NT; ++i)
#pragma unroll
                for (int q = 0; q < RE; ++q) {
                    const int e = lane + 32 * q;
                    kadd[i][q] = valid[i] && e < a.E ? __ldg(a.noise + (int64_t)t[i] * a.E + e) : 0.f;
                }
        }
        route_warp_n<RE, NT>(h, has_add, kadd, t, valid, lane, a, pacc);
    }
#pragma unroll
    for (int q = 0; q < RE; ++q) red[warp * 256 + lane + 32 * q] = pacc[q];
}

// Grid-wide barrier of the cooperative launch: every CTA counts itself once
// its phase A writes are done and waits (bounded) until all have. Returns the
// same result in every thread: true if all CTAs arrived and no bounded wait
// anywhere gave up (phase B may run), false otherwise.
__device__ __forceinline__ bool grid_barrier(int32_t *counter, uint32_t *status) {
    __shared__ int go_s;
    __syncthreads();  // every role of this CTA is done with phase A
    if (threadIdx.x == 0) {
        __threadfence();  // publishes the CTA's results (observed through the barrier above)
        atomicAdd(counter, 1);
        int go = 1;
        const uint64_t t0 = global_timer_ns();
        while (*reinterpret_cast<volatile int32_t *>(counter) < (int)gridDim.x) {
            if (*reinterpret_cast<volatile uint32_t *>(status) != kDevOk) {
                go = 0;
                break;
            }
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(status, kDevTimeout);
                go = 0;
                break;
            }
            __nanosleep(64);
        }
        __threadfence();  // the other CTAs' results are read after this
        if (*reinterpret_cast<volatile uint32_t *>(status) != kDevOk) go = 0;
        go_s = go;
    }
    __syncthreads();
    return go_s != 0;
}

template <int BN, int RE>
__global__ void __launch_bounds__(RCfg<BN>::kThreads, 1)
    router_fused_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                        const RouterFusedArgs a) {
    using C = RCfg<BN>;
    constexpr int kStages = C::kStages;
    constexpr int kEpiWarps = C::kEpiWarps;
    constexpr int HALF = BN / 2;      // expert rows of each plane this CTA stages
    constexpr int COLS = C::kCols;    // accumulator columns per epilogue thread
    extern __shared__ uint8_t smem_raw[];
    const RSmem s = rcarve<BN>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], 2);          // one forwarded arrival from each CTA
            mbar_init(&s.drained[i], kEpiWarps);  // this CTA's epilogue warps
        }
        mbar_init(s.mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(s.tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync_all();
    tc_fence_after_sync();
    const uint32_t tmem_base = *s.tmem_slot;

    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int total = a.n_mtiles * a.n_tiles * a.ksplit;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        uint32_t it = 0;
        for (int u = pair; u < total && ok; u += n_pairs) {
            const Unit un = unit_of(a, u);
            const int xrow = un.m * kTokTileR + static_cast<int>(rank) * kTokCta;
            const int wrow = un.n * BN + static_cast<int>(rank) * HALF;
            for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
                const int st = it % kStages;
                const uint32_t ph = (it / kStages) & 1u;
                int got = 1;
                if (lane == 0) got = mbar_wait(&s.empty[st], ph ^ 1u, a.status, a.wait_limit_ns) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) {
                    ok = false;
                    break;
                }
                // Self-test of the timeout path: the leader neither announces
                // nor loads this stage, so it never completes and the MMA
                // role's bounded wait runs out.
                if (lane == 0 && !(leader && static_cast<int>(it) == a.skip_stage)) {
                    if (leader) mbar_arrive_expect_tx(&s.full[st], 2u * C::kStage);
                    const uint32_t bar = mapa_shared(smem_u32(&s.full[st]), 0);
                    uint8_t *sA = s.stages + st * C::kStage;
                    tma_load_2d_pair(&map_x, bar, sA, kb * kBK, xrow);
#pragma unroll
                    for (int p = 0; p < 3; ++p)
                        tma_load_2d_pair(&map_w, bar, sA + C::kA + p * C::kBHalf, p * a.d + kb * kBK, wrow);
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA (leader)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(2 * kTokCta, BN);
            uint32_t it = 0, gcount = 0;
            for (int u = pair; u < total && ok; u += n_pairs) {
                const Unit un = unit_of(a, u);
                for (int g0 = un.kb0; g0 < un.kb1 && ok; g0 += kDrain, ++gcount) {
                    const uint32_t buf = gcount & 1u, use = gcount >> 1;
                    if (!mbar_wait(&s.tempty[buf], (use & 1u) ^ 1u, a.status, a.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t d_tmem = tmem_base + buf * BN;
                    const int g1 = min(g0 + kDrain, un.kb1);
                    for (int kb = g0; kb < g1; ++kb, ++it) {
                        const int st = it % kStages;
                        const uint32_t ph = (it / kStages) & 1u;
                        if (!mbar_wait(&s.full[st], ph, a.status, a.wait_limit_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t sa = smem_u32(s.stages + st * C::kStage);
                        const uint64_t ad = sw128_kmajor_desc(sa);
#pragma unroll
                        for (int p = 2; p >= 0; --p) {  // lo, mid, hi: the small products first
                            const uint64_t bd = sw128_kmajor_desc(sa + C::kA + p * C::kBHalf);
#pragma unroll
                            for (int kk = 0; kk < kBK / 16; ++kk)
                                tc_mma_bf16_pair(d_tmem, ad + 2u * kk, bd + 2u * kk, idesc,
                                                 (kb != g0 || p != 2 || kk != 0) ? 1u : 0u);
                        }
                        tc_commit_pair_mc(&s.empty[st], 0x3);
                    }
                    if (ok) tc_commit_pair_mc(&s.tfull[buf], 0x3);
                }
            }
            tc_commit_pair(s.mma_done);
            mbar_wait_drain(s.mma_done, 0u);
        }
    } else if (warp < 2 + kEpiWarps) {
        // ------------------------------------------------------------ epilogue (phase A)
        const int ew = warp - 2;
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int col0 = (ew >> 2) * COLS;       // this warp's columns of the expert tile
        uint32_t gcount = 0;
        for (int u = pair; u < total && ok; u += n_pairs) {
            const Unit un = unit_of(a, u);
            float sum[COLS];
#pragma unroll
            for (int j = 0; j < COLS; ++j) sum[j] = 0.f;
            for (int g0 = un.kb0; g0 < un.kb1; g0 += kDrain, ++gcount) {
                const uint32_t buf = gcount & 1u, use = gcount >> 1;
                int got = 1;
                if (lane == 0) got = mbar_wait(&s.tfull[buf], use & 1u, a.status, a.wait_limit_ns) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * BN + col0;
                // Columns per batch of loads (in flight together, one wait): up
                // to 32, or 16 when the thread already holds 64 running sums.
                constexpr int kBatch = COLS >= 64 ? 16 : (COLS < 32 ? COLS : 32);
#pragma unroll
                for (int c0 = 0; c0 < COLS; c0 += kBatch) {
                    uint32_t r[kBatch];
#pragma unroll
                    for (int c = 0; c < kBatch; c += 16)
                        tmem_ld_32x32b_x16(taddr + c0 + c, *reinterpret_cast<uint32_t(*)[16]>(&r[c]));
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < kBatch; ++j)
                        sum[c0 + j] =
                            g0 == un.kb0 ? __uint_as_float(r[j]) : __fadd_rn(sum[c0 + j], __uint_as_float(r[j]));
                }
                // The buffer is free once every epilogue warp of both CTAs has
                // read it: the warps arrive on this CTA's drained barrier and
                // one thread forwards a single arrival to the leader's tempty.
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.drained[buf]);
                if (ew == 0 && lane == 0) {
                    if (mbar_wait(&s.drained[buf], use & 1u, a.status, a.wait_limit_ns))
                        mbar_arrive_cluster(mapa_shared(smem_u32(&s.tempty[buf]), 0));
                    else
                        ok = false;
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
            }
            if (!ok) break;
            // The finished unit: the logits (bias added) when a token tile is
            // one unit, otherwise this split's partial sums.
            const int tl = static_cast<int>(rank) * kTokCta + q * 32 + lane;
            const int t = un.m * kTokTileR + tl;
            const int e0 = un.n * BN + col0;
            if (a.n_tiles * a.ksplit == 1) {
                if (t < a.T) {
                    float *lrow = a.logits + (int64_t)t * a.E + e0;
#pragma unroll
                    for (int j = 0; j < COLS; ++j)
                        if (e0 + j < a.E) lrow[j] = a.b_gate ? __fadd_rn(sum[j], __ldg(a.b_gate + e0 + j)) : sum[j];
                }
            } else {
                float4 *prow = reinterpret_cast<float4 *>(a.part + ((int64_t)u * kTokTileR + tl) * BN + col0);
#pragma unroll
                for (int j = 0; j < COLS; j += 4) prow[j / 4] = make_float4(sum[j], sum[j + 1], sum[j + 2], sum[j + 3]);
            }
        }
    }

    // A role that gave up may leave its own TMA loads in flight; give them a
    // millisecond to land before the pair meets.
    if (!ok || *reinterpret_cast<volatile uint32_t *>(a.status) != kDevOk) spin_ns(1000000ull);

    // ---------------------------------------------------------------- phase B
    if (grid_barrier(a.counters, a.status)) {
        const int nb = gridDim.x;
        const int chunk = (a.T + nb - 1) / nb;
        const int t_begin = min(a.T, (int)blockIdx.x * chunk), t_end = min(a.T, t_begin + chunk);
        route_tokens<BN, RE>(a, s.red, warp, C::kWarps, lane, t_begin, t_end);
        if (a.route) {
            __syncthreads();
            // This CTA's row of P sums: the warps' sums added in warp order.
            for (int e = threadIdx.x; e < a.E; e += C::kThreads) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < C::kWarps; ++w) v += s.red[w * 256 + e];
                a.psum_part[(int64_t)blockIdx.x * a.E + e] = v;
            }
        }
    }
    tc_fence_before_sync();
    cluster_sync_all();
    tc_fence_after_sync();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
}

template <int BN, int RE>
cudaError_t launch_cfg(const CUtensorMap &mx, const CUtensorMap &mw, const RouterFusedArgs &a, cudaStream_t s) {
    constexpr int kSmem = RCfg<BN>::kSmem;
    cudaError_t e = set_smem_limit_once<router_fused_kernel<BN, RE>>(kSmem);
    if (e != cudaSuccess) return e;
    const int total = a.n_mtiles * a.n_tiles * a.ksplit;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(router_fused_ctas(total, a.num_pairs), 1, 1);
    cfg.blockDim = dim3(RCfg<BN>::kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = s;
    // Cooperative: phase B starts after a grid-wide barrier, which needs every
    // CTA resident at once (the grid is at most the co-resident pairs).
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, router_fused_kernel<BN, RE>, mx, mw, a);
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap &mx, const CUtensorMap &mw, const RouterFusedArgs &a, cudaStream_t s) {
    if (a.E <= 32) return launch_cfg<BN, 1>(mx, mw, a, s);
    if (a.E <= 64) return launch_cfg<BN, 2>(mx, mw, a, s);
    if (a.E <= 128) return launch_cfg<BN, 4>(mx, mw, a, s);
    return launch_cfg<BN, 8>(mx, mw, a, s);
}

// W_g [E][d] fp32 -> [E_pad][3d] bf16 planes hi | mid | lo (rows >= E are zero).
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

}  // namespace

int router_fused_epad(int E) {
    int p = 32;
    while (p < E && p < 128) p <<= 1;
    return p < E ? 256 : p;
}

int router_fused_bn(int E) { return router_fused_epad(E) < 128 ? router_fused_epad(E) : 128; }

int router_fused_mtiles(int T) { return (T + kTokTileR - 1) / kTokTileR; }

// K splits: the fewest waves of units per unit of work, ceil(units ks / pairs) / ks,
// over ks = 1, 2, 4, 8 with at least one drain group per split; ties keep fewer
// splits.
int router_fused_ksplit(int T, int E, int d, int num_pairs) {
    const int units = router_fused_mtiles(T) * (router_fused_epad(E) / router_fused_bn(E));
    const int dblocks = d / kBK;
    if (units <= 0 || num_pairs <= 0) return 1;
    int best = 1;
    double best_cost = 1e30;
    for (int ks = 1; ks <= 8 && ks <= dblocks / kDrain; ks *= 2) {
        const double cost = (double)((units * ks + num_pairs - 1) / num_pairs) / ks;
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = ks;
        }
    }
    return best;
}

int router_fused_ctas(int units, int num_pairs) { return 2 * (units < num_pairs ? units : num_pairs); }

int router_fused_max_pairs(int num_sms) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    cfg.blockDim = dim3(RCfg<128>::kThreads, 1, 1);
    constexpr int kSmem = RCfg<128>::kSmem;  // the largest of the three layouts
    cfg.dynamicSmemBytes = kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kern = router_fused_kernel<128, 8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) return 0;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) return 0;
    return clusters < num_sms / 2 ? clusters : num_sms / 2;
}

cudaError_t launch_router_split(const float *w_gate, int E, int E_pad, int d, __nv_bfloat16 *w_split, int num_sms,
                                cudaStream_t s, int *launches) {
    const int64_t n = (int64_t)E_pad * d;
    int blocks = (int)((n + 255) / 256);
    if (blocks > num_sms * 16) blocks = num_sms * 16;
    router_split_kernel<<<blocks, 256, 0, s>>>(w_gate, E, E_pad, d, w_split);
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_router_fused(const CUtensorMap &map_x, const CUtensorMap &map_w, const RouterFusedArgs &a,
                                cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    if (a.num_pairs <= 0) return cudaErrorInvalidConfiguration;
    ++*launches;
    switch (a.BN) {
        case 32: return launch_bn<32>(map_x, map_w, a, s);
        case 64: return launch_bn<64>(map_x, map_w, a, s);
        case 128: return launch_bn<128>(map_x, map_w, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
