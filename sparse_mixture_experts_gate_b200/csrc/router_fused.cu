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
// Routing. Each CTA writes its finished unit (fp32 partial sums, or the logits
// themselves when a token tile is one unit) and counts it on its half tile's
// arrival counter; the CTA that completes a half tile (128 tokens) adds the
// partials in a fixed order (expert tile, then K split), adds the bias, writes
// the logits and routes the 128 tokens, a warp per token (route_common.cuh).
// Nothing waits for another CTA: the last to arrive does the work.
//
// Roles (320 threads per CTA): warp 0 loads (TMA), warp 1 owns TMEM and, in
// the leader, issues the MMAs; warps 2..9 drain the accumulators (two warps per
// TMEM lane quarter, BN/2 columns each) and route. Every wait is bounded; on a
// timeout the roles stop, in-flight copies and MMAs are drained, both CTAs meet
// at the cluster barrier and TMEM is freed.
#include "moe_common.cuh"
#include "moe_kernels.cuh"
#include "route_common.cuh"

namespace moe {
namespace {

constexpr int kTokCta = 128;      // token rows per CTA; the pair's M is 256
constexpr int kTokTileR = 256;    // tokens per unit
constexpr int kDrain = 2;         // K blocks of 64 per partial accumulator

// Epilogue warps: two per TMEM lane quarter (BN / 2 columns of running sums
// per thread).
template <int BN>
struct RCfg {
    static constexpr int kEpiWarps = 8;
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kA = kTokCta * kBK * 2;          // x rows of this CTA, one K block
    static constexpr int kBHalf = (BN / 2) * kBK * 2;     // one plane, this CTA's BN/2 expert rows
    static constexpr int kStage = kA + 3 * kBHalf;
    static constexpr int kStages = (200 * 1024) / kStage < 8 ? (200 * 1024) / kStage : 8;
    static constexpr int kTmemCols = 2 * BN;              // two partial buffers
    static constexpr int kRedBytes = kEpiWarps * 256 * 4;  // per-warp P sums of a half tile
    static constexpr int kCols = BN / (kEpiWarps / 4);     // accumulator columns per epilogue thread
    static constexpr int kSmem = 1024 + kStages * kStage + kRedBytes + 512;
    static_assert(BN == 32 || BN == 64 || BN == 128, "expert tile");
    static_assert(kBHalf % 1024 == 0, "plane tiles keep the 1024-byte swizzle alignment");
    static_assert(kSmem <= 232448, "exceeds the shared memory a CTA may use");
};

struct RSmem {
    uint8_t *stages;
    float *red;
    uint64_t *full, *empty, *tfull, *tempty, *mma_done, *epi_done, *route_go;
    uint32_t *tmem_slot;
    int32_t *flag;
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
    s.mma_done = s.tempty + 2;
    s.epi_done = s.mma_done + 1;
    s.route_go = s.epi_done + 1;
    s.tmem_slot = reinterpret_cast<uint32_t *>(s.route_go + 1);
    s.flag = reinterpret_cast<int32_t *>(s.tmem_slot + 2);
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

// Logits of the 128 tokens of half tile (m, rank) from the finished units
// (pieces > 1): sum over the K splits of each expert tile's partials, in split
// order, plus the bias, written to the logits output. All epilogue threads
// share the work, four experts of one token per item; a thread keeps up to 16
// loads in flight (several items' splits at once), so a half tile costs a few
// L2 round trips rather than one per item.
template <int BN>
__device__ __forceinline__ void merge_half_tile(const RouterFusedArgs &a, int m, int rank, int et) {
    constexpr int kEpiWarps = RCfg<BN>::kEpiWarps;
    constexpr int kNT = kEpiWarps * 32;
    // Loads in flight per thread: eight, or four with 128-expert tiles (whose
    // epilogue threads hold 64 running sums).
    constexpr int kL = BN == 128 ? 4 : 8;
    const int ks = a.ksplit;                       // 1, 2, 4 or 8
    const int per_batch = ks >= kL ? 1 : kL / ks;  // items per batch
    const int E4 = (a.E + 3) / 4;                  // items per token
    const bool vec_out = (a.E & 3) == 0;
    const int64_t stride = (int64_t)kTokTileR * BN / 4;  // float4s between two splits of a tile
    const int n_items = kTokCta * E4;
    const int t0 = m * kTokTileR + rank * kTokCta;
    for (int base = et; base < n_items; base += kNT * per_batch) {
        // Load slot j = (item base + (j / ks) * kNT, split j % ks); with more
        // splits than slots, the item's remaining splits are added below.
        float4 v[kL];
#pragma unroll
        for (int j = 0; j < kL; ++j) {
            const int item = base + (j / ks) * kNT;
            const int i = item / E4, e = (item - i * E4) * 4;
            if (item < n_items && t0 + i < a.T) {
                const int n = e / BN, c = e - n * BN;  // BN is a multiple of 4: one tile per item
                const float4 *src = reinterpret_cast<const float4 *>(
                    a.part + ((int64_t)((m * a.n_tiles + n) * ks) * kTokTileR + rank * kTokCta + i) * BN + c);
                if (j % ks < kL) v[j] = __ldcg(src + (j % ks) * stride);
            }
        }
        // Sums in split order; an item's logits are written after its last split.
        float4 h = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < kL; ++j) {
            const int sp = j % ks;
            if (sp == 0) {
                h = v[j];
            } else {
                h.x = __fadd_rn(h.x, v[j].x);
                h.y = __fadd_rn(h.y, v[j].y);
                h.z = __fadd_rn(h.z, v[j].z);
                h.w = __fadd_rn(h.w, v[j].w);
            }
            if (sp != ks - 1 && j != kL - 1) continue;
            const int item = base + (j / ks) * kNT;
            const int i = item / E4, e = (item - i * E4) * 4;
            if (item >= n_items || t0 + i >= a.T) continue;
            if (ks > kL) {  // the splits beyond the slots, in order
                const int n = e / BN, c = e - n * BN;
                const float4 *src = reinterpret_cast<const float4 *>(
                    a.part + ((int64_t)((m * a.n_tiles + n) * ks) * kTokTileR + rank * kTokCta + i) * BN + c);
                for (int sp2 = kL; sp2 < ks; ++sp2) {
                    const float4 w = __ldcg(src + sp2 * stride);
                    h.x = __fadd_rn(h.x, w.x);
                    h.y = __fadd_rn(h.y, w.y);
                    h.z = __fadd_rn(h.z, w.z);
                    h.w = __fadd_rn(h.w, w.w);
                }
            }
            float hv[4] = {h.x, h.y, h.z, h.w};
            if (a.b_gate)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (e + q < a.E) hv[q] = __fadd_rn(hv[q], __ldg(a.b_gate + e + q));
            float *row = a.logits + (int64_t)(t0 + i) * a.E + e;
            if (vec_out) {
                *reinterpret_cast<float4 *>(row) = make_float4(hv[0], hv[1], hv[2], hv[3]);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (e + q < a.E) row[q] = hv[q];
            }
        }
    }
}

// Routes the 128 tokens of half tile (m, rank) from their logits: a warp per
// token (route_common.cuh), the next token's logits (and noise) loaded before
// the current token is routed; a selection bias, the same for every token, is
// loaded once. Then this warp's per-expert P sums go to the shared rows.
template <int BN, int RE>
__device__ __forceinline__ void route_half_tile(const RouterFusedArgs &a, const RSmem &s, int m, int rank, int ew,
                                                int lane) {
    constexpr int kEpiWarps = RCfg<BN>::kEpiWarps;
    float pacc[RE];
#pragma unroll
    for (int q = 0; q < RE; ++q) pacc[q] = 0.f;
    const int t0 = m * kTokTileR + rank * kTokCta;
    const bool has_add = a.noise != nullptr || a.sel_bias != nullptr;
    float kadd[RE];
    if (!a.noise) key_addend<RE>(t0, lane, a, kadd);  // the selection bias (or nothing)
    auto load = [&](int i, float (&h)[RE], float (&nz)[RE]) -> bool {
        const int t = t0 + i;
        if (i >= kTokCta || t >= a.T) return false;
#pragma unroll
        for (int q = 0; q < RE; ++q) {
            const int e = lane + 32 * q;
            h[q] = e < a.E ? __ldcg(a.logits + (int64_t)t * a.E + e) : -INFINITY;
            if (a.noise) nz[q] = e < a.E ? __ldg(a.noise + (int64_t)t * a.E + e) : 0.f;
        }
        return true;
    };
    float h[RE], nz[RE];
    if constexpr (BN < 128) {  // the next token's loads in flight while this one is routed
        float h2[RE], nz2[RE];
        bool have = load(ew, h, nz);
        for (int i = ew; have; i += kEpiWarps) {
            const bool next = load(i + kEpiWarps, h2, nz2);
            if (a.noise) {
                route_warp<RE>(h, has_add, nz, t0 + i, lane, a, pacc);
            } else {
                route_warp<RE>(h, has_add, kadd, t0 + i, lane, a, pacc);
            }
#pragma unroll
            for (int q = 0; q < RE; ++q) {
                h[q] = h2[q];
                nz[q] = nz2[q];
            }
            have = next;
        }
    } else {  // 128-expert tiles: the registers go to the running sums; no prefetch
        for (int i = ew; load(i, h, nz); i += kEpiWarps) {
            if (a.noise) {
                route_warp<RE>(h, has_add, nz, t0 + i, lane, a, pacc);
            } else {
                route_warp<RE>(h, has_add, kadd, t0 + i, lane, a, pacc);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < RE; ++q) s.red[ew * 256 + lane + 32 * q] = pacc[q];
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
            mbar_init(&s.tempty[i], 2 * kEpiWarps);  // the epilogue warps of both CTAs
        }
        mbar_init(s.mma_done, 1);
        mbar_init(s.epi_done, kEpiWarps);
        mbar_init(s.route_go, 1);
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
                if (lane == 0) got = mbar_wait(&s.empty[st], ph ^ 1u, a.status) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
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
                    if (!mbar_wait(&s.tempty[buf], (use & 1u) ^ 1u, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t d_tmem = tmem_base + buf * BN;
                    const int g1 = min(g0 + kDrain, un.kb1);
                    for (int kb = g0; kb < g1; ++kb, ++it) {
                        const int st = it % kStages;
                        const uint32_t ph = (it / kStages) & 1u;
                        if (!mbar_wait(&s.full[st], ph, a.status)) {
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
    } else {
        // ------------------------------------------------------------ epilogue + routing
        const int ew = warp - 2;
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int col0 = (ew >> 2) * COLS;       // this warp's columns of the expert tile
        // Phases completed so far of epi_done (once per unit, once more per
        // routed half tile) and of route_go (once per unit).
        uint32_t gcount = 0, epi_n = 0, go_n = 0;
        for (int u = pair; u < total && ok; u += n_pairs, ++go_n) {
            const Unit un = unit_of(a, u);
            float sum[COLS];
#pragma unroll
            for (int j = 0; j < COLS; ++j) sum[j] = 0.f;
            for (int g0 = un.kb0; g0 < un.kb1; g0 += kDrain, ++gcount) {
                const uint32_t buf = gcount & 1u, use = gcount >> 1;
                int got = 1;
                if (lane == 0) got = mbar_wait(&s.tfull[buf], use & 1u, a.status) ? 1 : 0;
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
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.tempty[buf]), 0));
            }
            if (!ok) break;
            // The finished unit: logits (one unit per tile) or partial sums.
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
            // Count the unit on the half tile's counter once all epilogue warps
            // have written (their arrivals release the writes to the counting
            // thread, whose device-scope fence then publishes them all); the CTA
            // that completes the half tile routes it.
            __syncwarp();
            if (lane == 0) mbar_arrive(s.epi_done);
            if (ew == 0) {
                int flag = 0;
                if (lane == 0) {
                    if (mbar_wait(s.epi_done, epi_n & 1u, a.status)) {
                        __threadfence();
                        const int old = atomicAdd(a.counters + un.m * 2 + static_cast<int>(rank), 1);
                        flag = old == a.n_tiles * a.ksplit - 1 ? 1 : 0;
                        __threadfence();  // the other CTAs' partials are read after this
                    } else {
                        flag = -1;
                    }
                    *s.flag = flag;
                    mbar_arrive(s.route_go);
                }
            }
            ++epi_n;
            // Every lane acquires route_go: the routing below reads partials
            // that other CTAs wrote before their arrivals were counted.
            int flag = mbar_wait_all_lanes(s.route_go, go_n & 1u, a.status) ? *reinterpret_cast<volatile int32_t *>(s.flag)
                                                                            : -1;
            if (flag < 0) {
                ok = false;
                break;
            }
            if (flag) {
                if (a.n_tiles * a.ksplit > 1) {
                    merge_half_tile<BN>(a, un.m, static_cast<int>(rank), ew * 32 + lane);
                    // Every warp's logits written before any lane routes from them.
                    __threadfence_block();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s.epi_done);
                    const bool got = mbar_wait_all_lanes(s.epi_done, epi_n & 1u, a.status);
                    ++epi_n;
                    if (!got) {
                        ok = false;
                        break;
                    }
                }
                if (a.route) {
                    route_half_tile<BN, RE>(a, s, un.m, static_cast<int>(rank), ew, lane);
                    // The half tile's P sums: every warp's row, added in warp order
                    // (every lane acquires the rows the other warps wrote).
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s.epi_done);
                    const bool got = mbar_wait_all_lanes(s.epi_done, epi_n & 1u, a.status);
                    ++epi_n;
                    if (!got) {
                        ok = false;
                        break;
                    }
                    float *prow = a.psum_part + (int64_t)(un.m * 2 + static_cast<int>(rank)) * a.E;
                    for (int e = ew * 32 + lane; e < a.E; e += kEpiWarps * 32) {
                        float v = 0.f;
#pragma unroll
                        for (int w = 0; w < kEpiWarps; ++w) v += s.red[w * 256 + e];
                        prow[e] = v;
                    }
                    // s.red is written again only by a later routing, which
                    // starts after a route_go phase that needs every warp's
                    // epi_done arrival, made after this loop.
                }
            }
        }
    }

    // A role that gave up may leave its own TMA loads in flight; give them a
    // millisecond to land before the pair meets.
    if (!ok || *reinterpret_cast<volatile uint32_t *>(a.status) != kDevOk) spin_ns(1000000ull);
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
    const int pairs = total < a.num_pairs ? total : a.num_pairs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(RCfg<BN>::kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
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
