// gemm_pair.cu - grouped expert GEMM on CTA pairs (sm_100a tcgen05 cta_group::2).
//
// "Code Walkthrough - SER", gating / routing path: each selected expert runs its
// two-layer MLP, w1/b1 -> activation -> w2/b2, on the rows dispatched to it;
// shared experts ("Appendix C - Acronyms & Symbols", "Parameter accounting")
// run the same MLP on every token. Both layers of every expert are dense
// contractions, computed here as grouped GEMMs over the permuted row space:
//   out[row][f] = act( sum_k A[row][k] W[g][f][k] + b[g][f] ),  g = group of row.
// Layer 1: A = the routed token rows scattered into row order (dispatch.cu), or
// x itself for the shared experts, which read every token in order.
// Layer 2: A = the hidden activations H (already in row order).
// A forward runs both layers in one launch: layer 2's units of a token tile
// start as soon as every layer-1 unit of that tile has stored its rows of H
// (a per-tile counter, see the producer and the epilogue), so layer 2 fills
// layer 1's last wave. Expert parallelism runs one layer per launch.
//
// Operand roles. The tensor cores compute out^T: the MMA's M side is 256 output
// features (weights W[g], 128 per CTA of the pair) and its N side is a token
// tile of up to 256 rows of one expert. Each expert's rows are padded only to a
// multiple of 32 (the row space's block), instead of to the M extent, and the
// weight tile, the operand every token of the expert shares, is split across
// the pair so that each SM stages half of it.
//
// Units are handed out in index order from a global counter (see post_unit),
// so the pairs at work hold a contiguous run of units whatever their lengths:
// with a static round-robin the pairs drift apart over the ~140 waves of the
// E = 256 layer's first GEMM and the L2 reuse of the weight tiles collapses (it
// read 41.6 GB from DRAM instead of ~15 GB).
//
// Per CTA (192 threads): warp 0 loads (TMA, signalling the leader's stage
// barrier, which expects both CTAs' bytes), warp 1 owns TMEM (2 accumulators x
// 256 columns) and, in the leader, issues the pair MMAs and commits stages and
// accumulators to both CTAs at once; warps 2..5 drain this CTA's 128 features:
// each warp reads 32 features x 32 tokens from TMEM, adds the bias, applies the
// activation, pairs neighbouring lanes' values so that each lane holds two
// adjacent features of one token, and writes them into a shared box of 32
// tokens x 128 features (token-major, 256-byte rows) that the four warps fill
// together; one thread stores each box with a TMA tensor store. One epilogue
// thread takes each unit and waits for its accumulator, and the four warps
// agree on it at a named barrier, so all of them pass the same barriers and
// leave together. The epilogue releases an accumulator by arriving on the
// leader's barrier (one arrival per epilogue warp of both CTAs).
//
// Ragged last feature tile. When N leaves a last feature tile of at most 128
// features (d_ff = 1408 = 5.5 x 256, say), a unit of that tile would leave
// half of the pair's M side idle. Such units run transposed instead: the token
// tile is the MMA's M side (each CTA's half of the tokens on its 128 TMEM
// lanes) and the 128 features are its N side (64 weight rows staged per CTA),
// so the pair stages a quarter fewer bytes and issues half the MMA work for
// the same outputs. Their epilogue holds a token's 32 consecutive features per
// lane and writes them to global memory directly (64 bytes per token row).
//
// Every wait is bounded (mbar_wait); on a timeout the roles stop, the leader
// drains its MMAs, copies in flight are given time to land, both CTAs meet at
// the cluster barrier, and TMEM is freed.
#include <type_traits>

#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kEpiWarps = 4;                        // epilogue warps per CTA, one per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;
// Output stores: true, the four epilogue warps fill a shared box of 32 tokens
// x 128 features (256-byte rows) that one thread stores with a TMA tensor
// store; false, every lane stores its own 32-bit pairs (64-byte pieces of rows).
constexpr bool kWideStores = true;
constexpr int kFeatPair = 256;                     // MMA M: features per pair tile
constexpr int kFeatCta = 128;                      // features per CTA
constexpr int kOutBoxBytes = 32 * kFeatCta * 2;    // one staged output box: 32 tokens x 128 features
constexpr int kABytes = kFeatCta * kBK * 2;        // 16 KB: 128 weight rows x 64 K
constexpr int kAccCols = 256;
constexpr int kBoxTok = 32;                         // tokens per TMEM load of the epilogue
constexpr int kRowsPerLoad16 = 16;                  // rows of the narrow token box
constexpr int kRing = 8;            // unit-index ring between the leader's producer and the consumers
// leader: MMA thread + the epilogue (its one unit-taking thread with wide
// stores, else every epilogue warp); peer: producer + the epilogue
constexpr int kRingConsumers = kWideStores ? 4 : 2 * (1 + kEpiWarps);
static_assert(kTokTile == 256 && kTokTile % (2 * kRowsPerLoad16) == 0, "token tile layout");
static_assert(kNarrowTile % (2 * kRowsPerLoad16) == 0, "narrow token tile layout");

// Stage layout for token tiles of up to TILE rows (each CTA stages TILE / 2):
// 256-row tiles with 6 stages of 32 KB, or narrow 64-row tiles with 10 stages
// of 20 KB, which keeps 160 KB of weight tiles in flight per SM when the
// token tiles are short and the GEMM streams weights (one stage more of each
// when the outputs are stored from registers, without staging boxes).
template <int TILE>
struct PairCfg {
    static constexpr int kB = (TILE / 2) * kBK * 2;
    static constexpr int kStage = kABytes + kB;
    static constexpr int kStaging = kWideStores ? 2 * kOutBoxBytes : 0;
    static constexpr int kStages = (TILE == kTokTile ? 7 : 11) - (kWideStores ? 1 : 0);
    static constexpr int kSmem = 1024 + kStages * kStage + kStaging + 512;
    static_assert(kSmem <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
    static_assert(kB % 1024 == 0, "B stages keep the 1024-byte swizzle alignment");
};

struct Smem {
    uint8_t *sA, *sB, *staging;
    uint64_t *full, *empty, *tfull, *tempty, *mma_done, *ring_full, *ring_empty;
    uint32_t *tmem_slot;
    int32_t *ring;
    int32_t *epi_unit;  // [2] the unit the epilogue drains, by parity (wide stores)
};

template <int TILE>
__device__ __forceinline__ Smem carve(uint8_t *raw) {
    using C = PairCfg<TILE>;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    Smem s;
    s.sA = base;
    s.sB = base + C::kStages * kABytes;
    s.staging = base + C::kStages * C::kStage;
    s.full = reinterpret_cast<uint64_t *>(s.staging + C::kStaging);
    s.empty = s.full + C::kStages;
    s.tfull = s.empty + C::kStages;
    s.tempty = s.tfull + 2;
    s.mma_done = s.tempty + 2;
    s.ring_full = s.mma_done + 1;
    s.ring_empty = s.ring_full + kRing;
    s.tmem_slot = reinterpret_cast<uint32_t *>(s.ring_empty + kRing);
    s.ring = reinterpret_cast<int32_t *>(s.tmem_slot + 4);
    s.epi_unit = s.ring + kRing;
    return s;
}

// Named barrier 1 over the four epilogue warps (threads 64..191).
__device__ __forceinline__ void epi_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Layer 2 of a two-layer launch: its maps and arguments (a copy of layer 1's
// in a one-layer launch, unused there).
struct Layer2 {
    PairMaps m;
    PairGemmArgs a;
};

template <int ACT, int TILE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ PairMaps m1, const PairGemmArgs a,
                             const __grid_constant__ Layer2 l2) {
    const PairMaps &m2 = l2.m;
    const PairGemmArgs &b = l2.a;
    using C = PairCfg<TILE>;
    constexpr int kStages = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    const Smem s = carve<TILE>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const bool two = a.fuse2 != 0;  // layer 2 (b, m2) follows layer 1 (a, m1) in this launch

    if (threadIdx.x == 0) {
        for (int l = 0; l < (two ? 2 : 1); ++l) {
            const PairMaps &m = l ? m2 : m1;
            tma_prefetch_desc(&m.w);
            if ((l ? b : a).half_last) tma_prefetch_desc(&m.wh);
            tma_prefetch_desc(&m.t);
            tma_prefetch_desc(&m.t16);
            if ((l ? b : a).use_s) {
                tma_prefetch_desc(&m.s);
                tma_prefetch_desc(&m.s16);
            }
            if (kWideStores) tma_prefetch_desc(&m.out);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], 2 * kEpiWarps);  // the epilogue warps of both CTAs
        }
        mbar_init(s.mma_done, 1);
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&s.ring_full[i], 1);
            mbar_init(&s.ring_empty[i], kRingConsumers);  // used in the leader only
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(s.tmem_slot, 2 * kAccCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated in both
    tc_fence_after_sync();
    const uint32_t tmem_base = *s.tmem_slot;

    const int4 *tok_tiles = a.tok_tiles + (a.tile_base_word >= 0 ? a.ctrl[a.tile_base_word] : 0);
    const int n_tt = a.fixed_tiles > 0 ? a.fixed_tiles : min(a.ctrl[a.tiles_count_word], a.max_tok_tiles);
    // Units are numbered layer by layer: (token tile, feature tile) of layer
    // 1, then of layer 2, which reads layer 1's output rows.
    const int total1 = n_tt * a.n_ftiles;
    const int total = total1 + (two ? n_tt * b.n_ftiles : 0);
    // Layer of unit u, with its token tile and feature tile.
    auto decode = [&](int u, int &tt, int &j) -> int {
        const int l = u >= total1 ? 1 : 0;
        const int v = u - (l ? total1 : 0), nf = l ? b.n_ftiles : a.n_ftiles;
        tt = v / nf;
        j = v - tt * nf;
        return l;
    };
    // Weight-stack index of group g (shared groups may sit at another base).
    auto wgroup = [&](int g) { return g < a.E ? g : a.w_shared_base + (g - a.E); };
    // The last feature tile of a layer runs transposed (wide token tiles only).
    auto tr_tile = [&](int l) {
        const PairGemmArgs &P = l ? b : a;
        return (TILE == kTokTile && P.half_last) ? P.n_ftiles - 1 : -1;
    };
    bool ok = true;

    // Units are handed out in index order from a global counter, so the pairs
    // working at any moment hold a contiguous run of units and share their
    // weight and token tiles through L2, however unequal the units' lengths.
    // The leader's producer takes each unit and posts it to a ring in both
    // CTAs; every consumer reads entry i for its i-th unit and releases it on
    // the leader's ring_empty. -1 ends the work.
    auto post_unit = [&](uint32_t i) -> int {  // leader's producer, lane 0
        const uint32_t slot = i % kRing, ph = (i / kRing) & 1u;
        if (!mbar_wait_cluster(&s.ring_empty[slot], ph ^ 1u, a.status, a.wait_limit_ns)) return -2;
        int u = atomicAdd(a.work_counter, 1);
        if (u >= total) u = -1;
        s.ring[slot] = u;
        st_shared_cluster_u32(mapa_shared(smem_u32(&s.ring[slot]), 1), static_cast<uint32_t>(u));
        mbar_arrive(&s.ring_full[slot]);
        mbar_arrive_cluster(mapa_shared(smem_u32(&s.ring_full[slot]), 1));
        return u;
    };
    auto take_unit = [&](uint32_t i) -> int {  // one thread of each consumer
        const uint32_t slot = i % kRing, ph = (i / kRing) & 1u;
        if (!mbar_wait_cluster(&s.ring_full[slot], ph, a.status, a.wait_limit_ns)) return -2;
        const int u = *reinterpret_cast<volatile int32_t *>(&s.ring[slot]);
        mbar_arrive_cluster(mapa_shared(smem_u32(&s.ring_empty[slot]), 0));
        return u;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        uint32_t it = 0;
        for (uint32_t i = 0; ok; ++i) {
            int u = 0;
            if (lane == 0) u = leader ? post_unit(i) : take_unit(i);
            u = __shfl_sync(0xffffffffu, u, 0);
            if (u < 0) {
                ok = u == -1;
                break;
            }
            int tt, j;
            const int l = decode(u, tt, j);
            const PairGemmArgs &P = l ? b : a;
            const PairMaps &m = l ? m2 : m1;
            const int4 tile = tok_tiles[tt];  // {group, first row, rows, -}
            const int g = tile.x, ntok = tile.z;
            const CUtensorMap *mt = &m.t, *mt16 = &m.t16;
            int trow = tile.y + static_cast<int>(rank) * (ntok / 2);
            if (P.use_s && g >= a.E) {  // shared expert: rows of x in token order
                mt = &m.s;
                mt16 = &m.s16;
                trow -= a.group_start[g];
            }
            if (l == 1) {
                // Layer 2 reads the token tile's layer-1 outputs: wait until
                // every layer-1 unit of the tile has stored them (both CTAs
                // count), then order the tensor loads after that acquire.
                int got = 1;
                if (lane == 0)
                    got = wait_counter_geq(a.tile_done + tt, 2 * a.n_ftiles, a.status, a.wait_limit_ns) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) {
                    ok = false;
                    break;
                }
                fence_proxy_async_global();
            }
            const bool tr = j == tr_tile(l);  // 64 weight rows per CTA (the MMA's N side)
            const int wrow = wgroup(g) * P.N + j * kFeatPair + static_cast<int>(rank) * (tr ? kFeatCta / 2 : kFeatCta);
            const CUtensorMap *mw = tr ? &m.wh : &m.w;
            const uint32_t tx_bytes = (tr ? 1u : 2u) * kABytes + static_cast<uint32_t>(ntok) * kBK * 2u;
            const int n16 = ntok / (2 * kRowsPerLoad16);
            const int kblocks = P.K / kBK;
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                const int st = it % kStages;
                const uint32_t ph = (it / kStages) & 1u;
                int got = 1;
                if (lane == 0) got = mbar_wait(&s.empty[st], ph ^ 1u, a.status, a.wait_limit_ns) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) {
                    ok = false;
                    break;
                }
                if (lane == 0 && leader) mbar_arrive_expect_tx(&s.full[st], tx_bytes);
                __syncwarp();
                // Self-test of the timeout path: the leader announces this
                // stage's bytes but loads none of its own, so the stage never
                // completes and the MMA role's bounded wait runs out.
                if (leader && static_cast<int>(it) == a.skip_stage) continue;
                const uint32_t bar = mapa_shared(smem_u32(&s.full[st]), 0);
                uint8_t *sA = s.sA + st * kABytes, *sB = s.sB + st * C::kB;
                if (lane == 0) tma_load_2d_pair(mw, bar, sA, kb * kBK, wrow);
                if (ntok == kTokTile) {
                    if (lane == 1) tma_load_2d_pair(mt, bar, sB, kb * kBK, trow);
                } else if (lane < n16) {
                    tma_load_2d_pair(mt16, bar, sB + lane * kRowsPerLoad16 * 128, kb * kBK,
                                     trow + lane * kRowsPerLoad16);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA (leader)
        if (leader && lane == 0) {
            uint32_t it = 0;
            for (uint32_t tcount = 0; ok; ++tcount) {
                const int u = take_unit(tcount);
                if (u < 0) {
                    ok = u == -1;
                    break;
                }
                int tt, j;
                const int l = decode(u, tt, j);
                const int ntok = tok_tiles[tt].z;
                const int kblocks = (l ? b : a).K / kBK;
                // Transposed unit: A = the token tile (M = 256, each CTA's
                // ntok / 2 rows first), B = the 128 features (64 rows per CTA).
                const bool tr = j == tr_tile(l);
                const uint32_t idesc = tr ? idesc_bf16_f32(kTokTile, kFeatCta) : idesc_bf16_f32(kFeatPair, ntok);
                const uint32_t acc = tcount & 1u, use = tcount >> 1;
                if (!mbar_wait(&s.tempty[acc], (use & 1u) ^ 1u, a.status, a.wait_limit_ns)) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kAccCols;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int st = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(&s.full[st], ph, a.status, a.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t ad = sw128_kmajor_desc(smem_u32(s.sA + st * kABytes));
                    const uint64_t bd = sw128_kmajor_desc(smem_u32(s.sB + st * C::kB));
                    const uint64_t da = tr ? bd : ad, db = tr ? ad : bd;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma_bf16_pair(d_tmem, da + 2u * kk, db + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
                    tc_commit_pair_mc(&s.empty[st], 0x3);
                }
                if (ok) tc_commit_pair_mc(&s.tfull[acc], 0x3);
            }
            tc_commit_pair(s.mma_done);
            mbar_wait_drain(s.mma_done, 0u);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;        // TMEM lane quarter this warp may access
        const int ep = threadIdx.x - 64;  // 0..127 over the four epilogue warps
        uint32_t sub = 0;              // output boxes staged so far (buffer parity)
        // Two-layer launches: thread ep 0 publishes each layer-1 unit's outputs
        // one unit late, once the next unit's stores are under way (its own
        // bulk groups complete in order), so it rarely waits; the pending unit
        // is published at once when the next unit is a layer-2 one or the work
        // ends, before that unit's accumulator is awaited, so that no layer-2
        // producer of this pair can wait on it.
        int pend_tt = -1;
        auto publish = [&](int tile) {
            fence_proxy_async_global();
            red_release_add(a.tile_done + tile, 1);
        };
        // Drains one unit's accumulator with the activation ACT_C of its layer.
        auto drain = [&](auto act_c, const PairGemmArgs &P, const PairMaps &m, int tr, int u_tt, int j,
                         uint32_t acc) {
            constexpr int A = decltype(act_c)::value;
            const int4 tile = tok_tiles[u_tt];
            const int g = tile.x, row0 = tile.y, ntok = tile.z;
            const int fbase = j * kFeatPair + static_cast<int>(rank) * kFeatCta;
            const int fcol = fbase + q * 32;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
            if (j == tr) {
                // Transposed unit: TMEM lane = token (this CTA's ntok / 2
                // tokens first), column = feature. Each lane activates 32
                // consecutive features of its token and stores them as 64
                // bytes; chunks past N (N % 256 == 64) are not stored.
                const int half = ntok / 2, tok = q * 32 + lane;
                const int f0 = j * kFeatPair;
                __nv_bfloat16 *orow =
                    P.out + (static_cast<int64_t>(row0) + static_cast<int64_t>(rank) * half + tok) * P.N;
#pragma unroll 1
                for (int c = 0; c < kFeatCta && f0 + c < P.N; c += 32) {
                    const float bl = P.bias ? __ldg(P.bias + (int64_t)wgroup(g) * P.N + f0 + c + lane) : 0.f;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + c, r);
                    tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float z0 = activate_t<A>(__uint_as_float(r[2 * i]) + __shfl_sync(0xffffffffu, bl, 2 * i));
                        const float z1 =
                            activate_t<A>(__uint_as_float(r[2 * i + 1]) + __shfl_sync(0xffffffffu, bl, 2 * i + 1));
                        __nv_bfloat162 p2 = __floats2bfloat162_rn(z0, z1);
                        pk[i] = *reinterpret_cast<uint32_t *>(&p2);
                    }
                    if (tok < half) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + f0 + c);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    }
                }
                return;
            }
            // Lane = feature, register = token. Neighbouring lanes trade one
            // value per token pair, so the even lane holds features (f, f+1)
            // of token t and the odd lane those of token t+1: one bf16x2
            // conversion and one 32-bit store each. The last feature tile of
            // a ragged N leaves the warps past N idle.
            const bool valid = fcol < P.N;
            const float bv = valid && P.bias ? __ldg(P.bias + (int64_t)wgroup(g) * P.N + fcol + lane) : 0.f;
            const uint32_t odd = lane & 1u;
#pragma unroll 1
            for (int c = 0; c < ntok; c += kBoxTok) {
                uint32_t *dst;
                int64_t two_rows;  // the word stride of two token rows
                uint8_t *buf = nullptr;
                if constexpr (kWideStores) {
                    // The box staged two boxes ago has been read by its store.
                    buf = s.staging + (sub & 1u) * kOutBoxBytes;
                    if (ep == 0) bulk_wait_group_read<1>();
                    epi_bar_sync();
                    dst = reinterpret_cast<uint32_t *>(buf) + odd * (kFeatCta / 2) + q * 16 + (lane >> 1);
                    two_rows = kFeatCta;
                } else {
                    dst = reinterpret_cast<uint32_t *>(P.out + static_cast<int64_t>(row0 + c + static_cast<int>(odd)) * P.N +
                                                       fcol + (lane & ~1u));
                    two_rows = P.N;
                }
                if (valid) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int t = 0; t < 32; t += 2) {
                        const float z0 = activate_t<A>(__uint_as_float(r[t]) + bv);
                        const float z1 = activate_t<A>(__uint_as_float(r[t + 1]) + bv);
                        const float other = __shfl_xor_sync(0xffffffffu, odd ? z0 : z1, 1);
                        __nv_bfloat162 p = odd ? __floats2bfloat162_rn(other, z1) : __floats2bfloat162_rn(z0, other);
                        dst[(t / 2) * two_rows] = *reinterpret_cast<uint32_t *>(&p);
                    }
                }
                if constexpr (kWideStores) {
                    fence_proxy_async_smem();
                    epi_bar_sync();
                    if (ep == 0 && fbase < P.N) {  // columns past N are clipped by the store
                        tma_store_2d(&m.out, buf, fbase, row0 + c);
                        bulk_commit_group();
                    }
                    ++sub;
                }
            }
        };
        for (uint32_t tcount = 0;; ++tcount) {
            const uint32_t acc = tcount & 1u, use = tcount >> 1;
            int u;
            if constexpr (kWideStores) {
                // One thread takes the unit and waits for its accumulator; the
                // four warps agree on the outcome at a named barrier, so they
                // all pass the same barriers below and leave together.
                if (ep == 0) {
                    int v = take_unit(tcount);
                    if (two && pend_tt >= 0 && (v < 0 || v >= total1)) {
                        bulk_wait_group<0>();
                        publish(pend_tt);
                        pend_tt = -1;
                    }
                    if (v >= 0 && !mbar_wait_idle(&s.tfull[acc], use & 1u, a.status, a.wait_limit_ns)) v = -2;
                    s.epi_unit[tcount & 1u] = v;
                }
                epi_bar_sync();
                u = *reinterpret_cast<volatile int32_t *>(&s.epi_unit[tcount & 1u]);
                if (u < 0) break;
            } else {
                u = 0;
                if (lane == 0) u = take_unit(tcount);
                u = __shfl_sync(0xffffffffu, u, 0);
                if (u < 0) break;
                int got = 1;  // one lane waits; tcgen05.ld below is warp-collective
                if (lane == 0) got = mbar_wait_idle(&s.tfull[acc], use & 1u, a.status, a.wait_limit_ns) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, got, 0)) break;
            }
            tc_fence_after_sync();
            int tt, j;
            const int l = decode(u, tt, j);
            if (l == 0)
                drain(std::integral_constant<int, ACT>{}, a, m1, tr_tile(0), tt, j, acc);
            else
                drain(std::integral_constant<int, -1>{}, b, m2, tr_tile(1), tt, j, acc);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.tempty[acc]), 0));
            if constexpr (kWideStores) {
                if (two && l == 0) {
                    // This CTA's half of the unit's layer-1 outputs becomes
                    // the pending one: every warp's stores of it (the
                    // transposed unit's direct ones included) come before
                    // thread ep 0's later release. The previous pending unit
                    // is complete once at most this unit's own bulk groups
                    // are outstanding, and is published: a proxy fence and a
                    // release increment of its tile's counter.
                    epi_bar_sync();
                    if (ep == 0) {
                        if (pend_tt >= 0) {
                            const int4 tile = tok_tiles[tt];
                            const int fb = j * kFeatPair + static_cast<int>(rank) * kFeatCta;
                            const int nb = (j == tr_tile(0) || fb >= a.N) ? 0 : tile.z / kBoxTok;
                            bulk_wait_group_dyn(nb);
                            publish(pend_tt);
                        }
                        pend_tt = tt;
                    }
                }
            }
        }
        if (kWideStores && ep == 0) {
            bulk_wait_group<0>();  // all stores complete before exit
            if (two && pend_tt >= 0) publish(pend_tt);  // the loop ended on an error
        }
    }

    // A role that gave up may leave its own TMA loads in flight; they land
    // within microseconds, so give them a millisecond before the pair meets.
    if (!ok || *reinterpret_cast<volatile uint32_t *>(a.status) != kDevOk) spin_ns(1000000ull);
    tc_fence_before_sync();
    cluster_sync_all();
    tc_fence_after_sync();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, 2 * kAccCols);
    }
}

template <int ACT, int TILE>
cudaError_t launch_act(const PairMaps &m1, const PairMaps &m2, const PairGemmArgs &a, const PairGemmArgs &b,
                       cudaStream_t st) {
    constexpr int kSmem = PairCfg<TILE>::kSmem;
    auto kern = grouped_gemm_pair_kernel<ACT, TILE>;
    cudaError_t e = set_smem_limit_once<grouped_gemm_pair_kernel<ACT, TILE>>(kSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * a.num_pairs, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    Layer2 l2;
    l2.m = m2;
    l2.a = b;
    return cudaLaunchKernelEx(&cfg, kern, m1, a, l2);
}

}  // namespace

int gemm_pair_max_pairs(int num_sms) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    // The larger of the two stage layouts; both allow one CTA per SM.
    constexpr int kSmem = PairCfg<kNarrowTile>::kSmem > PairCfg<kTokTile>::kSmem ? PairCfg<kNarrowTile>::kSmem
                                                                                   : PairCfg<kTokTile>::kSmem;
    cfg.dynamicSmemBytes = kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kern = grouped_gemm_pair_kernel<-1, kTokTile>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) return 0;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) return 0;
    return clusters < num_sms / 2 ? clusters : num_sms / 2;
}

int gemm_pair_ftiles(int N) { return (N + kFeatPair - 1) / kFeatPair; }

int gemm_pair_half_last(int N) { return N % kFeatPair != 0 && N % kFeatPair <= kFeatCta ? 1 : 0; }

cudaError_t launch_gemm_pair(const PairMaps &m1, const PairGemmArgs &a, const PairMaps *m2, const PairGemmArgs *b,
                             cudaStream_t s, int *launches) {
    if (a.num_pairs <= 0) return cudaErrorInvalidConfiguration;
    // Two layers in one launch need the epilogue whose warps move together
    // (kWideStores), a counter per token tile and the same tile table.
    if ((m2 != nullptr) != (b != nullptr) || (b && (!kWideStores || !a.tile_done || b->narrow != a.narrow)))
        return cudaErrorInvalidValue;
    PairGemmArgs a1 = a;
    a1.fuse2 = b ? 1 : 0;
    const PairMaps &mm2 = m2 ? *m2 : m1;
    const PairGemmArgs &bb = b ? *b : a;
    ++*launches;
    if (a.narrow) {
        switch (a.act) {
            case 0: return launch_act<0, kNarrowTile>(m1, mm2, a1, bb, s);
            case 1: return launch_act<1, kNarrowTile>(m1, mm2, a1, bb, s);
            case 2: return launch_act<2, kNarrowTile>(m1, mm2, a1, bb, s);
            default: return launch_act<-1, kNarrowTile>(m1, mm2, a1, bb, s);
        }
    }
    switch (a.act) {
        case 0: return launch_act<0, kTokTile>(m1, mm2, a1, bb, s);
        case 1: return launch_act<1, kTokTile>(m1, mm2, a1, bb, s);
        case 2: return launch_act<2, kTokTile>(m1, mm2, a1, bb, s);
        default: return launch_act<-1, kTokTile>(m1, mm2, a1, bb, s);
    }
}

}  // namespace moe
