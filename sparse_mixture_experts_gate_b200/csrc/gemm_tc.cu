// gemm_tc.cu - grouped expert GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Code Walkthrough - SER", gating / routing path: each selected expert runs its
// two-layer MLP, w1/b1 -> activation -> w2/b2. Both layers of every expert are
// dense contractions over the rows dispatched to it, so they run as one grouped
// GEMM per layer over the permuted row space:
//   out[row][n] = act( sum_k A[row][k] * W[g][n][k] + b[g][n] ),  g = group of row.
// Layer 1: A = gathered x rows (routed) or x itself (shared experts), W = w1.
// Layer 2: A = the hidden activations, W = w2; the epilogue also writes, per row
// and N tile, the sum of squares of the fp32 outputs (for the credit norm).
//
// Design (one CTA per SM, persistent over 128 x BN output tiles, n fastest so
// concurrently running CTAs share A and B tiles through L2):
//   warp 0      TMA producer: A tile 128x64 and B tile BNx64 per stage, 128B
//               swizzle, NS-stage ring guarded by full/empty mbarriers;
//   warp 1      owns TMEM (512 columns = two fp32 accumulators of up to 256
//               columns); one lane issues tcgen05.mma M=128 N=BN K=16 and
//               tcgen05.commit to release stages and to publish accumulators;
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 16 columns, bias, activation,
//               bf16 store; accumulator ring of two so the epilogue of one tile
//               overlaps the mainloop of the next.
// Every wait is bounded (mbar_wait): on timeout the kernel flags the status
// word, drains its own copies and MMAs, frees TMEM and returns.
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kThreads = 192;
constexpr int kAccCols = 256;  // TMEM columns reserved per accumulator buffer

template <int BN>
struct TcCfg {
    static constexpr int A_BYTES = kBM * kBK * 2;
    static constexpr int B_BYTES = BN * kBK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NS = (200 * 1024) / STAGE < 8 ? (200 * 1024) / STAGE : 8;
    static constexpr int SMEM = 1024 + NS * STAGE + 256;
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA M=128 needs N % 16 == 0, 16..256");
    static_assert(B_BYTES % 1024 == 0, "B tile must keep 1024-byte swizzle alignment");
    static_assert(NS >= 2, "need at least two stages");
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_a1,
                           const __grid_constant__ CUtensorMap map_b, const GemmArgs a) {
    using C = TcCfg<BN>;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + NS * C::A_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + NS * C::STAGE);
    uint64_t *empty = full + NS;
    uint64_t *tfull = empty + NS;
    uint64_t *tempty = tfull + 2;
    uint64_t *mma_done = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 128);
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
        tma_prefetch_desc(&map_a0);
        tma_prefetch_desc(&map_a1);
        tma_prefetch_desc(&map_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * kAccCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    const int num_m = min(a.ctrl[kCtrlNumMTiles], a.max_mtiles);
    const int total = num_m * a.n_tiles;
    const int kblocks = a.K / kBK;
    uint32_t *status = a.status;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const int m = tile / a.n_tiles, n = tile - m * a.n_tiles;
                const int g = a.tile_group[m];
                const CUtensorMap *ma = &map_a0;
                int arow = m * kBM;
                if (a.use_a1 && g >= a.E) {
                    ma = &map_a1;
                    arow = m * kBM - a.group_start[g];
                }
                const int brow = g * a.N + n * BN;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % NS;
                    const uint32_t ph = (it / NS) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_2d(ma, &full[s], sA + s * C::A_BYTES, kb * kBK, arow);
                    tma_load_2d(&map_b, &full[s], sB + s * C::B_BYTES, kb * kBK, brow);
                }
            }
            // Drain: every issued copy must land before the CTA may exit. On the
            // normal path the consumer already waited for all of them.
            if (!ok) {
                for (uint32_t j = (it > (uint32_t)NS ? it - NS : 0u); j < it; ++j)
                    mbar_wait_drain(&full[j % NS], (j / NS) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tcount) {
                const uint32_t acc = tcount & 1u, use = tcount >> 1;
                if (!mbar_wait(&tempty[acc], (use & 1u) ^ 1u, status)) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kAccCols;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % NS;
                    const uint32_t ph = (it / NS) & 1u;
                    if (!mbar_wait(&full[s], ph, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + s * C::A_BYTES));
                    const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + s * C::B_BYTES));
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma_bf16(d_tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
                    tc_commit(&empty[s]);
                }
                if (ok) tc_commit(&tfull[acc]);
            }
            // All MMAs this thread issued are complete once mma_done flips.
            tc_commit(mma_done);
            mbar_wait_drain(mma_done, 0u);
        }
    } else {
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int lrow = q * 32 + lane;
        uint32_t tcount = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
            const int m = tile / a.n_tiles, n = tile - m * a.n_tiles;
            const uint32_t acc = tcount & 1u, use = tcount >> 1;
            // tcgen05.ld below is warp-collective: make the outcome warp-uniform.
            const bool got = mbar_wait(&tfull[acc], use & 1u, status);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after_sync();
            const int g = a.tile_group[m];
            const int grow = m * kBM + lrow;
            const bool valid = grow < a.group_start[g] + a.group_rows[g];
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
            const float *bias = a.bias ? a.bias + (int64_t)g * a.N + n * BN : nullptr;
            __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(a.out) + (int64_t)grow * a.N + n * BN;
            float ss = 0.f;
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(taddr + c, r);
                tmem_ld_wait();
                float v[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    float z = __uint_as_float(r[j]);
                    if (bias) z += __ldg(bias + c + j);
                    z = activate(a.act, z);
                    v[j] = z;
                    ss = fmaf(z, z, ss);
                }
                if (valid) {
                    uint4 pk[2];
                    uint32_t *pw = reinterpret_cast<uint32_t *>(pk);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
                        pw[j] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
                    dst[0] = pk[0];
                    dst[1] = pk[1];
                }
            }
            if (a.norm_part && valid) a.norm_part[(int64_t)grow * a.n_tiles + n] = ss;
            tc_fence_before_sync();
            mbar_arrive(&tempty[acc]);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, 2 * kAccCols);
    }
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap &m0, const CUtensorMap &m1, const CUtensorMap &mb, const GemmArgs &a,
                      cudaStream_t s) {
    using C = TcCfg<BN>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(grouped_gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    grouped_gemm_tc_kernel<BN><<<a.num_sms, kThreads, C::SMEM, s>>>(m0, m1, mb, a);
    return cudaGetLastError();
}

}  // namespace

int gemm_pick_bn(int N) {
    for (int bn = 256; bn >= 16; bn -= 16)
        if (N % bn == 0 && (bn == 256 || bn == 176 || bn == 128 || bn == 64 || bn == 32 || bn == 16)) return bn;
    return 0;
}

cudaError_t launch_gemm_tc(const CUtensorMap &m0, const CUtensorMap &m1, const CUtensorMap &mb, const GemmArgs &a,
                           int BN, cudaStream_t s, int *launches) {
    ++*launches;
    switch (BN) {
        case 256: return launch_bn<256>(m0, m1, mb, a, s);
        case 176: return launch_bn<176>(m0, m1, mb, a, s);
        case 128: return launch_bn<128>(m0, m1, mb, a, s);
        case 64: return launch_bn<64>(m0, m1, mb, a, s);
        case 32: return launch_bn<32>(m0, m1, mb, a, s);
        case 16: return launch_bn<16>(m0, m1, mb, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
