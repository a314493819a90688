// gemm_tc.cu - grouped expert GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Code Walkthrough - SER", gating / routing path: each selected expert runs its
// two-layer MLP, w1/b1 -> activation -> w2/b2. Both layers of every expert are
// dense contractions over the rows dispatched to it, so they run as one grouped
// GEMM per layer over the permuted row space:
//   out[row][n] = act( sum_k A[row][k] * W[g][n][k] + b[g][n] ),  g = group of row.
// Layer 1: A = the routed token rows scattered into row order (dispatch.cu), and
//   x itself for the shared experts, which read every token in order.
// Layer 2: A = the hidden activations H (already in row order);
//   the epilogue also writes, per row and N tile, the fp32 sum of squares of
//   the outputs (the credit's norm).
// The pipeline (tc_pipeline.cuh): persistent CTAs over 128 x BN tiles, n fastest
// so concurrently running CTAs share A and B tiles through L2; TMA producer
// warp, single-lane MMA issuer, four epilogue warps, TMEM double buffering.
// Epilogue: each warp turns its 32 accumulator rows into bf16 64 columns at a
// time, writes them to a 128B-swizzled shared staging buffer (two per warp,
// alternating) and one lane stores the 32 x 64 box with a TMA tensor store, so
// global writes are whole, coalesced lines and never stall the warp. Rows past
// an expert's kept count are padding rows of the row space (never read), so
// tiles are stored whole.
#include "moe_common.cuh"
#include "moe_kernels.cuh"
#include "tc_pipeline.cuh"

namespace moe {
namespace {

constexpr int kStoreCols = 64;                        // columns per staged store box (128 bytes)
constexpr int kStageBoxBytes = 32 * kStoreCols * 2;    // 32 rows x 128 bytes
constexpr int kStagingBytes = 4 * 2 * kStageBoxBytes;  // 4 epilogue warps x 2 buffers

template <int BN>
constexpr int gemm_smem_bytes() {
    return (1024 + TcLayout<BN>::NS * TcLayout<BN>::STAGE + 256 + 1023) / 1024 * 1024 + kStagingBytes;
}

template <int BN, int ACT, bool NORM>
__global__ void __launch_bounds__(kTcThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_a1,
                           const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_out,
                           const GemmArgs a) {
    static_assert(BN % kStoreCols == 0, "the N tile is stored in 64-column boxes");
    extern __shared__ uint8_t smem_raw[];
    const TcShared<BN> s = tc_carve<BN>(smem_raw);
    uint8_t *staging = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(s.tmem_slot) + 64 + 1023) & ~uintptr_t(1023));
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&map_a0);
        tma_prefetch_desc(&map_a1);
        tma_prefetch_desc(&map_b);
        tma_prefetch_desc(&map_out);
    }
    const uint32_t tmem_base = tc_setup<BN>(s);
    const int num_m = min(a.ctrl[kCtrlNumMTiles], a.max_mtiles);
    const int total = num_m * a.n_tiles;
    const int kblocks = a.K / kBK;
    const int warp = threadIdx.x >> 5;

    if (warp == 0) {
        const CUtensorMap *ma = &map_a0;
        int arow = 0, brow = 0;
        auto tile_begin = [&](int tile, int) {
            const int m = tile / a.n_tiles, n = tile - m * a.n_tiles;
            const int g = a.tile_group[m];
            brow = g * a.N + n * BN;
            ma = &map_a0;
            arow = m * kBM;
            if (a.use_a1 && g >= a.E) {  // shared expert: rows of x in token order
                ma = &map_a1;
                arow = m * kBM - a.group_start[g];
            }
        };
        auto load = [&](int, int kb, uint8_t *sA, uint8_t *sB, uint64_t *bar, int lane) {
            if (lane == 0) {
                tma_load_2d(ma, bar, sA, kb * kBK, arow);
                tma_load_2d(&map_b, bar, sB, kb * kBK, brow);
            }
        };
        tc_producer<BN>(s, total, kblocks, a.status, tile_begin, load);
    } else if (warp == 1) {
        if ((threadIdx.x & 31) == 0)
            tc_mma<BN>(s, tmem_base, total, kblocks, a.status,
                       [&](int tile) { return tile % a.n_tiles == a.n_tiles - 1 ? a.n_last : BN; });
    } else {
        uint8_t *my_stage = staging + (warp - 2) * 2 * kStageBoxBytes;
        uint32_t sub = 0;  // store boxes this warp has issued
        auto epi = [&](int tile, uint32_t taddr, int q, int lane) {
            const int m = tile / a.n_tiles, n = tile - m * a.n_tiles;
            const int g = a.tile_group[m];
            const int grow = m * kBM + q * 32 + lane;
            const float *bias = a.bias ? a.bias + (int64_t)g * a.N + n * BN : nullptr;
            const int ncols = n == a.n_tiles - 1 ? a.n_last : BN;
            float ss = 0.f;
#pragma unroll 1
            for (int c = 0; c < ncols; c += kStoreCols) {
                uint8_t *buf = my_stage + (sub & 1u) * kStageBoxBytes;
                if (lane == 0) bulk_wait_group_read<1>();  // the store that last used `buf` has read it
                __syncwarp();
                uint8_t *row = buf + lane * 128;
#pragma unroll 1
                for (int h = 0; h < kStoreCols; h += 32) {
                    float4 b4[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        b4[j] = bias ? __ldg(reinterpret_cast<const float4 *>(bias + c + h) + j)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + c + h, r);
                    tmem_ld_wait();
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float z0 = activate_t<ACT>(__uint_as_float(r[4 * j]) + b4[j].x);
                        const float z1 = activate_t<ACT>(__uint_as_float(r[4 * j + 1]) + b4[j].y);
                        const float z2 = activate_t<ACT>(__uint_as_float(r[4 * j + 2]) + b4[j].z);
                        const float z3 = activate_t<ACT>(__uint_as_float(r[4 * j + 3]) + b4[j].w);
                        if (NORM) {
                            ss = fmaf(z0, z0, ss);
                            ss = fmaf(z1, z1, ss);
                            ss = fmaf(z2, z2, ss);
                            ss = fmaf(z3, z3, ss);
                        }
                        __nv_bfloat162 p0 = __floats2bfloat162_rn(z0, z1), p1 = __floats2bfloat162_rn(z2, z3);
                        packed[2 * j] = *reinterpret_cast<uint32_t *>(&p0);
                        packed[2 * j + 1] = *reinterpret_cast<uint32_t *>(&p1);
                    }
                    // Row `lane`, 16-byte chunk j at chunk j ^ (row % 8): the 128B swizzle.
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int chunk = (h / 8) + j;
                        *reinterpret_cast<uint4 *>(row + ((chunk ^ (lane & 7)) << 4)) =
                            make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&map_out, buf, n * BN + c, m * kBM + q * 32);
                    bulk_commit_group();
                }
                ++sub;
            }
            if (NORM && grow < a.group_start[g] + a.group_rows[g])
                a.norm_part[(int64_t)grow * a.n_tiles + n] = ss;
        };
        tc_epilogue<BN>(s, tmem_base, total, a.status, epi);
        if ((threadIdx.x & 31) == 0) bulk_wait_group<0>();  // all stores complete before exit
    }
    tc_teardown<BN>(s, tmem_base);
}

template <int BN, int ACT, bool NORM>
cudaError_t launch_inst(const CUtensorMap &m0, const CUtensorMap &m1, const CUtensorMap &mb, const CUtensorMap &mo,
                        const GemmArgs &a, cudaStream_t s) {
    constexpr int smem = gemm_smem_bytes<BN>();
    static_assert(smem <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_tc_kernel<BN, ACT, NORM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    grouped_gemm_tc_kernel<BN, ACT, NORM><<<a.num_sms, kTcThreads, smem, s>>>(m0, m1, mb, mo, a);
    return cudaGetLastError();
}

// Layer 1 runs with the layer's activation and no norm; layer 2 with neither.
template <int BN>
cudaError_t launch_bn(const CUtensorMap &m0, const CUtensorMap &m1, const CUtensorMap &mb, const CUtensorMap &mo,
                      const GemmArgs &a, cudaStream_t s) {
    if (a.norm_part) return launch_inst<BN, -1, true>(m0, m1, mb, mo, a, s);
    switch (a.act) {
        case 0: return launch_inst<BN, 0, false>(m0, m1, mb, mo, a, s);
        case 1: return launch_inst<BN, 1, false>(m0, m1, mb, mo, a, s);
        case 2: return launch_inst<BN, 2, false>(m0, m1, mb, mo, a, s);
        default: return launch_inst<BN, -1, false>(m0, m1, mb, mo, a, s);
    }
}

}  // namespace

int gemm_pick_bn(int N) {
    if (N % 64 != 0 || N <= 0) return 0;
    if (N % 256 == 0 || N > 256) return 256;  // a ragged last tile is cheaper than a narrow BN
    return N % 128 == 0 ? 128 : 64;
}

cudaError_t launch_gemm_tc(const CUtensorMap &m0, const CUtensorMap &m1, const CUtensorMap &mb, const CUtensorMap &mo,
                           const GemmArgs &a, int BN, cudaStream_t s, int *launches) {
    ++*launches;
    switch (BN) {
        case 256: return launch_bn<256>(m0, m1, mb, mo, a, s);
        case 128: return launch_bn<128>(m0, m1, mb, mo, a, s);
        case 64: return launch_bn<64>(m0, m1, mb, mo, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
