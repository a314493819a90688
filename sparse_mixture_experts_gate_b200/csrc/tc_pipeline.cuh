// tc_pipeline.cuh - the one-CTA tcgen05 pipeline pieces of the tensor-core
// router (router_tc.cu): shared-memory layout of the stage ring, barrier and
// TMEM set-up and teardown, and the TMA producer role.
//
// One CTA per SM walks a static tile sequence (tile = blockIdx.x, += gridDim.x).
//   warp 0      producer: per K block, waits for a free stage, posts the
//               expected bytes and issues TMA loads (the kernel's load functor);
//   warp 1      owns TMEM (2 x 256 fp32 columns) and issues the MMAs;
//   other warps the kernel's epilogue.
// All waits are bounded (mbar_wait); on a timeout every role stops, in-flight
// copies and MMAs are drained, TMEM is freed and the kernel returns with the
// status word flagged.
#pragma once

#include "moe_common.cuh"

namespace moe {

constexpr int kTcThreads = 192;
constexpr int kTcAccCols = 256;  // TMEM columns per accumulator buffer

template <int BN>
struct TcLayout {
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
struct TcShared {
    uint8_t *sA, *sB;
    uint64_t *full, *empty, *tfull, *tempty, *mma_done;
    uint32_t *tmem_slot;
};

template <int BN>
__device__ __forceinline__ TcShared<BN> tc_carve(uint8_t *smem_raw) {
    using L = TcLayout<BN>;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    TcShared<BN> s;
    s.sA = smem;
    s.sB = smem + L::NS * L::A_BYTES;
    s.full = reinterpret_cast<uint64_t *>(smem + L::NS * L::STAGE);
    s.empty = s.full + L::NS;
    s.tfull = s.empty + L::NS;
    s.tempty = s.tfull + 2;
    s.mma_done = s.tempty + 2;
    s.tmem_slot = reinterpret_cast<uint32_t *>(s.mma_done + 1);
    return s;
}

// Barrier init (thread 0) and TMEM allocation (warp 1); returns the TMEM base.
// tempty_count: epilogue threads that release an accumulator (128 = 4 warps).
template <int BN>
__device__ __forceinline__ uint32_t tc_setup(const TcShared<BN> &s, uint32_t tempty_count = 128) {
    using L = TcLayout<BN>;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int i = 0; i < L::NS; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], tempty_count);
        }
        mbar_init(s.mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(s.tmem_slot, 2 * kTcAccCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    return *s.tmem_slot;
}

template <int BN>
__device__ __forceinline__ void tc_teardown(const TcShared<BN> &s, uint32_t tmem_base) {
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if ((threadIdx.x >> 5) == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, 2 * kTcAccCols);
    }
}

// Producer role, executed by all 32 lanes of warp 0. `load(tile, kb, sA, sB,
// bar, lane)` issues the stage's TMA loads (any lane may issue some of them);
// `tile_begin(tile, lane)` runs once per tile before its first K block. Lane 0
// owns the barrier protocol; the wait outcome is broadcast so the warp stays
// convergent. Tile `tile` covers K blocks [x, y) of krange(tile).
template <int BN, class TileBegin, class LoadFn, class KRange>
__device__ __forceinline__ void tc_producer_range(const TcShared<BN> &s, int total, uint32_t *status,
                                                  TileBegin tile_begin, LoadFn load, KRange krange) {
    using L = TcLayout<BN>;
    const int lane = threadIdx.x & 31;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        tile_begin(tile, lane);
        const int2 kr = krange(tile);
        for (int kb = kr.x; kb < kr.y; ++kb) {
            const int st = it % L::NS;
            const uint32_t ph = (it / L::NS) & 1u;
            int got = 1;
            if (lane == 0) got = mbar_wait(&s.empty[st], ph ^ 1u, status) ? 1 : 0;
            got = __shfl_sync(0xffffffffu, got, 0);
            if (!got) {
                ok = false;
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&s.full[st], L::STAGE);
            __syncwarp();
            load(tile, kb, s.sA + st * L::A_BYTES, s.sB + st * L::B_BYTES, &s.full[st], lane);
            ++it;
        }
    }
    // Every issued copy must land before the CTA exits; on the normal path the
    // MMA role has already waited for all of them.
    if (!ok && lane == 0) {
        for (uint32_t j = (it > (uint32_t)L::NS ? it - L::NS : 0u); j < it; ++j)
            mbar_wait_drain(&s.full[j % L::NS], (j / L::NS) & 1u);
    }
}

}  // namespace moe
