// moe_common.cuh - shared device helpers for the sm_100a MoE layer kernels:
// inline-PTX wrappers for mbarriers, TMA tensor loads and tcgen05 (TMEM
// allocation, UMMA issue, commit, TMEM loads), plus the bounded wait that every
// spin in these kernels goes through.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace moe {

// Rows (tokens) of the router's tensor-core M tile; also the rows of a full
// 128-row TMA box.
constexpr int kBM = 128;
// K extent of one pipeline stage: 64 bf16 = 128 bytes, one 128B-swizzle row.
constexpr int kBK = 64;
// Every expert's row segment in the permuted row space is padded to a multiple
// of kRowBlock rows; the expert GEMM covers a segment with token tiles of at
// most kTokTile rows (the MMA's N), each a multiple of kRowBlock.
constexpr int kRowBlock = 32;
constexpr int kTokTile = 256;

// Device status word values (bit flags, OR-ed together).
enum : uint32_t { kDevOk = 0u, kDevTimeout = 1u };

// A bounded wait gives up after this long (wall clock, %globaltimer ns).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// The shorter limit of the expert GEMM launch that the timeout self-test runs.
constexpr uint64_t kSelftestWaitNs = 20000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}

// Waits until the barrier phase with the given parity has completed. Returns
// false, without waiting further, once the shared status word is non-zero
// (another role or CTA gave up) or after kWaitLimitNs; in the latter case it
// sets kDevTimeout in the status word itself. Never traps, never spins forever.
// The status word (a global load) is only polled once the wait has lasted
// kStatusPollNs, so a normal short wait spins on the barrier alone.
constexpr uint64_t kStatusPollNs = 20000ull;
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *status,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        const uint64_t dt = global_timer_ns() - t0;
        if (dt > kStatusPollNs && *reinterpret_cast<volatile uint32_t *>(status) != kDevOk) return false;
        if (dt > limit_ns) {
            atomicOr(status, kDevTimeout);
            return false;
        }
    }
}

// mbar_wait in every lane of the warp. Each lane acquires the completed phase
// itself, so that every lane's later reads see what the arriving threads wrote
// before they arrived (a wait in one lane followed by a shuffle orders nothing
// for the other lanes' memory accesses). Returns the same result in all lanes.
__device__ __forceinline__ bool mbar_wait_all_lanes(uint64_t *bar, uint32_t parity, uint32_t *status) {
    const bool ok = mbar_wait(bar, parity, status);
    return __all_sync(0xffffffffu, ok);
}

// The same for a wait that is expected to be long and whose end is not
// latency-critical (an epilogue waiting for the next accumulator): after the
// first microsecond it sleeps between polls, leaving issue slots and shared
// memory bandwidth to the roles that are working.
__device__ __forceinline__ bool mbar_wait_idle(uint64_t *bar, uint32_t parity, uint32_t *status,
                                               uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        const uint64_t dt = global_timer_ns() - t0;
        if (dt > 1000ull) __nanosleep(256);
        if (dt > kStatusPollNs && *reinterpret_cast<volatile uint32_t *>(status) != kDevOk) return false;
        if (dt > limit_ns) {
            atomicOr(status, kDevTimeout);
            return false;
        }
    }
}

// Waits until the global counter *p reaches `target` (gpu-scope acquire
// loads, a short sleep between polls), bounded like mbar_wait.
__device__ __forceinline__ bool wait_counter_geq(const int32_t *p, int target, uint32_t *status,
                                                 uint64_t limit_ns = kWaitLimitNs) {
    auto load = [p]() {
        int v;
        asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        return v;
    };
    if (load() >= target) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        __nanosleep(64);
        if (load() >= target) return true;
        const uint64_t dt = global_timer_ns() - t0;
        if (dt > kStatusPollNs && *reinterpret_cast<volatile uint32_t *>(status) != kDevOk) return false;
        if (dt > limit_ns) {
            atomicOr(status, kDevTimeout);
            return false;
        }
    }
}

// Adds v to the global counter *p with gpu-scope release semantics.
__device__ __forceinline__ void red_release_add(int32_t *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Orders this thread's generic-proxy accesses of global memory with its
// async-proxy ones (TMA loads and stores) in both directions.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Drain wait used on the way out (own copies / MMAs still in flight): bounded
// by time only, so it still waits when the status word is already set.
constexpr uint64_t kDrainLimitNs = 200000000ull;
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > kDrainLimitNs) return false;
    }
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled tensor load into shared memory, completing on `bar` (complete_tx).
// c0 is the innermost (contiguous) coordinate in elements; it must be a
// multiple of 16 bytes' worth of elements.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint64_t *bar, void *dst, int32_t c0,
                                            int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// 2-D tiled tensor store from shared memory (bulk-group completion). The
// shared-memory source must have been made visible to the async proxy
// (fence_proxy_async_smem) by the threads that wrote it.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Waits until at most N of this thread's committed bulk groups still read
// shared memory (their sources may then be overwritten).
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Waits until at most N of this thread's committed bulk groups are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// bulk_wait_group with a run-time count (0..8; larger counts wait for 8).
__device__ __forceinline__ void bulk_wait_group_dyn(int n) {
    switch (n) {
        case 0: bulk_wait_group<0>(); break;
        case 1: bulk_wait_group<1>(); break;
        case 2: bulk_wait_group<2>(); break;
        case 3: bulk_wait_group<3>(); break;
        case 4: bulk_wait_group<4>(); break;
        case 5: bulk_wait_group<5>(); break;
        case 6: bulk_wait_group<6>(); break;
        case 7: bulk_wait_group<7>(); break;
        default: bulk_wait_group<8>(); break;
    }
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy accesses (TMA, tcgen05) of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation. Issued by
// one thread.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Each lane of the warp reads 16 consecutive 32-bit columns of its own TMEM
// lane (the warp's 32-lane quarter is fixed by warp index % 4).
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Each lane writes 16 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand tile stored the way a
// 128B-swizzled TMA load leaves it: rows of 128 bytes (64 bf16 of K), groups of
// 8 rows 1024 bytes apart (stride byte offset), tile base 1024-byte aligned.
// Fields: start address >> 4 in bits [0,14), leading byte offset (unused for
// swizzled K-major, 1) in [16,30), stride byte offset >> 4 in [32,46),
// descriptor version 1 in [46,48), layout type 2 = 128B swizzle in [61,64).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 D, both operands
// K-major, shape M x N: D format in bits [4,6) (1 = f32), A format [7,10) and
// B format [10,13) (1 = bf16), N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------- CTA pairs (cta_group::2)
//
// Two CTAs of a 2-CTA cluster run one MMA of M = 256 together: the leader
// (cluster rank 0) issues it, each CTA holds half of A (its 128 rows) and half
// of B (N/2 rows) in its own shared memory at the same offsets, and each CTA's
// TMEM receives its 128 rows of the accumulator.

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared::cluster address of the variable at shared::cta address `addr` in
// the cluster's CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// 32-bit store to a shared::cluster address (own or peer CTA).
__device__ __forceinline__ void st_shared_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// try_wait with cluster-scope acquire: data another CTA of the cluster wrote
// before its (release.cluster) arrive is visible once the phase completes.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}

// Bounded wait with cluster-scope acquire (same limits as mbar_wait).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, uint32_t *status,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        const uint64_t dt = global_timer_ns() - t0;
        if (dt > kStatusPollNs && *reinterpret_cast<volatile uint32_t *>(status) != kDevOk) return false;
        if (dt > limit_ns) {
            atomicOr(status, kDevTimeout);
            return false;
        }
    }
}

// Every thread of both CTAs arrives, then waits for all of them.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (own or peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}

// TMA load into this CTA's shared memory whose completion is signalled on an
// mbarrier of either CTA of the pair (the leader's, for the pair's MMA).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap *map, uint32_t bar_cluster_addr, void *dst,
                                                 int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// The pair's MMA, issued by one thread of the leader CTA.
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on the mbarrier at the same shared-memory offset in every CTA
// of `cta_mask` when the pair MMAs this thread issued so far have completed.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// As tc_commit, for pair MMAs, on this CTA's own barrier.
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Spins for about `ns` nanoseconds (used only on the way out after a timeout).
__device__ __forceinline__ void spin_ns(uint64_t ns) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < ns) {
    }
}

// ------------------------------------------------------------------ misc

// Raises kernel K's dynamic shared-memory limit once per device (the first
// launch), so that later launches, including ones captured into a CUDA graph,
// make no attribute call.
template <auto K>
inline cudaError_t set_smem_limit_once(int bytes) {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load() & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.fetch_or(bit);
    return e;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Activations of the expert MLP with the code fixed at compile time: 0 ReLU,
// 1 GELU (exact erf form), 2 Swish z * sigmoid(z) (fast exp and divide: their
// few-ulp fp32 error is far below the bf16 rounding of the result), other
// values the identity.
template <int ACT>
__device__ __forceinline__ float activate_t(float z) {
    if constexpr (ACT == 0) return z > 0.f ? z : 0.f;
    else if constexpr (ACT == 1) return 0.5f * z * (1.f + erff(z * 0.70710678118654752f));
    else if constexpr (ACT == 2) return __fdividef(z, 1.f + __expf(-z));
    else return z;
}

// The same with a run-time code (fp32 CUDA-core path: exact expf and divide).
__device__ __forceinline__ float activate(int act, float z) {
    if (act == 0) return z > 0.f ? z : 0.f;
    if (act == 1) return 0.5f * z * (1.f + erff(z * 0.70710678118654752f));
    if (act == 2) return z / (1.f + expf(-z));
    return z;
}

}  // namespace moe
