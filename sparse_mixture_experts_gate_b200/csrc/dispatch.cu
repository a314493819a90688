// dispatch.cu - capacity-capped dispatch of token assignments to expert buffers.
//
// "Appendix C - Acronyms & Symbols", table "Capacity & communication": each
// expert has a fixed buffer of C = ceil(C_f k T / E) tokens and the dispatch
// tensor D scatters tokens into those buffers; "Code Walkthrough - SER", "Load
// balancing": a hard per-expert cap drops overflow tokens. Priority inside an
// expert's buffer is ascending token index (a stable ranking), or, with
// rank-major priority, every token's first choice before any second choice.
//
// Instead of a dense one-hot D, the dispatch is a permutation into a compact row
// space: expert e owns rows [group_start[e], group_start[e] + kept_e), padded to
// a multiple of 32 rows, followed by one T-row segment per shared expert (also
// padded to 32). Two launches (one block for a batch of one chunk):
//   count  - per 256-token chunk, a histogram of selections (shared-memory
//            integer atomics: order-free, so deterministic); the CTA that
//            counts the last chunk then runs the scan:
//   scan   - per expert, exclusive prefix over chunks; kept = min(count, C);
//            the exclusive scan of the selection counts (pre_start);
//            exclusive scans of the padded kept counts and of their token
//            tiles -> segment starts, the 32-row block -> group table, the
//            token-tile table of the expert GEMM ({group, first row, rows},
//            at most 256 rows each) and the row and tile counts;
//   assign - per chunk, the stable rank of each assignment: chunk base +
//            assignments to the same expert in earlier warps + earlier lanes of
//            the same warp (a per-warp lane bitmask per expert, popcounted);
//            every selection's gate is also written at pre_start[e] + rank, so
//            each expert's gates lie together in token order (the importance
//            statistic sums them in that fixed order).
// Also the scatter of the routed token rows into the permuted row space, which
// the tensor-core expert GEMM then reads as plain TMA tiles.
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kChunk = 256;  // tokens per chunk = threads per block
constexpr int kMaxE = 256;

// The assignments in capacity-priority order: item i holds assignments
// t*k + r for r < k (token order, item = token t), or the single assignment
// (i mod T)*k + i/T (rank-major, item = r T + t).
__device__ __forceinline__ int items_per(const DispatchArgs &a) { return a.rank_major ? 1 : a.k; }
__device__ __forceinline__ int64_t assignment_of(const DispatchArgs &a, int i, int j) {
    return a.rank_major ? (int64_t)(i % a.T) * a.k + i / a.T : (int64_t)i * a.k + j;
}

// Per-chunk expert histogram (one block of kChunk threads per chunk).
__device__ __forceinline__ void dispatch_count(const DispatchArgs &a, int chunk) {
    __shared__ int cnt[kMaxE];
    for (int e = threadIdx.x; e < a.E; e += kChunk) cnt[e] = 0;
    __syncthreads();
    const int i = chunk * kChunk + threadIdx.x;
    if (i < a.n_items)
        for (int j = 0; j < items_per(a); ++j) atomicAdd(&cnt[a.idx[assignment_of(a, i, j)]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += kChunk) a.chunk_count[(int64_t)chunk * a.E + e] = cnt[e];
}


// Single CTA of kMaxE threads; thread e owns expert e.
__device__ __forceinline__ void dispatch_scan(const DispatchArgs &a) {
    __shared__ int sc_rows[kMaxE];
    __shared__ int sc_tiles[kMaxE];
    __shared__ int sc_pre[kMaxE];
    __shared__ int sc_nar[kMaxE];
    __shared__ int dropped_w[kMaxE / 32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    int pre = 0, kept = 0, padded = 0, tiles = 0, nars = 0;
    if (e < a.E) {
        // Exclusive prefix over chunks, loads batched so they are in flight together.
        const int32_t *__restrict__ cnt = a.chunk_count;
        int32_t *__restrict__ base = a.chunk_base;
        for (int c0 = 0; c0 < a.n_chunks; c0 += 32) {
            int v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = c0 + j < a.n_chunks ? __ldcg(cnt + (int64_t)(c0 + j) * a.E + e) : 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                if (c0 + j < a.n_chunks) base[(int64_t)(c0 + j) * a.E + e] = pre;
                pre += v[j];
            }
        }
        kept = (int64_t)pre < a.C ? pre : (int)a.C;
        padded = (kept + kRowBlock - 1) / kRowBlock * kRowBlock;
        tiles = (padded + kTokTile - 1) / kTokTile;
        nars = (padded + kNarrowTile - 1) / kNarrowTile;
    }
    // Inclusive scans of the padded rows and of the token tiles over the block
    // (Hillis-Steele in shared memory).
    sc_rows[e] = padded;
    sc_tiles[e] = tiles;
    sc_pre[e] = pre;
    sc_nar[e] = nars;
    __syncthreads();
    for (int off = 1; off < kMaxE; off <<= 1) {
        const int vr = e >= off ? sc_rows[e - off] : 0;
        const int vt = e >= off ? sc_tiles[e - off] : 0;
        const int vp = e >= off ? sc_pre[e - off] : 0;
        const int vn = e >= off ? sc_nar[e - off] : 0;
        __syncthreads();
        sc_rows[e] += vr;
        sc_tiles[e] += vt;
        sc_pre[e] += vp;
        sc_nar[e] += vn;
        __syncthreads();
    }
    const int start = sc_rows[e] - padded, tile0 = sc_tiles[e] - tiles;
    const int routed_rows = sc_rows[kMaxE - 1], routed_tiles = sc_tiles[kMaxE - 1], routed_nar = sc_nar[kMaxE - 1];
    int drop = pre - kept;
    for (int off = 16; off > 0; off >>= 1) drop += __shfl_xor_sync(0xffffffffu, drop, off);
    if (lane == 0) dropped_w[warp] = drop;
    if (e < a.E) {
        a.count_pre[e] = pre;
        a.count_kept[e] = kept;
        if (a.user_count_pre) a.user_count_pre[e] = pre;
        if (a.user_count_kept) a.user_count_kept[e] = kept;
        a.group_start[e] = start;
        a.group_rows[e] = kept;
        a.pre_start[e] = sc_pre[e] - pre;
        for (int b = start / kRowBlock; b < (start + padded) / kRowBlock; ++b) a.block_group[b] = e;
        for (int r = start + kept; r < start + padded; ++r) a.row_assign[r] = -1;
        for (int i = 0; i < tiles; ++i)
            a.tok_tiles[tile0 + i] = make_int4(e, start + i * kTokTile, min(kTokTile, padded - i * kTokTile), 0);
        if (a.narrow_tiles) {
            const int n0 = sc_nar[e] - nars;
            for (int i = 0; i < nars; ++i)
                a.narrow_tiles[n0 + i] =
                    make_int4(e, start + i * kNarrowTile, min(kNarrowTile, padded - i * kNarrowTile), 0);
        }
    }
    // Shared experts: one T_pad-row segment each, after the routed rows.
    const int shared_blocks = a.T_pad / kRowBlock;
    const int shared_tiles = (a.T_pad + kTokTile - 1) / kTokTile;
    for (int i = e; i < a.S * shared_blocks; i += kMaxE)
        a.block_group[routed_rows / kRowBlock + i] = a.E + i / shared_blocks;
    for (int i = e; i < a.S * shared_tiles; i += kMaxE) {
        const int sh = i / shared_tiles, j = i - sh * shared_tiles;
        a.tok_tiles[routed_tiles + i] = make_int4(a.E + sh, routed_rows + sh * a.T_pad + j * kTokTile,
                                                  min(kTokTile, a.T_pad - j * kTokTile), 0);
    }
    const int shared_nar = (a.T_pad + kNarrowTile - 1) / kNarrowTile;
    if (a.narrow_tiles)
        for (int i = e; i < a.S * shared_nar; i += kMaxE) {
            const int sh = i / shared_nar, j = i - sh * shared_nar;
            a.narrow_tiles[routed_nar + i] = make_int4(a.E + sh, routed_rows + sh * a.T_pad + j * kNarrowTile,
                                                       min(kNarrowTile, a.T_pad - j * kNarrowTile), 0);
        }
    if (e < a.S) {
        a.group_start[a.E + e] = routed_rows + e * a.T_pad;
        a.group_rows[a.E + e] = a.T;
    }
    if (a.tile_done)
        for (int i = e; i < a.n_tile_done; i += kMaxE) a.tile_done[i] = 0;
    __syncthreads();
    if (e == 0) {
        int d = 0;
        for (int w = 0; w < kMaxE / 32; ++w) d += dropped_w[w];
        const int total = routed_rows + a.S * a.T_pad;
        a.group_start[a.E + a.S] = total;
        a.ctrl[kCtrlNumRowBlocks] = total / kRowBlock;
        a.ctrl[kCtrlNumTokTiles] = routed_tiles + a.S * shared_tiles;
        a.ctrl[kCtrlRoutedTiles] = routed_tiles;
        a.ctrl[kCtrlNumNarrowTiles] = a.narrow_tiles ? routed_nar + a.S * shared_nar : 0;
        a.ctrl[kCtrlRoutedRows] = routed_rows;
        a.ctrl[kCtrlDropped] = d;
    }
}

// Count, then scan in the CTA that counts the last chunk (the other CTAs'
// counts are read from L2); the counter is left at zero again.
__global__ void __launch_bounds__(kChunk) dispatch_count_scan_kernel(DispatchArgs a) {
    __shared__ int last;
    dispatch_count(a, blockIdx.x);
    __syncthreads();  // the block's counts, then one device-scope fence publishes them
    if (threadIdx.x == 0) {
        __threadfence();
        const int old = atomicAdd(a.ctrl + kCtrlDispatchDone, 1);
        last = old == (int)gridDim.x - 1;
        if (last) {
            __threadfence();
            a.ctrl[kCtrlDispatchDone] = 0;
        }
    }
    __syncthreads();
    if (last) dispatch_scan(a);
}

// Stable ranks within the chunk on top of the chunk's per-expert bases; slot,
// row, row owner and the gate in expert order for every assignment.
__device__ __forceinline__ void dispatch_assign(const DispatchArgs &a, int chunk) {
    constexpr int W = kChunk / 32;
    __shared__ uint32_t mask[W][kMaxE];
    __shared__ int wbase[W][kMaxE];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < W * kMaxE; i += kChunk) (&mask[0][0])[i] = 0u;
    __syncthreads();
    const int item = chunk * kChunk + tid;
    if (item < a.n_items)
        for (int j = 0; j < items_per(a); ++j) atomicOr(&mask[warp][a.idx[assignment_of(a, item, j)]], 1u << lane);
    __syncthreads();
    for (int e = tid; e < a.E; e += kChunk) {
        int run = a.chunk_base[(int64_t)chunk * a.E + e];
        for (int w = 0; w < W; ++w) {
            wbase[w][e] = run;
            run += __popc(mask[w][e]);
        }
    }
    __syncthreads();
    if (item >= a.n_items) return;
    const uint32_t lt = (1u << lane) - 1u;
    for (int j = 0; j < items_per(a); ++j) {
        const int64_t ai = assignment_of(a, item, j);
        const int e = a.idx[ai];
        const int rank = wbase[warp][e] + __popc(mask[warp][e] & lt);
        a.gate_sorted[a.pre_start[e] + rank] = a.gates[ai];
        const bool kept = (int64_t)rank < a.C;
        a.slot[ai] = kept ? rank : -1;
        int row = -1;
        if (kept) {
            row = a.group_start[e] + rank;
            a.row_assign[row] = (int)ai;
        }
        a.row_of[ai] = row;
    }
}

__global__ void __launch_bounds__(kChunk) dispatch_assign_kernel(DispatchArgs a) { dispatch_assign(a, blockIdx.x); }

// A batch of one chunk: the three steps in one block, ordered by block
// barriers (which also order the block's global writes before its reads).
__global__ void __launch_bounds__(kChunk) dispatch_one_chunk_kernel(DispatchArgs a) {
    dispatch_count(a, 0);
    __syncthreads();
    dispatch_scan(a);
    __syncthreads();
    dispatch_assign(a, 0);
}

// Work item = (token, chunk of kScatterVec x 32 16-byte vectors of its row);
// one warp per item, so a short batch still spreads over every SM. The warp
// loads the chunk of x once (all of a lane's vectors in flight together) and
// writes it to the rows of every expert that kept the token. Padding rows of
// the row space are left as they are: the rows computed from them are never
// read.
constexpr int kScatterVec = 4;

__global__ void __launch_bounds__(256) scatter_rows_kernel(ScatterArgs a) {
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nvec = a.row_bytes / 16;
    const int nchunk = (nvec + 32 * kScatterVec - 1) / (32 * kScatterVec);
    const int64_t items = (int64_t)a.T * nchunk;
    for (int64_t it = warp; it < items; it += nwarps) {
        const int t = static_cast<int>(it / nchunk), j = static_cast<int>(it - (int64_t)t * nchunk);
        const int my_row = lane < a.k ? a.row_of[(int64_t)t * a.k + lane] : -1;  // k <= 16
        uint32_t live = __ballot_sync(0xffffffffu, my_row >= 0);
        if (live == 0) continue;
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const char *>(a.x) + (int64_t)t * a.row_bytes);
        const int v0 = j * 32 * kScatterVec + lane;
        uint4 val[kScatterVec];
#pragma unroll
        for (int u = 0; u < kScatterVec; ++u)
            if (v0 + 32 * u < nvec) val[u] = __ldg(src + v0 + 32 * u);
        while (live) {
            const int i = __ffs(live) - 1;
            live &= live - 1;
            const int row = __shfl_sync(0xffffffffu, my_row, i);
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<char *>(a.xp) + (int64_t)row * a.row_bytes);
#pragma unroll
            for (int u = 0; u < kScatterVec; ++u)
                if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = val[u];
        }
    }
}

}  // namespace

// Token tiles over rows received from G ranks: segment s = (source s / El,
// local expert s % El) holds recv_rows[s] rows (a multiple of 32), split into
// tiles of at most 256 rows. One CTA, thread s owns segment s (G El <= 256).
__global__ void __launch_bounds__(kMaxE) ep_tiles_kernel(EpTilesArgs a) {
    __shared__ int sc_rows[kMaxE];
    __shared__ int sc_tiles[kMaxE];
    const int s = threadIdx.x, nseg = a.G * a.El;
    const int rows = s < nseg ? a.recv_rows[s] : 0;
    const int tiles = (rows + kTokTile - 1) / kTokTile;
    sc_rows[s] = rows;
    sc_tiles[s] = tiles;
    __syncthreads();
    for (int off = 1; off < kMaxE; off <<= 1) {
        const int vr = s >= off ? sc_rows[s - off] : 0;
        const int vt = s >= off ? sc_tiles[s - off] : 0;
        __syncthreads();
        sc_rows[s] += vr;
        sc_tiles[s] += vt;
        __syncthreads();
    }
    const int row0 = sc_rows[s] - rows, tile0 = sc_tiles[s] - tiles;
    const bool fits = sc_rows[kMaxE - 1] <= a.R;  // a layout larger than the buffer runs nothing
    if (fits && s < nseg)
        for (int i = 0; i < tiles; ++i)
            a.tiles[tile0 + i] = make_int4(s % a.El, row0 + i * kTokTile, min(kTokTile, rows - i * kTokTile), 0);
    if (s < kCtrlWords) a.ctrl[s] = 0;
    __syncthreads();
    if (s == 0) a.ctrl[kCtrlNumTokTiles] = fits ? sc_tiles[kMaxE - 1] : 0;
}

cudaError_t launch_ep_tiles(const EpTilesArgs &a, cudaStream_t s, int *launches) {
    ep_tiles_kernel<<<1, kMaxE, 0, s>>>(a);
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    static_assert(kChunk == kMaxE, "the one-block path runs all three steps with the same threads");
    if (a.n_chunks == 1) {
        dispatch_one_chunk_kernel<<<1, kChunk, 0, s>>>(a);
        *launches += 1;
        return cudaGetLastError();
    }
    dispatch_count_scan_kernel<<<a.n_chunks, kChunk, 0, s>>>(a);
    dispatch_assign_kernel<<<a.n_chunks, kChunk, 0, s>>>(a);
    *launches += 2;
    return cudaGetLastError();
}

cudaError_t launch_scatter(const ScatterArgs &a, int num_sms, cudaStream_t s, int *launches) {
    if (a.T <= 0) return cudaSuccess;
    const int64_t nchunk = (a.row_bytes / 16 + 32 * kScatterVec - 1) / (32 * kScatterVec);
    const int64_t items = (int64_t)a.T * nchunk;
    const int blocks = (int)std::min<int64_t>((items + 7) / 8, (int64_t)num_sms * 8);
    scatter_rows_kernel<<<blocks, 256, 0, s>>>(a);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
