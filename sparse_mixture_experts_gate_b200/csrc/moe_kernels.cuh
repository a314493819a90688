// moe_kernels.cuh - argument blocks and host launchers of the MoE layer kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_common.cuh"

namespace moe {

// Router on fp32 CUDA cores (fp32 layers, and the MLP gate's output layer):
// logits h = W_g x + b, max, log-partition, selection key, top-k, gates.
struct RouterArgs {
    const void *x;          // [T][d] bf16 or fp32
    int x_bf16;
    const float *w_gate;    // [E][d]
    const float *b_gate;    // [E] or null
    const float *noise;     // [T][E] or null (added to the selection key only)
    const float *sel_bias;  // [E] or null (added to the selection key only)
    int T, d, E, k;
    float *logits;          // [T][E]
    int32_t *idx;           // [T][k]
    float *gates;           // [T][k]
    float *lse;             // [T]
    float *psum_part;       // [router_psum_blocks][E]: per-block sums of P over its tokens
    int x_relu;             // fp32 router only: relu(x) is the router's input (MLP gate output layer)
    int logits_only;        // fp32 router only: write logits (+ bias) and stop (MLP gate hidden layer)
};
int router_psum_blocks(int T);
cudaError_t launch_router(const RouterArgs &a, cudaStream_t s, int *launches);

// Router of bf16 layers in one cooperative kernel (router_fused.cu): logits on
// the tensor cores from three bf16 planes of W_g, then, after a grid-wide
// barrier, (route = 1) softmax, log-partition, keys, top-k, gates and a row of
// P sums per CTA. Units: token tiles of 256, expert tiles of BN, ksplit K
// splits.
struct RouterFusedArgs {
    const float *b_gate;    // [E] or null
    const float *noise;     // [T][E] or null (added to the selection key only)
    const float *sel_bias;  // [E] or null (added to the selection key only)
    int T, d, E, k;
    int BN, n_tiles, ksplit, n_mtiles;
    int route;              // 0: logits (+ bias) only, e.g. the MLP gate's hidden layer
    float *logits;          // [T][E]
    int32_t *idx;           // [T][k]
    float *gates;           // [T][k]
    float *lse;             // [T]
    float *psum_part;       // [router_fused_ctas][E]: P summed over each CTA's tokens
    float *part;            // [n_mtiles n_tiles ksplit][256][BN] partial sums when n_tiles ksplit > 1
    int32_t *counters;      // [1] grid-barrier counter, zero before the launch
    uint32_t *status;
    int num_pairs;          // CTA pairs to launch at most
    // Self-test of the bounded waits only (moe_selftest_router_timeout): every
    // leader's producer skips its loads of this pipeline stage (-1: none), and
    // every wait of the launch gives up after wait_limit_ns.
    int skip_stage = -1;
    uint64_t wait_limit_ns = kWaitLimitNs;
};
int router_fused_epad(int E);    // padded expert count (rows of the split planes): 32, 64, 128 or 256
int router_fused_bn(int E);      // expert tile: E_pad up to 128
int router_fused_mtiles(int T);  // token tiles of 256
int router_fused_ksplit(int T, int E, int d, int num_pairs);
int router_fused_max_pairs(int num_sms);
// CTAs the launch has for `units` units (2 per pair): the rows of psum_part.
int router_fused_ctas(int units, int num_pairs);
// W_g [E][d] fp32 -> w_split [E_pad][3d] bf16: planes hi | mid | lo, rows >= E zero.
cudaError_t launch_router_split(const float *w_gate, int E, int E_pad, int d, __nv_bfloat16 *w_split, int num_sms,
                                cudaStream_t s, int *launches);
// map_x: x [T][d] bf16, box 64 x 128; map_w: w_split, box 64 x BN/2.
cudaError_t launch_router_fused(const CUtensorMap &map_x, const CUtensorMap &map_w, const RouterFusedArgs &a,
                                cudaStream_t s, int *launches);

// Dispatch: histogram, scan, stable capacity-capped ranks, row map.
struct DispatchArgs {
    const int32_t *idx;     // [T][k]
    int T, E, k, S;
    int rank_major;         // capacity priority: 0 token order, 1 choice by choice (item = r T + t)
    int n_items;            // T (token order) or k T (rank-major)
    int64_t C;              // capacity
    int T_pad;              // T rounded up to kRowBlock (shared-expert segment length)
    int n_chunks;           // ceil(n_items / 256)
    int32_t *chunk_count;   // [n_chunks][E]
    int32_t *chunk_base;    // [n_chunks][E]
    int32_t *count_pre;     // [E]
    int32_t *count_kept;    // [E]
    int32_t *user_count_pre;   // [E] or null
    int32_t *user_count_kept;  // [E] or null
    int32_t *group_start;   // [E+S+1]
    int32_t *group_rows;    // [E+S]
    int32_t *block_group;   // [max_row_blocks]: group of each 32-row block
    int4 *tok_tiles;        // [max_tok_tiles]: {group, first row, rows, 0}
    int4 *narrow_tiles = nullptr;  // [max_narrow_tiles]: the same with at most kNarrowTile rows, or null
    int32_t *ctrl;          // control block (see kCtrl*)
    int32_t *slot;          // [T][k]
    int32_t *row_of;        // [T][k]
    int32_t *row_assign;    // [R_max]  t*k + r, or -1 on padding rows
    const float *gates;     // [T][k]
    int32_t *pre_start;     // [E]: exclusive scan of count_pre
    float *gate_sorted;     // [T*k]: every selection's gate, grouped by expert, token order
    int32_t *tile_done = nullptr;  // [n_tile_done] zeroed by the scan (the expert GEMM's per-tile counters)
    int n_tile_done = 0;
};
cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s, int *launches);

// Control block words.
enum {
    kCtrlStatus = 0,
    kCtrlNumRowBlocks = 1,
    kCtrlRoutedRows = 2,
    kCtrlDropped = 3,
    kCtrlNumTokTiles = 4,
    kCtrlWork1 = 5,  // unit counters of the two expert GEMM launches
    kCtrlWork2 = 6,
    kCtrlRoutedTiles = 7,  // token tiles of the routed experts (the shared experts' follow)
    kCtrlNumNarrowTiles = 8,
    kCtrlStatsDone = 9,      // CTAs of the statistics kernel done (its last CTA resets it)
    kCtrlDispatchDone = 10,  // chunks counted by the dispatch (its last CTA resets it)
    kCtrlWords = 11
};

// Rows of a narrow token tile: for short expert segments the expert GEMM
// stages at most kNarrowTile / 2 token rows per CTA, leaving room for a
// deeper pipeline of weight tiles.
constexpr int kNarrowTile = 64;

// Scatter of token rows into the permuted row space (rows of kept assignments).
struct ScatterArgs {
    const void *x;          // [T][d]
    void *xp;               // [R_routed_max][d]
    const int32_t *row_of;  // [T][k] row of each assignment, -1 if dropped
    int T, k;
    int row_bytes;          // d * element size (multiple of 16)
};
cudaError_t launch_scatter(const ScatterArgs &a, int num_sms, cudaStream_t s, int *launches);

// Grouped expert GEMM: out[row] = act(A[row] . W[g]^T + b[g]) for the rows of
// every group g (routed experts, then shared experts).
//
// bf16 tensor-core path on CTA pairs (gemm_pair.cu): work unit = (token tile,
// 256-feature tile). map_w: the weight stack [G*N][K] (box 64 x 128; map_wh
// the same with box 64 x 64); map_t / map_t16: the token rows in row order
// (box 64 x 128 and 64 x 16); map_s / map_s16: with use_s, the token rows of
// shared-expert groups (x itself, in token order); map_out: the output
// [rows][N] bf16 (box 128 x 32, no swizzle), also addressed directly through
// `out`. N and K must be multiples of 64.
// The tensor maps of one GEMM layer: weights (boxes of 128 and of 64 rows),
// token rows in row order (boxes of 128 and 16 rows), shared-expert token rows
// (x itself, with use_s) and the output (box 128 x 32).
struct PairMaps {
    CUtensorMap w, wh, t, t16, s, s16, out;
};

struct PairGemmArgs {
    const int4 *tok_tiles;       // [max_tok_tiles] {group, first row, rows, 0}
    const int32_t *group_start;  // [G+1]
    const int32_t *ctrl;         // kCtrlNumTokTiles, kCtrlStatus
    int max_tok_tiles;           // host bound (clamps the device count)
    int N, K;
    int n_ftiles;                // ceil(N / 256)
    int E;                       // groups >= E are shared experts
    int w_shared_base = 0;       // weight-stack index of the first shared group (E, or the local count)
    int tile_base_word = -1;     // ctrl word holding the index of the first tile to run, or -1 (tile 0)
    int fixed_tiles = 0;         // > 0: run this many tiles instead of ctrl[tiles_count_word]
    int tiles_count_word = kCtrlNumTokTiles;  // ctrl word holding the tile count
    int narrow = 0;              // 1: tok_tiles holds narrow tiles (at most kNarrowTile rows)
    int use_s;
    // 1: the last feature tile holds at most 128 features (N % 256 in {64, 128})
    // and its units run transposed (wide token tiles only), storing through `out`.
    int half_last = 0;
    // Two layers in one launch (set by launch_gemm_pair): layer 2's units of a
    // token tile wait until tile_done[tile] counts every layer-1 unit of it
    // (each CTA of a pair adds 1 once its outputs are stored). tile_done has
    // one zeroed int per token tile.
    int fuse2 = 0;
    int32_t *tile_done = nullptr;
    __nv_bfloat16 *out = nullptr;  // [rows][N] bf16 output (row space), the array map_out covers
    const float *bias;           // [G][N] or null
    int act;                     // activation code, -1 none
    uint32_t *status;            // device status word
    int32_t *work_counter;       // zero before the launch; units are handed out in order
    int num_pairs;               // clusters of 2 CTAs to launch
    // Self-test of the bounded waits only (moe_selftest_gemm_timeout): the
    // leader's producer skips its loads of this pipeline stage (-1: none), and
    // every wait of the launch gives up after wait_limit_ns.
    int skip_stage = -1;
    uint64_t wait_limit_ns = kWaitLimitNs;
};
int gemm_pair_max_pairs(int num_sms);
int gemm_pair_ftiles(int N);
int gemm_pair_half_last(int N);  // 1 when the last feature tile of N holds at most 128 features
// One launch of layer 1 (m1, a), or of layer 1 followed by layer 2 (m2, b:
// same token tiles, its token rows layer 1's outputs) when m2 and b are given.
cudaError_t launch_gemm_pair(const PairMaps &m1, const PairGemmArgs &a, const PairMaps *m2, const PairGemmArgs *b,
                             cudaStream_t s, int *launches);

// fp32 CUDA-core path: 32 x 32 output tiles over the 32-row blocks.
struct GemmSimtArgs {
    const int32_t *block_group;  // [max_row_blocks]
    const int32_t *group_start;  // [G+1]
    const int32_t *group_rows;   // [G]
    const int32_t *ctrl;         // kCtrlNumRowBlocks
    int max_row_blocks;
    int N, K, E, k;
    const int32_t *row_assign;   // [rows] t*k + r of each routed row (-1 padding)
    const float *bias;           // [G][N] or null
    float *out;                  // [rows][N]
    int act;
    const float *a;              // gather: x [T][K]; otherwise [rows][K]
    int gather;
    const float *w;              // [G][N][K]
};
cudaError_t launch_gemm_simt(const GemmSimtArgs &a, cudaStream_t s, int *launches);

// Gate-weighted combine with shared experts, plus credit.
struct CombineArgs {
    const void *o;          // [rows][O] expert outputs
    const float *row_norm2; // [rows] squared norms the credit uses instead of ||o||^2, or null
    const int32_t *row_of;  // [T][k]
    const float *gates;     // [T][k]
    const int32_t *group_start;
    int T, O, E, S, k;
    int bf16;
    void *y;                // [T][O]
    float *credit;          // [T][k]
};
cudaError_t launch_combine(const CombineArgs &a, int num_sms, cudaStream_t s, int *launches);

// Balancing and credit statistics: partial sums, then finalize.
struct StatsArgs {
    const float *psum_part;   // [n_chunks][E]: the router's per-block sums of P
    int n_chunks;
    const float *lse;         // [T]
    const int32_t *count_pre; // [E]
    const int32_t *group_start;
    const int32_t *group_rows;
    const int32_t *row_assign;
    const float *credit;      // [T][k]
    const float *token_loss;  // [T] or null
    const int32_t *ctrl;
    const int32_t *pre_start; // [E]
    const float *gate_sorted; // [T*k]
    int T, E, k;
    float *partials;          // [4E + 3] output
    int32_t *done_counter;    // zero; counts the CTAs done when the finalize is fused
};

struct FinalizeArgs {
    const float *partials;    // [4E + 3]
    int E, k;
    float alpha, beta;
    float *f, *p_mean, *l_aux, *l_z, *expert_loss;  // outputs (nullable)
    int32_t *n_dropped;
    float *importance, *cv_load, *cv_importance, *l_total;
};
// fin != null: the last CTA also forms the statistics (one launch in all).
cudaError_t launch_stat_partials(const StatsArgs &a, const FinalizeArgs *fin, cudaStream_t s, int *launches);
cudaError_t launch_stats_finalize(const FinalizeArgs &a, cudaStream_t s, int *launches);

// Expert parallelism: the token-tile table of rows received from G source
// ranks, laid out source-major, each source's rows grouped by local expert and
// padded to 32 rows (the sender's row space).
struct EpTilesArgs {
    const int32_t *recv_rows;  // [G][E_local] padded rows
    int G, El, R;
    int4 *tiles;               // out: {local expert, first row, rows, 0}
    int32_t *ctrl;             // out: kCtrlNumTokTiles (status and counters zeroed)
};
cudaError_t launch_ep_tiles(const EpTilesArgs &a, cudaStream_t s, int *launches);

// Squared norms of the routed rows of a [rows][n] matrix (H, for the credit's
// hidden-activation reading); padding rows are skipped.
struct RowNormArgs {
    const void *m;
    int n, bf16;
    const int32_t *row_assign;  // [rows], -1 on padding rows
    const int32_t *ctrl;        // kCtrlRoutedRows
    int max_rows;
    float *norm2;               // [rows]
};
cudaError_t launch_row_norms(const RowNormArgs &a, int num_sms, cudaStream_t s, int *launches);

// Panel (c) bookkeeping: EMA of the expert losses, mu <- softmax(mu + eta lhat),
// objective sum mu l.
struct DroArgs {
    const float *l;
    float *lhat, *mu, *objective;
    int E;
    float ema, eta;
};
cudaError_t launch_dro_update(const DroArgs &a, cudaStream_t s, int *launches);

// Aux-loss-free balancing: b_e += gamma sign(k T / E - load_e).
struct BiasUpdateArgs {
    const float *partials;     // [4E + 3] (loads and T from the sums) or null
    const int32_t *count_pre;  // [E], used when partials is null
    int T, E, k;
    float gamma;
    float *sel_bias;           // [E] in place
};
cudaError_t launch_bias_update(const BiasUpdateArgs &a, cudaStream_t s, int *launches);

// Sets the calling thread's last-error message; returns `code`.
int report_error(int code, const char *msg);

}  // namespace moe
