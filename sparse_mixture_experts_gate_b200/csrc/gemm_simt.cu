// gemm_simt.cu - grouped expert GEMM for fp32 layers on CUDA cores.
//
// The same operation as gemm_pair.cu ("Code Walkthrough - SER", gating /
// routing path: each expert's w1/b1 -> activation -> w2/b2 MLP over the rows
// dispatched to it) for layers stored in fp32, where bf16 tensor-core operands
// would not keep fp32 accuracy. 32 x 32 output tiles (one per 32-row block of
// the row space, which never straddles two groups), K staged through shared
// memory.
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kTile = 32;

__global__ void __launch_bounds__(256) grouped_gemm_simt_kernel(GemmSimtArgs a) {
    __shared__ float As[kTile][kTile + 1];
    __shared__ float Bs[kTile][kTile + 1];
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    const int r0 = blockIdx.y * kTile, n0 = blockIdx.x * kTile;
    static_assert(kTile == kRowBlock, "one output tile per row block");
    const int rows_total = min(a.ctrl[kCtrlNumRowBlocks], a.max_row_blocks) * kRowBlock;
    if (r0 >= rows_total) return;
    const int g = a.block_group[r0 / kRowBlock];
    const int rows_valid_end = a.group_start[g] + a.group_rows[g];
    const float *w = a.w + (int64_t)g * a.N * a.K;

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < a.K; k0 += kTile) {
        for (int i = ty; i < kTile; i += 8) {
            const int row = r0 + i, kk = k0 + tx;
            float v = 0.f;
            if (row < rows_valid_end && kk < a.K) {
                int64_t arow = row;  // row space itself
                if (a.gather) {      // token row of x: routed via the dispatch map, shared in order
                    arow = g < a.E ? a.row_assign[row] / a.k : row - a.group_start[g];
                }
                v = a.a[arow * a.K + kk];
            }
            As[i][tx] = v;
            const int n = n0 + i;
            Bs[i][tx] = (n < a.N && kk < a.K) ? w[(int64_t)n * a.K + kk] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kTile; ++kk) {
            const float b = Bs[tx][kk];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = fmaf(As[ty * 4 + j][kk], b, acc[j]);
        }
        __syncthreads();
    }
    const int n = n0 + tx;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int row = r0 + ty * 4 + j;
        if (row < rows_valid_end && n < a.N)
            a.out[(int64_t)row * a.N + n] = activate(a.act, acc[j] + (a.bias ? a.bias[(int64_t)g * a.N + n] : 0.f));
    }
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmSimtArgs &p, cudaStream_t s, int *launches) {
    dim3 grid((p.N + kTile - 1) / kTile, p.max_row_blocks);
    if (grid.y == 0) return cudaSuccess;
    grouped_gemm_simt_kernel<<<grid, dim3(32, 8), 0, s>>>(p);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
