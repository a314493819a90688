// gemm_simt.cu - grouped expert GEMM for fp32 layers on CUDA cores.
//
// The same operation as gemm_tc.cu ("Code Walkthrough - SER", gating / routing
// path: each expert's w1/b1 -> activation -> w2/b2 MLP over the rows dispatched
// to it) for layers stored in fp32, where bf16 tensor-core operands would not
// keep fp32 accuracy. 32 x 32 output tiles, K staged through shared memory;
// one warp covers 32 columns of four rows, so the per-row sum of squares for the
// credit norm is a warp reduction.
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kTile = 32;

__global__ void __launch_bounds__(256) grouped_gemm_simt_kernel(GemmSimtArgs p) {
    const GemmArgs &a = p.g;
    __shared__ float As[kTile][kTile + 1];
    __shared__ float Bs[kTile][kTile + 1];
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    const int r0 = blockIdx.y * kTile, n0 = blockIdx.x * kTile;
    const int rows_total = min(a.ctrl[kCtrlNumMTiles], a.max_mtiles) * kBM;
    if (r0 >= rows_total) return;
    const int g = a.tile_group[r0 / kBM];
    const int rows_valid_end = a.group_start[g] + a.group_rows[g];
    const float *w = p.w + (int64_t)g * a.N * a.K;

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < a.K; k0 += kTile) {
        for (int i = ty; i < kTile; i += 8) {
            const int row = r0 + i, kk = k0 + tx;
            float v = 0.f;
            if (row < rows_valid_end && kk < a.K) {
                int64_t arow = row;  // row space itself
                if (p.gather) {      // token row of x: routed via the dispatch map, shared in order
                    arow = g < a.E ? a.row_assign[row] / a.k : row - a.group_start[g];
                }
                v = p.a[arow * a.K + kk];
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
    float *out = static_cast<float *>(a.out);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int row = r0 + ty * 4 + j;
        float z = 0.f;
        if (n < a.N) {
            z = acc[j] + (a.bias ? a.bias[(int64_t)g * a.N + n] : 0.f);
            z = activate(a.act, z);
        }
        float ss = z * z;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (row < rows_valid_end) {
            if (n < a.N) out[(int64_t)row * a.N + n] = z;
            if (a.norm_part && tx == 0) a.norm_part[(int64_t)row * a.n_tiles + blockIdx.x] = ss;
        }
    }
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmSimtArgs &p, cudaStream_t s, int *launches) {
    dim3 grid((p.g.N + kTile - 1) / kTile, (p.max_rows + kTile - 1) / kTile);
    if (grid.y == 0) return cudaSuccess;
    grouped_gemm_simt_kernel<<<grid, dim3(32, 8), 0, s>>>(p);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
