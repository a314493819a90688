// selftest.cu - a self-check of the bounded-wait machinery.
//
// Every wait in the tcgen05 kernels goes through mbar_wait(): it spins on an
// mbarrier phase, and once the wait has lasted kWaitLimitNs it sets kDevTimeout
// in the forward's status word and returns false, so the kernel can drain and
// exit and the host reads the failure from moe_device_status. This entry point
// runs that path on purpose: one thread waits on a barrier that nothing ever
// arrives on. No copy, MMA or cluster peer is involved, so giving up leaves
// nothing in flight.
#include <cstring>

#include "moe.h"
#include "moe_common.cuh"

namespace moe {
int report_error(int code, const char *msg);
namespace {

__device__ uint32_t g_selftest_words[2];  // [0] status word, [1] outcome

__global__ void bounded_wait_selftest_kernel() {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        const bool got = mbar_wait(&bar, 0u, &g_selftest_words[0]);  // phase 0 never completes
        g_selftest_words[1] = got ? 1u : 2u;
    }
}

}  // namespace
}  // namespace moe

extern "C" int moe_selftest_bounded_wait(void *stream_v) {
    using namespace moe;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_v);
    void *words = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&words, g_selftest_words);
    if (e == cudaSuccess) e = cudaMemsetAsync(words, 0, sizeof(g_selftest_words), s);
    if (e == cudaSuccess) {
        bounded_wait_selftest_kernel<<<1, 32, 0, s>>>();
        e = cudaGetLastError();
    }
    uint32_t h[2] = {0u, 0u};
    if (e == cudaSuccess) e = cudaMemcpyAsync(h, words, sizeof(h), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return report_error(MOE_ERR_CUDA, cudaGetErrorString(e));
    if (h[1] != 2u || (h[0] & kDevTimeout) == 0u)
        return report_error(MOE_ERR_INTERNAL, "the bounded wait did not report its timeout");
    return MOE_OK;
}
