// moe_noalloc.cu - a layer forward that needs no caller workspace.
//
// Some callers cannot hand this library a workspace: a plugin inside a host
// application that owns every byte of device memory through its own pool and
// forbids side allocations, or a latency-critical loop that must never call
// cudaMalloc/cudaFree because those calls can synchronise the device. For them,
// moe_forward_noalloc runs the same forward as moe_forward, with its scratch in
// a fixed-size array that lives in this library's device image. The library
// allocates nothing at run time; the array exists on every GPU that loads the
// library, from module load until process exit.
#include <cstdio>
#include <mutex>

#include "moe.h"
#include "moe_common.cuh"
#include "moe_kernels.cuh"

namespace {

// The built-in scratch. In host code `g_noalloc_scratch` names a host-side
// stand-in, not the device array: only the address from cudaGetSymbolAddress
// (taken with the right device current) may be passed to kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of the built-in scratch on the current device, looked up once
// per device (the first call on a device does it, with that device current).
void *scratch_on_current_device(cudaError_t *err) {
    int dev = -1;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_addr[dev] = p;
    }
    return g_addr[dev];
}

}  // namespace

extern "C" {

MOE_API int moe_forward_noalloc(moe_layer_t *layer, const void *x, int32_t T, const float *logit_noise, void *y,
                                const moe_routing_t *routing, void *stream) {
    if (!layer) return moe::report_error(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (T < 0) return moe::report_error(MOE_ERR_INVALID_ARG, "T must be >= 0");
    const size_t need = moe_workspace_bytes(layer, T);
    if (need > (size_t)MOE_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "moe_forward_noalloc: T=%d needs %zu bytes of scratch, more than the built-in %zu bytes; "
                 "use fewer tokens per call or moe_forward with a caller workspace",
                 T, need, (size_t)MOE_NOALLOC_SCRATCH_BYTES);
        return moe::report_error(MOE_ERR_WORKSPACE, msg);
    }
    cudaError_t err = cudaSuccess;
    void *scratch = scratch_on_current_device(&err);
    if (!scratch) {
        char msg[256];
        snprintf(msg, sizeof msg, "moe_forward_noalloc: cudaGetSymbolAddress of the built-in scratch failed: %s",
                 cudaGetErrorString(err));
        return moe::report_error(MOE_ERR_CUDA, msg);
    }
    return moe_forward(layer, x, T, logit_noise, scratch, MOE_NOALLOC_SCRATCH_BYTES, y, routing, stream);
}

}  // extern "C"
