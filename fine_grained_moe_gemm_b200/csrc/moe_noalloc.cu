// moe_forward_noalloc (include/moe.h): moe_forward with its workspace in a
// static device array instead of caller memory, for callers that cannot
// allocate device memory at call time.  Nothing here allocates.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe.h"

namespace {

// The scratch: MOE_NOALLOC_MAX_BYTES on every GPU that loads the library,
// alive until the process exits.  In host code this name only stands for the
// symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_MAX_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up once per
// device, with that device current).  A device that is not sm_100 is refused
// before the lookup, as every other entry point refuses it.  The first lookup
// loads this file's device code on the device and so reserves the array there.
moe_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_UNSUPPORTED;
    }
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
        cudaGetLastError();
        return MOE_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();  // leave no sticky-looking error behind for the caller's next check
            return MOE_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_forward_noalloc(const moe_config* cfg, const moe_weights* w, const void* x,
                                          const float* bias, int T, void* y, moe_dtype y_dtype, int accumulate,
                                          moe_stream_t stream) {
    if (!cfg || T < 0) return MOE_ERR_INVALID_ARG;
    // moe_workspace_size is 0 for an invalid config; moe_forward reports that error itself
    if (moe_workspace_size(cfg, T) > MOE_NOALLOC_MAX_BYTES) return MOE_ERR_WORKSPACE;
    void* scratch = nullptr;
    moe_status st = scratch_address(&scratch);
    if (st != MOE_OK) return st;
    // moe_forward overwrites or zeroes every workspace region it later reads
    // (the fp32 combine buffer is cleared on the stream before the down GEMM)
    return moe_forward(cfg, w, x, bias, T, y, y_dtype, accumulate, scratch, MOE_NOALLOC_MAX_BYTES, stream);
}
