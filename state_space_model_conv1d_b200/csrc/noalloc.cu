// noalloc.cu -- ssm_scan_fwd for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: code running inside a
// CUDA-graph capture that must not allocate, runtimes whose memory pool is
// owned and fully reserved by another component, or plugins that are handed
// device buffers but no allocator.  ssm_scan_fwd needs a workspace for its
// device error word, the varlen schedule and (on the tensor-core Mamba-2
// path) the conv'd B / C tiles.  This entry point takes that workspace from a
// file-scope device array of fixed size instead, so the caller passes only
// its inputs and outputs.
//
// The array's name is a host-side stand-in in host code, not a device
// address, so its device address is fetched once per device with
// cudaGetSymbolAddress while that device is current, and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/ssm.h"

namespace {

constexpr int kMaxDevices = 64;

// The scratch every call shares (one copy per GPU that loads the library,
// held until the process exits).
__device__ __align__(256) unsigned char g_noalloc_scratch[SSM_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call for that device).  Returns a cudaError_t.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

ssm_status ssm_scan_fwd_noalloc(const ssm_scan_args *args, void *stream) {
    if (!args) return SSM_ERR_INVALID_ARG;
    size_t need = ssm_scan_workspace_size(args);
    ssm_scan_args whole;
    if (need > (size_t)SSM_NOALLOC_SCRATCH_BYTES && args->segments == 0) {
        // the library's choice of token segments keeps their states in the
        // workspace: without them the call may still fit the fixed scratch
        whole = *args;
        whole.segments = 1;
        need = ssm_scan_workspace_size(&whole);
        args = &whole;
    }
    if (need > (size_t)SSM_NOALLOC_SCRATCH_BYTES) return SSM_ERR_WORKSPACE;
    void *ws = nullptr;
    if (need > 0) {
        const cudaError_t e = scratch_address(&ws);
        if (e != cudaSuccess) return SSM_ERR_CUDA;
    }
    return ssm_scan_fwd(args, ws, need > 0 ? (size_t)SSM_NOALLOC_SCRATCH_BYTES : 0, stream);
}

}  // extern "C"
