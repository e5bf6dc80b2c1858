// launch.h -- host-side launchers behind the C ABI (internal to libssm).
// Arguments reaching these functions have already been validated by ssm_api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssm.h"

namespace ssm {

// Workspace layout of ssm_scan_fwd (all offsets 256-byte aligned):
//   [0, 256)            int32 device error word (SSM_DEVERR_*), then padding
//   [256, 256 + 4*n)    int32 sequence schedule (longest sequence first)
constexpr size_t kWsErrorOffset = 0;
constexpr size_t kWsOrderOffset = 256;
inline size_t varlen_workspace_bytes(int64_t nseqs) {
    return kWsOrderOffset + ((size_t)(nseqs > 0 ? nseqs : 1) * 4 + 255) / 256 * 256;
}

// Packed-sequence view shared by the scan launchers: sequence s spans tokens
// [cu[s], cu[s+1]) of batch row 0 when cu != nullptr, else row s spans
// [0, seqlen).  `order` (may be null) lists sequences longest first.
struct SeqView {
    const int32_t *cu;
    const int32_t *order;
    int32_t *err;
    int nseqs;
};

cudaError_t launch_conv1d(const ssm_conv_args &a, cudaStream_t st);
cudaError_t launch_varlen_plan(const int32_t *cu, int nseqs, int64_t total, int32_t *err, int32_t *order,
                               cudaStream_t st);
cudaError_t launch_scan_m1(const ssm_scan_args &a, const SeqView &sv, cudaStream_t st);
cudaError_t launch_scan_m2_simt(const ssm_scan_args &a, const SeqView &sv, cudaStream_t st);
cudaError_t launch_state_update(const ssm_update_args &a, cudaStream_t st);

// Largest dstate each path supports.
constexpr int64_t kMaxDstateM1 = 64;
constexpr int64_t kMaxDstateM2 = 256;
constexpr int64_t kMaxConvWidth = 8;

}  // namespace ssm
