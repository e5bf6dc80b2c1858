// launch.h -- host-side launchers behind the C ABI (internal to libssm).
// Arguments reaching these functions have already been validated by ssm_api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssm.h"

namespace ssm {

// Workspace layout of ssm_scan_fwd (all offsets 256-byte aligned):
//   [0, 256)            int32 device error word (SSM_DEVERR_*), then padding
//   [256, 256 + R)      varlen only: int32 sequence schedule (longest first), R = 4*nseqs rounded to 256
//   [256 + R, ...)      tensor-core Mamba-2 path only: conv'd bf16 B and C tiles
constexpr size_t kWsErrorOffset = 0;
constexpr size_t kWsOrderOffset = 256;
inline size_t order_bytes(int64_t nseqs) { return ((size_t)(nseqs > 0 ? nseqs : 1) * 4 + 255) / 256 * 256; }

// Packed-sequence view shared by the scan launchers: sequence s spans tokens
// [cu[s], cu[s+1]) of batch row 0 when cu != nullptr, else row s spans
// [0, seqlen).  `order` (may be null) lists sequences longest first.
struct SeqView {
    const int32_t *cu;
    const int32_t *order;
    int32_t *err;
    int nseqs;
};

// Intermediate-state extraction (prefix caching): after every `interval`
// tokens of a sequence, the state and conv history go to pool row
// slots[s * stride + k] (boundary k) when it lies in [0, nslots).  interval 0
// disables it.  `conv` is in the activation dtype, [nslots][conv_dim][K-1].
struct InterView {
    int64_t interval;
    const int32_t *slots;
    int64_t stride, nslots;
    float *states;
    void *conv;
    // pool row for the boundary that ends `done` tokens into sequence s, or -1
    __device__ __forceinline__ int64_t slot_after(int s, int64_t done) const {
        if (interval <= 0 || done <= 0 || done % interval != 0) return -1;
        const int64_t k = done / interval - 1;
        if (k >= stride) return -1;
        const int64_t r = slots[(int64_t)s * stride + k];
        return (r >= 0 && r < nslots) ? r : -1;
    }
};
inline InterView inter_view(const ssm_scan_args &a) {
    return InterView{a.state_interval, a.inter_slots, a.inter_stride, a.inter_nslots, a.inter_states, a.inter_conv};
}

// A causal depthwise conv over `channels` contiguous channels of a token-major
// tensor.  Carried states are [seq][...] with `state_stride` elements between
// sequences and K-1 values per channel (so a slice of a wider state works).
struct ConvJob {
    const void *x;
    int64_t x_bs, x_ts;
    const float *w, *b;                 // [channels][K], [channels] (already offset to the slice)
    const void *state_in;               // may be null
    void *state_out;                    // may be null
    int64_t state_stride;
    const int32_t *cu;
    int nseqs;
    int64_t batch, seqlen, channels, width;
    int act, dtype;
    void *out;
    int64_t o_bs, o_ts;
};

cudaError_t launch_conv1d(const ssm_conv_args &a, cudaStream_t st);
cudaError_t launch_conv_job(const ConvJob &j, cudaStream_t st);
cudaError_t launch_varlen_plan(const int32_t *cu, int nseqs, int64_t total, int32_t *err, int32_t *order,
                               cudaStream_t st);
cudaError_t launch_scan_m1(const ssm_scan_args &a, const SeqView &sv, cudaStream_t st);
cudaError_t launch_scan_m2_simt(const ssm_scan_args &a, const SeqView &sv, cudaStream_t st);
// Tensor-core (tcgen05) chunked Mamba-2 path: which shapes it takes, the
// workspace it needs for the conv'd B / C, and its launcher.
bool ssd_shape_ok(const ssm_scan_args &a);      // shapes only: decides the workspace size
bool ssd_supported(const ssm_scan_args &a);     // shapes and 16-byte alignment: decides the kernel
size_t ssd_workspace_bytes(const ssm_scan_args &a);
int ssd_segments(const ssm_scan_args &a);       // token segments per row (1 = rows stay whole)
cudaError_t launch_ssd(const ssm_scan_args &a, const SeqView &sv, void *ws_bc, cudaStream_t st);
// A [batch][tokens][channels] bf16 tensor (element strides ts, bs) as a 3-d
// TMA map with a 64-channel x box_rows-token box (128-byte swizzle or none).
bool make_map_box(CUtensorMap *m, const void *base, int64_t channels, int64_t tokens, int64_t batch, int64_t ts,
                  int64_t bs, bool swizzle, int box_rows);
cudaError_t launch_state_update(const ssm_update_args &a, cudaStream_t st);
// Backward scan: workspace bytes for the checkpoints and B / C accumulators
// (after the error word and the varlen order), and its launcher.
size_t scan_bwd_workspace_bytes(const ssm_scan_bwd_args &a);
cudaError_t launch_scan_bwd(const ssm_scan_bwd_args &a, const SeqView &sv, void *ws, cudaStream_t st);

// Sequence split across ranks (batch mode): the conv tail a segment hands on,
// the in-segment prefix sums of delta, the combine of the exchanged pairs,
// and the fix-up of y by the entering state.
cudaError_t launch_split_tail(const ssm_scan_args &a, void *tail, cudaStream_t st);
cudaError_t launch_split_cum_delta(const ssm_scan_args &a, float *cum, float *sum, cudaStream_t st);
cudaError_t launch_split_combine(const ssm_split_args &a, cudaStream_t st);
cudaError_t launch_split_fixup(const ssm_scan_args &a, const float *cum, const float *h_in, cudaStream_t st);
// The fix-up grids tile the tokens along grid.y (16 tokens per CTA row).
constexpr int64_t kMaxSplitSeqlen = 65535LL * 16;

// Device timing of the dominant kernel of a call (ssm_kernel_timing): a no-op
// unless enabled; otherwise records one event before and one after on `st`.
void timing_begin(cudaStream_t st);
void timing_end(cudaStream_t st);

// SM count of the current device (148 when none answers).
int sm_count();

// Largest dstate each path supports.
constexpr int64_t kMaxDstateM1 = 64;
constexpr int64_t kMaxDstateM2 = 256;
constexpr int64_t kMaxConvWidth = 8;

}  // namespace ssm
