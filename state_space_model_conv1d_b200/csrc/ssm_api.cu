// ssm_api.cu -- the C ABI of libssm.so: argument validation on the host, then
// the launch of the matching sm_100a kernel on the caller's stream.  Nothing
// here allocates device memory or synchronizes (except ssm_workspace_error,
// whose job is to read a device word back).
#include <cuda_runtime.h>

#include "../../include/ssm.h"
#include "common.cuh"
#include "launch.h"

#ifdef SSM_CHECK_BOUNDS
namespace ssm {
__device__ BoundsRecord g_ssm_bounds;
}
#endif

namespace {

thread_local int32_t g_last_cuda_error = 0;

ssm_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return SSM_OK;
    g_last_cuda_error = (int32_t)e;
    return SSM_ERR_CUDA;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }
size_t esize(int32_t dtype) { return dtype == SSM_BF16 ? 2 : 4; }
bool dtype_ok(int32_t d) { return d == SSM_F32 || d == SSM_BF16; }

// A token-major activation: row width w elements, strides in elements.
ssm_status check_act(const void *p, int64_t bs, int64_t ts, int64_t w, int64_t batch, int64_t seqlen, size_t es,
                     bool required) {
    if (!p) return required ? SSM_ERR_INVALID_ARG : SSM_OK;
    if (!aligned(p, es)) return SSM_ERR_ALIGNMENT;
    if (ts < 0 || bs < 0) return SSM_ERR_INVALID_ARG;
    if (seqlen > 1 && ts < w) return SSM_ERR_INVALID_ARG;          // token rows may not overlap
    if (batch > 1 && bs < ts * (seqlen - 1) + w) return SSM_ERR_INVALID_ARG;
    return SSM_OK;
}

#define SSM_TRY(expr)                      \
    do {                                   \
        ssm_status st_ = (expr);           \
        if (st_ != SSM_OK) return st_;     \
    } while (0)

ssm_status validate_conv(const ssm_conv_args *a) {
    if (!a) return SSM_ERR_INVALID_ARG;
    if (!dtype_ok(a->dtype) || a->batch < 0 || a->seqlen < 0 || a->channels < 1) return SSM_ERR_INVALID_ARG;
    if (a->width < 1 || a->width > ssm::kMaxConvWidth) return SSM_ERR_UNSUPPORTED;
    if (a->activation != 0 && a->activation != 1) return SSM_ERR_INVALID_ARG;
    if (!a->weight) return SSM_ERR_INVALID_ARG;
    if (a->cu_seqlens && (a->batch != 1 || a->nseqs < 0 || (a->nseqs == 0 && a->seqlen > 0)))
        return SSM_ERR_INVALID_ARG;
    if (a->seqlen > INT32_MAX || a->batch > 65535) return SSM_ERR_UNSUPPORTED;
    const size_t es = esize(a->dtype);
    const bool work = a->batch > 0 && a->seqlen > 0;
    SSM_TRY(check_act(a->x, a->x_batch_stride, a->x_token_stride, a->channels, a->batch, a->seqlen, es, work));
    SSM_TRY(check_act(a->out, a->out_batch_stride, a->out_token_stride, a->channels, a->batch, a->seqlen, es, work));
    if (!aligned(a->state_in, es) || !aligned(a->state_out, es)) return SSM_ERR_ALIGNMENT;
    if (!aligned(a->weight, 4) || !aligned(a->bias, 4)) return SSM_ERR_ALIGNMENT;
    return SSM_OK;
}

ssm_status validate_scan(const ssm_scan_args *a) {
    if (!a) return SSM_ERR_INVALID_ARG;
    if ((a->mode != SSM_MAMBA1 && a->mode != SSM_MAMBA2) || !dtype_ok(a->dtype)) return SSM_ERR_INVALID_ARG;
    if (a->batch < 0 || a->seqlen < 0 || a->d_inner < 1 || a->dstate < 1) return SSM_ERR_INVALID_ARG;
    if (a->delta_softplus != 0 && a->delta_softplus != 1) return SSM_ERR_INVALID_ARG;
    if (a->d_conv < 0 || a->d_conv > ssm::kMaxConvWidth) return a->d_conv < 0 ? SSM_ERR_INVALID_ARG : SSM_ERR_UNSUPPORTED;
    if (a->d_conv > 0 && !a->conv_w) return SSM_ERR_INVALID_ARG;
    if (a->seqlen > INT32_MAX || a->batch > 65535) return SSM_ERR_UNSUPPORTED;
    int64_t G, dtw;
    if (a->mode == SSM_MAMBA1) {
        if (a->ngroups > 1) return SSM_ERR_UNSUPPORTED;
        if (a->dstate > ssm::kMaxDstateM1) return SSM_ERR_UNSUPPORTED;
        G = 1;
        dtw = a->d_inner;
    } else {
        if (a->nheads < 1 || a->headdim < 1 || a->ngroups < 1) return SSM_ERR_INVALID_ARG;
        if (a->nheads * a->headdim != a->d_inner || a->nheads % a->ngroups != 0) return SSM_ERR_INVALID_ARG;
        if (a->dstate > ssm::kMaxDstateM2) return SSM_ERR_UNSUPPORTED;
        if (a->nheads * ((a->headdim + 31) / 32) > 2147483647LL) return SSM_ERR_UNSUPPORTED;
        G = a->ngroups;
        dtw = a->nheads;
    }
    if (a->cu_seqlens &&
        (a->batch != 1 || a->nseqs < 0 || a->nseqs > 65535 || (a->nseqs == 0 && a->seqlen > 0)))
        return SSM_ERR_INVALID_ARG;
    const size_t es = esize(a->dtype);
    const bool work = a->batch > 0 && a->seqlen > 0;
    SSM_TRY(check_act(a->x, a->x_batch_stride, a->x_token_stride, a->d_inner, a->batch, a->seqlen, es, work));
    SSM_TRY(check_act(a->z, a->z_batch_stride, a->z_token_stride, a->d_inner, a->batch, a->seqlen, es, false));
    SSM_TRY(check_act(a->dt, a->dt_batch_stride, a->dt_token_stride, dtw, a->batch, a->seqlen, es, work));
    SSM_TRY(check_act(a->B, a->B_batch_stride, a->B_token_stride, G * a->dstate, a->batch, a->seqlen, es, work));
    SSM_TRY(check_act(a->C, a->C_batch_stride, a->C_token_stride, G * a->dstate, a->batch, a->seqlen, es, work));
    SSM_TRY(check_act(a->y, a->y_batch_stride, a->y_token_stride, a->d_inner, a->batch, a->seqlen, es, work));
    if (!a->A) return SSM_ERR_INVALID_ARG;
    if (!aligned(a->A, 4) || !aligned(a->D, 4) || !aligned(a->dt_bias, 4) || !aligned(a->h0, 4) ||
        !aligned(a->h_final, 4) || !aligned(a->conv_w, 4) || !aligned(a->conv_b, 4) || !aligned(a->cu_seqlens, 4))
        return SSM_ERR_ALIGNMENT;
    if (!aligned(a->conv_state_in, es) || !aligned(a->conv_state_out, es)) return SSM_ERR_ALIGNMENT;
    if (a->chunk < 0 || a->segments < 0) return SSM_ERR_INVALID_ARG;
    if (a->state_interval != 0) {
        if (a->state_interval < 0 || a->state_interval % 64 != 0 || !a->inter_slots || a->inter_stride < 0 ||
            a->inter_nslots < 0 || (!a->inter_states && !a->inter_conv))
            return SSM_ERR_INVALID_ARG;
        if (!aligned(a->inter_slots, 4) || !aligned(a->inter_states, 4) || !aligned(a->inter_conv, es))
            return SSM_ERR_ALIGNMENT;
    }
    return SSM_OK;
}

ssm_status validate_update(const ssm_update_args *a) {
    if (!a) return SSM_ERR_INVALID_ARG;
    if ((a->mode != SSM_MAMBA1 && a->mode != SSM_MAMBA2) || !dtype_ok(a->dtype)) return SSM_ERR_INVALID_ARG;
    if (a->delta_softplus != 0 && a->delta_softplus != 1) return SSM_ERR_INVALID_ARG;
    if (a->batch < 0 || a->batch > 65535 || a->d_inner < 1 || a->dstate < 1) return SSM_ERR_INVALID_ARG;
    if (a->d_conv < 0 || a->d_conv > ssm::kMaxConvWidth) return a->d_conv < 0 ? SSM_ERR_INVALID_ARG : SSM_ERR_UNSUPPORTED;
    if (a->d_conv > 0 && (!a->conv_w || !a->conv_state || a->conv_state_len < a->d_conv - 1)) return SSM_ERR_INVALID_ARG;
    if (a->mode == SSM_MAMBA2) {
        if (a->nheads < 1 || a->headdim < 1 || a->ngroups < 1) return SSM_ERR_INVALID_ARG;
        if (a->nheads * a->headdim != a->d_inner || a->nheads % a->ngroups != 0) return SSM_ERR_INVALID_ARG;
        if (a->ngroups > 65535) return SSM_ERR_UNSUPPORTED;
        // one CTA keeps its group's conv outputs in shared memory
        if ((a->nheads / a->ngroups) * (a->headdim + 2) + 2 * a->dstate > 48 * 1024) return SSM_ERR_UNSUPPORTED;
    } else if (a->ngroups > 1) {
        return SSM_ERR_UNSUPPORTED;
    }
    if (a->batch == 0) return SSM_OK;
    if (!a->state || !a->x || !a->dt || !a->A || !a->B || !a->C || !a->y) return SSM_ERR_INVALID_ARG;
    if (!a->state_batch_indices && a->nslots < a->batch) return SSM_ERR_INVALID_ARG;
    if (a->nslots < 0) return SSM_ERR_INVALID_ARG;
    const size_t es = esize(a->dtype);
    if (!aligned(a->x, es) || !aligned(a->z, es) || !aligned(a->dt, es) || !aligned(a->B, es) || !aligned(a->C, es) ||
        !aligned(a->y, es) || !aligned(a->conv_state, es))
        return SSM_ERR_ALIGNMENT;
    if (!aligned(a->state, a->dstate % 4 == 0 ? 16 : 4) || !aligned(a->A, 4) || !aligned(a->D, 4) ||
        !aligned(a->dt_bias, 4) || !aligned(a->conv_w, 4) || !aligned(a->conv_b, 4) ||
        !aligned(a->state_batch_indices, 4))
        return SSM_ERR_ALIGNMENT;
    const int64_t gw = (a->mode == SSM_MAMBA2 ? a->ngroups : 1) * a->dstate;
    const int64_t dtw = a->mode == SSM_MAMBA2 ? a->nheads : a->d_inner;
    if (a->batch > 1 && (a->x_batch_stride < a->d_inner || a->y_batch_stride < a->d_inner ||
                         a->dt_batch_stride < dtw || a->B_batch_stride < gw || a->C_batch_stride < gw ||
                         (a->z && a->z_batch_stride < a->d_inner)))
        return SSM_ERR_INVALID_ARG;
    return SSM_OK;
}

}  // namespace

extern "C" {

int32_t ssm_abi_version(void) { return SSM_ABI_VERSION; }

const char *ssm_status_string(ssm_status s) {
    switch (s) {
        case SSM_OK: return "ok";
        case SSM_ERR_INVALID_ARG: return "invalid argument";
        case SSM_ERR_UNSUPPORTED: return "unsupported configuration";
        case SSM_ERR_ALIGNMENT: return "misaligned pointer";
        case SSM_ERR_WORKSPACE: return "workspace missing or too small";
        case SSM_ERR_CUDA: return "CUDA error";
        case SSM_ERR_DEVICE: return "device-side validation failed";
    }
    return "unknown status";
}

int32_t ssm_last_cuda_error(void) { return g_last_cuda_error; }

ssm_status ssm_conv1d_fwd(const ssm_conv_args *args, void *stream) {
    SSM_TRY(validate_conv(args));
    if (args->batch == 0 || (args->seqlen == 0 && !args->state_out)) return SSM_OK;
    return cuda_status(ssm::launch_conv1d(*args, (cudaStream_t)stream));
}

namespace {
struct WsPlan {
    size_t order_off, bc_off, total;
    bool ssd;
};
// The workspace depends on shapes only (a call whose pointers rule out the
// tensor-core path still finds its error word and schedule in the same place).
WsPlan plan_workspace(const ssm_scan_args *a) {
    WsPlan p{0, 0, 0, false};
    const bool ssd_shape = ssm::ssd_shape_ok(*a);
    p.ssd = ssd_shape && ssm::ssd_supported(*a);
    size_t off = 0;
    if (a->cu_seqlens || ssd_shape) off = ssm::kWsOrderOffset;      // error word
    if (a->cu_seqlens) {
        p.order_off = off;
        off += ssm::order_bytes(a->nseqs);
    }
    if (ssd_shape) {
        p.bc_off = off;
        off += ssm::ssd_workspace_bytes(*a);
    }
    p.total = off;
    return p;
}
}  // namespace

namespace {
// The backward validates its forward description with y standing in as dy
// (same shape, strides and dtype), then its own outputs.
ssm_status validate_bwd(const ssm_scan_bwd_args *b) {
    if (!b) return SSM_ERR_INVALID_ARG;
    ssm_scan_args f = b->fwd;
    f.y = const_cast<void *>(b->dy);
    f.y_batch_stride = b->dy_batch_stride;
    f.y_token_stride = b->dy_token_stride;
    f.state_interval = 0;
    SSM_TRY(validate_scan(&f));
    if (!b->dx || !b->ddt || !b->dB || !b->dC || !b->dA || !b->dh0) return SSM_ERR_INVALID_ARG;
    if (f.z && !b->dz) return SSM_ERR_INVALID_ARG;
    const float *outs[] = {b->dx, b->dz, b->ddt, b->dB, b->dC, b->dA, b->dD, b->ddt_bias, b->dh0,
                           b->dconv_w, b->dconv_b, b->dconv_state_in, b->dh_final};
    for (const float *o : outs)
        if (!aligned(o, 4)) return SSM_ERR_ALIGNMENT;
    if (!aligned(b->dconv_state_out, esize(f.dtype))) return SSM_ERR_ALIGNMENT;
    return SSM_OK;
}
size_t bwd_ws_prefix(const ssm_scan_args &f) {
    return ssm::kWsOrderOffset + (f.cu_seqlens ? ssm::order_bytes(f.nseqs) : 0);
}
}  // namespace

size_t ssm_scan_bwd_workspace_size(const ssm_scan_bwd_args *args) {
    if (!args) return 0;
    const ssm_scan_args &f = args->fwd;
    if (f.batch < 0 || f.seqlen < 0 || f.nseqs < 0 || f.ngroups < 0 || f.dstate < 1 || f.d_inner < 1) return 0;
    return bwd_ws_prefix(f) + ssm::scan_bwd_workspace_bytes(*args);
}

ssm_status ssm_scan_bwd(const ssm_scan_bwd_args *args, void *workspace, size_t ws_bytes, void *stream) {
    SSM_TRY(validate_bwd(args));
    const ssm_scan_args &f = args->fwd;
    const cudaStream_t st = (cudaStream_t)stream;
    const size_t need = bwd_ws_prefix(f) + ssm::scan_bwd_workspace_bytes(*args);
    char *ws = static_cast<char *>(workspace);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return SSM_ERR_WORKSPACE;
    ssm::SeqView sv{nullptr, nullptr, reinterpret_cast<int32_t *>(ws + ssm::kWsErrorOffset), (int)f.batch};
    if (f.cu_seqlens) {
        sv.cu = f.cu_seqlens;
        sv.nseqs = f.nseqs;
        // validates cu_seqlens into the error word (the schedule it also writes is not used here)
        SSM_TRY(cuda_status(ssm::launch_varlen_plan(f.cu_seqlens, f.nseqs, f.seqlen, sv.err,
                                                    reinterpret_cast<int32_t *>(ws + ssm::kWsOrderOffset), st)));
    } else {
        SSM_TRY(cuda_status(cudaMemsetAsync(sv.err, 0, sizeof(int32_t), st)));
    }
    return cuda_status(ssm::launch_scan_bwd(*args, sv, ws + bwd_ws_prefix(f), st));
}

size_t ssm_scan_workspace_size(const ssm_scan_args *args) {
    if (!args || args->batch < 0 || args->seqlen < 0 || args->nseqs < 0 || args->ngroups < 0 || args->dstate < 0 ||
        args->segments < 0)
        return 0;
    return plan_workspace(args).total;
}

int64_t ssm_scan_segments(const ssm_scan_args *args) {
    if (validate_scan(args) != SSM_OK) return 0;
    if (args->mode != SSM_MAMBA2 || !plan_workspace(args).ssd) return 1;
    return ssm::ssd_segments(*args);
}

ssm_status ssm_scan_fwd(const ssm_scan_args *args, void *workspace, size_t ws_bytes, void *stream) {
    SSM_TRY(validate_scan(args));
    const cudaStream_t st = (cudaStream_t)stream;
    ssm::SeqView sv{nullptr, nullptr, nullptr, (int)args->batch};
    const WsPlan plan = plan_workspace(args);
    char *ws = static_cast<char *>(workspace);
    if (plan.total > 0) {
        if (!workspace || ws_bytes < plan.total || !aligned(workspace, 256)) return SSM_ERR_WORKSPACE;
        sv.err = reinterpret_cast<int32_t *>(ws + ssm::kWsErrorOffset);
    }
    if (args->cu_seqlens) {
        sv.cu = args->cu_seqlens;
        sv.order = reinterpret_cast<int32_t *>(ws + plan.order_off);
        sv.nseqs = args->nseqs;
        SSM_TRY(cuda_status(ssm::launch_varlen_plan(args->cu_seqlens, args->nseqs, args->seqlen, sv.err,
                                                    const_cast<int32_t *>(sv.order), st)));
    } else if (sv.err) {
        SSM_TRY(cuda_status(cudaMemsetAsync(sv.err, 0, sizeof(int32_t), st)));
    }
    if (args->mode == SSM_MAMBA1) return cuda_status(ssm::launch_scan_m1(*args, sv, st));
    if (plan.ssd) return cuda_status(ssm::launch_ssd(*args, sv, ws + plan.bc_off, st));
    return cuda_status(ssm::launch_scan_m2_simt(*args, sv, st));
}

ssm_status ssm_state_update(const ssm_update_args *args, void *stream) {
    SSM_TRY(validate_update(args));
    return cuda_status(ssm::launch_state_update(*args, (cudaStream_t)stream));
}

namespace {
// The split entry points take the segment's ssm_scan_fwd description: batch
// mode only, and token counts the fix-up grids can tile.
ssm_status validate_split_scan(const ssm_scan_args *a) {
    SSM_TRY(validate_scan(a));
    if (a->cu_seqlens) return SSM_ERR_UNSUPPORTED;
    if (a->seqlen > ssm::kMaxSplitSeqlen) return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}
}  // namespace

ssm_status ssm_split_conv_tail(const ssm_scan_args *args, void *tail, void *stream) {
    SSM_TRY(validate_split_scan(args));
    if (args->d_conv < 2 || !tail) return SSM_ERR_INVALID_ARG;
    if (!aligned(tail, esize(args->dtype))) return SSM_ERR_ALIGNMENT;
    return cuda_status(ssm::launch_split_tail(*args, tail, (cudaStream_t)stream));
}

ssm_status ssm_split_cum_delta(const ssm_scan_args *args, float *cum_delta, float *sum_delta, void *stream) {
    SSM_TRY(validate_split_scan(args));
    if (!sum_delta) return SSM_ERR_INVALID_ARG;
    if (!aligned(cum_delta, 4) || !aligned(sum_delta, 4)) return SSM_ERR_ALIGNMENT;
    return cuda_status(ssm::launch_split_cum_delta(*args, cum_delta, sum_delta, (cudaStream_t)stream));
}

ssm_status ssm_split_combine(const ssm_split_args *a, void *stream) {
    if (!a) return SSM_ERR_INVALID_ARG;
    if (a->mode != SSM_MAMBA1 && a->mode != SSM_MAMBA2) return SSM_ERR_INVALID_ARG;
    if (a->nranks < 1 || a->rank < 0 || a->rank >= a->nranks) return SSM_ERR_INVALID_ARG;
    if (a->batch < 0 || a->d_inner < 1 || a->dstate < 1) return SSM_ERR_INVALID_ARG;
    if (a->mode == SSM_MAMBA2 &&
        (a->nheads < 1 || a->headdim < 1 || a->nheads * a->headdim != a->d_inner))
        return SSM_ERR_INVALID_ARG;
    if (!a->A || !a->sum_delta || !a->h_local) return SSM_ERR_INVALID_ARG;
    if (!aligned(a->A, 4) || !aligned(a->sum_delta, 4) || !aligned(a->h_local, 4) || !aligned(a->h_in, 4) ||
        !aligned(a->h_out, 4))
        return SSM_ERR_ALIGNMENT;
    const int64_t U = a->mode == SSM_MAMBA2 ? a->nheads : a->d_inner;
    const int64_t S = a->d_inner * a->dstate;
    if (a->sum_delta_rank_stride < 0 || (a->sum_delta_rank_stride > 0 && a->sum_delta_rank_stride < a->batch * U) ||
        a->h_local_rank_stride < 0 || (a->h_local_rank_stride > 0 && a->h_local_rank_stride < a->batch * S) ||
        a->sum_delta_rank_stride % 4 != 0 || a->h_local_rank_stride % 4 != 0)
        return SSM_ERR_INVALID_ARG;
    if (S > INT32_MAX || a->batch > 65535) return SSM_ERR_UNSUPPORTED;   // 32-bit indices in the kernel
    return cuda_status(ssm::launch_split_combine(*a, (cudaStream_t)stream));
}

ssm_status ssm_split_fixup(const ssm_scan_args *args, const float *cum_delta, const float *h_in, void *stream) {
    SSM_TRY(validate_split_scan(args));
    if (args->batch == 0 || args->seqlen == 0) return SSM_OK;   // a segment with no tokens has no y to fix
    if (!cum_delta || !h_in) return SSM_ERR_INVALID_ARG;
    if (!aligned(cum_delta, 4) || !aligned(h_in, 4)) return SSM_ERR_ALIGNMENT;
    return cuda_status(ssm::launch_split_fixup(*args, cum_delta, h_in, (cudaStream_t)stream));
}

int32_t ssm_check_bounds_enabled(void) {
#ifdef SSM_CHECK_BOUNDS
    return 1;
#else
    return 0;
#endif
}

ssm_status ssm_bounds_record(int32_t *code, int32_t *site, int64_t *index, int64_t *extent, int32_t clear) {
#ifdef SSM_CHECK_BOUNDS
    SSM_TRY(cuda_status(cudaDeviceSynchronize()));
    ssm::BoundsRecord r{};
    SSM_TRY(cuda_status(cudaMemcpyFromSymbol(&r, ssm::g_ssm_bounds, sizeof(r))));
    if (code) *code = r.code;
    if (site) *site = r.site;
    if (index) *index = r.index;
    if (extent) *extent = r.extent;
    if (clear) {
        const ssm::BoundsRecord z{};
        SSM_TRY(cuda_status(cudaMemcpyToSymbol(ssm::g_ssm_bounds, &z, sizeof(z))));
    }
    return SSM_OK;
#else
    (void)code; (void)site; (void)index; (void)extent; (void)clear;
    return SSM_ERR_UNSUPPORTED;
#endif
}

ssm_status ssm_workspace_error(const void *workspace, int32_t *code, void *stream) {
    if (!workspace) return SSM_ERR_INVALID_ARG;
    SSM_TRY(cuda_status(cudaStreamSynchronize((cudaStream_t)stream)));
    int32_t v = 0;
    SSM_TRY(cuda_status(cudaMemcpy(&v, static_cast<const char *>(workspace) + ssm::kWsErrorOffset, sizeof(v),
                                   cudaMemcpyDeviceToHost)));
    if (code) *code = v;
    return v == SSM_DEVERR_NONE ? SSM_OK : SSM_ERR_DEVICE;
}

}  // extern "C"
