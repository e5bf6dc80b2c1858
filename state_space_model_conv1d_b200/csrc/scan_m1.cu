// scan_m1.cu -- Mamba-1 selective scan (diagonal A[d, n]) with the causal conv
// + SiLU fused into its prologue.
//
//   delta = softplus(dt + dt_bias)
//   h_t[d, n] = exp(delta_t[d] A[d, n]) h_{t-1}[d, n] + delta_t[d] B_t[n] xc_t[d]
//   y_t[d] = (sum_n C_t[n] h_t[d, n] + D[d] xc_t[d]) * silu(z_t[d])
// with h_0 = h0 and xc the conv output ("Adding Initial Value Support to
// Selective Scan Forward Kernel", state-spaces/mamba issue 285: the step and
// the (exp(delta*A), h) pair seeded with (1, h0); llama.cpp issue 6758:
// GGML_OP_SSM_CONV / GGML_OP_SSM_SCAN shapes, final state returned).
//
// Design (sm_100a, SIMT): one CTA owns one sequence and DB = 32 channels and
// walks the tokens in chunks of TC.  Per chunk the raw x / dt / z / B / C rows
// are staged in shared memory (16-byte vector loads, 64-byte rows per
// tensor), a cooperative prologue computes conv + SiLU, delta, delta*x and the
// gate once per (token, channel), then 4 lanes per channel each advance
// N/4 states held in registers.  The carry across chunks is simply the fp32
// state staying in registers, seeded from h0 -- the (1, h0) seed of the pair
// scan.  The K-1 raw rows before each chunk sit in a shared halo that also
// becomes conv_state_out.  Every input element crosses HBM once.
//
// The per-(token, channel, state) work is one exp on the MUFU pipe plus four
// FP32 ops; with dstate 16 this kernel is bound by the MUFU exp rate, not HBM.
#include "common.cuh"
#include "launch.h"
#include "tile_io.cuh"

namespace ssm {
namespace {

constexpr int kDB = 32;             // channels per CTA
constexpr int kLanes = 4;           // lanes per channel
constexpr int kThreads = kDB * kLanes;
constexpr int kTC = 64;             // tokens per chunk
constexpr int kHalo = kMaxConvWidth - 1;

struct M1Args {
    const void *x, *z, *dt, *B, *C;
    void *y;
    int64_t x_bs, x_ts, z_bs, z_ts, dt_bs, dt_ts, B_bs, B_ts, C_bs, C_ts, y_bs, y_ts;
    const float *A, *D, *dt_bias, *h0, *conv_w, *conv_b;
    float *h_final;
    const void *conv_state_in;
    void *conv_state_out;
    int64_t Dn, N, seqlen;
    int K, softplus;
    bool vec_x, vec_z, vec_dt, vec_B, vec_C, vec_y;
    SeqView sv;
};

template <int SPT>
struct SmemM1 {
    static constexpr int NP = kLanes * SPT;             // padded dstate
    float xraw[kHalo + kTC][kDB];
    float dl[kTC][kDB];       // dt, then delta
    float zg[kTC][kDB];       // z, then the gate silu(z)
    float xc[kTC][kDB];       // conv output, then y
    float dx[kTC][kDB];       // delta * xc
    float Bs[kTC][NP];
    float Cs[kTC][NP];
};

template <typename T, int SPT>
__global__ void __launch_bounds__(kThreads)
scan_m1_kernel(const M1Args a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<SmemM1<SPT> *>(smem_raw);
    constexpr int NP = SmemM1<SPT>::NP;
    constexpr int VW = SPT < 4 ? SPT : 4;     // states per shared-memory vector
    constexpr int NJ = SPT / VW;

    if (a.sv.err && *a.sv.err != 0) return;
    const int tid = threadIdx.x;
    const int64_t d0 = (int64_t)blockIdx.x * kDB;
    const int si = blockIdx.y;
    const int s = a.sv.order ? a.sv.order[si] : si;
    int64_t start = 0, len = a.seqlen, row = s;
    if (a.sv.cu) {
        const int64_t c0 = min(max((int64_t)a.sv.cu[s], (int64_t)0), a.seqlen);
        const int64_t c1 = min(max((int64_t)a.sv.cu[s + 1], c0), a.seqlen);
        start = c0; len = c1 - c0; row = 0;
    }
    const T *xg = static_cast<const T *>(a.x) + row * a.x_bs + start * a.x_ts;
    const T *dtg = static_cast<const T *>(a.dt) + row * a.dt_bs + start * a.dt_ts;
    const T *zg = a.z ? static_cast<const T *>(a.z) + row * a.z_bs + start * a.z_ts : nullptr;
    const T *Bg = static_cast<const T *>(a.B) + row * a.B_bs + start * a.B_ts;
    const T *Cg = static_cast<const T *>(a.C) + row * a.C_bs + start * a.C_ts;
    T *yg = static_cast<T *>(a.y) + row * a.y_bs + start * a.y_ts;
    const int K = a.K;
    const int64_t Dn = a.Dn, N = a.N;

    // ---- prologue-role constants: channel pd = tid % 32, tokens tid/32 + 4i
    const int pd = tid % kDB;
    const int64_t pch = d0 + pd;
    const bool pvalid = pch < Dn;
    float cw[kMaxConvWidth], cb = 0.f, dtb = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxConvWidth; ++k) cw[k] = (pvalid && k < K) ? a.conv_w[pch * K + k] : 0.f;
    if (pvalid && a.conv_b) cb = a.conv_b[pch];
    if (pvalid && a.dt_bias) dtb = a.dt_bias[pch];

    // ---- scan-role constants: channel sd = tid / 4, lane q = tid % 4
    const int sd = tid / kLanes, q = tid % kLanes;
    const int64_t sch = d0 + sd;
    const bool svalid = sch < Dn;
    float A2[SPT], h[SPT];
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
        for (int e = 0; e < VW; ++e) {
            const int64_t n = (int64_t)VW * (q + kLanes * j) + e;
            const bool ok = svalid && n < N;
            A2[j * VW + e] = ok ? a.A[sch * N + n] * kLog2e : 0.f;
            h[j * VW + e] = (ok && a.h0) ? a.h0[((int64_t)s * Dn + sch) * N + n] : 0.f;
        }
    const float Dd = (svalid && a.D) ? a.D[sch] : 0.f;

    // ---- conv halo: the K-1 raw inputs before the first token
    if (K > 1) {
        const T *csi = static_cast<const T *>(a.conv_state_in);
        for (int idx = tid; idx < (K - 1) * kDB; idx += kThreads) {
            const int j = idx / kDB, d = idx % kDB;
            const int64_t ch = d0 + d;
            sm.xraw[kHalo - (K - 1) + j][d] =
                (csi && ch < Dn) ? Elem<T>::ld(csi + ((int64_t)s * Dn + ch) * (K - 1) + j) : 0.f;
        }
    }

    const int ncols = (int)min((int64_t)kDB, Dn - d0);
    for (int64_t t0 = 0; t0 < len || t0 == 0; t0 += kTC) {
        const int nv = (int)min((int64_t)kTC, len - t0);    // may be 0 for an empty sequence
        if (nv > 0) {
            load_tile_f32<T, kThreads>(&sm.xraw[kHalo][0], kDB, xg + t0 * a.x_ts, a.x_ts, kTC, nv, d0, kDB, Dn, a.vec_x);
            load_tile_f32<T, kThreads>(&sm.dl[0][0], kDB, dtg + t0 * a.dt_ts, a.dt_ts, kTC, nv, d0, kDB, Dn, a.vec_dt);
            if (zg) load_tile_f32<T, kThreads>(&sm.zg[0][0], kDB, zg + t0 * a.z_ts, a.z_ts, kTC, nv, d0, kDB, Dn, a.vec_z);
            load_tile_f32<T, kThreads>(&sm.Bs[0][0], NP, Bg + t0 * a.B_ts, a.B_ts, kTC, nv, 0, NP, N, a.vec_B);
            load_tile_f32<T, kThreads>(&sm.Cs[0][0], NP, Cg + t0 * a.C_ts, a.C_ts, kTC, nv, 0, NP, N, a.vec_C);
        }
        __syncthreads();
        if (nv > 0) {
            // prologue: conv + SiLU, delta, delta * xc, gate -- once per (token, channel)
            for (int t = tid / kDB; t < kTC; t += kThreads / kDB) {
                float xcv = 0.f, dlt = 0.f, g = 1.f;
                if (t < nv && pvalid) {
                    if (K > 0) {
                        float acc = cb;
#pragma unroll
                        for (int k = 0; k < kMaxConvWidth; ++k)
                            if (k < K) acc = fmaf(cw[k], sm.xraw[kHalo + t - (K - 1) + k][pd], acc);
                        xcv = silu(acc);
                    } else {
                        xcv = sm.xraw[kHalo + t][pd];
                    }
                    const float u = sm.dl[t][pd] + dtb;
                    dlt = a.softplus ? softplus(u) : u;
                    if (zg) g = silu(sm.zg[t][pd]);
                }
                sm.xc[t][pd] = xcv;
                sm.dl[t][pd] = dlt;             // delta = 0 past the end: the state stays put
                sm.dx[t][pd] = dlt * xcv;
                sm.zg[t][pd] = g;
            }
        }
        __syncthreads();
        if (nv > 0) {
            // recurrence: 4 lanes per channel, SPT states each, sequential over tokens
            for (int t = 0; t < kTC; ++t) {
                const float dl = sm.dl[t][sd], dxv = sm.dx[t][sd];
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    float bv[VW], cv[VW];
                    const int n0 = VW * (q + kLanes * j);
                    if constexpr (VW == 4) {
                        const float4 b4 = *reinterpret_cast<const float4 *>(&sm.Bs[t][n0]);
                        const float4 c4 = *reinterpret_cast<const float4 *>(&sm.Cs[t][n0]);
                        bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
                        cv[0] = c4.x; cv[1] = c4.y; cv[2] = c4.z; cv[3] = c4.w;
                    } else if constexpr (VW == 2) {
                        const float2 b2 = *reinterpret_cast<const float2 *>(&sm.Bs[t][n0]);
                        const float2 c2 = *reinterpret_cast<const float2 *>(&sm.Cs[t][n0]);
                        bv[0] = b2.x; bv[1] = b2.y; cv[0] = c2.x; cv[1] = c2.y;
                    } else {
                        bv[0] = sm.Bs[t][n0]; cv[0] = sm.Cs[t][n0];
                    }
#pragma unroll
                    for (int e = 0; e < VW; ++e) {
                        const float dA = ex2(dl * A2[j * VW + e]);
                        h[j * VW + e] = fmaf(dA, h[j * VW + e], dxv * bv[e]);
                        acc = fmaf(cv[e], h[j * VW + e], acc);
                    }
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (q == 0) sm.xc[t][sd] = (acc + Dd * sm.xc[t][sd]) * sm.zg[t][sd];
            }
        }
        __syncthreads();
        if (nv > 0) {
            store_tile_f32<T, kThreads>(yg + t0 * a.y_ts, a.y_ts, &sm.xc[0][0], kDB, nv, d0, ncols, Dn, a.vec_y);
            // slide the conv halo: the last K-1 raw rows (halo rows included when nv < K-1)
            if (K > 1 && nv == kTC) {
                constexpr int kRowsPerPass = kThreads / kDB;
                constexpr int kPasses = (kHalo + kRowsPerPass - 1) / kRowsPerPass;
                float keep[kPasses];
                const int d = tid % kDB;
#pragma unroll
                for (int i = 0; i < kPasses; ++i) {
                    const int j = tid / kDB + i * kRowsPerPass;
                    if (j < K - 1) keep[i] = sm.xraw[kHalo + kTC - (K - 1) + j][d];
                }
                __syncthreads();
#pragma unroll
                for (int i = 0; i < kPasses; ++i) {
                    const int j = tid / kDB + i * kRowsPerPass;
                    if (j < K - 1) sm.xraw[kHalo - (K - 1) + j][d] = keep[i];
                }
            }
        }
        __syncthreads();
        if (nv < kTC) {
            // final chunk: the halo-relative window of the last K-1 raw inputs
            if (K > 1 && a.conv_state_out) {
                T *cso = static_cast<T *>(a.conv_state_out);
                for (int idx = tid; idx < (K - 1) * kDB; idx += kThreads) {
                    const int j = idx / kDB, d = idx % kDB;
                    const int64_t ch = d0 + d;
                    if (ch < Dn)
                        Elem<T>::st(cso + ((int64_t)s * Dn + ch) * (K - 1) + j, sm.xraw[kHalo + nv - (K - 1) + j][d]);
                }
            }
            break;
        }
        if (t0 + kTC == len) {
            // the sequence ended exactly on a chunk boundary: halo already slid
            if (K > 1 && a.conv_state_out) {
                T *cso = static_cast<T *>(a.conv_state_out);
                for (int idx = tid; idx < (K - 1) * kDB; idx += kThreads) {
                    const int j = idx / kDB, d = idx % kDB;
                    const int64_t ch = d0 + d;
                    if (ch < Dn)
                        Elem<T>::st(cso + ((int64_t)s * Dn + ch) * (K - 1) + j, sm.xraw[kHalo - (K - 1) + j][d]);
                }
            }
            break;
        }
    }
    if (a.h_final && svalid) {
#pragma unroll
        for (int j = 0; j < NJ; ++j)
#pragma unroll
            for (int e = 0; e < VW; ++e) {
                const int64_t n = (int64_t)VW * (q + kLanes * j) + e;
                if (n < N) a.h_final[((int64_t)s * Dn + sch) * N + n] = h[j * VW + e];
            }
    }
}

template <typename T, int SPT>
cudaError_t launch_spt(const M1Args &a, int nseqs, cudaStream_t st) {
    const size_t smem = sizeof(SmemM1<SPT>);
    auto kern = scan_m1_kernel<T, SPT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.Dn + kDB - 1) / kDB), (unsigned)nseqs);
    kern<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const M1Args &a, int nseqs, cudaStream_t st) {
    if (a.N <= 4) return launch_spt<T, 1>(a, nseqs, st);
    if (a.N <= 8) return launch_spt<T, 2>(a, nseqs, st);
    if (a.N <= 16) return launch_spt<T, 4>(a, nseqs, st);
    if (a.N <= 32) return launch_spt<T, 8>(a, nseqs, st);
    return launch_spt<T, 16>(a, nseqs, st);
}

inline bool vec_ok(const void *p, int64_t bs, int64_t ts, size_t es) {
    return p == nullptr || ((uintptr_t)p % 16 == 0 && (bs * (int64_t)es) % 16 == 0 && (ts * (int64_t)es) % 16 == 0);
}

}  // namespace

cudaError_t launch_scan_m1(const ssm_scan_args &s, const SeqView &sv, cudaStream_t st) {
    M1Args a;
    a.x = s.x; a.z = s.z; a.dt = s.dt; a.B = s.B; a.C = s.C; a.y = s.y;
    a.x_bs = s.x_batch_stride; a.x_ts = s.x_token_stride;
    a.z_bs = s.z_batch_stride; a.z_ts = s.z_token_stride;
    a.dt_bs = s.dt_batch_stride; a.dt_ts = s.dt_token_stride;
    a.B_bs = s.B_batch_stride; a.B_ts = s.B_token_stride;
    a.C_bs = s.C_batch_stride; a.C_ts = s.C_token_stride;
    a.y_bs = s.y_batch_stride; a.y_ts = s.y_token_stride;
    a.A = s.A; a.D = s.D; a.dt_bias = s.dt_bias; a.h0 = s.h0; a.h_final = s.h_final;
    a.conv_w = s.conv_w; a.conv_b = s.conv_b; a.conv_state_in = s.conv_state_in; a.conv_state_out = s.conv_state_out;
    a.Dn = s.d_inner; a.N = s.dstate; a.seqlen = s.seqlen;
    a.K = (int)s.d_conv; a.softplus = s.delta_softplus;
    const size_t es = s.dtype == SSM_BF16 ? 2 : 4;
    a.vec_x = vec_ok(s.x, s.x_batch_stride, s.x_token_stride, es) && s.d_inner % 8 == 0;
    a.vec_z = vec_ok(s.z, s.z_batch_stride, s.z_token_stride, es) && s.d_inner % 8 == 0;
    a.vec_dt = vec_ok(s.dt, s.dt_batch_stride, s.dt_token_stride, es) && s.d_inner % 8 == 0;
    a.vec_y = vec_ok(s.y, s.y_batch_stride, s.y_token_stride, es) && s.d_inner % 8 == 0;
    a.vec_B = vec_ok(s.B, s.B_batch_stride, s.B_token_stride, es);
    a.vec_C = vec_ok(s.C, s.C_batch_stride, s.C_token_stride, es);
    a.sv = sv;
    const int nseqs = s.cu_seqlens ? s.nseqs : (int)s.batch;
    if (nseqs == 0) return cudaSuccess;
    return s.dtype == SSM_BF16 ? launch_typed<__nv_bfloat16>(a, nseqs, st) : launch_typed<float>(a, nseqs, st);
}

}  // namespace ssm
