// scan_m2_simt.cu -- Mamba-2 selective scan (scalar A per head, B/C shared by
// contiguous groups of heads) with the causal conv over x | B | C fused in
// front, evaluated as the token-sequential recurrence on CUDA cores.
//
//   delta_t[h] = softplus(dt_t[h] + dt_bias[h]),  a_t[h] = exp(delta_t[h] A[h])
//   S_t[h, p, n] = a_t[h] S_{t-1}[h, p, n] + delta_t[h] x_t[h, p] B_t[g(h), n]
//   y_t[h, p] = (sum_n C_t[g(h), n] S_t[h, p, n] + D[h] x_t[h, p]) * silu(z_t[h, p])
// with g(h) = h / (H / G) ("Tensor-parallel SSM", Fast-LLM PR 333: groups of
// heads as contiguous repeat_interleave blocks) and S_0 = h0 ("Adding Initial
// Value Support to Selective Scan Forward Kernel", state-spaces/mamba issue
// 285: the (1, h0) seed of the running prefix).
//
// One CTA owns (sequence, head, 32 channels of the head) and walks tokens in
// chunks of TC.  Per chunk the raw x / B / C rows (with a K-1 row halo), dt and
// z are staged in shared memory; a cooperative prologue runs the conv + SiLU
// over the x channels of this block and the B / C channels of its group, and
// computes delta and the decay once per token; then 8 lanes per channel
// advance N/8 states each in registers.  This path serves every shape the
// tensor-core SSD kernel does not take (odd dstate / headdim, fp32 inputs,
// short sequences) and is the reference point for it.
#include "common.cuh"
#include "launch.h"
#include "tile_io.cuh"

namespace ssm {
namespace {

constexpr int kPB = 32;            // channels (p) per CTA
constexpr int kLanes = 8;          // lanes per channel
constexpr int kThreads = kPB * kLanes;
constexpr int kTC = 32;            // tokens per chunk
constexpr int kHalo = kMaxConvWidth - 1;

struct M2Args {
    const void *x, *z, *dt, *B, *C;
    void *y;
    int64_t x_bs, x_ts, z_bs, z_ts, dt_bs, dt_ts, B_bs, B_ts, C_bs, C_ts, y_bs, y_ts;
    const float *A, *D, *dt_bias, *h0, *conv_w, *conv_b;
    float *h_final;
    const void *conv_state_in;
    void *conv_state_out;
    int64_t H, P, G, N, seqlen;
    int K, softplus, npb;
    bool vec_x, vec_z, vec_B, vec_C, vec_y;
    SeqView sv;
    InterView iv;
};

template <int SPT>
struct SmemM2 {
    static constexpr int NP = kLanes * SPT;
    float xraw[kHalo + kTC][kPB];
    float braw[kHalo + kTC][NP];
    float craw[kHalo + kTC][NP];
    float xc[kTC][kPB];           // conv(x), then y
    float zg[kTC][kPB];           // z, then gate
    float Bc[kTC][NP];
    float Cc[kTC][NP];
    float dl[kTC];                // delta
    float da[kTC];                // exp(delta * A)
};

// Conv + SiLU of one channel column of a raw tile (halo rows included).
SSM_DEVINL float conv_col(const float *raw, int ld, int t, int col, const float *w, float b, int K) {
    float acc = b;
#pragma unroll
    for (int k = 0; k < kMaxConvWidth; ++k)
        if (k < K) acc = fmaf(w[k], raw[(kHalo + t - (K - 1) + k) * ld + col], acc);
    return silu(acc);
}

template <typename T, int SPT>
__global__ void __launch_bounds__(kThreads)
scan_m2_simt_kernel(const M2Args a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<SmemM2<SPT> *>(smem_raw);
    constexpr int NP = SmemM2<SPT>::NP;
    constexpr int VW = SPT < 4 ? SPT : 4;
    constexpr int NJ = SPT / VW;

    if (a.sv.err && *a.sv.err != 0) return;
    const int tid = threadIdx.x;
    const int64_t H = a.H, P = a.P, G = a.G, N = a.N, Dn = H * P;
    const int hh = blockIdx.x / a.npb, pb = blockIdx.x % a.npb;
    const int64_t g = hh / (H / G);
    const int64_t p0 = (int64_t)pb * kPB;
    const int si = blockIdx.y;
    const int s = a.sv.order ? a.sv.order[si] : si;
    int64_t start = 0, len = a.seqlen, row = s;
    if (a.sv.cu) {
        const int64_t c0 = min(max((int64_t)a.sv.cu[s], (int64_t)0), a.seqlen);
        const int64_t c1 = min(max((int64_t)a.sv.cu[s + 1], c0), a.seqlen);
        start = c0; len = c1 - c0; row = 0;
    }
    const int K = a.K;
    const int64_t cdim = Dn + 2 * G * N;
    const T *xg = static_cast<const T *>(a.x) + row * a.x_bs + start * a.x_ts + hh * P;
    const T *dtg = static_cast<const T *>(a.dt) + row * a.dt_bs + start * a.dt_ts + hh;
    const T *zg = a.z ? static_cast<const T *>(a.z) + row * a.z_bs + start * a.z_ts + hh * P : nullptr;
    const T *Bg = static_cast<const T *>(a.B) + row * a.B_bs + start * a.B_ts + g * N;
    const T *Cg = static_cast<const T *>(a.C) + row * a.C_bs + start * a.C_ts + g * N;
    T *yg = static_cast<T *>(a.y) + row * a.y_bs + start * a.y_ts + hh * P;
    // bounds-checked build: the CTA's ranges (uniform, so the whole CTA returns together)
    if (!SSM_BOUNDS(len > 0 ? start + len - 1 : 0, a.seqlen > 0 ? a.seqlen : 1, BS_M2S_SEQ) ||
        !SSM_BOUNDS((int64_t)hh * P + p0, Dn, BS_M2S_HEAD) || !SSM_BOUNDS(s, a.sv.nseqs, BS_M2S_STATE))
        return;
    const int ncols = (int)min((int64_t)kPB, P - p0);
    // conv channel indices of this block's x columns and of the group's B / C
    const int64_t xch0 = hh * P + p0, bch0 = Dn + g * N, cch0 = Dn + G * N + g * N;

    // scan role: channel sp = tid / 8, lane q = tid % 8
    const int sp = tid / kLanes, q = tid % kLanes;
    const int64_t pch = p0 + sp;
    const bool svalid = pch < P;
    float h[SPT];
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
        for (int e = 0; e < VW; ++e) {
            const int64_t n = (int64_t)VW * (q + kLanes * j) + e;
            h[j * VW + e] = (svalid && n < N && a.h0) ? a.h0[(((int64_t)s * H + hh) * P + pch) * N + n] : 0.f;
        }
    const float A2 = a.A[hh] * kLog2e;
    const float Dh = a.D ? a.D[hh] : 0.f;
    const float dtb = a.dt_bias ? a.dt_bias[hh] : 0.f;

    // conv halo (x columns of this block, B / C of the group)
    if (K > 1) {
        const T *csi = static_cast<const T *>(a.conv_state_in);
        for (int idx = tid; idx < (K - 1) * (kPB + 2 * NP); idx += kThreads) {
            const int j = idx % (K - 1), c = idx / (K - 1);
            float v = 0.f;
            int64_t ch;
            float *dst;
            if (c < kPB) { ch = (p0 + c < P) ? xch0 + c : -1; dst = &sm.xraw[kHalo - (K - 1) + j][c]; }
            else if (c < kPB + NP) { const int n = c - kPB; ch = n < N ? bch0 + n : -1; dst = &sm.braw[kHalo - (K - 1) + j][n]; }
            else { const int n = c - kPB - NP; ch = n < N ? cch0 + n : -1; dst = &sm.craw[kHalo - (K - 1) + j][n]; }
            if (csi && ch >= 0) v = Elem<T>::ld(csi + ((int64_t)s * cdim + ch) * (K - 1) + j);
            *dst = v;
        }
    }

    for (int64_t t0 = 0; t0 < len || t0 == 0; t0 += kTC) {
        const int nv = (int)min((int64_t)kTC, len - t0);
        if (nv > 0) {
            load_tile_f32<T, kThreads>(&sm.xraw[kHalo][0], kPB, xg + t0 * a.x_ts, a.x_ts, kTC, nv, p0, kPB, P, a.vec_x);
            load_tile_f32<T, kThreads>(&sm.braw[kHalo][0], NP, Bg + t0 * a.B_ts, a.B_ts, kTC, nv, 0, NP, N, a.vec_B);
            load_tile_f32<T, kThreads>(&sm.craw[kHalo][0], NP, Cg + t0 * a.C_ts, a.C_ts, kTC, nv, 0, NP, N, a.vec_C);
            if (zg) load_tile_f32<T, kThreads>(&sm.zg[0][0], kPB, zg + t0 * a.z_ts, a.z_ts, kTC, nv, p0, kPB, P, a.vec_z);
            for (int t = tid; t < kTC; t += kThreads) sm.dl[t] = t < nv ? Elem<T>::ld(dtg + (t0 + t) * a.dt_ts) : 0.f;
        }
        __syncthreads();
        if (nv > 0) {
            for (int t = tid; t < kTC; t += kThreads) {
                float dlt = 0.f;
                if (t < nv) {
                    const float u = sm.dl[t] + dtb;
                    dlt = a.softplus ? softplus(u) : u;
                }
                sm.dl[t] = dlt;                   // 0 past the end: decay 1, no input
                sm.da[t] = ex2(dlt * A2);
            }
            for (int idx = tid; idx < kTC * kPB; idx += kThreads) {
                const int t = idx / kPB, c = idx % kPB;
                float v = 0.f, gte = 1.f;
                if (t < nv && p0 + c < P) {
                    if (K > 0) {
                        float w[kMaxConvWidth];
                        for (int k = 0; k < K; ++k) w[k] = a.conv_w[(xch0 + c) * K + k];
                        v = conv_col(&sm.xraw[0][0], kPB, t, c, w, a.conv_b ? a.conv_b[xch0 + c] : 0.f, K);
                    } else {
                        v = sm.xraw[kHalo + t][c];
                    }
                    if (zg) gte = silu(sm.zg[t][c]);
                }
                sm.xc[t][c] = v;
                sm.zg[t][c] = gte;
            }
            for (int idx = tid; idx < kTC * NP; idx += kThreads) {
                const int t = idx / NP, n = idx % NP;
                float vb = 0.f, vc = 0.f;
                if (t < nv && n < N) {
                    if (K > 0) {
                        float wb[kMaxConvWidth], wc[kMaxConvWidth];
                        for (int k = 0; k < K; ++k) {
                            wb[k] = a.conv_w[(bch0 + n) * K + k];
                            wc[k] = a.conv_w[(cch0 + n) * K + k];
                        }
                        vb = conv_col(&sm.braw[0][0], NP, t, n, wb, a.conv_b ? a.conv_b[bch0 + n] : 0.f, K);
                        vc = conv_col(&sm.craw[0][0], NP, t, n, wc, a.conv_b ? a.conv_b[cch0 + n] : 0.f, K);
                    } else {
                        vb = sm.braw[kHalo + t][n];
                        vc = sm.craw[kHalo + t][n];
                    }
                }
                sm.Bc[t][n] = vb;
                sm.Cc[t][n] = vc;
            }
        }
        __syncthreads();
        if (nv > 0) {
            for (int t = 0; t < kTC; ++t) {
                const float dA = sm.da[t];
                const float xv = sm.xc[t][sp];
                const float dxv = sm.dl[t] * xv;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    float bv[VW], cv[VW];
                    const int n0 = VW * (q + kLanes * j);
                    if constexpr (VW == 4) {
                        const float4 b4 = *reinterpret_cast<const float4 *>(&sm.Bc[t][n0]);
                        const float4 c4 = *reinterpret_cast<const float4 *>(&sm.Cc[t][n0]);
                        bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
                        cv[0] = c4.x; cv[1] = c4.y; cv[2] = c4.z; cv[3] = c4.w;
                    } else if constexpr (VW == 2) {
                        const float2 b2 = *reinterpret_cast<const float2 *>(&sm.Bc[t][n0]);
                        const float2 c2 = *reinterpret_cast<const float2 *>(&sm.Cc[t][n0]);
                        bv[0] = b2.x; bv[1] = b2.y; cv[0] = c2.x; cv[1] = c2.y;
                    } else {
                        bv[0] = sm.Bc[t][n0]; cv[0] = sm.Cc[t][n0];
                    }
#pragma unroll
                    for (int e = 0; e < VW; ++e) {
                        h[j * VW + e] = fmaf(dA, h[j * VW + e], dxv * bv[e]);
                        acc = fmaf(cv[e], h[j * VW + e], acc);
                    }
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                __syncwarp();
                if (q == 0) sm.xc[t][sp] = (acc + Dh * xv) * sm.zg[t][sp];
            }
        }
        __syncthreads();
        // intermediate state after this chunk when it closes a state interval: the
        // lanes' register states, and the last K-1 raw rows of the tiles (before the slide)
        if (a.iv.interval > 0 && nv == kTC) {
            const int64_t slot = a.iv.slot_after(s, t0 + kTC);
            if (slot >= 0) {
                if (a.iv.states && svalid) {
                    float *dst = a.iv.states + ((slot * H + hh) * P + pch) * N;
#pragma unroll
                    for (int j = 0; j < NJ; ++j)
#pragma unroll
                        for (int e = 0; e < VW; ++e) {
                            const int64_t n = (int64_t)VW * (q + kLanes * j) + e;
                            if (n < N) dst[n] = h[j * VW + e];
                        }
                }
                if (a.iv.conv && K > 1) {
                    T *cdst = static_cast<T *>(a.iv.conv) + slot * cdim * (K - 1);
                    const bool bc_owner = (hh % (H / G) == 0) && pb == 0;   // one writer per group
                    for (int idx = tid; idx < (K - 1) * (kPB + 2 * NP); idx += kThreads) {
                        const int j = idx % (K - 1), c = idx / (K - 1);
                        const int r = kHalo + kTC - (K - 1) + j;
                        if (c < kPB) {
                            if (p0 + c < P) Elem<T>::st(cdst + (xch0 + c) * (K - 1) + j, sm.xraw[r][c]);
                        } else if (bc_owner && c < kPB + NP) {
                            const int n = c - kPB;
                            if (n < N) Elem<T>::st(cdst + (bch0 + n) * (K - 1) + j, sm.braw[r][n]);
                        } else if (bc_owner) {
                            const int n = c - kPB - NP;
                            if (n < N) Elem<T>::st(cdst + (cch0 + n) * (K - 1) + j, sm.craw[r][n]);
                        }
                    }
                }
            }
        }
        if (nv > 0) {
            store_tile_f32<T, kThreads>(yg + t0 * a.y_ts, a.y_ts, &sm.xc[0][0], kPB, nv, p0, ncols, P, a.vec_y);
            if (K > 1 && nv == kTC) {
                // slide the halo: rows kTC-(K-1).. of the raw tiles become the next halo
                const int per = kPB + 2 * NP;
                float keep[((kHalo * (kPB + 2 * NP)) + kThreads - 1) / kThreads];
                int cnt = 0;
                for (int idx = tid; idx < (K - 1) * per; idx += kThreads, ++cnt) {
                    const int j = idx / per, c = idx % per;
                    const int r = kHalo + kTC - (K - 1) + j;
                    keep[cnt] = c < kPB ? sm.xraw[r][c] : (c < kPB + NP ? sm.braw[r][c - kPB] : sm.craw[r][c - kPB - NP]);
                }
                __syncthreads();
                cnt = 0;
                for (int idx = tid; idx < (K - 1) * per; idx += kThreads, ++cnt) {
                    const int j = idx / per, c = idx % per;
                    const int r = kHalo - (K - 1) + j;
                    if (c < kPB) sm.xraw[r][c] = keep[cnt];
                    else if (c < kPB + NP) sm.braw[r][c - kPB] = keep[cnt];
                    else sm.craw[r][c - kPB - NP] = keep[cnt];
                }
            }
        }
        __syncthreads();
        const bool last = nv < kTC || t0 + kTC == len;
        if (last) {
            if (K > 1 && a.conv_state_out) {
                // halo-relative rows of the last K-1 raw inputs
                const int base = (nv < kTC) ? kHalo + nv - (K - 1) : kHalo - (K - 1);
                T *cso = static_cast<T *>(a.conv_state_out);
                const bool bc_owner = (hh % (H / G) == 0) && pb == 0;   // one writer per group
                for (int idx = tid; idx < (K - 1) * (kPB + 2 * NP); idx += kThreads) {
                    const int j = idx % (K - 1), c = idx / (K - 1);
                    const int r = base + j;
                    if (c < kPB) {
                        if (p0 + c < P) Elem<T>::st(cso + ((int64_t)s * cdim + xch0 + c) * (K - 1) + j, sm.xraw[r][c]);
                    } else if (bc_owner && c < kPB + NP) {
                        const int n = c - kPB;
                        if (n < N) Elem<T>::st(cso + ((int64_t)s * cdim + bch0 + n) * (K - 1) + j, sm.braw[r][n]);
                    } else if (bc_owner) {
                        const int n = c - kPB - NP;
                        if (n < N) Elem<T>::st(cso + ((int64_t)s * cdim + cch0 + n) * (K - 1) + j, sm.craw[r][n]);
                    }
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
                if (n < N) a.h_final[(((int64_t)s * H + hh) * P + pch) * N + n] = h[j * VW + e];
            }
    }
}

template <typename T, int SPT>
cudaError_t launch_spt(const M2Args &a, int nseqs, cudaStream_t st) {
    const size_t smem = sizeof(SmemM2<SPT>);
    auto kern = scan_m2_simt_kernel<T, SPT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(a.H * a.npb), (unsigned)nseqs);
    timing_begin(st);
    kern<<<grid, kThreads, smem, st>>>(a);
    timing_end(st);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const M2Args &a, int nseqs, cudaStream_t st) {
    if (a.N <= 8) return launch_spt<T, 1>(a, nseqs, st);
    if (a.N <= 16) return launch_spt<T, 2>(a, nseqs, st);
    if (a.N <= 32) return launch_spt<T, 4>(a, nseqs, st);
    if (a.N <= 64) return launch_spt<T, 8>(a, nseqs, st);
    if (a.N <= 128) return launch_spt<T, 16>(a, nseqs, st);
    return launch_spt<T, 32>(a, nseqs, st);
}

inline bool vec_ok(const void *p, int64_t bs, int64_t ts, size_t es, int64_t colstep) {
    return p == nullptr || ((uintptr_t)p % 16 == 0 && (bs * (int64_t)es) % 16 == 0 && (ts * (int64_t)es) % 16 == 0 &&
                            (colstep * (int64_t)es) % 16 == 0);
}

}  // namespace

cudaError_t launch_scan_m2_simt(const ssm_scan_args &s, const SeqView &sv, cudaStream_t st) {
    M2Args a;
    a.x = s.x; a.z = s.z; a.dt = s.dt; a.B = s.B; a.C = s.C; a.y = s.y;
    a.x_bs = s.x_batch_stride; a.x_ts = s.x_token_stride;
    a.z_bs = s.z_batch_stride; a.z_ts = s.z_token_stride;
    a.dt_bs = s.dt_batch_stride; a.dt_ts = s.dt_token_stride;
    a.B_bs = s.B_batch_stride; a.B_ts = s.B_token_stride;
    a.C_bs = s.C_batch_stride; a.C_ts = s.C_token_stride;
    a.y_bs = s.y_batch_stride; a.y_ts = s.y_token_stride;
    a.A = s.A; a.D = s.D; a.dt_bias = s.dt_bias; a.h0 = s.h0; a.h_final = s.h_final;
    a.conv_w = s.conv_w; a.conv_b = s.conv_b; a.conv_state_in = s.conv_state_in; a.conv_state_out = s.conv_state_out;
    a.H = s.nheads; a.P = s.headdim; a.G = s.ngroups; a.N = s.dstate; a.seqlen = s.seqlen;
    a.K = (int)s.d_conv; a.softplus = s.delta_softplus;
    a.npb = (int)((s.headdim + kPB - 1) / kPB);
    const size_t es = s.dtype == SSM_BF16 ? 2 : 4;
    // each head's columns start at h*P (x, z, y) and each group's at g*N (B, C)
    a.vec_x = vec_ok(s.x, s.x_batch_stride, s.x_token_stride, es, s.headdim);
    a.vec_z = vec_ok(s.z, s.z_batch_stride, s.z_token_stride, es, s.headdim);
    a.vec_y = vec_ok(s.y, s.y_batch_stride, s.y_token_stride, es, s.headdim);
    a.vec_B = vec_ok(s.B, s.B_batch_stride, s.B_token_stride, es, s.dstate);
    a.vec_C = vec_ok(s.C, s.C_batch_stride, s.C_token_stride, es, s.dstate);
    a.sv = sv;
    a.iv = inter_view(s);
    const int nseqs = s.cu_seqlens ? s.nseqs : (int)s.batch;
    if (nseqs == 0) return cudaSuccess;
    return s.dtype == SSM_BF16 ? launch_typed<__nv_bfloat16>(a, nseqs, st) : launch_typed<float>(a, nseqs, st);
}

}  // namespace ssm
