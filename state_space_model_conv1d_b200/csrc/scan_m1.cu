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
// Design (sm_100a, CUDA cores).  One CTA owns one sequence and DB = 32
// channels and walks the tokens in chunks of TC.  Raw x / dt / z / B / C
// chunk tiles are staged in shared memory with 16-byte cp.async copies, two
// chunks ahead of the compute (double buffer), so HBM latency hides behind
// the scan.  A cooperative prologue computes conv + SiLU, delta, delta*x and
// the gate once per (token, channel) into fp32 tiles.  Then 4 lanes per
// channel advance N/4 states each in registers; the carry across chunks is
// the fp32 state staying in registers, seeded from h0 (the (1, h0) seed of
// the pair scan).  The 4 lanes' partial read-outs of 4 consecutive tokens
// are combined by a two-level shuffle reduce-scatter, so each lane finishes
// one token's y.  The K-1 raw rows before each chunk live in a small
// double-buffered halo, which is also what conv_state_out receives.
//
// Per (token, channel, state) the work is one MUFU exp plus four FP32 ops:
// with dstate 16 the kernel is bound by the MUFU exp rate, not by HBM.
#include "common.cuh"
#include "launch.h"

namespace ssm {
namespace {

constexpr int kDB = 32;             // channels per CTA
constexpr int kLanes = 4;           // lanes per channel
constexpr int kThreads = kDB * kLanes;
constexpr int kTC = 32;             // tokens per chunk
constexpr int kHalo = kMaxConvWidth - 1;
constexpr int kRowsPerThread = kTC * kDB / kThreads;   // prologue rows per thread (8)

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
    bool async_act, async_bc, vec_y;
    SeqView sv;
};

template <typename T, int SPT>
struct SmemM1 {
    static constexpr int NP = kLanes * SPT;             // padded dstate
    T rx[2][kTC][kDB];
    T rdt[2][kTC][kDB];
    T rz[2][kTC][kDB];
    T rB[2][kTC][NP];
    T rC[2][kTC][NP];
    float halo[2][kHalo][kDB];
    float xc[kTC][kDB];
    float2 dd[kTC][kDB];      // (delta, delta * xc)
    float g[kTC][kDB];
    float y[kTC][kDB];
    float Bf[kTC][NP];
    float Cf[kTC][NP];
};

SSM_DEVINL void cp_async16(void *smem, const void *gmem) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
SSM_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
SSM_DEVINL void cp_async_wait1() { asm volatile("cp.async.wait_group 1;\n" ::); }

// Stage rows [0, nv) x cols [col0, col0 + ncols) of a token-major tensor into
// dst[kTC][ld] (raw dtype).  16-byte cp.async when `async` (every row start
// 16-byte aligned, ncols * sizeof(T) a multiple of 16), else plain loads.
template <typename T>
SSM_DEVINL void stage_tile(T *dst, int ld, const T *src, int64_t ts, int nv, int64_t col0, int ncols,
                           int64_t col_end, bool async) {
    constexpr int E = 16 / sizeof(T);
    if (async) {
        const int per_row = ncols / E;
        for (int i = threadIdx.x; i < nv * per_row; i += kThreads) {
            const int r = i / per_row, v = i % per_row;
            const int64_t c = col0 + (int64_t)v * E;
            if (c + E <= col_end) cp_async16(dst + r * ld + v * E, src + r * ts + c);
        }
    } else {
        for (int i = threadIdx.x; i < nv * ncols; i += kThreads) {
            const int r = i / ncols, v = i % ncols;
            const int64_t c = col0 + v;
            if (c < col_end) dst[r * ld + v] = src[r * ts + c];
        }
    }
}

template <typename T, int SPT>
__global__ void __launch_bounds__(kThreads)
scan_m1_kernel(const M1Args a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<SmemM1<T, SPT> *>(smem_raw);
    constexpr int NP = SmemM1<T, SPT>::NP;
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
    const int nchunks = (int)((len + kTC - 1) / kTC);

    auto stage = [&](int c) {
        const int buf = c & 1;
        const int64_t t0 = (int64_t)c * kTC;
        const int nv = (int)min((int64_t)kTC, len - t0);
        if (nv > 0) {
            stage_tile<T>(&sm.rx[buf][0][0], kDB, xg + t0 * a.x_ts, a.x_ts, nv, d0, kDB, Dn, a.async_act);
            stage_tile<T>(&sm.rdt[buf][0][0], kDB, dtg + t0 * a.dt_ts, a.dt_ts, nv, d0, kDB, Dn, a.async_act);
            if (zg) stage_tile<T>(&sm.rz[buf][0][0], kDB, zg + t0 * a.z_ts, a.z_ts, nv, d0, kDB, Dn, a.async_act);
            stage_tile<T>(&sm.rB[buf][0][0], NP, Bg + t0 * a.B_ts, a.B_ts, nv, 0, (int)N, N, a.async_bc);
            stage_tile<T>(&sm.rC[buf][0][0], NP, Cg + t0 * a.C_ts, a.C_ts, nv, 0, (int)N, N, a.async_bc);
        }
        cp_async_commit();
    };
    stage(0);
    stage(1);

    // ---- prologue role: channel pd = tid % 32, rows [pr0, pr0 + 8)
    const int pd = tid % kDB;
    const int pr0 = (tid / kDB) * kRowsPerThread;
    const int64_t pch = d0 + pd;
    const bool pvalid = pch < Dn;
    // conv taps right-aligned: wr[kHalo] multiplies the current token, wr[kHalo - m]
    // the input m tokens back; unused leading taps are 0, so every index is static
    float wr[kMaxConvWidth], cb = 0.f, dtb = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxConvWidth; ++j) {
        const int k = K - kMaxConvWidth + j;                  // tap index in [0, K)
        wr[j] = (pvalid && k >= 0) ? a.conv_w[pch * K + k] : 0.f;
    }
    if (pvalid && a.conv_b) cb = a.conv_b[pch];
    if (pvalid && a.dt_bias) dtb = a.dt_bias[pch];

    // ---- scan role: channel sd = tid / 4, lane q = tid % 4
    const int sd = tid / kLanes, q = tid % kLanes;
    const int64_t sch = d0 + sd;
    const bool svalid = sch < Dn;
    // states of this lane: n = VW * (q + 4 j) + e; kept as fp32 pairs (h2, A2p)
    // for the packed path, or scalars when a lane holds a single state
    constexpr int NPAIR = SPT >= 2 ? SPT / 2 : 1;
    float A2[SPT], h[SPT];
    float2 A2p[NPAIR], h2[NPAIR];
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
        for (int e = 0; e < VW; ++e) {
            const int64_t n = (int64_t)VW * (q + kLanes * j) + e;
            const bool ok = svalid && n < N;
            A2[j * VW + e] = ok ? a.A[sch * N + n] * kLog2e : 0.f;
            h[j * VW + e] = (ok && a.h0) ? a.h0[((int64_t)s * Dn + sch) * N + n] : 0.f;
        }
#pragma unroll
    for (int p = 0; p < NPAIR; ++p) {
        if constexpr (SPT >= 2) {
            A2p[p] = make_float2(A2[2 * p], A2[2 * p + 1]);
            h2[p] = make_float2(h[2 * p], h[2 * p + 1]);
        }
    }
    const float Dd = (svalid && a.D) ? a.D[sch] : 0.f;

    // ---- conv halo of chunk 0: the carried state (the K-1 raw inputs before the first token)
    if (K > 1) {
        const T *csi = static_cast<const T *>(a.conv_state_in);
        for (int idx = tid; idx < (K - 1) * kDB; idx += kThreads) {
            const int j = idx / kDB, d = idx % kDB;
            const int64_t ch = d0 + d;
            sm.halo[0][kHalo - (K - 1) + j][d] =
                (csi && ch < Dn) ? Elem<T>::ld(csi + ((int64_t)s * Dn + ch) * (K - 1) + j) : 0.f;
        }
    }

    for (int c = 0; c < nchunks || c == 0; ++c) {
        const int buf = c & 1;
        const int64_t t0 = (int64_t)c * kTC;
        const int nv = (int)max((int64_t)0, min((int64_t)kTC, len - t0));
        cp_async_wait1();
        __syncthreads();                                               // chunk c staged, halo[buf] ready

        // ---------------- prologue: once per (token, channel)
        {
            float win[kHalo];                                           // raw rows t-7 .. t-1
            auto raw_at = [&](int v) -> float {                         // v: row relative to the chunk
                return v >= 0 ? Elem<T>::ld(&sm.rx[buf][v][pd]) : sm.halo[buf][kHalo + v][pd];
            };
#pragma unroll
            for (int j = 0; j < kHalo; ++j)                             // only the last K-1 are live
                win[j] = (j >= kHalo - (K - 1) && pvalid) ? raw_at(pr0 - kHalo + j) : 0.f;
#pragma unroll
            for (int i = 0; i < kRowsPerThread; ++i) {
                const int t = pr0 + i;
                float xcv = 0.f, dlt = 0.f, gv = 1.f;
                if (t < nv && pvalid) {
                    const float cur = Elem<T>::ld(&sm.rx[buf][t][pd]);
                    if (K > 0) {
                        float acc = fmaf(wr[kHalo], cur, cb);
#pragma unroll
                        for (int j = 0; j < kHalo; ++j) acc = fmaf(wr[j], win[j], acc);
                        xcv = silu_fast<T>(acc);
                    } else {
                        xcv = cur;
                    }
#pragma unroll
                    for (int j = 0; j + 1 < kHalo; ++j) win[j] = win[j + 1];
                    win[kHalo - 1] = cur;
                    const float u = Elem<T>::ld(&sm.rdt[buf][t][pd]) + dtb;
                    dlt = a.softplus ? softplus(u) : u;
                    if (zg) gv = silu_fast<T>(Elem<T>::ld(&sm.rz[buf][t][pd]));
                }
                sm.xc[t][pd] = xcv;
                sm.dd[t][pd] = make_float2(dlt, dlt * xcv);   // delta = 0 past the end: the state stays put
                sm.g[t][pd] = gv;
            }
            // next halo: the last K-1 raw inputs up to this chunk's end
            if (K > 1 && tid < kDB)
                for (int j = 0; j < K - 1; ++j) {
                    const int v = nv - (K - 1) + j;
                    sm.halo[buf ^ 1][kHalo - (K - 1) + j][pd] = pvalid ? raw_at(v) : 0.f;
                }
            // B and C to fp32, zero past the end of the sequence and of dstate
            for (int i = tid; i < kTC * NP; i += kThreads) {
                const int t = i / NP, n = i % NP;
                const bool ok = t < nv && n < N;
                sm.Bf[t][n] = ok ? Elem<T>::ld(&sm.rB[buf][t][n]) : 0.f;
                sm.Cf[t][n] = ok ? Elem<T>::ld(&sm.rC[buf][t][n]) : 0.f;
            }
        }
        __syncthreads();                                               // raw[buf] consumed
        stage(c + 2);                                                  // prefetch two chunks ahead

        // ---------------- recurrence, 4 tokens per step of the loop
#pragma unroll 2
        for (int t4 = 0; t4 < kTC; t4 += 4) {
            float acc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = t4 + i;
                const float2 dd = sm.dd[t][sd];                      // (delta, delta * xc)
                if constexpr (VW >= 2) {
                    // packed fp32x2: two states per FMUL2 / FFMA2 instruction
                    const float2 dl2 = make_float2(dd.x, dd.x), dx2 = make_float2(dd.y, dd.y);
                    float2 ac2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int n0 = VW * (q + kLanes * j);
#pragma unroll
                        for (int e = 0; e < VW; e += 2) {
                            const float2 b2 = *reinterpret_cast<const float2 *>(&sm.Bf[t][n0 + e]);
                            const float2 c2 = *reinterpret_cast<const float2 *>(&sm.Cf[t][n0 + e]);
                            const int pi = (j * VW + e) / 2;
                            const float2 arg = __fmul2_rn(dl2, A2p[pi]);
                            const float2 dA = make_float2(ex2(arg.x), ex2(arg.y));
                            h2[pi] = __ffma2_rn(dA, h2[pi], __fmul2_rn(dx2, b2));
                            ac2 = __ffma2_rn(c2, h2[pi], ac2);
                        }
                    }
                    acc[i] = ac2.x + ac2.y;
                } else {
                    float ac = 0.f;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int n0 = q + kLanes * j;
                        const float dA = ex2(dd.x * A2[j]);
                        h[j] = fmaf(dA, h[j], dd.y * sm.Bf[t][n0]);
                        ac = fmaf(sm.Cf[t][n0], h[j], ac);
                    }
                    acc[i] = ac;
                }
            }
            // reduce-scatter over the 4 lanes of the channel: lane q ends with token t4 + q
            const bool hi = (q & 2) != 0;
            const float s0 = hi ? acc[0] : acc[2], s1 = hi ? acc[1] : acc[3];
            const float k0 = hi ? acc[2] : acc[0], k1 = hi ? acc[3] : acc[1];
            const float r0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 2);
            const float r1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 2);
            const bool odd = (q & 1) != 0;
            const float tot = (odd ? r1 : r0) + __shfl_xor_sync(0xffffffffu, odd ? r0 : r1, 1);
            const int t = t4 + q;
            sm.y[t][sd] = (tot + Dd * sm.xc[t][sd]) * sm.g[t][sd];
        }
        __syncthreads();                                               // y tile complete

        if (nv > 0) {
            // y tile -> global, 16-byte stores when aligned
            constexpr int E = 16 / sizeof(T);
            if (a.vec_y && d0 + kDB <= Dn) {
                for (int i = tid; i < nv * (kDB / 8); i += kThreads) {
                    const int r = i / (kDB / 8), v = i % (kDB / 8);
                    float o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = sm.y[r][v * 8 + e];
                    Vec8<T>::st(yg + (t0 + r) * a.y_ts + d0 + v * 8, o);
                }
            } else {
                for (int i = tid; i < nv * kDB; i += kThreads) {
                    const int r = i / kDB, v = i % kDB;
                    if (d0 + v < Dn) Elem<T>::st(yg + (t0 + r) * a.y_ts + d0 + v, sm.y[r][v]);
                }
            }
            (void)E;
        }
        if (c + 1 >= nchunks) {
            // carried conv state: the halo written by this (last) chunk's prologue
            if (K > 1 && a.conv_state_out) {
                T *cso = static_cast<T *>(a.conv_state_out);
                for (int idx = tid; idx < (K - 1) * kDB; idx += kThreads) {
                    const int j = idx / kDB, d = idx % kDB;
                    const int64_t ch = d0 + d;
                    if (ch < Dn)
                        Elem<T>::st(cso + ((int64_t)s * Dn + ch) * (K - 1) + j, sm.halo[buf ^ 1][kHalo - (K - 1) + j][d]);
                }
            }
            break;
        }
    }
    asm volatile("cp.async.wait_all;\n" ::);
    if constexpr (SPT >= 2) {
#pragma unroll
        for (int p = 0; p < NPAIR; ++p) {
            h[2 * p] = h2[p].x;
            h[2 * p + 1] = h2[p].y;
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
    const size_t smem = sizeof(SmemM1<T, SPT>);
    auto kern = scan_m1_kernel<T, SPT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.Dn + kDB - 1) / kDB), (unsigned)nseqs);
    kern<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(M1Args a, int nseqs, cudaStream_t st) {
    constexpr int E = 16 / sizeof(T);
    // B / C rows go through 16-byte copies only when dstate fills whole vectors
    // and the padded row (4 * SPT elements) keeps every row 16-byte aligned.
    auto bc_ok = [&](int np) { return a.async_bc && a.N % E == 0 && (np * (int)sizeof(T)) % 16 == 0; };
    if (a.N <= 4) { a.async_bc = bc_ok(4); return launch_spt<T, 1>(a, nseqs, st); }
    if (a.N <= 8) { a.async_bc = bc_ok(8); return launch_spt<T, 2>(a, nseqs, st); }
    if (a.N <= 16) { a.async_bc = bc_ok(16); return launch_spt<T, 4>(a, nseqs, st); }
    if (a.N <= 32) { a.async_bc = bc_ok(32); return launch_spt<T, 8>(a, nseqs, st); }
    a.async_bc = bc_ok(64);
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
    // x / dt / z tiles: 32-channel rows starting at multiples of 32 channels
    a.async_act = vec_ok(s.x, s.x_batch_stride, s.x_token_stride, es) &&
                  vec_ok(s.dt, s.dt_batch_stride, s.dt_token_stride, es) &&
                  vec_ok(s.z, s.z_batch_stride, s.z_token_stride, es) && s.d_inner % (16 / es) == 0;
    a.async_bc = vec_ok(s.B, s.B_batch_stride, s.B_token_stride, es) &&
                 vec_ok(s.C, s.C_batch_stride, s.C_token_stride, es);
    a.vec_y = vec_ok(s.y, s.y_batch_stride, s.y_token_stride, es);
    a.sv = sv;
    const int nseqs = s.cu_seqlens ? s.nseqs : (int)s.batch;
    if (nseqs == 0) return cudaSuccess;
    return s.dtype == SSM_BF16 ? launch_typed<__nv_bfloat16>(a, nseqs, st) : launch_typed<float>(a, nseqs, st);
}

}  // namespace ssm
