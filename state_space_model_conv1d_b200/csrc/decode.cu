// decode.cu -- single-token state update, in place ("Clean up SSM ops
// directory structure", Megatron-LM PR 6444: causal_conv1d_update followed by
// selective_state_update; slot-indexed state rows as in intermediate_extraction).
//
// Per batch row r (state slot s = idx ? idx[r] : r):
//   conv window: conv_state[s][c] rolled left by one, the new raw input
//   appended; xc[c] = silu(b[c] + sum_k w[c, k] * window[L-K+k])
//   delta[h] = softplus(dt[h] + dt_bias[h]);  a = exp(delta A)
//   S[h, p, n] = a S[h, p, n] + delta xc[h, p] B[g(h), n]        (in place)
//   y[h, p] = (sum_n C[g(h), n] S[h, p, n] + D[h] xc[h, p]) * silu(z[h, p])
// Mamba-1 is the same with one channel per "head" (P = 1), A[d, n] per state
// and B / C taken as given (the conv covers x only).
//
// HBM-bound: the fp32 state is read and written once (16-byte vectors, one
// warp per 128-state row for dstate 128), the conv state once each way; B / C
// are loaded once per (row, group).  One CTA owns (batch row, group) for
// Mamba-2 -- so the group's B / C conv state is rolled exactly once -- and
// (batch row, 256 channels) for Mamba-1.
#include "common.cuh"
#include "launch.h"

namespace ssm {
namespace {

constexpr int kThreads = 512;          // two CTAs of 16 warps per SM: one's prologue overlaps the other's streaming
constexpr int kM1Channels = 256;

struct DecArgs {
    float *state;
    void *conv_state;
    const float *conv_w, *conv_b;
    const void *x, *z, *dt, *B, *C;
    void *y;
    int64_t x_bs, z_bs, dt_bs, B_bs, C_bs, y_bs;
    const float *A, *D, *dt_bias;
    const int32_t *idx;
    int64_t nslots, Dn, H, P, G, N, Ls;
    int K, softplus, mode;
};

// Roll one channel's conv window and return silu(conv) of the new input.
template <typename T>
SSM_DEVINL float conv_roll(T *cs, int64_t Ls, const float *w, float b, int K, float u) {
    float win[kMaxConvWidth];
    float acc = b;
    // the last K-1 stored inputs, oldest first, then the new input
    for (int k = 0; k < K - 1; ++k) win[k] = Elem<T>::ld(cs + Ls - (K - 1) + k);
    for (int k = 0; k < K - 1; ++k) acc = fmaf(w[k], win[k], acc);
    acc = fmaf(w[K - 1], u, acc);
    for (int64_t k = 0; k + 1 < Ls; ++k) Elem<T>::st(cs + k, Elem<T>::ld(cs + k + 1));
    if (Ls > 0) Elem<T>::st(cs + Ls - 1, u);
    return silu(acc);
}

// Fast path for bf16 with a 4-wide window: one 8-byte load and store.
// wr holds the taps right-aligned (wr[7] multiplies the new input, wr[7 - m]
// the input m steps back, zeros before the first tap), so no index is dynamic.
SSM_DEVINL float conv_roll4_bf16(__nv_bfloat16 *cs, const float (&wr)[kMaxConvWidth], float b, float u) {
    uint2 r = *reinterpret_cast<const uint2 *>(cs);
    float s0 = __uint_as_float(r.x << 16), s1 = __uint_as_float(r.x & 0xffff0000u);
    float s2 = __uint_as_float(r.y << 16), s3 = __uint_as_float(r.y & 0xffff0000u);
    float acc = fmaf(wr[7], u, b);
    acc = fmaf(wr[6], s3, acc);
    acc = fmaf(wr[5], s2, acc);
    acc = fmaf(wr[4], s1, acc);
    acc = fmaf(wr[3], s0, acc);
    __nv_bfloat162 lo = __floats2bfloat162_rn(s1, s2);
    __nv_bfloat162 hi = __floats2bfloat162_rn(s3, u);   // u is a bf16 value already: exact
    r.x = *reinterpret_cast<uint32_t *>(&lo);
    r.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(cs) = r;
    return silu(acc);
}

SSM_DEVINL int64_t hh_first(int unit, int64_t hpg) { return (int64_t)unit * hpg; }

// Rows [0, nrows) of one Mamba-2 group: row = (local head, p), state row at
// stb + (c0 + row) * N, N = 128 * NV.  Lane l owns states 4 * (l + 32 v) .. +3.
// dxr[row] = delta * x and dar[row] = exp(delta A) of the row's head.  The R
// rows a warp has in flight are summed with a reduce-scatter: lanes exchange
// halves of their partial sums until each lane holds one row's, then finish
// that row with a butterfly, and lane 32 / R * i writes row i.
template <int NV, typename T>
SSM_DEVINL void stream_rows(float *stb, int64_t c0, int64_t h0, int64_t nrows, int64_t P, const float *xs,
                            const float *Bs, const float *Cs, const float *dxr, const float *dar, const float *Dp,
                            const T *zr, T *yr, int warp, int lane) {
    constexpr int64_t N = 128 * NV;
    constexpr int R = NV == 1 ? 4 : 2;         // rows in flight per warp (within 64 registers)
    float2 Bv[NV][2], Cv[NV][2];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        const float4 b4 = *reinterpret_cast<const float4 *>(Bs + 4 * (lane + 32 * v));
        const float4 c4 = *reinterpret_cast<const float4 *>(Cs + 4 * (lane + 32 * v));
        Bv[v][0] = make_float2(b4.x, b4.y); Bv[v][1] = make_float2(b4.z, b4.w);
        Cv[v][0] = make_float2(c4.x, c4.y); Cv[v][1] = make_float2(c4.z, c4.w);
    }
    constexpr int kWarps = kThreads / 32;
    for (int64_t row0 = (int64_t)warp * R; row0 < nrows; row0 += (int64_t)kWarps * R) {
        float4 sv[R][NV];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int64_t row = row0 + i;
            if (row < nrows) {
                const float *srow = stb + (c0 + row) * N;
#pragma unroll
                for (int v = 0; v < NV; ++v) sv[i][v] = __ldcs(reinterpret_cast<const float4 *>(srow + 4 * (lane + 32 * v)));
            }
        }
        float acc[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int64_t row = row0 + i;
            acc[i] = 0.f;
            if (row < nrows) {
                const float2 dA = make_float2(dar[row], dar[row]);
                const float2 dx = make_float2(dxr[row], dxr[row]);
                float *srow = stb + (c0 + row) * N;
                float2 ac = make_float2(0.f, 0.f);
#pragma unroll
                for (int v = 0; v < NV; ++v) {
                    float2 lo = make_float2(sv[i][v].x, sv[i][v].y), hi = make_float2(sv[i][v].z, sv[i][v].w);
                    lo = __ffma2_rn(dA, lo, __fmul2_rn(dx, Bv[v][0]));
                    hi = __ffma2_rn(dA, hi, __fmul2_rn(dx, Bv[v][1]));
                    __stcs(reinterpret_cast<float4 *>(srow + 4 * (lane + 32 * v)), make_float4(lo.x, lo.y, hi.x, hi.y));
                    ac = __ffma2_rn(Cv[v][0], lo, ac);
                    ac = __ffma2_rn(Cv[v][1], hi, ac);
                }
                acc[i] = ac.x + ac.y;
            }
        }
        // reduce-scatter over the R rows, then a butterfly over the remaining lanes
#pragma unroll
        for (int o = 16, w = R / 2; w >= 1; o >>= 1, w >>= 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int k = 0; k < w; ++k) {
                const float keep = up ? acc[w + k] : acc[k];
                const float send = up ? acc[k] : acc[w + k];
                acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
#pragma unroll
        for (int o = 32 / R / 2; o >= 1; o >>= 1) acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], o);
        // lane bits 4, 3 (R = 4) or bit 4 (R = 2) name the row this lane now holds
        int q = 0;
#pragma unroll
        for (int o = 16, w = R / 2; w >= 1; o >>= 1, w >>= 1) q += (lane & o) ? w : 0;
        if ((lane & (32 / R - 1)) == 0) {
            const int64_t row = row0 + q;
            if (row < nrows) {
                const int64_t hl = row / P, ch = c0 + row;
                float yv = acc[0] + (Dp ? Dp[h0 + hl] : 0.f) * xs[row];
                if (zr) yv *= silu(Elem<T>::ld(zr + ch));
                Elem<T>::st(yr + ch, yv);
            }
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecArgs a) {
    extern __shared__ __align__(16) float sm[];
    const int r = blockIdx.y;
    const int unit = blockIdx.x;
    const bool m2 = a.mode == SSM_MAMBA2;
    const int64_t N = a.N, P = m2 ? a.P : 1;
    const int64_t hpg = m2 ? a.H / a.G : 0;
    // channels owned by this CTA: [c0, c0 + nx) of x; Mamba-2 also B / C of group `unit`
    const int64_t c0 = m2 ? unit * hpg * P : (int64_t)unit * kM1Channels;
    const int64_t nx = m2 ? hpg * P : min((int64_t)kM1Channels, a.Dn - c0);
    const int64_t h0 = m2 ? unit * hpg : c0;            // first head (Mamba-1: channel)
    const int64_t nh = m2 ? hpg : nx;
    int64_t slot = a.idx ? (int64_t)a.idx[r] : r;
    const T *xr = static_cast<const T *>(a.x) + r * a.x_bs;
    T *yr = static_cast<T *>(a.y) + r * a.y_bs;
    // bounds-checked build: the CTA's channel range (uniform, so the whole CTA returns together)
    if (!SSM_BOUNDS(c0 + nx - 1, a.Dn, BS_DEC_CHANNEL) || !SSM_BOUNDS(r, (int64_t)gridDim.y, BS_DEC_ROW)) return;
    if (slot < 0 || slot >= a.nslots) {                 // padding row: y = 0, nothing else touched
        for (int64_t i = threadIdx.x; i < nx; i += kThreads) Elem<T>::st(yr + c0 + i, 0.f);
        return;
    }
    float *xs = sm;                    // [nx] conv output of x (padded to 4 for 16-byte alignment)
    float *Bs = xs + ((nx + 3) & ~(int64_t)3);   // [N]
    float *Cs = Bs + N;                // [N]
    float *dls = Cs + N;               // [nh] delta
    float *das = dls + nh;             // [nh] exp(delta A)   (Mamba-2 only)
    float *dxr = das + nh;             // [nx] delta * x per state row (Mamba-2 streaming path)
    float *dar = dxr + nx;             // [nx] exp(delta A) per state row
    const int64_t cdim = m2 ? a.Dn + 2 * a.G * N : a.Dn;
    T *csb = static_cast<T *>(a.conv_state) + slot * cdim * a.Ls;
    const T *Br = static_cast<const T *>(a.B) + r * a.B_bs + (m2 ? unit * N : 0);
    const T *Cr = static_cast<const T *>(a.C) + r * a.C_bs + (m2 ? unit * N : 0);
    const int K = a.K;
    const int64_t nconv = nx + (m2 ? 2 * N : 0);

    for (int64_t i = threadIdx.x; i < nconv; i += kThreads) {
        int64_t ch;
        float u;
        if (i < nx) { ch = c0 + i; u = Elem<T>::ld(xr + c0 + i); }
        else if (i < nx + N) { ch = a.Dn + unit * N + (i - nx); u = Elem<T>::ld(Br + (i - nx)); }
        else { ch = a.Dn + a.G * N + unit * N + (i - nx - N); u = Elem<T>::ld(Cr + (i - nx - N)); }
        float v = u;
        if (K > 0) {
            const float *w = a.conv_w + ch * K;
            const float b = a.conv_b ? a.conv_b[ch] : 0.f;
            T *cs = csb + ch * a.Ls;
            if constexpr (sizeof(T) == 2) {
                if (a.Ls == 4 && K <= 5 && ((uintptr_t)cs & 7) == 0) {
                    float wr[kMaxConvWidth];
#pragma unroll
                    for (int j = 0; j < kMaxConvWidth; ++j) {
                        const int k = K - kMaxConvWidth + j;
                        wr[j] = k >= 0 ? a.conv_w[ch * K + k] : 0.f;
                    }
                    v = conv_roll4_bf16(reinterpret_cast<__nv_bfloat16 *>(cs), wr, b, u);
                } else {
                    v = conv_roll<T>(cs, a.Ls, w, b, K, u);
                }
            } else {
                v = conv_roll<T>(cs, a.Ls, w, b, K, u);
            }
        }
        if (i < nx) xs[i] = v;
        else if (i < nx + N) Bs[i - nx] = v;
        else Cs[i - nx - N] = v;
    }
    if (!m2) {
        for (int64_t n = threadIdx.x; n < N; n += kThreads) {
            Bs[n] = Elem<T>::ld(Br + n);
            Cs[n] = Elem<T>::ld(Cr + n);
        }
    }
    const T *dtr = static_cast<const T *>(a.dt) + r * a.dt_bs;
    for (int64_t i = threadIdx.x; i < nh; i += kThreads) {
        const int64_t hh = h0 + i;
        const float u = Elem<T>::ld(dtr + hh) + (a.dt_bias ? a.dt_bias[hh] : 0.f);
        const float dl = a.softplus ? softplus(u) : u;
        dls[i] = dl;
        das[i] = m2 ? ex2(dl * a.A[hh] * kLog2e) : 0.f;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const T *zr = a.z ? static_cast<const T *>(a.z) + r * a.z_bs : nullptr;
    float *stb = a.state + slot * a.Dn * N;
    if (m2 && (N == 128 || N == 256)) {
        for (int64_t i = threadIdx.x; i < nx; i += kThreads) {
            const int64_t hl = i / P;
            dxr[i] = dls[hl] * xs[i];
            dar[i] = das[hl];
        }
        __syncthreads();
        // Streaming fast path: one warp per 128-state row segment, each lane one
        // float4 per 128 states; four rows in flight per warp; B / C held in
        // registers for the whole group.
        if (N == 128) stream_rows<1, T>(stb, c0, hh_first(unit, hpg), nh * P, P, xs, Bs, Cs, dxr, dar, a.D, zr, yr, warp, lane);
        else stream_rows<2, T>(stb, c0, hh_first(unit, hpg), nh * P, P, xs, Bs, Cs, dxr, dar, a.D, zr, yr, warp, lane);
        return;
    }

    // state rows: (head, p) pairs of this CTA, N states each; LPR lanes per row
    const bool vec = (N % 4 == 0);
    int lpr = 1;                                                        // lanes per row, a power of two
    if (vec)
        while (lpr * 2 <= 32 && lpr * 2 * 4 <= N) lpr *= 2;
    const int rpw = 32 / lpr;                                          // rows per warp pass
    const int sub = lane / lpr, sl = lane % lpr;
    const int64_t nrows = nh * P;
    for (int64_t row0 = (int64_t)warp * rpw; row0 < nrows; row0 += (int64_t)(kThreads / 32) * rpw) {
        const int64_t row = row0 + sub;
        const bool rv = row < nrows && vec;
        const int64_t hl = row / P;                  // local head index
        const int64_t ch = c0 + row;                 // x channel
        float acc = 0.f;
        if (rv) {
            const float dl = dls[hl];
            const float xv = xs[row];
            const float dxv = dl * xv;
            float *srow = stb + ch * N;
            if (m2) {
                const float dA = das[hl];
                for (int64_t n = (int64_t)sl * 4; n < N; n += (int64_t)lpr * 4) {
                    float4 s4 = *reinterpret_cast<float4 *>(srow + n);
                    s4.x = fmaf(dA, s4.x, dxv * Bs[n]);
                    s4.y = fmaf(dA, s4.y, dxv * Bs[n + 1]);
                    s4.z = fmaf(dA, s4.z, dxv * Bs[n + 2]);
                    s4.w = fmaf(dA, s4.w, dxv * Bs[n + 3]);
                    *reinterpret_cast<float4 *>(srow + n) = s4;
                    acc = fmaf(Cs[n], s4.x, acc);
                    acc = fmaf(Cs[n + 1], s4.y, acc);
                    acc = fmaf(Cs[n + 2], s4.z, acc);
                    acc = fmaf(Cs[n + 3], s4.w, acc);
                }
            } else {
                const float *Arow = a.A + ch * N;
                for (int64_t n = (int64_t)sl * 4; n < N; n += (int64_t)lpr * 4) {
                    float4 s4 = *reinterpret_cast<float4 *>(srow + n);
                    const float4 A4 = make_float4(Arow[n], Arow[n + 1], Arow[n + 2], Arow[n + 3]);
                    s4.x = fmaf(ex2(dl * A4.x * kLog2e), s4.x, dxv * Bs[n]);
                    s4.y = fmaf(ex2(dl * A4.y * kLog2e), s4.y, dxv * Bs[n + 1]);
                    s4.z = fmaf(ex2(dl * A4.z * kLog2e), s4.z, dxv * Bs[n + 2]);
                    s4.w = fmaf(ex2(dl * A4.w * kLog2e), s4.w, dxv * Bs[n + 3]);
                    *reinterpret_cast<float4 *>(srow + n) = s4;
                    acc = fmaf(Cs[n], s4.x, acc);
                    acc = fmaf(Cs[n + 1], s4.y, acc);
                    acc = fmaf(Cs[n + 2], s4.z, acc);
                    acc = fmaf(Cs[n + 3], s4.w, acc);
                }
            }
        } else if (row < nrows && sl == 0) {
            // dstate not a multiple of 4: one lane walks the row
            const float dl = dls[hl], xv = xs[row], dxv = dl * xv;
            float *srow = stb + ch * N;
            for (int64_t n = 0; n < N; ++n) {
                const float dA = m2 ? das[hl] : ex2(dl * a.A[ch * N + n] * kLog2e);
                const float sv = fmaf(dA, srow[n], dxv * Bs[n]);
                srow[n] = sv;
                acc = fmaf(Cs[n], sv, acc);
            }
        }
        for (int off = lpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (row < nrows && sl == 0) {
            const int64_t hh = h0 + hl;
            float yv = acc + (a.D ? a.D[hh] : 0.f) * xs[row];
            if (zr) yv *= silu(Elem<T>::ld(zr + ch));
            Elem<T>::st(yr + ch, yv);
        }
    }
}

template <typename T>
cudaError_t launch_typed(const DecArgs &a, int64_t batch, cudaStream_t st) {
    const bool m2 = a.mode == SSM_MAMBA2;
    const int64_t units = m2 ? a.G : (a.Dn + kM1Channels - 1) / kM1Channels;
    const int64_t nx = m2 ? (a.H / a.G) * a.P : kM1Channels;
    const int64_t nh = m2 ? a.H / a.G : kM1Channels;
    const size_t smem = (size_t)(((nx + 3) & ~(int64_t)3) + 2 * a.N + 2 * nh + 2 * nx) * sizeof(float);
    auto kern = decode_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)units, (unsigned)batch);
    timing_begin(st);
    kern<<<grid, kThreads, smem, st>>>(a);
    timing_end(st);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const ssm_update_args &u, cudaStream_t st) {
    if (u.batch == 0) return cudaSuccess;
    DecArgs a;
    a.state = u.state; a.conv_state = u.conv_state; a.conv_w = u.conv_w; a.conv_b = u.conv_b;
    a.x = u.x; a.z = u.z; a.dt = u.dt; a.B = u.B; a.C = u.C; a.y = u.y;
    a.x_bs = u.x_batch_stride; a.z_bs = u.z_batch_stride; a.dt_bs = u.dt_batch_stride;
    a.B_bs = u.B_batch_stride; a.C_bs = u.C_batch_stride; a.y_bs = u.y_batch_stride;
    a.A = u.A; a.D = u.D; a.dt_bias = u.dt_bias; a.idx = u.state_batch_indices;
    a.nslots = u.nslots; a.Dn = u.d_inner; a.N = u.dstate; a.Ls = u.conv_state_len;
    a.mode = u.mode; a.K = (int)u.d_conv; a.softplus = u.delta_softplus;
    if (u.mode == SSM_MAMBA2) { a.H = u.nheads; a.P = u.headdim; a.G = u.ngroups; }
    else { a.H = u.d_inner; a.P = 1; a.G = 1; }
    return u.dtype == SSM_BF16 ? launch_typed<__nv_bfloat16>(a, u.batch, st) : launch_typed<float>(a, u.batch, st);
}

}  // namespace ssm
