// seq_split.cu -- joining a batch of sequences whose tokens were scanned in
// contiguous segments, one per rank: the conv tail a segment hands to the
// next, the in-segment prefix sums of delta, the combine of every segment's
// (decay, end state) pair, and the fix-up of y by the state entering the
// segment.
//
// The scan element (exp(delta*A), h) composes associatively with seed
// (1, h0) ("Adding Initial Value Support to Selective Scan Forward Kernel",
// state-spaces/mamba issue 285).  A segment scanned from a zero state ends in
// h_loc; started from h_in it ends in exp(A * sum delta) h_in + h_loc, and
// its state at token t differs from the zero-start one by exp(A cs_t) h_in,
// cs_t the in-segment prefix sum of delta.  The read-out is linear in the
// state, so y_t differs by silu(z_t) * C_t . (exp(A cs_t) h_in).
#include "common.cuh"
#include "launch.h"

namespace ssm {
namespace {

// ---------------------------------------------------------------- tail
// The activation tensors the conv channels come from: channels [0, w0) of
// p[0], the next w1 of p[1], the rest of p[2] (Mamba-2 x | B | C; Mamba-1
// uses p[0] only).
struct ConvSrc {
    const void *p[3];
    int64_t bs[3], ts[3];
    int64_t w0, w1;
};

// One thread per (row, conv channel): the K-1 raw inputs that end the
// segment, oldest first; positions before its first token read the carried
// state (or 0).
template <typename T>
__global__ void split_tail_kernel(ConvSrc s, const T *__restrict__ state_in, T *__restrict__ tail, int64_t batch,
                                  int64_t seqlen, int64_t cdim, int K) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= batch * cdim) return;
    const int64_t b = i / cdim, c = i % cdim;
    const int j = c < s.w0 ? 0 : (c < s.w0 + s.w1 ? 1 : 2);
    const int64_t col = j == 0 ? c : (j == 1 ? c - s.w0 : c - s.w0 - s.w1);
    const void *base = j == 0 ? s.p[0] : (j == 1 ? s.p[1] : s.p[2]);
    const int64_t bs = j == 0 ? s.bs[0] : (j == 1 ? s.bs[1] : s.bs[2]);
    const int64_t ts = j == 0 ? s.ts[0] : (j == 1 ? s.ts[1] : s.ts[2]);
    const T *src = static_cast<const T *>(base) + b * bs + col;
    for (int q = 0; q < K - 1; ++q) {
        const int64_t tau = seqlen - (K - 1) + q;
        float v = 0.f;
        if (tau >= 0)
            v = Elem<T>::ld(src + tau * ts);
        else if (state_in)
            v = Elem<T>::ld(state_in + i * (K - 1) + (tau + K - 1));
        Elem<T>::st(tail + i * (K - 1) + q, v);
    }
}

// ----------------------------------------------------------- cum delta
// A CTA owns 32 delta units of one row and walks the tokens in tiles of
// 8 warps x 32 tokens: each lane issues its 32 loads, then sums its unit over
// its warp's 32 tokens in registers; the warps' totals go through shared
// memory, and a running carry joins the tiles.  Loads and stores are 32
// consecutive units wide.
constexpr int kCdWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kCdWarps * 32)
split_cum_delta_kernel(const T *__restrict__ dt, int64_t dbs, int64_t dts, const float *__restrict__ dt_bias,
                       int softplus_on, int64_t U, int64_t seqlen, float *__restrict__ cum,
                       float *__restrict__ sum) {
    __shared__ float tot[kCdWarps][32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t u = (int64_t)blockIdx.x * 32 + lane;
    const int64_t b = blockIdx.y;
    const bool ok = u < U;
    const float bias = (ok && dt_bias) ? dt_bias[u] : 0.f;
    const T *src = dt + b * dbs + u;
    float carry = 0.f;
    for (int64_t t0 = 0; t0 < seqlen; t0 += 32 * kCdWarps) {
        const int64_t tw = t0 + 32 * w;
        const int nv = ok ? (int)max((int64_t)0, min((int64_t)32, seqlen - tw)) : 0;
        const T *p = src + tw * dts;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = i < nv ? Elem<T>::ld(p + i * dts) : 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i < nv) {
                const float r = v[i] + bias;
                v[i] = softplus_on ? softplus(r) : r;
            }
        }
#pragma unroll
        for (int i = 1; i < 32; ++i) v[i] += v[i - 1];
        tot[w][lane] = v[31];
        __syncthreads();
        float off = carry, all = 0.f;
#pragma unroll
        for (int k = 0; k < kCdWarps; ++k) {
            const float x = tot[k][lane];
            if (k < w) off += x;
            all += x;
        }
        __syncthreads();                                  // tot is rewritten by the next tile
        carry += all;
        if (cum && ok) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (tw + i < seqlen) cum[(b * seqlen + tw + i) * U + u] = v[i] + off;
        }
    }
    if (ok && w == 0) sum[b * U + u] = carry;
}

// ------------------------------------------------------------- combine
// One thread per (row, state element): the pairs of segments 0..rank folded
// in order.  `per_unit` state elements share one delta unit (N for Mamba-1,
// P*N for Mamba-2); Mamba-1 A is indexed like the state, Mamba-2 A per head.
__global__ void split_combine_kernel(const float *__restrict__ A, int m2, const float *__restrict__ sd,
                                     const float *__restrict__ hl, float *__restrict__ h_in,
                                     float *__restrict__ h_out, int rank, int64_t batch, int64_t S, int64_t U,
                                     int64_t per_unit) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= batch * S) return;
    const int64_t b = i / S, e = i % S;
    const int64_t u = e / per_unit;
    const float a = m2 ? A[u] : A[e];
    float H = hl[i];
    float before = 0.f;
    for (int k = 1; k <= rank; ++k) {
        before = H;
        const float decay = ex2(a * sd[((int64_t)k * batch + b) * U + u] * kLog2e);
        H = fmaf(decay, H, hl[(int64_t)k * batch * S + i]);
    }
    if (h_in) h_in[i] = before;
    if (h_out) h_out[i] = H;
}

// ------------------------------------------------------- fix-up, Mamba-1
// A CTA covers 128 channels x 16 tokens of one row.  The C rows of the 16
// tokens sit in shared memory; each thread keeps its channel's 16 prefix
// sums and partial corrections in registers and walks the states.
constexpr int kF1Tok = 16;
constexpr int kF1Threads = 128;

struct FixArgs {
    const void *y; int64_t ybs, yts;
    const void *z; int64_t zbs, zts;
    const void *C; int64_t cbs, cts;
    const float *A, *cum, *h_in;
    const float *conv_w, *conv_b;
    const void *conv_state_in;
    int64_t seqlen, D, N, H, P, G, K, cdim;
};

template <typename T>
__global__ void __launch_bounds__(kF1Threads) split_fixup_m1_kernel(FixArgs f) {
    __shared__ float crow[kF1Tok][kMaxDstateM1];
    const int64_t d = (int64_t)blockIdx.x * kF1Threads + threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.y * kF1Tok;
    const int64_t b = blockIdx.z;
    const int N = (int)f.N;
    const int nt = (int)min((int64_t)kF1Tok, f.seqlen - t0);
    const T *Cb = static_cast<const T *>(f.C) + b * f.cbs;
    for (int idx = threadIdx.x; idx < nt * N; idx += kF1Threads) {
        const int t = idx / N, n = idx % N;
        crow[t][n] = Elem<T>::ld(Cb + (t0 + t) * f.cts + n);
    }
    __syncthreads();
    if (d >= f.D) return;
    float cs[kF1Tok], acc[kF1Tok];
#pragma unroll
    for (int t = 0; t < kF1Tok; ++t) {
        cs[t] = t < nt ? f.cum[(b * f.seqlen + t0 + t) * f.D + d] * kLog2e : 0.f;
        acc[t] = 0.f;
    }
    const float *Ad = f.A + d * N;
    const float *hd = f.h_in + (b * f.D + d) * N;
#pragma unroll 4
    for (int n = 0; n < N; ++n) {
        const float a = Ad[n], hv = hd[n];
#pragma unroll
        for (int t = 0; t < kF1Tok; ++t) acc[t] = fmaf(crow[t][n] * ex2(a * cs[t]), hv, acc[t]);
    }
    T *yb = static_cast<T *>(const_cast<void *>(f.y)) + b * f.ybs + d;
    const T *zb = f.z ? static_cast<const T *>(f.z) + b * f.zbs + d : nullptr;
#pragma unroll
    for (int t = 0; t < kF1Tok; ++t) {
        if (t >= nt) break;
        const float g = zb ? silu(Elem<T>::ld(zb + (t0 + t) * f.zts)) : 1.f;
        T *yp = yb + (t0 + t) * f.yts;
        Elem<T>::st(yp, fmaf(g, acc[t], Elem<T>::ld(yp)));
    }
}

// ------------------------------------------------------- fix-up, Mamba-2
// A CTA covers 64 tokens of one (row, group) and walks the group's heads.
// The group's raw C rows (from K-1 tokens before the tile, the carried conv
// state where those precede the segment) are staged once, then convolved
// (+ SiLU) into the 64 C rows; per head and per 64 head channels, the
// entering state is staged transposed ([n][p], row stride 65: the coalesced
// fill and the reads are both conflict-free).  Every staging loop keeps 8 or
// 16 loads in flight per thread.  Warp w owns tokens 16w..16w+15, lane l
// channels l and l+32: 32 accumulators per thread, C read as broadcast float4
// along n when N % 4 == 0.
constexpr int kF2Tok = 64;
constexpr int kF2P = 64;
constexpr int kF2Stride = kF2P + 1;
constexpr int kF2Threads = 128;
constexpr int kF2TokPerWarp = kF2Tok / (kF2Threads / 32);

// C rows, then one region that first holds the staged raw C rows (at most
// kF2Tok + 7 of them) and later the transposed state
inline size_t fixup_m2_smem(int64_t N) {
    return (size_t)(kF2Tok * N + N * (kF2Tok + kMaxConvWidth - 1 > kF2Stride ? kF2Tok + kMaxConvWidth - 1 : kF2Stride)) *
           sizeof(float);
}

template <typename T, bool V4>
__global__ void __launch_bounds__(kF2Threads) split_fixup_m2_kernel(FixArgs f) {
    extern __shared__ __align__(16) float sm[];
    const int N = (int)f.N;
    float *Cs = sm;                      // [kF2Tok][N]
    float *Hs = sm + kF2Tok * N;         // [N][kF2Stride]
    float *Rs = Hs;                      // [kF2Tok + K - 1][N] raw rows, before the first head
    const int64_t g = blockIdx.x;
    const int64_t t0 = (int64_t)blockIdx.y * kF2Tok;
    const int64_t b = blockIdx.z;
    const int64_t hpg = f.H / f.G;
    const int nt = (int)min((int64_t)kF2Tok, f.seqlen - t0);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const T *Cb = static_cast<const T *>(f.C) + b * f.cbs;
    const T *si = static_cast<const T *>(f.conv_state_in);
    const int K = (int)f.K;
    const int Ke = K > 0 ? K : 1;                    // rows of history per output (no conv: the row itself)
    const int R = kF2Tok + Ke - 1;                   // staged raw rows: tokens t0-Ke+1 .. t0+kF2Tok-1
    for (int n = lane; n < N; n += 32) {
        const int64_t col = g * N + n;
        const int64_t ch = f.H * f.P + f.G * N + col;   // conv channel of this C column
        for (int r0 = warp; r0 < R; r0 += 8 * (kF2Threads / 32)) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = r0 + j * (kF2Threads / 32);
                const int64_t tau = t0 - (Ke - 1) + r;
                float u = 0.f;
                if (r < R && tau < f.seqlen) {
                    if (tau >= 0)
                        u = Elem<T>::ld(Cb + tau * f.cts + col);
                    else if (si)
                        u = Elem<T>::ld(si + (b * f.cdim + ch) * (K - 1) + (tau + K - 1));
                }
                v[j] = u;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = r0 + j * (kF2Threads / 32);
                if (r < R) Rs[r * N + n] = v[j];
            }
        }
    }
    __syncthreads();
    for (int n = lane; n < N; n += 32) {
        const int64_t ch = f.H * f.P + f.G * N + g * N + n;
        float w[kMaxConvWidth];
#pragma unroll
        for (int k = 0; k < kMaxConvWidth; ++k) w[k] = (k < K) ? f.conv_w[ch * K + k] : 0.f;
        const float bias = (K > 0 && f.conv_b) ? f.conv_b[ch] : 0.f;
        for (int t = warp; t < kF2Tok; t += kF2Threads / 32) {
            float v = 0.f;
            if (t < nt) {
                if (K > 0) {
                    float acc = bias;
#pragma unroll
                    for (int k = 0; k < kMaxConvWidth; ++k)
                        if (k < K) acc = fmaf(w[k], Rs[(t + k) * N + n], acc);
                    v = silu(acc);
                } else {
                    v = Rs[t * N + n];
                }
            }
            Cs[t * N + n] = v;
        }
    }
    const int tb = warp * kF2TokPerWarp;
    for (int64_t hi = 0; hi < hpg; ++hi) {
        const int64_t h = g * hpg + hi;
        const float ah = f.A[h] * kLog2e;
        const float *hb = f.h_in + (b * f.H + h) * f.P * N;
        T *yb = static_cast<T *>(const_cast<void *>(f.y)) + b * f.ybs + h * f.P;
        const T *zb = f.z ? static_cast<const T *>(f.z) + b * f.zbs + h * f.P : nullptr;
        for (int64_t p0 = 0; p0 < f.P; p0 += kF2P) {
            __syncthreads();                              // Cs built (Rs consumed) / the previous Hs consumed
            for (int n = lane; n < N; n += 32) {
                constexpr int kRows = kF2P / (kF2Threads / 32);
                float v[kRows];
#pragma unroll
                for (int j = 0; j < kRows; ++j) {
                    const int p = warp + j * (kF2Threads / 32);
                    v[j] = (p0 + p < f.P) ? hb[(p0 + p) * N + n] : 0.f;
                }
#pragma unroll
                for (int j = 0; j < kRows; ++j) Hs[n * kF2Stride + warp + j * (kF2Threads / 32)] = v[j];
            }
            __syncthreads();
            float a0[kF2TokPerWarp], a1[kF2TokPerWarp];
#pragma unroll
            for (int i = 0; i < kF2TokPerWarp; ++i) a0[i] = a1[i] = 0.f;
            if constexpr (V4) {
                for (int n = 0; n < N; n += 4) {
                    float h0v[4], h1v[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        h0v[j] = Hs[(n + j) * kF2Stride + lane];
                        h1v[j] = Hs[(n + j) * kF2Stride + lane + 32];
                    }
#pragma unroll
                    for (int i = 0; i < kF2TokPerWarp; ++i) {
                        const float4 c = *reinterpret_cast<const float4 *>(&Cs[(tb + i) * N + n]);
                        a0[i] = fmaf(c.x, h0v[0], a0[i]); a1[i] = fmaf(c.x, h1v[0], a1[i]);
                        a0[i] = fmaf(c.y, h0v[1], a0[i]); a1[i] = fmaf(c.y, h1v[1], a1[i]);
                        a0[i] = fmaf(c.z, h0v[2], a0[i]); a1[i] = fmaf(c.z, h1v[2], a1[i]);
                        a0[i] = fmaf(c.w, h0v[3], a0[i]); a1[i] = fmaf(c.w, h1v[3], a1[i]);
                    }
                }
            } else {
                for (int n = 0; n < N; ++n) {
                    const float h0v = Hs[n * kF2Stride + lane], h1v = Hs[n * kF2Stride + lane + 32];
#pragma unroll
                    for (int i = 0; i < kF2TokPerWarp; ++i) {
                        const float c = Cs[(tb + i) * N + n];
                        a0[i] = fmaf(c, h0v, a0[i]);
                        a1[i] = fmaf(c, h1v, a1[i]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kF2TokPerWarp; ++i) {
                const int t = tb + i;
                if (t >= nt) break;
                const float e = ex2(ah * f.cum[(b * f.seqlen + t0 + t) * f.H + h]);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int64_t p = p0 + lane + 32 * half;
                    if (p >= f.P) continue;
                    const float gz = zb ? silu(Elem<T>::ld(zb + (t0 + t) * f.zts + p)) : 1.f;
                    T *yp = yb + (t0 + t) * f.yts + p;
                    Elem<T>::st(yp, fmaf(gz * e, half ? a1[i] : a0[i], Elem<T>::ld(yp)));
                }
            }
        }
    }
}

template <typename T>
cudaError_t tail_typed(const ssm_scan_args &a, void *tail, cudaStream_t st) {
    const bool m2 = a.mode == SSM_MAMBA2;
    const int64_t gn = (m2 ? a.ngroups : 0) * a.dstate;
    const int64_t cdim = a.d_inner + 2 * gn;
    ConvSrc s{{a.x, a.B, a.C},
              {a.x_batch_stride, a.B_batch_stride, a.C_batch_stride},
              {a.x_token_stride, a.B_token_stride, a.C_token_stride},
              a.d_inner, gn};
    const int64_t n = a.batch * cdim;
    if (n == 0) return cudaSuccess;
    split_tail_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        s, static_cast<const T *>(a.conv_state_in), static_cast<T *>(tail), a.batch, a.seqlen, cdim, (int)a.d_conv);
    return cudaGetLastError();
}

template <typename T>
cudaError_t cum_delta_typed(const ssm_scan_args &a, float *cum, float *sum, cudaStream_t st) {
    const int64_t U = a.mode == SSM_MAMBA2 ? a.nheads : a.d_inner;
    if (a.batch == 0) return cudaSuccess;
    dim3 grid((unsigned)((U + 31) / 32), (unsigned)a.batch);
    split_cum_delta_kernel<T><<<grid, kCdWarps * 32, 0, st>>>(static_cast<const T *>(a.dt), a.dt_batch_stride,
                                                              a.dt_token_stride, a.dt_bias, a.delta_softplus, U,
                                                              a.seqlen, cum, sum);
    return cudaGetLastError();
}

template <typename T>
cudaError_t fixup_typed(const ssm_scan_args &a, const float *cum, const float *h_in, cudaStream_t st) {
    if (a.batch == 0 || a.seqlen == 0) return cudaSuccess;
    const bool m2 = a.mode == SSM_MAMBA2;
    FixArgs f;
    f.y = a.y; f.ybs = a.y_batch_stride; f.yts = a.y_token_stride;
    f.z = a.z; f.zbs = a.z_batch_stride; f.zts = a.z_token_stride;
    f.C = a.C; f.cbs = a.C_batch_stride; f.cts = a.C_token_stride;
    f.A = a.A; f.cum = cum; f.h_in = h_in;
    f.conv_w = a.conv_w; f.conv_b = a.conv_b; f.conv_state_in = a.conv_state_in;
    f.seqlen = a.seqlen; f.D = a.d_inner; f.N = a.dstate;
    f.H = m2 ? a.nheads : 1; f.P = m2 ? a.headdim : 1; f.G = m2 ? a.ngroups : 1;
    f.K = a.d_conv; f.cdim = a.d_inner + (m2 ? 2 * a.ngroups * a.dstate : 0);
    if (!m2) {
        dim3 grid((unsigned)((a.d_inner + kF1Threads - 1) / kF1Threads), (unsigned)((a.seqlen + kF1Tok - 1) / kF1Tok),
                  (unsigned)a.batch);
        timing_begin(st);
        split_fixup_m1_kernel<T><<<grid, kF1Threads, 0, st>>>(f);
        timing_end(st);
        return cudaGetLastError();
    }
    const size_t smem = fixup_m2_smem(a.dstate);
    dim3 grid((unsigned)a.ngroups, (unsigned)((a.seqlen + kF2Tok - 1) / kF2Tok), (unsigned)a.batch);
    const bool v4 = a.dstate % 4 == 0;
    auto kern = v4 ? split_fixup_m2_kernel<T, true> : split_fixup_m2_kernel<T, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)fixup_m2_smem(kMaxDstateM2));
    if (e != cudaSuccess) return e;
    timing_begin(st);
    kern<<<grid, kF2Threads, smem, st>>>(f);
    timing_end(st);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_split_tail(const ssm_scan_args &a, void *tail, cudaStream_t st) {
    return a.dtype == SSM_BF16 ? tail_typed<__nv_bfloat16>(a, tail, st) : tail_typed<float>(a, tail, st);
}

cudaError_t launch_split_cum_delta(const ssm_scan_args &a, float *cum, float *sum, cudaStream_t st) {
    return a.dtype == SSM_BF16 ? cum_delta_typed<__nv_bfloat16>(a, cum, sum, st)
                               : cum_delta_typed<float>(a, cum, sum, st);
}

cudaError_t launch_split_combine(const ssm_split_args &a, cudaStream_t st) {
    const bool m2 = a.mode == SSM_MAMBA2;
    const int64_t S = a.d_inner * a.dstate;
    const int64_t n = a.batch * S;
    if (n == 0) return cudaSuccess;
    split_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        a.A, m2, a.sum_delta, a.h_local, a.h_in, a.h_out, a.rank, a.batch, S, m2 ? a.nheads : a.d_inner,
        m2 ? a.headdim * a.dstate : a.dstate);
    return cudaGetLastError();
}

cudaError_t launch_split_fixup(const ssm_scan_args &a, const float *cum, const float *h_in, cudaStream_t st) {
    return a.dtype == SSM_BF16 ? fixup_typed<__nv_bfloat16>(a, cum, h_in, st) : fixup_typed<float>(a, cum, h_in, st);
}

}  // namespace ssm
