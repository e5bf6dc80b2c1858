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
#include <string.h>

#include "common.cuh"
#include "launch.h"
#include "tc05.cuh"

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

// In parallel over token blocks of 32 * kCdWarps tokens, when cs is wanted:
// (1) each CTA the in-block prefix of one block (the loop body above, no
// carry); (2) one thread per (row, unit) turns the blocks' last entries into
// the prefix up to there, in order, and writes the total; (3) each CTA of a
// later block adds the prefix that ends the block before it to its other
// entries.  Every entry is written by one thread of one launch, so the
// result does not depend on scheduling.
constexpr int kCdBlock = 32 * kCdWarps;

template <typename T>
__global__ void __launch_bounds__(kCdWarps * 32)
split_cum_local_kernel(const T *__restrict__ dt, int64_t dbs, int64_t dts, const float *__restrict__ dt_bias,
                       int softplus_on, int64_t U, int64_t seqlen, float *__restrict__ cum) {
    __shared__ float tot[kCdWarps][32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t u = (int64_t)blockIdx.x * 32 + lane;
    const int64_t b = blockIdx.y;
    const bool ok = u < U;
    const float bias = (ok && dt_bias) ? dt_bias[u] : 0.f;
    const int64_t tw = (int64_t)blockIdx.z * kCdBlock + 32 * w;
    const int nv = ok ? (int)max((int64_t)0, min((int64_t)32, seqlen - tw)) : 0;
    const T *p = dt + b * dbs + u + tw * dts;
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
    float off = 0.f;
#pragma unroll
    for (int k = 0; k < kCdWarps; ++k)
        if (k < w) off += tot[k][lane];
    if (ok) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < nv) cum[(b * seqlen + tw + i) * U + u] = v[i] + off;
    }
}

__global__ void split_cum_ends_kernel(int64_t batch, int64_t U, int64_t seqlen, float *__restrict__ cum,
                                      float *__restrict__ sum) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= batch * U) return;
    const int64_t b = i / U, u = i % U;
    const int64_t nblk = (seqlen + kCdBlock - 1) / kCdBlock;
    float run = 0.f;
    for (int64_t k0 = 0; k0 < nblk; k0 += 16) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int64_t k = k0 + j;
            const int64_t e = min((k + 1) * kCdBlock, seqlen) - 1;
            v[j] = k < nblk ? cum[(b * seqlen + e) * U + u] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int64_t k = k0 + j;
            if (k < nblk) {
                run += v[j];
                cum[(b * seqlen + min((k + 1) * kCdBlock, seqlen) - 1) * U + u] = run;
            }
        }
    }
    sum[b * U + u] = run;
}

__global__ void __launch_bounds__(kCdWarps * 32)
split_cum_offset_kernel(int64_t U, int64_t seqlen, float *__restrict__ cum) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t u = (int64_t)blockIdx.x * 32 + lane;
    const int64_t b = blockIdx.y;
    const int64_t blk = (int64_t)blockIdx.z + 1;            // blocks after the first
    if (u >= U) return;
    const int64_t t0 = blk * kCdBlock, tend = min(t0 + kCdBlock, seqlen) - 1;   // tend already holds its prefix
    const float off = cum[(b * seqlen + t0 - 1) * U + u];
    const int64_t tw = t0 + 32 * w;
    float v[32];                                          // every load before any store
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = tw + i < tend ? cum[(b * seqlen + tw + i) * U + u] : 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
        if (tw + i < tend) cum[(b * seqlen + tw + i) * U + u] = v[i] + off;
}

// ------------------------------------------------------------- combine
// One thread per (row, 4 consecutive state elements; the grid's y is the
// row): the pairs of segments 0..rank folded in order.  `per_unit` state
// elements share one delta unit (N for Mamba-1, P*N for Mamba-2, both
// multiples of 4 on the vector path); Mamba-1 A is indexed like the state,
// Mamba-2 A per head.  Rank k's sum_delta / h_local start sd_rs / hl_rs
// elements after rank k-1's.  Element indices within a row fit 32 bits (the
// API refuses larger states).
__global__ void split_combine_kernel(const float *__restrict__ A, int m2, const float *__restrict__ sd,
                                     const float *__restrict__ hl, float *__restrict__ h_in,
                                     float *__restrict__ h_out, int rank, uint32_t S, uint32_t U, uint32_t per_unit,
                                     int64_t sd_rs, int64_t hl_rs, bool vec4) {
    const uint32_t b = blockIdx.y;
    const int64_t row = (int64_t)b * S;
    const float *sdr = sd + (int64_t)b * U;
    if (vec4) {
        const uint32_t e = (blockIdx.x * blockDim.x + threadIdx.x) * 4u;
        if (e >= S) return;
        const uint32_t u = e / per_unit;                  // the same unit for all 4
        float4 a4;
        if (m2) a4 = make_float4(A[u], A[u], A[u], A[u]);
        else a4 = *reinterpret_cast<const float4 *>(A + e);
        float4 H = *reinterpret_cast<const float4 *>(hl + row + e);
        float4 before = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 1; k <= rank; ++k) {
            before = H;
            const float sdk = sdr[(int64_t)k * sd_rs + u] * kLog2e;
            const float4 l = *reinterpret_cast<const float4 *>(hl + (int64_t)k * hl_rs + row + e);
            H.x = fmaf(ex2(a4.x * sdk), H.x, l.x);
            H.y = fmaf(ex2(a4.y * sdk), H.y, l.y);
            H.z = fmaf(ex2(a4.z * sdk), H.z, l.z);
            H.w = fmaf(ex2(a4.w * sdk), H.w, l.w);
        }
        if (h_in) *reinterpret_cast<float4 *>(h_in + row + e) = before;
        if (h_out) *reinterpret_cast<float4 *>(h_out + row + e) = H;
        return;
    }
    const uint32_t e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= S) return;
    const uint32_t u = e / per_unit;
    const float a = m2 ? A[u] : A[e];
    float H = hl[row + e];
    float before = 0.f;
    for (int k = 1; k <= rank; ++k) {
        before = H;
        const float decay = ex2(a * sdr[(int64_t)k * sd_rs + u] * kLog2e);
        H = fmaf(decay, H, hl[(int64_t)k * hl_rs + row + e]);
    }
    if (h_in) h_in[row + e] = before;
    if (h_out) h_out[row + e] = H;
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

// ------------------------------------------- fix-up, Mamba-2 on the tensor cores
// The same fix-up as a matrix product per head: for a tile of 128 tokens of
// one (row, group), Yh = C' h_in^T with C' the group's conv'd C rows (128 x N,
// bf16, K-major) and h_in^T (N x P, bf16, MN-major), one tcgen05 chain of
// eight K = 16 MMAs into a 128 x 64 fp32 tensor-memory accumulator; then
// y_t += exp(A cs_t) silu(z_t) Yh_t.  Shapes of the tensor-core scan (bf16,
// P = 64, N = 128).  The CTA builds C' once (raw rows staged in shared memory,
// conv + SiLU into the 128-byte-swizzled operand tile) and walks the group's
// heads.  Per head the y and z tiles (128 tokens x 64 channels) come in and y
// goes out by TMA (rows past the segment are zero-filled on the way in and
// clipped on the way out; y double-buffered), so each thread updates its
// token's row in shared memory.  While head h's epilogue runs, head h+1's
// state is already on its way into registers and its z and y tiles into
// shared memory; its state tile is written, and its MMAs issued, right after.
// A wait that runs out (two seconds; not expected) stores the tile's y as NaN
// instead of fixing it.
constexpr int kFtTok = 128;                       // tokens per CTA (the MMA's M)
constexpr int kFtP = 64, kFtN = 128;
constexpr int kFtThreads = 256;
constexpr uint32_t FT_OFF_A = 0;                  // C' tile: two K-atoms of 128 rows x 64 n (16 KB each)
constexpr uint32_t FT_OFF_B = 32768;              // h_in^T tile: 128 n rows x 64 p (16 KB)
constexpr uint32_t FT_OFF_R = 32768;              // raw C rows, bf16 [kFtTok + K - 1][N], before the tiles below
constexpr uint32_t FT_OFF_Z = 49152;              // z tile, 128 rows x 64 p (128-byte swizzle)
constexpr uint32_t FT_OFF_Y = 65536;              // two y tiles, same layout
constexpr uint32_t FT_OFF_AUX = 98304;
static_assert(FT_OFF_R + (kFtTok + kMaxConvWidth - 1) * kFtN * 2 <= FT_OFF_AUX, "raw rows overflow");
enum { FB_MMA0, FB_MMA1, FB_Z, FB_Y0, FB_Y1, FB_DRAIN, kNumFtBar };
struct FtAux {
    uint32_t tmem;
    int abort;
    uint64_t mb[kNumFtBar];
};
constexpr size_t kFtSmemBytes = FT_OFF_AUX + sizeof(FtAux) + 1024;
constexpr uint32_t ID_FT = tc::idesc_bf16(128, 64, 0, 1);

SSM_DEVINL bool ft_wait(FtAux &ax, int i, uint32_t parity) {
    if (tc::mbar_try_wait(&ax.mb[i], parity)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    for (;;) {
        if (*reinterpret_cast<volatile int *>(&ax.abort)) return false;
        if (tc::mbar_try_wait(&ax.mb[i], parity)) return true;
        if (tc::globaltimer_ns() - t0 > 2000000000ull) break;
    }
    *reinterpret_cast<volatile int *>(&ax.abort) = 1;
    return false;
}

__global__ void __launch_bounds__(kFtThreads, 2)
split_fixup_tc_kernel(const FixArgs f, const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_z) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    FtAux &ax = *reinterpret_cast<FtAux *>(smem + FT_OFF_AUX);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t g = blockIdx.x, b = blockIdx.z;
    const int64_t t0 = (int64_t)blockIdx.y * kFtTok;
    const int nt = (int)min((int64_t)kFtTok, f.seqlen - t0);
    const int64_t hpg = f.H / f.G;
    const int K = (int)f.K, Ke = K > 0 ? K : 1;
    const bool zg = f.z != nullptr;
    if (!SSM_BOUNDS(t0 + nt - 1, f.seqlen, BS_SPLIT_ROW) || !SSM_BOUNDS((g + 1) * kFtN - 1, f.G * kFtN, BS_SPLIT_CHANNEL))
        return;
    const __nv_bfloat16 *Cb = static_cast<const __nv_bfloat16 *>(f.C) + b * f.cbs + g * kFtN;
    const __nv_bfloat16 *si = static_cast<const __nv_bfloat16 *>(f.conv_state_in);
    if (tid == 0) {
        ax.abort = 0;
        for (int i = 0; i < kNumFtBar; ++i) tc::mbar_init(&ax.mb[i], 1);
        tc::mbar_init_fence();
        tc::prefetch_map(&tm_y);
        if (zg) tc::prefetch_map(&tm_z);
    }
    if (warp == 0) tc::tmem_alloc(&ax.tmem, 128);
    // raw C rows of the tile: tokens t0 - (Ke - 1) .. t0 + kFtTok - 1, 16 bytes (8 channels) per load,
    // every load of a thread issued before its stores
    const int R = kFtTok + Ke - 1;
    unsigned char *raw = smem + FT_OFF_R;
    {
        constexpr int kMaxIt = ((kFtTok + kMaxConvWidth - 1) * (kFtN / 8) + kFtThreads - 1) / kFtThreads;
        uint4 v[kMaxIt];
#pragma unroll
        for (int it = 0; it < kMaxIt; ++it) {
            const int i = tid + it * kFtThreads;
            const int r = i / (kFtN / 8), c8 = i % (kFtN / 8);
            const int64_t tau = t0 - (Ke - 1) + r;
            v[it] = make_uint4(0, 0, 0, 0);
            if (r < R) {
                if (tau >= 0 && tau < f.seqlen) {
                    v[it] = *reinterpret_cast<const uint4 *>(Cb + tau * f.cts + c8 * 8);
                } else if (tau < 0 && si) {
                    // before the segment: the carried conv state [row][channel][K-1]
                    alignas(16) __nv_bfloat16 e[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int64_t ch = f.H * f.P + f.G * kFtN + g * kFtN + c8 * 8 + j;
                        e[j] = si[(b * f.cdim + ch) * (K - 1) + (tau + K - 1)];
                    }
                    v[it] = *reinterpret_cast<const uint4 *>(e);
                }
            }
        }
#pragma unroll
        for (int it = 0; it < kMaxIt; ++it) {
            const int i = tid + it * kFtThreads;
            const int r = i / (kFtN / 8), c8 = i % (kFtN / 8);
            if (r < R) *reinterpret_cast<uint4 *>(raw + r * (kFtN * 2) + c8 * 16) = v[it];
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ax.tmem;
    // C' = SiLU(conv(C)) (or C itself without a conv): thread -> 8 channels c8 of rows tid / 16 + 16 i;
    // rows past the segment are zero
    {
        const int c8 = tid % (kFtN / 8);
        float w[kMaxConvWidth][8], bias[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t ch = f.H * f.P + f.G * kFtN + g * kFtN + c8 * 8 + j;
#pragma unroll
            for (int k = 0; k < kMaxConvWidth; ++k) w[k][j] = k < K ? f.conv_w[ch * K + k] : 0.f;
            bias[j] = (K > 0 && f.conv_b) ? f.conv_b[ch] : 0.f;
        }
        for (int t = tid / (kFtN / 8); t < kFtTok; t += kFtThreads / (kFtN / 8)) {
            float o[8];
            if (K > 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j) o[j] = bias[j];
#pragma unroll
                for (int k = 0; k < kMaxConvWidth; ++k) {
                    if (k < K) {
                        float v[8];
                        tc::unpack_bf16x8(*reinterpret_cast<const uint4 *>(raw + (t + k) * (kFtN * 2) + c8 * 16), v);
#pragma unroll
                        for (int j = 0; j < 8; ++j) o[j] = fmaf(w[k][j], v[j], o[j]);
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) o[j] = silu_fast<__nv_bfloat16>(o[j]);
            } else {
                tc::unpack_bf16x8(*reinterpret_cast<const uint4 *>(raw + t * (kFtN * 2) + c8 * 16), o);
            }
            if (t >= nt) {
#pragma unroll
                for (int j = 0; j < 8; ++j) o[j] = 0.f;
            }
            *reinterpret_cast<uint4 *>(smem + FT_OFF_A + tc::off_sw128(t, c8 * 8, 16384)) = tc::pack_bf16x8(o);
        }
    }
    // the raw rows are consumed: the state, z and y tiles may take their space
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    auto load_z = [&](int64_t h) {
        if (!zg) return;
        tc::mbar_expect_tx(&ax.mb[FB_Z], kFtTok * kFtP * 2);
        tc::tma_load_3d(smem + FT_OFF_Z, &tm_z, (int)(h * kFtP), (int)t0, (int)b, &ax.mb[FB_Z]);
    };
    auto load_y = [&](int64_t h, int yb) {
        tc::mbar_expect_tx(&ax.mb[FB_Y0 + yb], kFtTok * kFtP * 2);
        tc::tma_load_3d(smem + FT_OFF_Y + yb * 16384, &tm_y, (int)(h * kFtP), (int)t0, (int)b, &ax.mb[FB_Y0 + yb]);
    };
    if (tid == 0) {
        load_z(g * hpg);
        load_y(g * hpg, 0);
    }
    // h_in^T of one head: rows n, 64 p (MN-major).  Lanes over n keep the loads
    // coalesced; a thread's 32 loads are issued together (fetch), converted and
    // stored once the tile is free (put).
    constexpr int kIt = kFtN * (kFtP / 8) / kFtThreads;
    float hv[kIt][8];
    auto fetch_state = [&](int64_t h) {
        const float *hb = f.h_in + (b * f.H + h) * kFtP * kFtN;
#pragma unroll
        for (int it = 0; it < kIt; ++it) {
            const int i = tid + it * kFtThreads, n = i % kFtN, p8 = i / kFtN;
#pragma unroll
            for (int j = 0; j < 8; ++j) hv[it][j] = hb[(int64_t)(p8 * 8 + j) * kFtN + n];
        }
    };
    auto put_state = [&]() {
#pragma unroll
        for (int it = 0; it < kIt; ++it) {
            const int i = tid + it * kFtThreads, n = i % kFtN, p8 = i / kFtN;
            *reinterpret_cast<uint4 *>(smem + FT_OFF_B + tc::off_sw128(n, p8 * 8, 8192)) = tc::pack_bf16x8(hv[it]);
        }
    };
    const uint32_t sbase = tc::smem_u32(smem);
    const uint64_t dA = tc::desc_sw128(sbase + FT_OFF_A, 16, 1024);
    const uint64_t dB = tc::desc_sw128(sbase + FT_OFF_B, 8192, 1024);
    auto issue = [&](int bb) {
#pragma unroll
        for (int kk = 0; kk < kFtN / 16; ++kk)
            tc::mma_bf16(tmem + bb * 64, dA + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), dB + kk * 128, ID_FT, kk > 0);
        tc::mma_commit(&ax.mb[FB_MMA0 + bb]);
    };
    fetch_state(g * hpg);
    put_state();
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) issue(0);

    // epilogue mapping: warp quarter q4 -> tokens 32 q4 .. 32 q4 + 31 (lane = token), half -> p 32 half ..
    const int q4 = warp & 3, half = warp >> 2;
    const int t = q4 * 32 + lane;
    const float *cum_t = f.cum + (b * f.seqlen + t0 + t) * f.H;
    float cum_next = t < nt ? cum_t[g * hpg] : 0.f;
    for (int64_t hi = 0; hi < hpg; ++hi) {
        const int64_t h = g * hpg + hi;
        const int bb = (int)(hi & 1), yb = (int)(hi & 1);
        const bool more = hi + 1 < hpg;
        const float cum_h = cum_next;
        if (more) {
            if (t < nt) cum_next = cum_t[h + 1];
            fetch_state(h + 1);                  // in flight during this head's epilogue
        }
        bool ok = ft_wait(ax, FB_MMA0 + bb, (uint32_t)(hi >> 1) & 1u);
        ok = ft_wait(ax, FB_Y0 + yb, (uint32_t)(hi >> 1) & 1u) && ok;
        if (zg) ok = ft_wait(ax, FB_Z, (uint32_t)hi & 1u) && ok;
        ok = __all_sync(0xffffffffu, ok);
        tc::fence_after_sync();
        const float e = ex2(f.A[h] * kLog2e * cum_h);
        float acc[32];
        if (ok) tc::tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + bb * 64 + half * 32, acc);
        unsigned char *ytile = smem + FT_OFF_Y + yb * 16384;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t off = (uint32_t)(t >> 3) * 1024u + (uint32_t)(t & 7) * 128u +
                                 ((uint32_t)((half * 4 + q) ^ (t & 7)) << 4);
            float yv[8], zv[8], o[8];
            tc::unpack_bf16x8(*reinterpret_cast<const uint4 *>(ytile + off), yv);
            if (zg) tc::unpack_bf16x8(*reinterpret_cast<const uint4 *>(smem + FT_OFF_Z + off), zv);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                o[j] = ok ? fmaf(e * (zg ? silu_fast<__nv_bfloat16>(zv[j]) : 1.f), acc[q * 8 + j], yv[j])
                          : __int_as_float(0x7fc00000);
            *reinterpret_cast<uint4 *>(ytile + off) = tc::pack_bf16x8(o);
        }
        // head hi+1's state tile (MMA(hi) has read the previous one)
        if (more) put_state();
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (tid == 0) {
            tc::tma_store_3d(&tm_y, (int)(h * kFtP), (int)t0, (int)b, ytile);
            if (more) {
                load_z(h + 1);                    // the epilogue has read z
                if (!*reinterpret_cast<volatile int *>(&ax.abort)) issue(bb ^ 1);
                tc::bulk_wait_read_1();           // y tile yb ^ 1 (stored one head ago) has been read
                load_y(h + 1, yb ^ 1);
            }
        }
    }
    if (tid == 0) {
        tc::bulk_wait_all();
        if (*reinterpret_cast<volatile int *>(&ax.abort)) {
            tc::mma_commit(&ax.mb[FB_DRAIN]);
            tc::mbar_wait(&ax.mb[FB_DRAIN], 0, 1u << 22);
            tc::mbar_wait(&ax.mb[FB_Z], (uint32_t)(hpg - 1) & 1u, 1u << 22);
            tc::mbar_wait(&ax.mb[FB_Y0 + (int)((hpg - 1) & 1)], (uint32_t)((hpg - 1) >> 1) & 1u, 1u << 22);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 128);
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
    const int64_t nblk = (a.seqlen + kCdBlock - 1) / kCdBlock;
    if (cum && nblk > 1 && nblk <= 65535) {
        const dim3 g1((unsigned)((U + 31) / 32), (unsigned)a.batch, (unsigned)nblk);
        split_cum_local_kernel<T><<<g1, kCdWarps * 32, 0, st>>>(static_cast<const T *>(a.dt), a.dt_batch_stride,
                                                               a.dt_token_stride, a.dt_bias, a.delta_softplus, U,
                                                               a.seqlen, cum);
        const int64_t n = a.batch * U;
        split_cum_ends_kernel<<<(unsigned)((n + 127) / 128), 128, 0, st>>>(a.batch, U, a.seqlen, cum, sum);
        const dim3 g3((unsigned)((U + 31) / 32), (unsigned)a.batch, (unsigned)(nblk - 1));
        split_cum_offset_kernel<<<g3, kCdWarps * 32, 0, st>>>(U, a.seqlen, cum);
        return cudaGetLastError();
    }
    dim3 grid((unsigned)((U + 31) / 32), (unsigned)a.batch);
    split_cum_delta_kernel<T><<<grid, kCdWarps * 32, 0, st>>>(static_cast<const T *>(a.dt), a.dt_batch_stride,
                                                              a.dt_token_stride, a.dt_bias, a.delta_softplus, U,
                                                              a.seqlen, cum, sum);
    return cudaGetLastError();
}

// The tensor-core fix-up takes the tensor-core scan's shapes with 16-byte
// aligned C, y and z rows (its loads and stores move 8 channels at a time).
bool fixup_tc_ok(const ssm_scan_args &a) {
    auto al16 = [](const void *p) { return p == nullptr || ((uintptr_t)p & 15) == 0; };
    auto st8 = [](int64_t v) { return v % 8 == 0; };
    return a.mode == SSM_MAMBA2 && a.dtype == SSM_BF16 && a.headdim == kFtP && a.dstate == kFtN &&
           a.d_conv <= kMaxConvWidth && al16(a.C) && al16(a.y) && al16(a.z) && st8(a.C_token_stride) &&
           st8(a.C_batch_stride) && st8(a.y_token_stride) && st8(a.y_batch_stride) &&
           (a.z == nullptr || (st8(a.z_token_stride) && st8(a.z_batch_stride)));
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
    if (fixup_tc_ok(a)) {
        CUtensorMap tm_y, tm_z;
        memset(&tm_y, 0, sizeof(tm_y));
        memset(&tm_z, 0, sizeof(tm_z));
        if (!make_map_box(&tm_y, a.y, a.d_inner, a.seqlen, a.batch, a.y_token_stride, a.y_batch_stride, true, kFtTok) ||
            (a.z && !make_map_box(&tm_z, a.z, a.d_inner, a.seqlen, a.batch, a.z_token_stride, a.z_batch_stride, true,
                                  kFtTok)))
            return cudaErrorInvalidValue;
        cudaError_t e = cudaFuncSetAttribute(split_fixup_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kFtSmemBytes);
        if (e != cudaSuccess) return e;
        dim3 grid((unsigned)a.ngroups, (unsigned)((a.seqlen + kFtTok - 1) / kFtTok), (unsigned)a.batch);
        timing_begin(st);
        split_fixup_tc_kernel<<<grid, kFtThreads, kFtSmemBytes, st>>>(f, tm_y, tm_z);
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
    const int64_t U = m2 ? a.nheads : a.d_inner;
    const int64_t per_unit = m2 ? a.headdim * a.dstate : a.dstate;
    if (a.batch * S == 0) return cudaSuccess;
    const int64_t sd_rs = a.sum_delta_rank_stride > 0 ? a.sum_delta_rank_stride : a.batch * U;
    const int64_t hl_rs = a.h_local_rank_stride > 0 ? a.h_local_rank_stride : a.batch * S;
    // 16-byte accesses when every row and rank block starts on a 16-byte boundary
    // and 4 consecutive elements share their delta unit
    const bool vec4 = per_unit % 4 == 0 && S % 4 == 0 && hl_rs % 4 == 0 && ((uintptr_t)a.h_local % 16) == 0 &&
                      ((uintptr_t)a.h_in % 16) == 0 && ((uintptr_t)a.h_out % 16) == 0 &&
                      (m2 || ((uintptr_t)a.A % 16) == 0);
    const int64_t per_row = vec4 ? S / 4 : S;
    const dim3 grid((unsigned)((per_row + 255) / 256), (unsigned)a.batch);
    split_combine_kernel<<<grid, 256, 0, st>>>(a.A, m2, a.sum_delta, a.h_local, a.h_in, a.h_out, a.rank,
                                               (uint32_t)S, (uint32_t)U, (uint32_t)per_unit, sd_rs, hl_rs, vec4);
    return cudaGetLastError();
}

cudaError_t launch_split_fixup(const ssm_scan_args &a, const float *cum, const float *h_in, cudaStream_t st) {
    return a.dtype == SSM_BF16 ? fixup_typed<__nv_bfloat16>(a, cum, h_in, st) : fixup_typed<float>(a, cum, h_in, st);
}

}  // namespace ssm
