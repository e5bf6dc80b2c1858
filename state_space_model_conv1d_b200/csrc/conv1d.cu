// conv1d.cu -- standalone causal depthwise conv (GGML_OP_SSM_CONV semantics).
//
// out[t, c] = act( bias[c] + sum_{k<K} w[c, k] * u[t-K+1+k, c] ), where u before
// a sequence's first token comes from that sequence's carried state (the last
// K-1 raw inputs, oldest first) and w[c, K-1] multiplies the current token
// ("ggml : add GPU support for Mamba models", llama.cpp issue 6758:
// SSM_CONV shapes and the concat-in-front-of-the-tokens reply).
//
// HBM-bound streaming kernel.  Each thread owns VEC consecutive channels
// (one 16-byte load of bf16, two of fp32) and a run of TT consecutive tokens,
// keeping the K-1 previous rows in registers, so every input element is read
// once from DRAM (plus a (K-1)/TT halo re-read) and every output written once.
// A warp covers 256 contiguous channels of one token: 512-byte coalesced rows.
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace ssm {
namespace {

constexpr int kThreads = 128;
constexpr int kTokensPerThread = 4;
constexpr int kRunsPerThread = 8;      // consecutive 4-token runs per thread: taps loaded once, history carried

// four CTAs per SM: short runs keep the rows in flight per thread small, and
// the extra resident warps keep more rows in flight per SM
template <typename T, int VEC, int K>
__global__ void __launch_bounds__(kThreads, 4)
conv1d_kernel(const T *__restrict__ x, int64_t x_bs, int64_t x_ts, const float *__restrict__ w,
              const float *__restrict__ bias, const T *__restrict__ state_in, int64_t ss, T *__restrict__ out,
              int64_t o_bs, int64_t o_ts, const int32_t *__restrict__ cu, int nseqs, int64_t seqlen,
              int64_t channels, int act, int vpc) {
    // a CTA covers vpc channel vectors x (kThreads / vpc) groups of token runs
    const int64_t cv = (int64_t)blockIdx.x * vpc + threadIdx.x % vpc;
    const int64_t c0 = cv * VEC;
    if (c0 >= channels) return;
    const int row = blockIdx.z;
    const int64_t grp = (int64_t)blockIdx.y * (kThreads / vpc) + threadIdx.x / vpc;
    const int64_t tr0 = grp * kTokensPerThread * kRunsPerThread;
    if (tr0 >= seqlen) return;

    float wk[K][VEC], bb[VEC];
    const bool w4 = K == 4 && ((uintptr_t)w & 15) == 0;       // each channel's 4 taps as one 16-byte load
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        if (w4) {
            const float4 q = *reinterpret_cast<const float4 *>(w + (c0 + v) * 4);
            wk[0][v] = q.x; wk[1 % K][v] = q.y; wk[2 % K][v] = q.z; wk[3 % K][v] = q.w;
        } else {
#pragma unroll
            for (int k = 0; k < K; ++k) wk[k][v] = w[(c0 + v) * K + k];
        }
        bb[v] = bias ? bias[c0 + v] : 0.f;
    }
    const T *xr = x + row * x_bs;
    T *orow = out + row * o_bs;
    float hist[K > 1 ? K - 1 : 1][VEC];
    // Offsets are clamped into [0, seqlen] so a malformed cu_seqlens can give
    // wrong values but never an out-of-bounds access.
    int s = cu ? seq_of_token(cu, nseqs, tr0) : row;
    // bounds-checked build: this thread's channels and sequence
    if (!SSM_BOUNDS(c0 + VEC - 1 < channels ? c0 + VEC - 1 : c0, channels, BS_CONV_CHANNEL) ||
        !SSM_BOUNDS(s, cu ? nseqs : (int)gridDim.z, BS_CONV_STATE))
        return;
    int64_t start = cu ? min(max((int64_t)cu[s], (int64_t)0), seqlen) : 0;
    int64_t end = cu ? min(max((int64_t)cu[s + 1], start), seqlen) : seqlen;
    auto load_hist = [&](int64_t t) {
#pragma unroll
        for (int j = 0; j < K - 1; ++j) {          // hist[j] holds time t-(K-1)+j
            const int64_t tau = t - (K - 1) + j;
            if (tau >= start) {
                if constexpr (VEC == 8) {
                    Vec8<T>::ld(xr + tau * x_ts + c0, hist[j]);
                } else {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) hist[j][v] = Elem<T>::ld(xr + tau * x_ts + c0 + v);
                }
            } else {
                const int64_t q = tau - start + (K - 1);   // index into the carried state
#pragma unroll
                for (int v = 0; v < VEC; ++v)
                    hist[j][v] = (state_in && q >= 0) ? Elem<T>::ld(state_in + (int64_t)s * ss + (c0 + v) * (K - 1) + q) : 0.f;
            }
        }
    };
    bool have_hist = false;                    // hist holds the K-1 rows before t0 of sequence s
  for (int run = 0; run < kRunsPerThread; ++run) {
    const int64_t t0 = tr0 + (int64_t)run * kTokensPerThread;
    if (t0 >= seqlen) break;
    const int64_t t1 = min(t0 + (int64_t)kTokensPerThread, seqlen);
    if (cu && t0 >= end) {                     // the run starts in a later sequence
        while (s + 1 < nseqs && cu[s + 1] <= t0) ++s;
        start = min(max((int64_t)cu[s], (int64_t)0), seqlen);
        end = min(max((int64_t)cu[s + 1], start), seqlen);
        have_hist = false;
    }
    if (!have_hist) load_hist(t0);
    have_hist = true;
    if (!cu || t1 <= end) {
        // the whole run lies in one sequence: issue every row's load before any
        // math; rows are held in their raw 16-byte form (bf16 rows take half the
        // registers of fp32 ones) and widened when used
        using Row = typename std::conditional<VEC == 8, uint4[sizeof(T) == 2 ? 1 : 2], float[VEC]>::type;
        Row cur[kTokensPerThread];
#pragma unroll
        for (int i = 0; i < kTokensPerThread; ++i) {
            if (t0 + i < t1) {
                const T *src = xr + (t0 + i) * x_ts + c0;
                if constexpr (VEC == 8) {
                    cur[i][0] = *reinterpret_cast<const uint4 *>(src);
                    if constexpr (sizeof(T) == 4) cur[i][1] = *reinterpret_cast<const uint4 *>(src + 4);
                } else {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) cur[i][v] = Elem<T>::ld(src + v);
                }
            }
        }
        auto widen = [&](const Row &r, float (&f)[VEC]) {
            if constexpr (VEC == 8 && sizeof(T) == 2) {
                const uint32_t w[4] = {r[0].x, r[0].y, r[0].z, r[0].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    f[2 * q] = __uint_as_float(w[q] << 16);
                    f[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
                }
            } else if constexpr (VEC == 8) {
                const uint4 a0 = r[0], a1 = r[1];
                f[0] = __uint_as_float(a0.x); f[1] = __uint_as_float(a0.y); f[2] = __uint_as_float(a0.z); f[3] = __uint_as_float(a0.w);
                f[4] = __uint_as_float(a1.x); f[5] = __uint_as_float(a1.y); f[6] = __uint_as_float(a1.z); f[7] = __uint_as_float(a1.w);
            } else {
#pragma unroll
                for (int v = 0; v < VEC; ++v) f[v] = r[v];
            }
        };
#pragma unroll
        for (int i = 0; i < kTokensPerThread; ++i) {
            if (t0 + i >= t1) break;
            float cf[VEC];
            widen(cur[i], cf);
            float o[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                float acc = bb[v];
#pragma unroll
                for (int k = 0; k < K - 1; ++k) acc = fmaf(wk[k][v], hist[k][v], acc);
                acc = fmaf(wk[K - 1][v], cf[v], acc);
                o[v] = act ? silu(acc) : acc;
            }
            if constexpr (VEC == 8) {
                Vec8<T>::st(orow + (t0 + i) * o_ts + c0, o);
            } else {
#pragma unroll
                for (int v = 0; v < VEC; ++v) Elem<T>::st(orow + (t0 + i) * o_ts + c0 + v, o[v]);
            }
#pragma unroll
            for (int k = 0; k + 1 < K - 1; ++k)
#pragma unroll
                for (int v = 0; v < VEC; ++v) hist[k][v] = hist[k + 1][v];
            if (K > 1)
#pragma unroll
                for (int v = 0; v < VEC; ++v) hist[K > 1 ? K - 2 : 0][v] = cf[v];
        }
        continue;
    }
    for (int64_t t = t0; t < t1; ++t) {
        if (cu && t >= end) {                      // next (non-empty) sequence of the packed row
            while (s + 1 < nseqs && cu[s + 1] <= t) ++s;
            start = min(max((int64_t)cu[s], (int64_t)0), seqlen);
            end = min(max((int64_t)cu[s + 1], start), seqlen);
            if (t < start || t >= end) return;     // malformed offsets: stop, stay in bounds
            load_hist(t);
        }
        float cur[VEC];
        if constexpr (VEC == 8) {
            Vec8<T>::ld(xr + t * x_ts + c0, cur);
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) cur[v] = Elem<T>::ld(xr + t * x_ts + c0 + v);
        }
        float o[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            float acc = bb[v];
#pragma unroll
            for (int k = 0; k < K - 1; ++k) acc = fmaf(wk[k][v], hist[k][v], acc);
            acc = fmaf(wk[K - 1][v], cur[v], acc);
            o[v] = act ? silu(acc) : acc;
        }
        if constexpr (VEC == 8) {
            Vec8<T>::st(orow + t * o_ts + c0, o);
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) Elem<T>::st(orow + t * o_ts + c0 + v, o[v]);
        }
#pragma unroll
        for (int k = 0; k + 1 < K - 1; ++k)
#pragma unroll
            for (int v = 0; v < VEC; ++v) hist[k][v] = hist[k + 1][v];
        if (K > 1)
#pragma unroll
            for (int v = 0; v < VEC; ++v) hist[K > 1 ? K - 2 : 0][v] = cur[v];
    }
  }
}

// Carried state after the sequence: the last K-1 raw inputs of
// concat(state_in, x_seq).  One thread per (sequence, channel); all reads
// happen before the writes, so state_out may alias state_in.
template <typename T>
__global__ void conv_state_out_kernel(const T *__restrict__ x, int64_t x_bs, int64_t x_ts, const T *state_in,
                                      T *state_out, int64_t ss, const int32_t *__restrict__ cu, int nseq,
                                      int64_t seqlen, int64_t channels, int K) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)nseq * channels) return;
    const int s = (int)(i / channels);
    const int64_t c = i % channels;
    const int64_t start = cu ? min(max((int64_t)cu[s], (int64_t)0), seqlen) : 0;
    const int64_t end = cu ? min(max((int64_t)cu[s + 1], start), seqlen) : seqlen;
    const T *xr = x + (cu ? 0 : (int64_t)s * x_bs);
    float v[kMaxConvWidth];
    for (int p = 0; p < K - 1; ++p) {
        const int64_t tau = end - (K - 1) + p;
        if (tau >= start) {
            v[p] = Elem<T>::ld(xr + tau * x_ts + c);
        } else {
            const int64_t q = tau - start + (K - 1);
            v[p] = (state_in && q >= 0) ? Elem<T>::ld(state_in + (int64_t)s * ss + c * (K - 1) + q) : 0.f;
        }
    }
    for (int p = 0; p < K - 1; ++p) Elem<T>::st(state_out + (int64_t)s * ss + c * (K - 1) + p, v[p]);
}

template <typename T, int VEC>
cudaError_t launch_typed_vec(const ConvJob &a, cudaStream_t st) {
    const int64_t nvec = (a.channels + VEC - 1) / VEC;
    // narrow tensors (few channel vectors) put several token-run groups in one CTA
    int vpc = kThreads;
    while (vpc / 2 >= nvec && vpc > 1) vpc /= 2;
    const int64_t per_cta = (int64_t)kTokensPerThread * kRunsPerThread * (kThreads / vpc);
    dim3 grid((unsigned)((nvec + vpc - 1) / vpc), (unsigned)((a.seqlen + per_cta - 1) / per_cta), (unsigned)a.batch);
    const T *x = static_cast<const T *>(a.x);
    const T *si = static_cast<const T *>(a.state_in);
    T *o = static_cast<T *>(a.out);
    const int ns = a.cu ? a.nseqs : (int)a.batch;
    if (grid.y > 0) {
#define SSM_CONV_CASE(KK)                                                                                    \
    case KK:                                                                                                \
        conv1d_kernel<T, VEC, KK><<<grid, kThreads, 0, st>>>(x, a.x_bs, a.x_ts, a.w, a.b, si, a.state_stride, o, \
                                                             a.o_bs, a.o_ts, a.cu, ns, a.seqlen, a.channels,   \
                                                             a.act, vpc);                                      \
        break;
        switch (a.width) {
            SSM_CONV_CASE(1) SSM_CONV_CASE(2) SSM_CONV_CASE(3) SSM_CONV_CASE(4)
            SSM_CONV_CASE(5) SSM_CONV_CASE(6) SSM_CONV_CASE(7) SSM_CONV_CASE(8)
            default: return cudaErrorInvalidValue;
        }
#undef SSM_CONV_CASE
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.state_out && a.width > 1 && ns > 0) {
        const int64_t n = (int64_t)ns * a.channels;
        conv_state_out_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            x, a.x_bs, a.x_ts, si, static_cast<T *>(a.state_out), a.state_stride, a.cu, ns, a.seqlen, a.channels,
            (int)a.width);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_typed(const ConvJob &a, cudaStream_t st) {
    const size_t es = sizeof(T);
    const bool vec_ok = a.channels % 8 == 0 && ((uintptr_t)a.x % 16 == 0) && ((uintptr_t)a.out % 16 == 0) &&
                        (a.x_ts * es) % 16 == 0 && (a.x_bs * es) % 16 == 0 &&
                        (a.o_ts * es) % 16 == 0 && (a.o_bs * es) % 16 == 0;
    return vec_ok ? launch_typed_vec<T, 8>(a, st) : launch_typed_vec<T, 1>(a, st);
}

}  // namespace

cudaError_t launch_conv_job(const ConvJob &j, cudaStream_t st) {
    return j.dtype == SSM_BF16 ? launch_typed<__nv_bfloat16>(j, st) : launch_typed<float>(j, st);
}

cudaError_t launch_conv1d(const ssm_conv_args &a, cudaStream_t st) {
    ConvJob j;
    j.x = a.x; j.x_bs = a.x_batch_stride; j.x_ts = a.x_token_stride;
    j.w = a.weight; j.b = a.bias;
    j.state_in = a.state_in; j.state_out = a.state_out; j.state_stride = a.channels * (a.width - 1);
    j.cu = a.cu_seqlens; j.nseqs = a.nseqs; j.batch = a.batch; j.seqlen = a.seqlen;
    j.channels = a.channels; j.width = a.width; j.act = a.activation; j.dtype = a.dtype;
    j.out = a.out; j.o_bs = a.out_batch_stride; j.o_ts = a.out_token_stride;
    return launch_conv_job(j, st);
}

}  // namespace ssm
