// common.cuh -- small device helpers shared by the sm_100a kernels of libssm.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssm.h"

#define SSM_DEVINL __device__ __forceinline__

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// 2^x on the MUFU unit (ex2.approx, flush-to-zero).
SSM_DEVINL float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// log2(x) on the MUFU unit.
SSM_DEVINL float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
SSM_DEVINL float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(u) = log(1 + e^u).  Three regimes of the same function:
//   u > 15        : u + log(1 + e^-u) = u to within 3e-7 relative;
//   u < -5        : e^u (1 - e^u / 2), the first two series terms
//                   (relative error below e^(2u)/3 < 1.6e-5);
//   otherwise     : log2(1 + 2^(u log2 e)) * ln 2, where 1 + e^u >= 1.0067
//                   keeps the rounding of the sum below 2e-5 relative.
SSM_DEVINL float softplus(float u) {
    if (u > 15.f) return u;
    float e = ex2(u * kLog2e);
    if (u < -5.f) return e * (1.f - 0.5f * e);
    return lg2(1.f + e) * kLn2;
}

// silu(v) = v * sigmoid(v) = v / (1 + e^-v).  For v << 0 the exponential
// overflows to +inf and the reciprocal gives 0, the correct limit.
SSM_DEVINL float silu(float v) { return v * rcp(1.f + ex2(-v * kLog2e)); }

// tanh on the MUFU unit (tanh.approx: relative error about 2^-11).
SSM_DEVINL float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// silu for a given activation dtype.  bf16 data (whose own rounding is 2^-9)
// takes sigmoid(v) = (1 + tanh(v/2)) / 2 on one MUFU op; fp32 data keeps the
// exp + reciprocal form above.
template <typename T>
SSM_DEVINL float silu_fast(float v) {
    if constexpr (sizeof(T) == 2) {
        const float hv = 0.5f * v;
        return fmaf(hv, tanh_approx(hv), hv);
    } else {
        return silu(v);
    }
}

// ----------------------------------------------------------- bounds checks
// In the bounds-checked build (SSM_CHECK_BOUNDS) SSM_BOUNDS(index, extent,
// site) tests 0 <= index < extent; a failing test records the first failure
// (SSM_DEVERR_BOUNDS, the site, the index, the extent) in one device-wide
// record and yields false, so the caller skips the access.  Nothing traps.
// In the normal build it is the constant true and costs nothing.
enum BoundsSite {
    BS_SSD_SEQ = 1, BS_SSD_HEAD, BS_SSD_GROUP, BS_SSD_STATE, BS_SSD_CONV_STATE, BS_SSD_Y, BS_SSD_POOL, BS_SSD_RAW_BC,
    BS_BC_ROW, BS_BC_CHANNEL, BS_BC_STATE,
    BS_M1_SEQ, BS_M1_CHANNEL, BS_M1_STATE, BS_M1_CONV_STATE, BS_M1_Y, BS_M1_POOL,
    BS_M2S_SEQ, BS_M2S_HEAD, BS_M2S_STATE,
    BS_DEC_ROW, BS_DEC_SLOT, BS_DEC_CHANNEL,
    BS_CONV_TOKEN, BS_CONV_CHANNEL, BS_CONV_STATE,
    BS_BWD_SEQ, BS_BWD_CHANNEL, BS_SPLIT_ROW, BS_SPLIT_CHANNEL, BS_SSD_SEGMENT,
};
#ifdef SSM_CHECK_BOUNDS
struct BoundsRecord {
    int32_t code, site;
    long long index, extent;
};
extern __device__ BoundsRecord g_ssm_bounds;
SSM_DEVINL bool bounds_ok(int64_t index, int64_t extent, int site) {
    if (index >= 0 && index < extent) return true;
    if (atomicCAS(&g_ssm_bounds.code, 0, SSM_DEVERR_BOUNDS) == 0) {
        g_ssm_bounds.site = site;
        g_ssm_bounds.index = (long long)index;
        g_ssm_bounds.extent = (long long)extent;
        __threadfence();
    }
    return false;
}
#define SSM_BOUNDS(index, extent, site) ::ssm::bounds_ok((int64_t)(index), (int64_t)(extent), (int)(site))
#else
#define SSM_BOUNDS(index, extent, site) true
#endif

// ----------------------------------------------------------- element I/O
template <typename T> struct Elem;
template <> struct Elem<float> {
    static SSM_DEVINL float ld(const float *p) { return *p; }
    static SSM_DEVINL void st(float *p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
    static SSM_DEVINL float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static SSM_DEVINL void st(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

// Eight consecutive elements <-> eight floats, one or two 16-byte accesses.
template <typename T> struct Vec8;
template <> struct Vec8<float> {
    static SSM_DEVINL void ld(const float *p, float (&v)[8]) {
        float4 a = *reinterpret_cast<const float4 *>(p);
        float4 b = *reinterpret_cast<const float4 *>(p + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    static SSM_DEVINL void st(float *p, const float (&v)[8]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
};
template <> struct Vec8<__nv_bfloat16> {
    static SSM_DEVINL void ld(const __nv_bfloat16 *p, float (&v)[8]) {
        uint4 r = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static SSM_DEVINL void st(__nv_bfloat16 *p, const float (&v)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&b);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// Sequence that owns packed token t: the largest s with cu[s] <= t, among
// sequences 0..nseqs-1 (binary search; cu is non-decreasing).
SSM_DEVINL int seq_of_token(const int32_t *cu, int nseqs, int64_t t) {
    int lo = 0, hi = nseqs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

}  // namespace ssm
