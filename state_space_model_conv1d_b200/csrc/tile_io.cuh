// tile_io.cuh -- cooperative global <-> shared tile movers used by the scan kernels.
#pragma once

#include "common.cuh"

namespace ssm {

// Load rows [0, rows) x cols [col0, col0 + ncols) of a token-major tensor into
// a dense fp32 shared tile dst[rows][ldd].  Rows >= valid_rows and columns
// >= col_end are filled with zeros.  vec: every 8-column group starting at a
// multiple of 8 may use one 16-byte (bf16) or two 16-byte (fp32) loads.
template <typename T, int NT>
SSM_DEVINL void load_tile_f32(float *dst, int ldd, const T *src, int64_t ts, int rows, int valid_rows,
                              int64_t col0, int ncols, int64_t col_end, bool vec) {
    const int nv = (ncols + 7) / 8;
    for (int idx = threadIdx.x; idx < rows * nv; idx += NT) {
        const int r = idx / nv, cv = idx % nv;
        const int64_t c = col0 + cv * 8;
        float v[8];
        if (r < valid_rows && vec && c + 8 <= col_end) {
            Vec8<T>::ld(src + r * ts + c, v);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                v[e] = (r < valid_rows && c + e < col_end) ? Elem<T>::ld(src + r * ts + c + e) : 0.f;
        }
        float *d = dst + r * ldd + cv * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (cv * 8 + e < ncols) d[e] = v[e];
    }
}

// Store rows [0, valid_rows) x cols [0, ncols) of a dense fp32 shared tile to
// a token-major tensor (columns >= col_end - col0 are skipped).
template <typename T, int NT>
SSM_DEVINL void store_tile_f32(T *dst, int64_t ts, const float *src, int lds, int valid_rows, int64_t col0,
                               int ncols, int64_t col_end, bool vec) {
    const int nv = (ncols + 7) / 8;
    for (int idx = threadIdx.x; idx < valid_rows * nv; idx += NT) {
        const int r = idx / nv, cv = idx % nv;
        const int64_t c = col0 + cv * 8;
        const float *s = src + r * lds + cv * 8;
        if (vec && c + 8 <= col_end && cv * 8 + 8 <= ncols) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = s[e];
            Vec8<T>::st(dst + r * ts + c, v);
        } else {
            for (int e = 0; e < 8; ++e)
                if (cv * 8 + e < ncols && c + e < col_end) Elem<T>::st(dst + r * ts + c + e, s[e]);
        }
    }
}

}  // namespace ssm
