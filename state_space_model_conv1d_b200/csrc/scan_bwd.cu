// scan_bwd.cu -- backward of the fused causal conv + selective scan.
//
// Gradients of L = sum(dy y) + sum(dh_final h_final) + sum(dconv_state_out
// conv_state_out) for both forms.  The step
//   h_t = a_t h_{t-1} + delta_t B_t xc_t,   a_t = exp(delta_t A),
//   y_t = (C_t . h_t + D xc_t) silu(z_t)
// is differentiated as it stands: with g = dL/dh_t,
//   g += dy_t silu(z_t) C_t;  dB_t += g delta_t xc_t;  dxc_t += g . B_t delta_t;
//   ddelta_t += g . (h_{t-1} a_t A + B_t xc_t);  dA += g h_{t-1} a_t delta_t;
//   g *= a_t  (then the next token back), and dh0 is the g left after the
// first token ("Adding Initial Value Support to Selective Scan Forward
// Kernel", state-spaces/mamba issue 285: the backward carries dh back through
// exp(delta A) to the initial state).  The conv gradients follow from
// xc = silu(b + sum_k w_k u_{t-K+1+k}) with u before the sequence taken from
// the carried conv state.
//
// Work layout (SIMT, correctness first): one CTA per (sequence, block of
// channels) -- for Mamba-2 the block lies inside one head.  L lanes per
// channel hold NS states each.  Pass A walks the sequence forward in chunks of
// TC tokens and stores each chunk's start state in the workspace; pass B
// walks the chunks backwards, recomputes the chunk's states from its
// checkpoint into shared memory and runs the reverse recurrence.  Gradients
// summed over channels (B, C and, for Mamba-2, delta and A) go through
// shared-memory then global float atomics.  The Mamba-2 B / C conv backward
// runs afterwards, once per (sequence, B / C channel), on the summed
// gradients of the conv outputs.
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace ssm {
namespace {

constexpr int kBT = 128;     // threads per CTA
constexpr int kTCb = 16;     // tokens per chunk

struct BwdArgs {
    const void *x, *z, *dt, *B, *C;
    int64_t x_bs, x_ts, z_bs, z_ts, dt_bs, dt_ts, B_bs, B_ts, C_bs, C_ts;
    const float *A, *D, *dt_bias, *h0, *conv_w, *conv_b;
    const void *conv_state_in;
    const void *dy;
    int64_t dy_bs, dy_ts;
    const float *dh_final;
    const void *dcs_out;
    float *dx, *dz, *ddt, *dB, *dC, *dA, *dD, *ddt_bias, *dh0, *dconv_w, *dconv_b, *dcs_in;
    float *ckpt;            // [slots][Dn][NP] chunk-start states
    float *dBc, *dCc;       // Mamba-2: [b*T][G*N] gradients of the conv'd B / C
    int64_t Dn, H, P, G, N, T, rows, slots_per_row;
    int K, softplus, mode, L, CPB, NP, units_per_head;
    SeqView sv;
};

SSM_DEVINL float sigmoidf_(float v) { return rcp(1.f + ex2(-v * kLog2e)); }
SSM_DEVINL float dsilu(float v) {
    const float s = sigmoidf_(v);
    return s * (1.f + v * (1.f - s));
}

// sequence bounds of CTA row `si` (packed or batched)
struct Seq {
    int s;
    int64_t start, len, row, slot0;
};
SSM_DEVINL Seq seq_bounds(const BwdArgs &a, int si) {
    Seq q;
    q.s = si;
    q.start = 0; q.len = a.T; q.row = si;
    if (a.sv.cu) {
        const int64_t c0 = min(max((int64_t)a.sv.cu[si], (int64_t)0), a.T);
        const int64_t c1 = min(max((int64_t)a.sv.cu[si + 1], c0), a.T);
        q.start = c0; q.len = c1 - c0; q.row = 0;
        q.slot0 = si + c0 / kTCb;              // disjoint per sequence (see the workspace sizing)
    } else {
        q.slot0 = (int64_t)si * a.slots_per_row;
    }
    return q;
}

template <typename T, int NS, int LT>
__global__ void __launch_bounds__(kBT) scan_bwd_kernel(const BwdArgs a) {
    extern __shared__ __align__(16) float smb[];
    const int tid = threadIdx.x;
    constexpr int L = LT, CPB = kBT / LT, NP = LT * NS;
    const int K = a.K;
    const bool m1 = a.mode == SSM_MAMBA1;
    const int j = tid / L, l = tid % L;
    const Seq q = seq_bounds(a, blockIdx.y);
    // channels of this CTA
    int64_t hh, p0;
    if (m1) { hh = 0; p0 = (int64_t)blockIdx.x * CPB; }
    else { hh = blockIdx.x / a.units_per_head; p0 = (int64_t)(blockIdx.x % a.units_per_head) * CPB; }
    const int64_t P = m1 ? a.Dn : a.P;
    const int64_t pj = p0 + j;
    const bool cvalid = j < CPB && pj < P;
    const int64_t ch = m1 ? pj : hh * a.P + pj;            // x channel
    const int64_t g = m1 ? 0 : hh / (a.H / a.G);
    const int64_t N = a.N, Dn = a.Dn, GN = a.G * a.N;
    const int64_t cdim = m1 ? Dn : Dn + 2 * GN;
    // bounds-checked build: the CTA's ranges (uniform, so the whole CTA returns together)
    if (!SSM_BOUNDS(q.len > 0 ? q.start + q.len - 1 : 0, a.T > 0 ? a.T : 1, BS_BWD_SEQ) ||
        !SSM_BOUNDS(m1 ? p0 : hh * a.P + p0, Dn, BS_BWD_CHANNEL))
        return;

    // shared memory
    float *hs = smb;                                         // [TC+1][kBT][NS]
    float *xc = hs + (kTCb + 1) * kBT * NS;                  // [TC][CPB] each below
    float *pre = xc + kTCb * CPB;
    float *dl = pre + kTCb * CPB;
    float *spd = dl + kTCb * CPB;
    float *gate = spd + kTCb * CPB;
    float *dgate = gate + kTCb * CPB;
    float *dyv = dgate + kTCb * CPB;
    float *dxc = dyv + kTCb * CPB;
    float *Bt = dxc + kTCb * CPB;                            // [TC][NP]
    float *Ct = Bt + kTCb * NP;
    float *sdB = Ct + kTCb * NP;
    float *sdC = sdB + kTCb * NP;
    float *sddt = sdC + kTCb * NP;                           // [TC]
    float *carry = sddt + kTCb;                              // [CPB][kMaxConvWidth]
    float *dcw = carry + CPB * kMaxConvWidth;                // [CPB][kMaxConvWidth]
    float *rawx = dcw + CPB * kMaxConvWidth;                 // [TC + K-1][CPB] raw x rows t0-(K-1) ..
    float *wts = rawx + (kTCb + kMaxConvWidth - 1) * CPB;    // [CPB][kMaxConvWidth] conv taps of the x channels
    float *dcb = wts + CPB * kMaxConvWidth;                  // [CPB] conv bias gradient of the x channels

    const T *xg = static_cast<const T *>(a.x);
    const T *csi = static_cast<const T *>(a.conv_state_in);
    // raw conv input of conv channel cc at position pos of the sequence (pos < 0: carried state)
    auto raw_at = [&](const T *src, int64_t bs, int64_t ts, int64_t col, int64_t cc, int64_t pos) -> float {
        if (pos >= 0) return Elem<T>::ld(src + q.row * bs + (q.start + pos) * ts + col);
        const int64_t qq = pos + (K - 1);
        return (csi && qq >= 0) ? Elem<T>::ld(csi + ((int64_t)q.s * cdim + cc) * (K - 1) + qq) : 0.f;
    };
    auto conv_pre = [&](const T *src, int64_t bs, int64_t ts, int64_t col, int64_t cc, int64_t pos) -> float {
        float acc = a.conv_b ? a.conv_b[cc] : 0.f;
        for (int k = 0; k < K; ++k) acc = fmaf(a.conv_w[cc * K + k], raw_at(src, bs, ts, col, cc, pos - (K - 1) + k), acc);
        return acc;
    };

    const int nch = (int)((q.len + kTCb - 1) / kTCb);
    // Stage chunk c into shared memory.  Every thread first issues all of its
    // global loads (compile-time trip counts), then does the math, so the load
    // latencies overlap.  FULL = false (the checkpoint pass) skips what only
    // the reverse pass reads: z, dy, C and the softplus derivative.
    constexpr int kRawIt = ((kTCb + kMaxConvWidth - 1) * CPB + kBT - 1) / kBT;
    constexpr int kTokIt = (kTCb * CPB + kBT - 1) / kBT;
    constexpr int kStIt = (kTCb * NP + kBT - 1) / kBT;
    const T *dtp = static_cast<const T *>(a.dt), *zp = static_cast<const T *>(a.z), *dyp = static_cast<const T *>(a.dy);
    const T *Bs = static_cast<const T *>(a.B), *Cs = static_cast<const T *>(a.C);
    // Staging is split in two: issue(c) loads chunk c's inputs into registers,
    // finish(c) writes / computes them into shared memory.  issue runs one
    // chunk ahead, so the load latency hides behind the current chunk's work.
    float rv[kRawIt], rdt[kTokIt], rz[kTokIt], rdy[kTokIt], rb[kStIt], rc[kStIt];
    const bool bc_raw = m1 || K == 0;
    auto issue = [&](int c, auto full_tag) {
        constexpr bool FULL = decltype(full_tag)::value;
        const int64_t t0 = (int64_t)c * kTCb;
        const int nv = (int)min((int64_t)kTCb, q.len - t0);
        const int KW = K > 0 ? K - 1 : 0;
#pragma unroll
        for (int i = 0; i < kRawIt; ++i) {
            const int idx = tid + i * kBT;
            const int r = idx / CPB, jj = idx % CPB;
            const int64_t pp = p0 + jj, pos = t0 - KW + r;
            rv[i] = 0.f;
            if (r < kTCb + KW && pp < P && pos < q.len) {
                const int64_t cc = m1 ? pp : hh * a.P + pp;
                rv[i] = raw_at(xg, a.x_bs, a.x_ts, cc, cc, pos);
            }
        }
#pragma unroll
        for (int i = 0; i < kTokIt; ++i) {
            const int idx = tid + i * kBT;
            const int t = idx / CPB, jj = idx % CPB;
            const int64_t pp = p0 + jj;
            rdt[i] = 0.f; rz[i] = 0.f; rdy[i] = 0.f;
            if (t < nv && pp < P) {
                const int64_t cc = m1 ? pp : hh * a.P + pp;
                const int64_t tok = q.start + t0 + t;
                rdt[i] = Elem<T>::ld(dtp + q.row * a.dt_bs + tok * a.dt_ts + (m1 ? cc : hh));
                if (FULL) {
                    if (zp) rz[i] = Elem<T>::ld(zp + q.row * a.z_bs + tok * a.z_ts + cc);
                    rdy[i] = Elem<T>::ld(dyp + q.row * a.dy_bs + tok * a.dy_ts + cc);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kStIt; ++i) {
            const int idx = tid + i * kBT;
            const int t = idx / NP, n = idx % NP;
            rb[i] = 0.f; rc[i] = 0.f;
            if (bc_raw && t < nv && n < N) {
                const int64_t tok = q.start + t0 + t;
                rb[i] = Elem<T>::ld(Bs + q.row * a.B_bs + tok * a.B_ts + g * N + n);
                if (FULL) rc[i] = Elem<T>::ld(Cs + q.row * a.C_bs + tok * a.C_ts + g * N + n);
            }
        }
    };
    auto stage = [&](int c, auto full_tag) {
        constexpr bool FULL = decltype(full_tag)::value;
        const int64_t t0 = (int64_t)c * kTCb;
        const int nv = (int)min((int64_t)kTCb, q.len - t0);
        const int KW = K > 0 ? K - 1 : 0;
#pragma unroll
        for (int i = 0; i < kRawIt; ++i) {
            const int idx = tid + i * kBT;
            if (idx < (kTCb + KW) * CPB) rawx[idx] = rv[i];
        }
        __syncthreads();                                    // rawx complete
#pragma unroll
        for (int i = 0; i < kTokIt; ++i) {
            const int idx = tid + i * kBT;
            if (idx >= kTCb * CPB) break;
            const int t = idx / CPB, jj = idx % CPB;
            const int64_t pp = p0 + jj;
            float vxc = 0.f, vpre = 0.f, vdl = 0.f, vsp = 0.f, vg = 1.f, vdg = 0.f;
            if (t < nv && pp < P) {
                const int64_t cc = m1 ? pp : hh * a.P + pp;
                if (K > 0) {
                    float acc = a.conv_b ? a.conv_b[cc] : 0.f;
                    for (int k = 0; k < K; ++k) acc = fmaf(wts[jj * kMaxConvWidth + k], rawx[(t + k) * CPB + jj], acc);
                    vpre = acc;
                    vxc = silu(vpre);
                } else {
                    vxc = rawx[t * CPB + jj];
                }
                const int64_t dcol = m1 ? cc : hh;
                const float u = rdt[i] + (a.dt_bias ? a.dt_bias[dcol] : 0.f);
                vdl = a.softplus ? softplus(u) : u;
                if (FULL) {
                    vsp = a.softplus ? sigmoidf_(u) : 1.f;
                    if (zp) {
                        vg = silu(rz[i]);
                        vdg = dsilu(rz[i]);
                    }
                }
            }
            xc[t * CPB + jj] = vxc; dl[t * CPB + jj] = vdl;
            if (FULL) {
                pre[t * CPB + jj] = vpre; spd[t * CPB + jj] = vsp;
                gate[t * CPB + jj] = vg; dgate[t * CPB + jj] = vdg; dyv[t * CPB + jj] = rdy[i];
            }
        }
#pragma unroll
        for (int i = 0; i < kStIt; ++i) {
            const int idx = tid + i * kBT;
            if (idx >= kTCb * NP) break;
            const int t = idx / NP, n = idx % NP;
            float vb = rb[i], vc = rc[i];
            if (!bc_raw && t < nv && n < N) {
                vb = silu(conv_pre(Bs, a.B_bs, a.B_ts, g * N + n, Dn + g * N + n, t0 + t));
                if (FULL) vc = silu(conv_pre(Cs, a.C_bs, a.C_ts, g * N + n, Dn + GN + g * N + n, t0 + t));
            }
            Bt[t * NP + n] = vb;
            if (FULL) Ct[t * NP + n] = vc;
        }
    };
    using FullT = std::integral_constant<bool, true>;
    using LightT = std::integral_constant<bool, false>;
    auto A_of = [&](int e) -> float {
        const int64_t n = (int64_t)l * NS + e;
        if (n >= N || !cvalid) return 0.f;
        return m1 ? a.A[ch * N + n] : a.A[hh];
    };
    float An[NS];
#pragma unroll
    for (int e = 0; e < NS; ++e) An[e] = A_of(e);

    for (int idx = tid; idx < CPB * kMaxConvWidth; idx += kBT) {
        const int jj = idx / kMaxConvWidth, k = idx % kMaxConvWidth;
        const int64_t pp = p0 + jj;
        const int64_t cc = m1 ? pp : hh * a.P + pp;
        wts[idx] = (pp < P && k < K) ? a.conv_w[cc * K + k] : 0.f;
    }
    // ---- pass A: forward, storing chunk-start states
    float h[NS];
    const int64_t hbase = ((int64_t)q.s * Dn + ch) * N;
#pragma unroll
    for (int e = 0; e < NS; ++e) {
        const int64_t n = (int64_t)l * NS + e;
        h[e] = (cvalid && n < N && a.h0) ? a.h0[hbase + n] : 0.f;
    }
    if (nch > 0) issue(0, LightT{});
    for (int c = 0; c < nch; ++c) {
        if (cvalid) {
            float *dst = a.ckpt + ((q.slot0 + c) * Dn + ch) * NP + (int64_t)l * NS;
#pragma unroll
            for (int e = 0; e < NS; ++e) dst[e] = h[e];
        }
        __syncthreads();
        stage(c, LightT{});
        __syncthreads();
        if (c + 1 < nch) issue(c + 1, LightT{});
        const int nv = (int)min((int64_t)kTCb, q.len - (int64_t)c * kTCb);
        if (cvalid)
            for (int t = 0; t < nv; ++t) {
                const float d = dl[t * CPB + j], xv = xc[t * CPB + j];
#pragma unroll
                for (int e = 0; e < NS; ++e) h[e] = fmaf(__expf(d * An[e]), h[e], d * Bt[t * NP + l * NS + e] * xv);
            }
    }

    // ---- pass B: reverse
    float gr[NS], dAa[NS];
#pragma unroll
    for (int e = 0; e < NS; ++e) {
        const int64_t n = (int64_t)l * NS + e;
        gr[e] = (cvalid && n < N && a.dh_final) ? a.dh_final[hbase + n] : 0.f;
        dAa[e] = 0.f;
    }
    float dDa = 0.f, dbias_a = 0.f;
    if (tid < CPB) {
        for (int k = 0; k < kMaxConvWidth; ++k) { carry[tid * kMaxConvWidth + k] = 0.f; dcw[tid * kMaxConvWidth + k] = 0.f; }
        dcb[tid] = 0.f;
    }
    const float Dv = (cvalid && a.D) ? a.D[m1 ? ch : hh] : 0.f;
    const unsigned gmask = L >= 32 ? 0xffffffffu : (((1u << L) - 1u) << ((threadIdx.x & 31) / L * L));
    auto lane_sum = [&](float v) {
        for (int o = L / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(gmask, v, o);
        return v;
    };
    const T *dcso = static_cast<const T *>(a.dcs_out);

    if (nch > 0) issue(nch - 1, FullT{});
    for (int c = nch - 1; c >= 0; --c) {
        const int64_t t0 = (int64_t)c * kTCb;
        const int nv = (int)min((int64_t)kTCb, q.len - t0);
        __syncthreads();
        stage(c, FullT{});
        if (c > 0) issue(c - 1, FullT{});
        for (int idx = tid; idx < kTCb * NP; idx += kBT) { sdB[idx] = 0.f; sdC[idx] = 0.f; }
        if (tid < kTCb) sddt[tid] = 0.f;
        __syncthreads();
        // states of the chunk from its checkpoint
        {
            const float *src = a.ckpt + ((q.slot0 + c) * Dn + (cvalid ? ch : 0)) * NP + (int64_t)l * NS;
#pragma unroll
            for (int e = 0; e < NS; ++e) h[e] = cvalid ? src[e] : 0.f;
#pragma unroll
            for (int e = 0; e < NS; ++e) hs[tid * NS + e] = h[e];
            for (int t = 0; t < nv; ++t) {
                const float d = dl[t * CPB + (cvalid ? j : 0)], xv = cvalid ? xc[t * CPB + j] : 0.f;
#pragma unroll
                for (int e = 0; e < NS; ++e) {
                    h[e] = fmaf(__expf(d * An[e]), h[e], d * Bt[t * NP + l * NS + e] * xv);
                    hs[((t + 1) * kBT + tid) * NS + e] = h[e];
                }
            }
        }
        // reverse recurrence over the chunk
        for (int t = nv - 1; t >= 0; --t) {
            const int jj = cvalid ? j : 0;
            const float d = dl[t * CPB + jj], xv = xc[t * CPB + jj];
            float yb = 0.f;
#pragma unroll
            for (int e = 0; e < NS; ++e) yb = fmaf(Ct[t * NP + l * NS + e], hs[((t + 1) * kBT + tid) * NS + e], yb);
            yb = lane_sum(yb) + Dv * xv;
            const float dyt = dyv[t * CPB + jj];
            const float dyb = dyt * gate[t * CPB + jj];
            float dxp = 0.f, ddp = 0.f;
            float vals[2 * NS];                                 // this lane's dB (e) and dC (NS + e) terms
#pragma unroll
            for (int e = 0; e < NS; ++e) {
                const int n = l * NS + e;
                const float hc = hs[((t + 1) * kBT + tid) * NS + e], hp = hs[(t * kBT + tid) * NS + e];
                vals[NS + e] = cvalid ? dyb * hc : 0.f;
                gr[e] = fmaf(dyb, Ct[t * NP + n], gr[e]);
                const float av = __expf(d * An[e]);
                vals[e] = cvalid ? gr[e] * d * xv : 0.f;
                dxp = fmaf(gr[e] * d, Bt[t * NP + n], dxp);
                ddp = fmaf(gr[e], hp * av * An[e] + Bt[t * NP + n] * xv, ddp);
                dAa[e] = fmaf(gr[e], hp * av * d, dAa[e]);
                gr[e] *= av;
            }
            // sum over the warp's channels (lane bits above the L state lanes): halve the
            // values at each level until one is left, then plain butterflies; each
            // (dB / dC, state) sum lands on one lane, which adds it to the chunk tile
            {
                int base = 0, cnt = 2 * NS;
                bool writer = true;
#pragma unroll
                for (int o = 16; o >= LT; o >>= 1) {
                    const bool up = (threadIdx.x & o) != 0;
                    if (cnt >= 2) {
                        const int hlf = cnt / 2;
#pragma unroll
                        for (int k = 0; k < 2 * NS / 2; ++k) {
                            if (k < hlf) {
                                const float keep = up ? vals[hlf + k] : vals[k];
                                const float send = up ? vals[k] : vals[hlf + k];
                                vals[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                            }
                        }
                        base += up ? hlf : 0;
                        cnt = hlf;
                    } else {
                        vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], o);
                        writer = writer && !up;
                    }
                }
                if (writer) {
#pragma unroll
                    for (int k = 0; k < 2 * NS; ++k) {
                        if (k < cnt) {
                            const int idx = base + k;
                            float *dst = idx < NS ? sdB : sdC;
                            atomicAdd(&dst[t * NP + l * NS + (idx % NS)], vals[k]);
                        }
                    }
                }
            }
            dxp = lane_sum(dxp);
            ddp = lane_sum(ddp);
            if (cvalid && l == 0) {
                const int64_t tok = q.start + t0 + t;
                const int64_t rt = q.row * a.T + tok;
                if (a.z) a.dz[rt * Dn + ch] = dyt * yb * dgate[t * CPB + j];
                dDa = fmaf(dyb, xv, dDa);
                dxc[t * CPB + j] = dxp + dyb * Dv;
                const float dd = ddp * spd[t * CPB + j];
                if (m1) {
                    a.ddt[rt * Dn + ch] = dd;
                    dbias_a += dd;
                } else {
                    atomicAdd(&sddt[t], dd);
                }
            }
        }
        __syncthreads();
        // chunk sums over this CTA's channels -> global
        for (int idx = tid; idx < kTCb * NP; idx += kBT) {
            const int t = idx / NP, n = idx % NP;
            if (t < nv && n < N) {
                const int64_t rt = q.row * a.T + q.start + t0 + t;
                if (m1) {
                    atomicAdd(&a.dB[rt * N + n], sdB[idx]);
                    atomicAdd(&a.dC[rt * N + n], sdC[idx]);
                } else {
                    atomicAdd(&a.dBc[rt * GN + g * N + n], sdB[idx]);
                    atomicAdd(&a.dCc[rt * GN + g * N + n], sdC[idx]);
                }
            }
        }
        if (!m1 && tid < nv) {
            const int64_t rt = q.row * a.T + q.start + t0 + tid;
            atomicAdd(&a.ddt[rt * a.H + hh], sddt[tid]);
            dbias_a += sddt[tid];                 // summed below by threads < kTCb
        }
        // conv backward of this chunk's x channels, spread over the CTA:
        // dpre per (token, channel), then d raw per (token, channel), the tap
        // gradients per (channel, tap), and the carried dpre of this chunk's
        // first K-1 tokens for the chunk before it
        __syncthreads();                                  // dxc of every channel written
        for (int idx = tid; idx < kTCb * CPB; idx += kBT) {
            if (idx / CPB < nv && K > 0) dxc[idx] = dxc[idx] * dsilu(pre[idx]);
        }
        __syncthreads();
        auto dp_at = [&](int jj, int64_t x) -> float {    // dpre at sequence position x >= t0
            if (x < t0 + nv) return dxc[(x - t0) * CPB + jj];
            const int64_t i = x - (t0 + nv);
            return (x < q.len && i < kMaxConvWidth) ? carry[jj * kMaxConvWidth + i] : 0.f;
        };
        for (int idx = tid; idx < kTCb * CPB; idx += kBT) {
            const int t = idx / CPB, jj = idx % CPB;
            if (t >= nv || p0 + jj >= P) continue;
            const int64_t cc = m1 ? p0 + jj : hh * a.P + p0 + jj;
            const int64_t pos = t0 + t;
            float v;
            if (K > 0) {
                v = 0.f;
                for (int k = 0; k < K; ++k) v = fmaf(dp_at(jj, pos + (K - 1) - k), wts[jj * kMaxConvWidth + k], v);
            } else {
                v = dxc[idx];
            }
            if (dcso && K > 1 && pos >= q.len - (K - 1))
                v += Elem<T>::ld(dcso + ((int64_t)q.s * cdim + cc) * (K - 1) + (pos - (q.len - (K - 1))));
            a.dx[(q.row * a.T + q.start + pos) * Dn + cc] = v;
        }
        if (K > 0)
            for (int idx = tid; idx < CPB * K; idx += kBT) {
                const int jj = idx / K, k = idx % K;
                if (p0 + jj >= P) continue;
                float sw = 0.f, sb = 0.f;
                for (int t = 0; t < nv; ++t) {
                    const float dp = dxc[t * CPB + jj];
                    sw = fmaf(dp, rawx[(t + k) * CPB + jj], sw);
                    sb += dp;
                }
                dcw[jj * kMaxConvWidth + k] += sw;
                if (k == 0) dcb[jj] += sb;
            }
        __syncthreads();                                  // the old carry has been read
        for (int idx = tid; idx < CPB * (kMaxConvWidth - 1); idx += kBT) {
            const int jj = idx / (kMaxConvWidth - 1), i = idx % (kMaxConvWidth - 1);
            if (i < K - 1) carry[jj * kMaxConvWidth + i] = dp_at(jj, t0 + i);
        }
    }
    __syncthreads();
    // carried-state gradients, dh0, and the sums over the whole sequence
    if (tid < CPB && p0 + tid < P && K > 1 && a.dcs_in) {
        const int jj = tid;
        const int64_t cc = m1 ? p0 + jj : hh * a.P + p0 + jj;
        const float *cr = carry + jj * kMaxConvWidth;
        for (int qq = 0; qq < K - 1; ++qq) {
            const int64_t pos = qq - (K - 1);                  // history position
            float v = 0.f;
            for (int k = 0; k < K; ++k) {
                const int64_t x = pos + (K - 1) - k;
                if (x >= 0 && x < q.len && x < K - 1) v = fmaf(cr[x], a.conv_w[cc * K + k], v);
            }
            if (dcso && pos >= q.len - (K - 1))
                v += Elem<T>::ld(dcso + ((int64_t)q.s * cdim + cc) * (K - 1) + (pos - (q.len - (K - 1))));
            a.dcs_in[((int64_t)q.s * cdim + cc) * (K - 1) + qq] = v;
        }
    }
    if (tid < CPB && p0 + tid < P && K > 0) {
        const int64_t cc = m1 ? p0 + tid : hh * a.P + p0 + tid;
        if (a.dconv_w)
            for (int k = 0; k < K; ++k) atomicAdd(&a.dconv_w[cc * K + k], dcw[tid * kMaxConvWidth + k]);
        if (a.dconv_b) atomicAdd(&a.dconv_b[cc], dcb[tid]);
    }
    if (cvalid) {
#pragma unroll
        for (int e = 0; e < NS; ++e) {
            const int64_t n = (int64_t)l * NS + e;
            if (n < N) {
                a.dh0[hbase + n] = gr[e];
                if (m1) atomicAdd(&a.dA[ch * N + n], dAa[e]);
            }
        }
        if (!m1) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < NS; ++e) s += dAa[e];
            atomicAdd(&a.dA[hh], s);
        }
        if (l == 0) {
            if (a.dD && a.D) atomicAdd(&a.dD[m1 ? ch : hh], dDa);
            if (m1 && a.ddt_bias && a.dt_bias) atomicAdd(&a.ddt_bias[ch], dbias_a);
        }
    }
    if (!m1 && tid < kTCb && a.ddt_bias && a.dt_bias) atomicAdd(&a.ddt_bias[hh], dbias_a);
}

// Mamba-2 B / C conv backward: one thread per (sequence, B / C channel), walking
// the sequence backwards over the summed gradients of the conv outputs.
template <typename T>
__global__ void bc_conv_bwd_kernel(const BwdArgs a) {
    const int64_t GN = a.G * a.N, Dn = a.Dn, cdim = Dn + 2 * GN;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int nseq = a.sv.cu ? a.sv.nseqs : (int)a.rows;
    if (i >= (int64_t)nseq * 2 * GN) return;
    const int si = (int)(i / (2 * GN));
    const int64_t cc2 = i % (2 * GN);
    const int which = (int)(cc2 / GN);
    const int64_t col = cc2 % GN;
    const int64_t cc = Dn + which * GN + col;                 // conv channel
    const Seq q = seq_bounds(a, si);
    const int K = a.K;
    const T *src = static_cast<const T *>(which ? a.C : a.B);
    const int64_t bs = which ? a.C_bs : a.B_bs, ts = which ? a.C_ts : a.B_ts;
    const float *gin = which ? a.dCc : a.dBc;
    float *gout = which ? a.dC : a.dB;
    const T *csi = static_cast<const T *>(a.conv_state_in);
    const T *dcso = static_cast<const T *>(a.dcs_out);
    auto raw_at = [&](int64_t pos) -> float {
        if (pos >= 0) return Elem<T>::ld(src + q.row * bs + (q.start + pos) * ts + col);
        const int64_t qq = pos + (K - 1);
        return (csi && qq >= 0) ? Elem<T>::ld(csi + ((int64_t)q.s * cdim + cc) * (K - 1) + qq) : 0.f;
    };
    auto dout_at = [&](int64_t pos) -> float { return gin[(q.row * a.T + q.start + pos) * GN + col]; };
    auto dcso_at = [&](int64_t pos) -> float {
        return (dcso && K > 1 && pos >= q.len - (K - 1))
                   ? Elem<T>::ld(dcso + ((int64_t)q.s * cdim + cc) * (K - 1) + (pos - (q.len - (K - 1))))
                   : 0.f;
    };
    if (K == 0) {
        for (int64_t pos = 0; pos < q.len; ++pos) gout[(q.row * a.T + q.start + pos) * GN + col] = dout_at(pos);
        return;
    }
    float w[kMaxConvWidth], dw[kMaxConvWidth], ring[kMaxConvWidth];   // ring: dpre at pos+1 .. pos+K-1
    for (int k = 0; k < kMaxConvWidth; ++k) { w[k] = k < K ? a.conv_w[cc * K + k] : 0.f; dw[k] = 0.f; ring[k] = 0.f; }
    const float bias = a.conv_b ? a.conv_b[cc] : 0.f;
    float db = 0.f;
    for (int64_t pos = q.len - 1; pos >= -(int64_t)(K - 1); --pos) {
        float dp = 0.f;
        if (pos >= 0) {
            float pre = bias;
            for (int k = 0; k < K; ++k) pre = fmaf(w[k], raw_at(pos - (K - 1) + k), pre);
            dp = dout_at(pos) * dsilu(pre);
            db += dp;
            for (int k = 0; k < K; ++k) dw[k] += dp * raw_at(pos - (K - 1) + k);
        }
        // d raw(pos) = sum_k dpre(pos + K-1-k) w[k]; dpre(pos) is dp, dpre(pos + m) is ring[m-1]
        float v = dp * w[K - 1];
        for (int k = 0; k + 1 < K; ++k) v = fmaf(ring[K - 2 - k], w[k], v);
        v += dcso_at(pos);
        if (pos >= 0) gout[(q.row * a.T + q.start + pos) * GN + col] = v;
        else if (a.dcs_in) a.dcs_in[((int64_t)q.s * cdim + cc) * (K - 1) + (pos + (K - 1))] = v;
        for (int m = kMaxConvWidth - 1; m >= 1; --m) ring[m] = ring[m - 1];
        ring[0] = dp;
    }
    if (a.dconv_w)
        for (int k = 0; k < K; ++k) atomicAdd(&a.dconv_w[cc * K + k], dw[k]);
    if (a.dconv_b) atomicAdd(&a.dconv_b[cc], db);
}

}  // namespace

// The kernel instance for (states per lane, lanes per channel).
template <typename T, typename Run>
cudaError_t dispatch(Run &&run, int NS, int L) {
    if (NS == 8) return run(scan_bwd_kernel<T, 8, 32>);
    switch (L) {
        case 1: return run(scan_bwd_kernel<T, 4, 1>);
        case 2: return run(scan_bwd_kernel<T, 4, 2>);
        case 4: return run(scan_bwd_kernel<T, 4, 4>);
        case 8: return run(scan_bwd_kernel<T, 4, 8>);
        case 16: return run(scan_bwd_kernel<T, 4, 16>);
        default: return run(scan_bwd_kernel<T, 4, 32>);
    }
}

// Lanes per channel and states per lane for dstate N.
static void bwd_layout(int64_t N, int *L, int *NS) {
    *NS = N > 128 ? 8 : 4;
    int l = 1;
    while (l * *NS < N) l *= 2;
    *L = l;
}

size_t scan_bwd_workspace_bytes(const ssm_scan_bwd_args &b) {
    const ssm_scan_args &s = b.fwd;
    int L, NS;
    bwd_layout(s.dstate, &L, &NS);
    const int64_t NP = (int64_t)L * NS;
    const int64_t nseq = s.cu_seqlens ? s.nseqs : s.batch;
    const int64_t slots = s.cu_seqlens ? (int64_t)nseq + (s.seqlen + kTCb - 1) / kTCb + 1
                                       : s.batch * ((s.seqlen + kTCb - 1) / kTCb);
    size_t bytes = ((size_t)slots * (size_t)s.d_inner * (size_t)NP * 4 + 255) / 256 * 256;
    if (s.mode == SSM_MAMBA2)
        bytes += 2 * (((size_t)s.batch * (size_t)s.seqlen * (size_t)(s.ngroups * s.dstate) * 4 + 255) / 256 * 256);
    return bytes;
}

cudaError_t launch_scan_bwd(const ssm_scan_bwd_args &b, const SeqView &sv, void *ws, cudaStream_t st) {
    const ssm_scan_args &s = b.fwd;
    const bool m1 = s.mode == SSM_MAMBA1;
    int L, NS;
    bwd_layout(s.dstate, &L, &NS);
    BwdArgs a;
    a.x = s.x; a.z = s.z; a.dt = s.dt; a.B = s.B; a.C = s.C;
    a.x_bs = s.x_batch_stride; a.x_ts = s.x_token_stride; a.z_bs = s.z_batch_stride; a.z_ts = s.z_token_stride;
    a.dt_bs = s.dt_batch_stride; a.dt_ts = s.dt_token_stride; a.B_bs = s.B_batch_stride; a.B_ts = s.B_token_stride;
    a.C_bs = s.C_batch_stride; a.C_ts = s.C_token_stride;
    a.A = s.A; a.D = s.D; a.dt_bias = s.dt_bias; a.h0 = s.h0; a.conv_w = s.conv_w; a.conv_b = s.conv_b;
    a.conv_state_in = s.conv_state_in;
    a.dy = b.dy; a.dy_bs = b.dy_batch_stride; a.dy_ts = b.dy_token_stride;
    a.dh_final = b.dh_final; a.dcs_out = b.dconv_state_out;
    a.dx = b.dx; a.dz = b.dz; a.ddt = b.ddt; a.dB = b.dB; a.dC = b.dC; a.dA = b.dA; a.dD = b.dD;
    a.ddt_bias = b.ddt_bias; a.dh0 = b.dh0; a.dconv_w = b.dconv_w; a.dconv_b = b.dconv_b; a.dcs_in = b.dconv_state_in;
    a.Dn = s.d_inner; a.N = s.dstate; a.T = s.seqlen; a.rows = s.batch;
    a.H = m1 ? s.d_inner : s.nheads; a.P = m1 ? 1 : s.headdim; a.G = m1 ? 1 : s.ngroups;
    a.slots_per_row = (s.seqlen + kTCb - 1) / kTCb;
    a.K = (int)s.d_conv; a.softplus = s.delta_softplus; a.mode = s.mode;
    a.L = L; a.NP = L * NS; a.CPB = kBT / L;
    a.units_per_head = m1 ? 0 : (int)((s.headdim + a.CPB - 1) / a.CPB);
    a.sv = sv;
    const int64_t nseq = s.cu_seqlens ? s.nseqs : s.batch;
    const int64_t slots = s.cu_seqlens ? nseq + (s.seqlen + kTCb - 1) / kTCb + 1 : s.batch * a.slots_per_row;
    char *w = static_cast<char *>(ws);
    a.ckpt = reinterpret_cast<float *>(w);
    w += ((size_t)slots * (size_t)s.d_inner * (size_t)a.NP * 4 + 255) / 256 * 256;
    const size_t bc_bytes = (size_t)s.batch * (size_t)s.seqlen * (size_t)(a.G * s.dstate) * 4;
    a.dBc = a.dCc = nullptr;
    if (!m1) {
        a.dBc = reinterpret_cast<float *>(w);
        a.dCc = reinterpret_cast<float *>(w + (bc_bytes + 255) / 256 * 256);
    }
    // accumulated outputs start at zero
    auto zero = [&](void *p, size_t bytes) { return p ? cudaMemsetAsync(p, 0, bytes, st) : cudaSuccess; };
    const int64_t K = s.d_conv, cdim = m1 ? s.d_inner : s.d_inner + 2 * a.G * s.dstate;
    cudaError_t e;
    if ((e = zero(b.dA, (size_t)(m1 ? s.d_inner * s.dstate : s.nheads) * 4)) != cudaSuccess) return e;
    if ((e = zero(b.dD, (size_t)a.H * 4)) != cudaSuccess) return e;
    if ((e = zero(b.ddt_bias, (size_t)a.H * 4)) != cudaSuccess) return e;
    if (K > 0) {
        if ((e = zero(b.dconv_w, (size_t)(cdim * K) * 4)) != cudaSuccess) return e;
        if ((e = zero(b.dconv_b, (size_t)cdim * 4)) != cudaSuccess) return e;
    }
    if (m1) {
        if ((e = zero(b.dB, bc_bytes)) != cudaSuccess) return e;
        if ((e = zero(b.dC, bc_bytes)) != cudaSuccess) return e;
    } else {
        if ((e = zero(b.ddt, (size_t)s.batch * (size_t)s.seqlen * (size_t)s.nheads * 4)) != cudaSuccess) return e;
        if ((e = zero(a.dBc, bc_bytes)) != cudaSuccess) return e;
        if ((e = zero(a.dCc, bc_bytes)) != cudaSuccess) return e;
    }
    const size_t smem = (size_t)((kTCb + 1) * kBT * NS + 8 * kTCb * a.CPB + 4 * kTCb * a.NP + kTCb +
                                 3 * a.CPB * kMaxConvWidth + (kTCb + kMaxConvWidth - 1) * a.CPB + a.CPB) * 4;
    const unsigned gx = m1 ? (unsigned)((s.d_inner + a.CPB - 1) / a.CPB) : (unsigned)(s.nheads * a.units_per_head);
    dim3 grid(gx, (unsigned)nseq);
    if (nseq > 0) {
        auto run = [&](auto kern) -> cudaError_t {
            cudaError_t ee = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (ee != cudaSuccess) return ee;
            timing_begin(st);
            kern<<<grid, kBT, smem, st>>>(a);
            timing_end(st);
            return cudaGetLastError();
        };
        if (s.dtype == SSM_BF16) e = dispatch<__nv_bfloat16>(run, NS, L);
        else e = dispatch<float>(run, NS, L);
        if (e != cudaSuccess) return e;
        if (!m1) {
            const int64_t n = nseq * 2 * a.G * s.dstate;
            const unsigned blocks = (unsigned)((n + 127) / 128);
            if (s.dtype == SSM_BF16) bc_conv_bwd_kernel<__nv_bfloat16><<<blocks, 128, 0, st>>>(a);
            else bc_conv_bwd_kernel<float><<<blocks, 128, 0, st>>>(a);
            e = cudaGetLastError();
        }
    }
    return e;
}

}  // namespace ssm
