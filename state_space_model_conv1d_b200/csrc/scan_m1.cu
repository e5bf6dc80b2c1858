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
// chunk tiles are staged in shared memory with 16-byte cp.async copies into
// a 3-deep ring.  A cooperative prologue computes conv + SiLU, delta,
// delta*x, D*x and the gate once per (token, channel) into fp32 tiles (two
// slots).  Then 4 lanes per channel advance N/4 states each in registers;
// the carry across chunks is the fp32 state staying in registers, seeded
// from h0 (the (1, h0) seed of the pair scan).  The 4 lanes' partial
// read-outs of 4 consecutive tokens are combined by a two-level shuffle
// reduce-scatter, so each lane finishes one token's y.
//
// Software pipeline, one CTA barrier per chunk: iteration c scans chunk c,
// stores y of chunk c-1, runs the prologue of chunk c+1 and issues the copies
// of chunk c+3.  Warps drift freely inside an iteration, so the MUFU-heavy
// scan of one warp overlaps the load / convert work of another.  The K-1 raw
// rows before each chunk live in a double-buffered halo, which is also what
// conv_state_out receives.
//
// Per (token, channel, state) the work is one MUFU exp plus four FP32 ops:
// with dstate 16 the kernel is bound by the MUFU exp rate, not by HBM.
//
// A second, time-parallel form (further down) spreads the tokens of a chunk
// over the lanes of a warp and joins them with a warp-shuffle prefix of the
// scan element (exp(delta A), h).  It does more work per update (two walks
// and the shuffle scan) but has more independent warps, so the launcher picks
// it when the sequential form would leave the SMs short of warps (few
// sequences or channels).
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
    InterView iv;
};

SSM_DEVINL void cp_async16(void *smem, const void *gmem) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
SSM_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
SSM_DEVINL void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Stage rows [0, nv) x cols [col0, col0 + NCOLS) of a token-major tensor into
// dst[kTC][NCOLS] (raw dtype), columns >= col_end skipped.  16-byte cp.async
// when `async` (row starts 16-byte aligned and col_end - col0 a multiple of
// 16 bytes), else plain element copies.  NCOLS is a compile-time width so the
// thread -> (row, vector) map is shifts and masks.
template <typename T, int NCOLS>
SSM_DEVINL void stage_tile(T *dst, const T *src, int64_t ts, int nv, int64_t col0, int64_t col_end, bool async) {
    constexpr int E = 16 / sizeof(T);
    constexpr int PER_ROW = NCOLS / E;
    static_assert(NCOLS % E == 0, "tile rows must be whole 16-byte vectors");
    if (async) {
#pragma unroll
        for (int i0 = 0; i0 < kTC * PER_ROW; i0 += kThreads) {
            const int i = i0 + threadIdx.x;
            const int r = i / PER_ROW, v = i % PER_ROW;
            const int64_t c = col0 + (int64_t)v * E;
            if ((kTC * PER_ROW) % kThreads == 0 || i < kTC * PER_ROW)
                if (r < nv && c + E <= col_end) cp_async16(dst + r * NCOLS + v * E, src + r * ts + c);
        }
    } else {
        for (int i = threadIdx.x; i < nv * NCOLS; i += kThreads) {
            const int r = i / NCOLS, v = i % NCOLS;
            const int64_t c = col0 + v;
            if (c < col_end) dst[r * NCOLS + v] = src[r * ts + c];
        }
    }
}

template <typename T, int SPT>
struct SmemM1 {
    static constexpr int NP = kLanes * SPT;             // padded dstate
    static constexpr int E = 16 / sizeof(T);
    static constexpr int NPR = (NP + E - 1) / E * E;    // raw B / C row: whole 16-byte vectors
    T rx[3][kTC][kDB];
    T rdt[3][kTC][kDB];
    T rz[3][kTC][kDB];
    T rB[3][kTC][NPR];
    T rC[3][kTC][NPR];
    float halo[2][kHalo][kDB];
    float2 dd[2][kTC][kDB];   // (delta, delta * xc)
    float2 ep[2][kTC][kDB];   // (D * xc, gate)
    float Bf[2][kTC][NP];
    float Cf[2][kTC][NP];
    float y[2][kTC][kDB];
};

// INTER: the intermediate-state stores are compiled in (a separate instance,
// so the plain scan's register allocation is not perturbed by them).
template <typename T, int SPT, int KT, bool INTER>
__global__ void __launch_bounds__(kThreads, 3)
scan_m1_kernel(const M1Args a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<SmemM1<T, SPT> *>(smem_raw);
    constexpr int NP = SmemM1<T, SPT>::NP;
    constexpr int NPR = SmemM1<T, SPT>::NPR;
    constexpr int VW = SPT < 4 ? SPT : 4;     // states per shared-memory vector
    constexpr int NJ = SPT / VW;
    constexpr int KW = KT - 1;                // conv window of previous raw rows

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
    // bounds-checked build: the CTA's ranges (uniform, so the whole CTA returns together)
    if (!SSM_BOUNDS(len > 0 ? start + len - 1 : 0, a.seqlen > 0 ? a.seqlen : 1, BS_M1_SEQ) ||
        !SSM_BOUNDS(d0, a.Dn, BS_M1_CHANNEL) || !SSM_BOUNDS(s, a.sv.nseqs, BS_M1_STATE))
        return;
    const int K = a.K;
    const int64_t Dn = a.Dn, N = a.N;
    const int nchunks = max(1, (int)((len + kTC - 1) / kTC));   // an empty sequence still passes its state through
    auto chunk_len = [&](int c) { return (int)max((int64_t)0, min((int64_t)kTC, len - (int64_t)c * kTC)); };

    // raw tiles of chunk c -> ring slot c % 3 (one cp.async group per chunk, empty past the end)
    auto stage = [&](int c) {
        const int rb = c % 3;
        const int64_t t0 = (int64_t)c * kTC;
        const int nv = chunk_len(c);
        if (nv > 0) {
            stage_tile<T, kDB>(&sm.rx[rb][0][0], xg + t0 * a.x_ts, a.x_ts, nv, d0, Dn, a.async_act);
            stage_tile<T, kDB>(&sm.rdt[rb][0][0], dtg + t0 * a.dt_ts, a.dt_ts, nv, d0, Dn, a.async_act);
            if (zg) stage_tile<T, kDB>(&sm.rz[rb][0][0], zg + t0 * a.z_ts, a.z_ts, nv, d0, Dn, a.async_act);
            stage_tile<T, NPR>(&sm.rB[rb][0][0], Bg + t0 * a.B_ts, a.B_ts, nv, 0, N, a.async_bc);
            stage_tile<T, NPR>(&sm.rC[rb][0][0], Cg + t0 * a.C_ts, a.C_ts, nv, 0, N, a.async_bc);
        }
        cp_async_commit();
    };

    // ---- prologue role: channel pd = tid % 32, rows [pr0, pr0 + 8)
    const int pd = tid % kDB;
    const int pr0 = (tid / kDB) * kRowsPerThread;
    const int64_t pch = d0 + pd;
    const bool pvalid = pch < Dn;
    // conv taps right-aligned in KT slots: wr[KT-1] multiplies the current
    // token, wr[KT-1-m] the input m tokens back; unused leading taps are 0, so
    // every index is static (KT = 4 covers widths up to 4, KT = 8 the rest)
    float wr[KT], cb = 0.f, dtb = 0.f;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
        const int k = K - KT + j;                             // tap index in [0, K)
        wr[j] = (pvalid && k >= 0) ? a.conv_w[pch * K + k] : 0.f;
    }
    if (pvalid && a.conv_b) cb = a.conv_b[pch];
    if (pvalid && a.dt_bias) dtb = a.dt_bias[pch];
    const float Dp = (pvalid && a.D) ? a.D[pch] : 0.f;

    // prologue of chunk c: raw slot c % 3 + halo slot c % 2 -> work slot c % 2,
    // and the halo of chunk c + 1
    auto prologue = [&](int c) {
        const int rb = c % 3, wb = c & 1;
        const int nv = chunk_len(c);
        float win[KW];                                              // raw rows t-KW .. t-1
        auto raw_at = [&](int v) -> float {                         // v: row relative to the chunk
            return v >= 0 ? Elem<T>::ld(&sm.rx[rb][v][pd]) : sm.halo[wb][kHalo + v][pd];
        };
#pragma unroll
        for (int j = 0; j < KW; ++j)                                // only the last K-1 are live
            win[j] = (j >= KW - (K - 1) && pvalid) ? raw_at(pr0 - KW + j) : 0.f;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
            const int t = pr0 + i;
            float xcv = 0.f, dlt = 0.f, gv = 1.f;
            if (t < nv && pvalid) {
                const float cur = Elem<T>::ld(&sm.rx[rb][t][pd]);
                if (K > 0) {
                    float acc = fmaf(wr[KW], cur, cb);
#pragma unroll
                    for (int j = 0; j < KW; ++j) acc = fmaf(wr[j], win[j], acc);
                    xcv = silu_fast<T>(acc);
                } else {
                    xcv = cur;
                }
#pragma unroll
                for (int j = 0; j + 1 < KW; ++j) win[j] = win[j + 1];
                if (KW > 0) win[KW - 1] = cur;
                const float u = Elem<T>::ld(&sm.rdt[rb][t][pd]) + dtb;
                dlt = a.softplus ? softplus(u) : u;
                if (zg) gv = silu_fast<T>(Elem<T>::ld(&sm.rz[rb][t][pd]));
            }
            sm.dd[wb][t][pd] = make_float2(dlt, dlt * xcv);         // delta = 0 past the end: the state stays put
            sm.ep[wb][t][pd] = make_float2(Dp * xcv, gv);
        }
        // halo of the next chunk: the last K-1 raw inputs up to this chunk's end
        if (K > 1 && tid < kDB)
            for (int j = 0; j < K - 1; ++j) {
                const int v = nv - (K - 1) + j;
                sm.halo[wb ^ 1][kHalo - (K - 1) + j][pd] = pvalid ? raw_at(v) : 0.f;
            }
        // B and C to fp32, zero past the end of the sequence and of dstate
        for (int i = tid; i < kTC * NP; i += kThreads) {
            const int t = i / NP, n = i % NP;
            const bool ok = t < nv && n < N;
            sm.Bf[wb][t][n] = ok ? Elem<T>::ld(&sm.rB[rb][t][n]) : 0.f;
            sm.Cf[wb][t][n] = ok ? Elem<T>::ld(&sm.rC[rb][t][n]) : 0.f;
        }
    };

    // y of chunk c (ysm slot c % 2) -> global, 16-byte stores when aligned
    auto store_y = [&](int c) {
        const int yb = c & 1;
        const int nv = chunk_len(c);
        const int64_t t0 = (int64_t)c * kTC;
        if (a.vec_y && d0 + kDB <= Dn) {
            for (int i = tid; i < nv * (kDB / 8); i += kThreads) {
                const int r = i / (kDB / 8), v = i % (kDB / 8);
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = sm.y[yb][r][v * 8 + e];
                if (SSM_BOUNDS(start + t0 + r, a.seqlen, BS_M1_Y)) Vec8<T>::st(yg + (t0 + r) * a.y_ts + d0 + v * 8, o);
            }
        } else {
            for (int i = tid; i < nv * kDB; i += kThreads) {
                const int r = i / kDB, v = i % kDB;
                if (d0 + v < Dn && SSM_BOUNDS(start + t0 + r, a.seqlen, BS_M1_Y))
                    Elem<T>::st(yg + (t0 + r) * a.y_ts + d0 + v, sm.y[yb][r][v]);
            }
        }
    };

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

    // recurrence over chunk c (work slot c % 2), y into ysm slot c % 2
    auto scan = [&](int c) {
        const int wb = c & 1;
#pragma unroll
        for (int t4 = 0; t4 < kTC; t4 += kLanes) {
            float acc[kLanes];
#pragma unroll
            for (int i = 0; i < kLanes; ++i) {
                const int t = t4 + i;
                const float2 dd = sm.dd[wb][t][sd];                  // (delta, delta * xc)
                if constexpr (VW >= 2) {
                    // packed fp32x2: two states per FMUL2 / FFMA2 instruction
                    const float2 dl2 = make_float2(dd.x, dd.x), dx2 = make_float2(dd.y, dd.y);
                    float2 ac2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int n0 = VW * (q + kLanes * j);
                        float2 bp[VW / 2], cp[VW / 2];
                        if constexpr (VW == 4) {
                            const float4 b4 = *reinterpret_cast<const float4 *>(&sm.Bf[wb][t][n0]);
                            const float4 c4 = *reinterpret_cast<const float4 *>(&sm.Cf[wb][t][n0]);
                            bp[0] = make_float2(b4.x, b4.y); bp[1] = make_float2(b4.z, b4.w);
                            cp[0] = make_float2(c4.x, c4.y); cp[1] = make_float2(c4.z, c4.w);
                        } else {
                            bp[0] = *reinterpret_cast<const float2 *>(&sm.Bf[wb][t][n0]);
                            cp[0] = *reinterpret_cast<const float2 *>(&sm.Cf[wb][t][n0]);
                        }
#pragma unroll
                        for (int e = 0; e < VW / 2; ++e) {
                            const int pi = j * (VW / 2) + e;
                            const float2 arg = __fmul2_rn(dl2, A2p[pi]);
                            const float2 dA = make_float2(ex2(arg.x), ex2(arg.y));
                            h2[pi] = __ffma2_rn(dA, h2[pi], __fmul2_rn(dx2, bp[e]));
                            ac2 = __ffma2_rn(cp[e], h2[pi], ac2);
                        }
                    }
                    acc[i] = ac2.x + ac2.y;
                } else {
                    float ac = 0.f;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int n0 = q + kLanes * j;
                        const float dA = ex2(dd.x * A2[j]);
                        h[j] = fmaf(dA, h[j], dd.y * sm.Bf[wb][t][n0]);
                        ac = fmaf(sm.Cf[wb][t][n0], h[j], ac);
                    }
                    acc[i] = ac;
                }
            }
            // reduce-scatter over the lanes of the channel: at each level a lane keeps
            // half of its partial sums (upper half when its bit is set) and adds the
            // partner's copy of that half; lane q ends with the sum of token t4 + q
#pragma unroll
            for (int o = kLanes / 2; o >= 1; o >>= 1) {
                const bool up = (q & o) != 0;
#pragma unroll
                for (int k = 0; k < o; ++k) {
                    const float keep = up ? acc[o + k] : acc[k];
                    const float send = up ? acc[k] : acc[o + k];
                    acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
            const float tot = acc[0];
            const int t = t4 + q;
            const float2 e2 = sm.ep[wb][t][sd];                      // (D * xc, gate)
            sm.y[wb][t][sd] = (tot + e2.x) * e2.y;
        }
    };

    // ---- intermediate state after chunk c when it closes a state interval: the
    // lanes' register states, and the conv history, which is the halo of chunk
    // c + 1 (written by the prologue of chunk c)
    auto inter_store = [&](int c) {
        const int64_t slot = a.iv.slot_after(s, (int64_t)(c + 1) * kTC);
        if (slot < 0 || !SSM_BOUNDS(slot, a.iv.nslots, BS_M1_POOL)) return;
        if (a.iv.states && svalid) {
            float *dst = a.iv.states + (slot * Dn + sch) * N;
#pragma unroll
            for (int j = 0; j < NJ; ++j)
#pragma unroll
                for (int e = 0; e < VW; ++e) {
                    const int64_t n = (int64_t)VW * (q + kLanes * j) + e;
                    float v;
                    if constexpr (SPT >= 2) {
                        const int i = j * VW + e;
                        v = (i & 1) ? h2[i / 2].y : h2[i / 2].x;
                    } else {
                        v = h[j * VW + e];
                    }
                    if (n < N) dst[n] = v;
                }
        }
        if (a.iv.conv && K > 1) {
            T *cdst = static_cast<T *>(a.iv.conv) + slot * Dn * (K - 1);
            const int hb = (c + 1) & 1;
            for (int idx = tid; idx < (K - 1) * kDB; idx += kThreads) {
                const int j = idx / kDB, d = idx % kDB;
                const int64_t ch = d0 + d;
                if (ch < Dn) Elem<T>::st(cdst + ch * (K - 1) + j, sm.halo[hb][kHalo - (K - 1) + j][d]);
            }
        }
    };

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
    stage(0);
    stage(1);
    stage(2);
    cp_async_wait<2>();                                   // chunk 0 landed (own copies)
    __syncthreads();                                      // ... everyone's copies, halo 0
    prologue(0);
    cp_async_wait<1>();                                   // chunk 1 landed
    __syncthreads();

    for (int c = 0; c < nchunks; ++c) {
        scan(c);                                          // work slot c % 2 -> ysm slot c % 2
        if constexpr (INTER) {
            if (chunk_len(c) == kTC) inter_store(c);
        }
        if (c > 0) store_y(c - 1);                        // ysm slot (c-1) % 2
        if (c + 1 < nchunks) prologue(c + 1);             // raw slot (c+1) % 3 -> work slot (c+1) % 2
        stage(c + 3);                                     // raw slot c % 3, read by prologue(c) last iteration
        cp_async_wait<1>();                               // chunk c + 2 landed
        __syncthreads();
    }
    store_y(nchunks - 1);
    // carried conv state: the halo written by the last chunk's prologue
    if (K > 1 && a.conv_state_out) {
        T *cso = static_cast<T *>(a.conv_state_out);
        const int hb = nchunks & 1;
        for (int idx = tid; idx < (K - 1) * kDB; idx += kThreads) {
            const int j = idx / kDB, d = idx % kDB;
            const int64_t ch = d0 + d;
            if (ch < Dn) Elem<T>::st(cso + ((int64_t)s * Dn + ch) * (K - 1) + j, sm.halo[hb][kHalo - (K - 1) + j][d]);
        }
    }
    cp_async_wait<0>();
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
    auto kern = a.iv.interval > 0 ? scan_m1_kernel<T, SPT, kMaxConvWidth, true>
                : a.K <= 4          ? scan_m1_kernel<T, SPT, 4, false>
                                    : scan_m1_kernel<T, SPT, kMaxConvWidth, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.Dn + kDB - 1) / kDB), (unsigned)nseqs);
    timing_begin(st);
    kern<<<grid, kThreads, smem, st>>>(a);
    timing_end(st);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(M1Args a, int nseqs, cudaStream_t st) {
    constexpr int E = 16 / sizeof(T);
    // B / C rows go through 16-byte copies only when dstate fills whole vectors
    // and the padded row (4 * SPT elements) keeps every row 16-byte aligned.
    auto bc_ok = [&](int np) { return a.async_bc && a.N % E == 0 && (np * (int)sizeof(T)) % 16 == 0; };
    if (a.N <= kLanes * 1) { a.async_bc = bc_ok(kLanes * 1); return launch_spt<T, 1>(a, nseqs, st); }
    if (a.N <= kLanes * 2) { a.async_bc = bc_ok(kLanes * 2); return launch_spt<T, 2>(a, nseqs, st); }
    if (a.N <= kLanes * 4) { a.async_bc = bc_ok(kLanes * 4); return launch_spt<T, 4>(a, nseqs, st); }
    if (a.N <= kLanes * 8) { a.async_bc = bc_ok(kLanes * 8); return launch_spt<T, 8>(a, nseqs, st); }
    a.async_bc = bc_ok(kLanes * 16);
    return launch_spt<T, 16>(a, nseqs, st);
}

// ===================================================================== time-parallel form
// Mamba-1 scan with the tokens of a chunk spread over the lanes of a warp and
// joined by a warp-shuffle prefix of the scan element (exp(delta A), h)
// ("Adding Initial Value Support to Selective Scan Forward Kernel",
// state-spaces/mamba issue 285: the pair, composed associatively, seeded with
// (1, h0) and carried across chunks in fp32).
//
// One CTA owns one sequence and DB = 16 channels (8 when 16 would leave SMs
// without a CTA); 8 warps; chunks of TP_TC = 64 tokens.  In the scan, warp w
// takes channels 2w and 2w + 1 in turn (channel w when DB = 8), and lane
// l = 4 r + q takes the run of tokens 8r .. 8r+7 and the four
// states 16 g + 4 q .. 16 g + 4 q + 3 of state group g.  Per (channel, group):
//   1. each lane walks its run from the identity (1, 0):
//      a_t = exp(delta_t A), P = prod a_t, Q = a_t Q + delta_t x_t B_t
//      (a_t and delta_t x_t B_t are kept for step 3);
//   2. an inclusive shuffle scan over the 8 runs composes (P, Q) pairs,
//      (P2, Q2) o (P1, Q1) = (P2 P1, P2 Q1 + Q2);
//   3. the lane's entering state h = P_excl carry + Q_excl (carry = the
//      state at the chunk start, h0 for the first chunk) and a second walk
//      h = a_t h + delta_t x_t B_t with the read-out C_t . h;
//   4. the chunk's end state (run 7's inclusive pair applied to the carry) is
//      the next carry.
// Each lane holds the partial read-out of its four states; a two-level
// shuffle reduce-scatter over the four state lanes sums them (two tokens per
// lane), then y = (sum + D xc) silu(z).
//
// A cooperative prologue per chunk (thread = channel x 4 or 2 tokens) computes the
// conv + SiLU, delta = softplus(dt + dt_bias), delta xc, D xc and the gate,
// and widens B / C to fp32, into shared-memory layouts padded so that both
// the prologue's writes (lanes = channels) and the scan's reads (lanes = runs)
// are free of bank conflicts.  Software pipeline, one barrier per chunk:
// iteration c scans chunk c, stores y of chunk c-1, runs the prologue of chunk
// c+1 and issues the copies of chunk c+2 (raw tiles double-buffered).
constexpr int TP_TC = 64;            // tokens per chunk
constexpr int TP_THREADS = 256;
constexpr int TP_RUNS = 8;           // runs of 8 tokens per chunk (one per 4 lanes)
// DD / EP rows: per channel 8 runs of 9 float2 (8 tokens + 1 pad), + 1 float2
constexpr int TP_RUN_F2 = 9;
constexpr int TP_CH_F2 = TP_RUNS * TP_RUN_F2 + 1;   // 73 float2 = 584 bytes
SSM_DEVINL int tp_dd(int c, int t) { return c * TP_CH_F2 + (t >> 3) * TP_RUN_F2 + (t & 7); }
// B / C rows (fp32, N wide): every 8 rows are followed by 16 pad floats
template <int N>
SSM_DEVINL int tp_bc(int t, int n) { return t * N + (t >> 3) * 16 + n; }

template <typename T, int N, int DB>
struct SmemTP {
    static constexpr int BCROWS = TP_TC * N + (TP_TC / 8) * 16;
    T rx[2][TP_TC][DB];
    T rdt[2][TP_TC][DB];
    T rz[2][TP_TC][DB];
    T rB[2][TP_TC][N];
    T rC[2][TP_TC][N];
    float halo[2][kHalo][DB];
    float2 dd[2][DB * TP_CH_F2];      // (delta, delta * xc)
    float2 ep[2][DB * TP_CH_F2];      // (D * xc, gate)
    alignas(16) float Bf[2][BCROWS];
    alignas(16) float Cf[2][BCROWS];
    float y[2][TP_TC][DB + 1];        // +1: conflict-free column writes
    alignas(16) float carry[DB][N];   // state at the chunk start
    alignas(16) float A2[DB][N];      // A * log2(e)
};

// rows [0, nv) x NCOLS columns of a token-major tensor -> dst[TP_TC][NCOLS]
template <typename T, int NCOLS>
SSM_DEVINL void tp_stage(T *dst, const T *src, int64_t ts, int nv, int64_t col0, int64_t col_end, bool async) {
    constexpr int E = 16 / sizeof(T);
    constexpr int PER_ROW = NCOLS / E;
    static_assert(NCOLS % E == 0, "tile rows must be whole 16-byte vectors");
    if (async) {
        for (int i = threadIdx.x; i < TP_TC * PER_ROW; i += TP_THREADS) {
            const int r = i / PER_ROW, v = i % PER_ROW;
            const int64_t c = col0 + (int64_t)v * E;
            if (r < nv && c + E <= col_end) cp_async16(dst + r * NCOLS + v * E, src + r * ts + c);
        }
    } else {
        for (int i = threadIdx.x; i < nv * NCOLS; i += TP_THREADS) {
            const int r = i / NCOLS, v = i % NCOLS;
            const int64_t c = col0 + v;
            if (c < col_end) dst[r * NCOLS + v] = src[r * ts + c];
        }
    }
}

template <typename T, int N, int DB, bool INTER>
__global__ void __launch_bounds__(TP_THREADS, 2)
scan_m1_tp_kernel(const M1Args a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<SmemTP<T, N, DB> *>(smem_raw);
    constexpr int TPR = TP_TC * DB / TP_THREADS;     // prologue tokens per thread
    constexpr int CPW = DB / (TP_THREADS / 32);       // channels per warp in the scan
    constexpr int NG = N / 16;               // state groups of 16 (4 lanes x 4 states)
    if (a.sv.err && *a.sv.err != 0) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t d0 = (int64_t)blockIdx.x * DB;
    const int s = a.sv.order ? a.sv.order[blockIdx.y] : (int)blockIdx.y;
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
    // bounds-checked build: the CTA's ranges (uniform, so the whole CTA returns together)
    if (!SSM_BOUNDS(len > 0 ? start + len - 1 : 0, a.seqlen > 0 ? a.seqlen : 1, BS_M1_SEQ) ||
        !SSM_BOUNDS(d0, a.Dn, BS_M1_CHANNEL) || !SSM_BOUNDS(s, a.sv.nseqs, BS_M1_STATE))
        return;
    const int K = a.K;
    const int64_t Dn = a.Dn;
    const int nchunks = max(1, (int)((len + TP_TC - 1) / TP_TC));   // an empty sequence still passes its state through
    auto chunk_len = [&](int c) { return (int)max((int64_t)0, min((int64_t)TP_TC, len - (int64_t)c * TP_TC)); };

    auto stage = [&](int c) {
        const int rb = c & 1;
        const int64_t t0 = (int64_t)c * TP_TC;
        const int nv = chunk_len(c);
        if (nv > 0) {
            tp_stage<T, DB>(&sm.rx[rb][0][0], xg + t0 * a.x_ts, a.x_ts, nv, d0, Dn, a.async_act);
            tp_stage<T, DB>(&sm.rdt[rb][0][0], dtg + t0 * a.dt_ts, a.dt_ts, nv, d0, Dn, a.async_act);
            if (zg) tp_stage<T, DB>(&sm.rz[rb][0][0], zg + t0 * a.z_ts, a.z_ts, nv, d0, Dn, a.async_act);
            tp_stage<T, N>(&sm.rB[rb][0][0], Bg + t0 * a.B_ts, a.B_ts, nv, 0, N, a.async_bc);
            tp_stage<T, N>(&sm.rC[rb][0][0], Cg + t0 * a.C_ts, a.C_ts, nv, 0, N, a.async_bc);
        }
        cp_async_commit();
    };

    // ---- prologue role: channel pc = tid % DB, tokens TPR * (tid / DB) .. + TPR - 1
    const int pc = tid % DB;
    const int pt0 = (tid / DB) * TPR;
    const int64_t pch = d0 + pc;
    const bool pvalid = pch < Dn;
    float wr[4], cb = 0.f, dtb = 0.f;                  // taps right-aligned: wr[3] multiplies the current token
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k = K - 4 + j;
        wr[j] = (pvalid && k >= 0) ? a.conv_w[pch * K + k] : 0.f;
    }
    if (pvalid && a.conv_b) cb = a.conv_b[pch];
    if (pvalid && a.dt_bias) dtb = a.dt_bias[pch];
    const float Dp = (pvalid && a.D) ? a.D[pch] : 0.f;

    auto prologue = [&](int c) {
        const int rb = c & 1, wb = c & 1;
        const int nv = chunk_len(c);
        auto raw_at = [&](int v) -> float {             // v: row relative to the chunk
            return v >= 0 ? Elem<T>::ld(&sm.rx[rb][v][pc]) : sm.halo[wb][kHalo + v][pc];
        };
        float w0 = 0.f, w1 = 0.f, w2 = 0.f;               // raw rows t-3, t-2, t-1
        if (pvalid) {
            if (K > 3) w0 = raw_at(pt0 - 3);
            if (K > 2) w1 = raw_at(pt0 - 2);
            if (K > 1) w2 = raw_at(pt0 - 1);
        }
#pragma unroll
        for (int i = 0; i < TPR; ++i) {
            const int t = pt0 + i;
            float xcv = 0.f, dlt = 0.f, gv = 1.f;
            float cur = 0.f;
            if (t < nv && pvalid) {
                cur = Elem<T>::ld(&sm.rx[rb][t][pc]);
                if (K > 0) {
                    float acc = fmaf(wr[3], cur, cb);
                    acc = fmaf(wr[2], w2, acc);
                    acc = fmaf(wr[1], w1, acc);
                    acc = fmaf(wr[0], w0, acc);
                    xcv = silu_fast<T>(acc);
                } else {
                    xcv = cur;
                }
                const float u = Elem<T>::ld(&sm.rdt[rb][t][pc]) + dtb;
                dlt = a.softplus ? softplus(u) : u;
                if (zg) gv = silu_fast<T>(Elem<T>::ld(&sm.rz[rb][t][pc]));
            }
            w0 = w1; w1 = w2; w2 = cur;
            sm.dd[wb][tp_dd(pc, t)] = make_float2(dlt, dlt * xcv);   // delta = 0 past the end: the state stays put
            sm.ep[wb][tp_dd(pc, t)] = make_float2(Dp * xcv, gv);
        }
        // halo of the next chunk: the last K-1 raw inputs up to this chunk's end
        if (K > 1 && tid < DB)
            for (int j = 0; j < K - 1; ++j) {
                const int v = nv - (K - 1) + j;
                sm.halo[wb ^ 1][kHalo - (K - 1) + j][pc] = pvalid ? raw_at(v) : 0.f;
            }
        // B and C to fp32 (zero past the end of the sequence)
        for (int i = tid; i < TP_TC * N; i += TP_THREADS) {
            const int t = i / N, n = i % N;
            const bool ok = t < nv;
            sm.Bf[wb][tp_bc<N>(t, n)] = ok ? Elem<T>::ld(&sm.rB[rb][t][n]) : 0.f;
            sm.Cf[wb][tp_bc<N>(t, n)] = ok ? Elem<T>::ld(&sm.rC[rb][t][n]) : 0.f;
        }
    };

    // y of chunk c -> global, 16-byte stores when aligned
    auto store_y = [&](int c) {
        const int yb = c & 1;
        const int nv = chunk_len(c);
        const int64_t t0 = (int64_t)c * TP_TC;
        if (a.vec_y && d0 + DB <= Dn) {
            for (int i = tid; i < nv * (DB / 8); i += TP_THREADS) {
                const int r = i / (DB / 8), v = i % (DB / 8);
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = sm.y[yb][r][v * 8 + e];
                if (SSM_BOUNDS(start + t0 + r, a.seqlen, BS_M1_Y)) Vec8<T>::st(yg + (t0 + r) * a.y_ts + d0 + v * 8, o);
            }
        } else {
            for (int i = tid; i < nv * DB; i += TP_THREADS) {
                const int r = i / DB, v = i % DB;
                if (d0 + v < Dn && SSM_BOUNDS(start + t0 + r, a.seqlen, BS_M1_Y))
                    Elem<T>::st(yg + (t0 + r) * a.y_ts + d0 + v, sm.y[yb][r][v]);
            }
        }
    };

    // ---- scan role: lane = 4 r + q (run r, state quarter q), channels CPW warp .. CPW warp + CPW - 1
    const int r = lane >> 2, q = lane & 3;
    // where the reduce-scatter leaves this lane's two tokens: 8 r + jb, 8 r + jb + 1
    const int jb = (q & 1) * 4 + (q & 2);

    auto scan = [&](int c) {
        const int wb = c & 1;
#pragma unroll 1
        for (int cc = 0; cc < CPW; ++cc) {
            const int ch = warp * CPW + cc;
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const int n0 = 16 * g + 4 * q;
                const float4 A4 = *reinterpret_cast<const float4 *>(&sm.A2[ch][n0]);
                const float2 Aa = make_float2(A4.x, A4.y), Ab = make_float2(A4.z, A4.w);
                // 1. walk the run from (1, 0)
                float2 aa[8], ab[8], ba[8], bb[8];         // a_t and delta_t x_t B_t, states (0,1) and (2,3)
                float2 Pa = make_float2(1.f, 1.f), Pb = Pa, Qa = make_float2(0.f, 0.f), Qb = Qa;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = r * 8 + j;
                    const float2 dd = sm.dd[wb][tp_dd(ch, t)];
                    const float4 b4 = *reinterpret_cast<const float4 *>(&sm.Bf[wb][tp_bc<N>(t, n0)]);
                    const float2 dl = make_float2(dd.x, dd.x), dx = make_float2(dd.y, dd.y);
                    const float2 ea = __fmul2_rn(dl, Aa), eb = __fmul2_rn(dl, Ab);
                    aa[j] = make_float2(ex2(ea.x), ex2(ea.y));
                    ab[j] = make_float2(ex2(eb.x), ex2(eb.y));
                    ba[j] = __fmul2_rn(dx, make_float2(b4.x, b4.y));
                    bb[j] = __fmul2_rn(dx, make_float2(b4.z, b4.w));
                    Qa = __ffma2_rn(aa[j], Qa, ba[j]);
                    Qb = __ffma2_rn(ab[j], Qb, bb[j]);
                    Pa = __fmul2_rn(Pa, aa[j]);
                    Pb = __fmul2_rn(Pb, ab[j]);
                }
                // 2. inclusive scan over the runs (lanes 4 apart)
#pragma unroll
                for (int o = 1; o < TP_RUNS; o <<= 1) {
                    const float pax = __shfl_up_sync(0xffffffffu, Pa.x, 4 * o), pay = __shfl_up_sync(0xffffffffu, Pa.y, 4 * o);
                    const float pbx = __shfl_up_sync(0xffffffffu, Pb.x, 4 * o), pby = __shfl_up_sync(0xffffffffu, Pb.y, 4 * o);
                    const float qax = __shfl_up_sync(0xffffffffu, Qa.x, 4 * o), qay = __shfl_up_sync(0xffffffffu, Qa.y, 4 * o);
                    const float qbx = __shfl_up_sync(0xffffffffu, Qb.x, 4 * o), qby = __shfl_up_sync(0xffffffffu, Qb.y, 4 * o);
                    if (r >= o) {
                        Qa = __ffma2_rn(Pa, make_float2(qax, qay), Qa);
                        Qb = __ffma2_rn(Pb, make_float2(qbx, qby), Qb);
                        Pa = __fmul2_rn(Pa, make_float2(pax, pay));
                        Pb = __fmul2_rn(Pb, make_float2(pbx, pby));
                    }
                }
                // 3. the run's entering state from the exclusive prefix and the chunk carry
                const float4 cr4 = *reinterpret_cast<const float4 *>(&sm.carry[ch][n0]);
                const float2 ca = make_float2(cr4.x, cr4.y), cb2 = make_float2(cr4.z, cr4.w);
                float2 ha = __ffma2_rn(Pa, ca, Qa), hb = __ffma2_rn(Pb, cb2, Qb);   // state at the run's end
                {
                    const float hax = __shfl_up_sync(0xffffffffu, ha.x, 4), hay = __shfl_up_sync(0xffffffffu, ha.y, 4);
                    const float hbx = __shfl_up_sync(0xffffffffu, hb.x, 4), hby = __shfl_up_sync(0xffffffffu, hb.y, 4);
                    // 4. the chunk's end state (run 7) is the next carry
                    const float ex = __shfl_sync(0xffffffffu, ha.x, 28 + q), ey = __shfl_sync(0xffffffffu, ha.y, 28 + q);
                    const float fx = __shfl_sync(0xffffffffu, hb.x, 28 + q), fy = __shfl_sync(0xffffffffu, hb.y, 28 + q);
                    ha = r > 0 ? make_float2(hax, hay) : ca;
                    hb = r > 0 ? make_float2(hbx, hby) : cb2;
                    __syncwarp();
                    if (r == 0) *reinterpret_cast<float4 *>(&sm.carry[ch][n0]) = make_float4(ex, ey, fx, fy);
                }
                // second walk with the read-out
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = r * 8 + j;
                    const float4 c4 = *reinterpret_cast<const float4 *>(&sm.Cf[wb][tp_bc<N>(t, n0)]);
                    ha = __ffma2_rn(aa[j], ha, ba[j]);
                    hb = __ffma2_rn(ab[j], hb, bb[j]);
                    const float2 s2 = __ffma2_rn(make_float2(c4.z, c4.w), hb, __fmul2_rn(make_float2(c4.x, c4.y), ha));
                    acc[j] += s2.x + s2.y;
                }
            }
            // reduce-scatter over the four state lanes: lane q keeps tokens jb, jb + 1 of its run
            {
                const bool up1 = (q & 1) != 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float keep = up1 ? acc[4 + k] : acc[k];
                    const float send = up1 ? acc[k] : acc[4 + k];
                    acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                }
                const bool up2 = (q & 2) != 0;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float keep = up2 ? acc[2 + k] : acc[k];
                    const float send = up2 ? acc[k] : acc[2 + k];
                    acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                }
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = r * 8 + jb + k;
                const float2 e2 = sm.ep[wb][tp_dd(ch, t)];          // (D * xc, gate)
                sm.y[wb][t][ch] = (acc[k] + e2.x) * e2.y;
            }
        }
    };

    // ---- intermediate state after chunk c when it closes a state interval:
    // the carry (the state at the end of chunk c) and the conv history, which
    // is the halo the prologue of chunk c left for chunk c + 1
    auto inter_store = [&](int c) {
        const int64_t slot = a.iv.slot_after(s, (int64_t)(c + 1) * TP_TC);
        if (slot < 0 || !SSM_BOUNDS(slot, a.iv.nslots, BS_M1_POOL)) return;
        if (a.iv.states)
            for (int i = tid; i < DB * N; i += TP_THREADS) {
                const int cidx = i / N, n = i % N;
                if (d0 + cidx < Dn) a.iv.states[(slot * Dn + d0 + cidx) * N + n] = sm.carry[cidx][n];
            }
        if (a.iv.conv && K > 1) {
            T *cdst = static_cast<T *>(a.iv.conv) + slot * Dn * (K - 1);
            const int hb = (c + 1) & 1;
            for (int idx = tid; idx < (K - 1) * DB; idx += TP_THREADS) {
                const int j = idx / DB, dd = idx % DB;
                if (d0 + dd < Dn) Elem<T>::st(cdst + (d0 + dd) * (K - 1) + j, sm.halo[hb][kHalo - (K - 1) + j][dd]);
            }
        }
    };

    // ---- initial state, A, conv halo of chunk 0
    for (int i = tid; i < DB * N; i += TP_THREADS) {
        const int cidx = i / N, n = i % N;
        const int64_t ch = d0 + cidx;
        const bool ok = ch < Dn;
        sm.A2[cidx][n] = ok ? a.A[ch * N + n] * kLog2e : 0.f;
        sm.carry[cidx][n] = (ok && a.h0) ? a.h0[((int64_t)s * Dn + ch) * N + n] : 0.f;
    }
    if (K > 1) {
        const T *csi = static_cast<const T *>(a.conv_state_in);
        for (int idx = tid; idx < (K - 1) * DB; idx += TP_THREADS) {
            const int j = idx / DB, dd = idx % DB;
            const int64_t ch = d0 + dd;
            sm.halo[0][kHalo - (K - 1) + j][dd] =
                (csi && ch < Dn) ? Elem<T>::ld(csi + ((int64_t)s * Dn + ch) * (K - 1) + j) : 0.f;
        }
    }
    stage(0);
    stage(1);
    cp_async_wait<1>();                                   // chunk 0 landed (own copies)
    __syncthreads();                                      // ... everyone's copies, halo 0, carry, A
    prologue(0);
    __syncthreads();
    for (int c = 0; c < nchunks; ++c) {
        scan(c);                                          // work slot c % 2 -> y slot c % 2, carry
        if (c > 0) store_y(c - 1);                        // y slot (c-1) % 2
        cp_async_wait<0>();                               // chunk c + 1 landed (own copies)
        __syncthreads();                                  // everyone's copies; the carry of chunk c
        if constexpr (INTER) {
            if (chunk_len(c) == TP_TC) inter_store(c);
        }
        if (c + 1 < nchunks) prologue(c + 1);             // raw slot (c+1) % 2 -> work slot (c+1) % 2
        stage(c + 2);                                     // raw slot c % 2, read by prologue(c) last iteration
        __syncthreads();
    }
    store_y(nchunks - 1);
    // carried conv state: the halo written by the last chunk's prologue
    if (K > 1 && a.conv_state_out) {
        T *cso = static_cast<T *>(a.conv_state_out);
        const int hb = nchunks & 1;
        for (int idx = tid; idx < (K - 1) * DB; idx += TP_THREADS) {
            const int j = idx / DB, dd = idx % DB;
            const int64_t ch = d0 + dd;
            if (ch < Dn) Elem<T>::st(cso + ((int64_t)s * Dn + ch) * (K - 1) + j, sm.halo[hb][kHalo - (K - 1) + j][dd]);
        }
    }
    cp_async_wait<0>();
    if (a.h_final)
        for (int i = tid; i < DB * N; i += TP_THREADS) {
            const int cidx = i / N, n = i % N;
            const int64_t ch = d0 + cidx;
            if (ch < Dn) a.h_final[((int64_t)s * Dn + ch) * N + n] = sm.carry[cidx][n];
        }
}

template <typename T, int N, int DB>
cudaError_t launch_tp_n(const M1Args &a, int nseqs, cudaStream_t st) {
    const size_t smem = sizeof(SmemTP<T, N, DB>);
    auto kern = a.iv.interval > 0 ? scan_m1_tp_kernel<T, N, DB, true> : scan_m1_tp_kernel<T, N, DB, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.Dn + DB - 1) / DB), (unsigned)nseqs);
    timing_begin(st);
    kern<<<grid, TP_THREADS, smem, st>>>(a);
    timing_end(st);
    return cudaGetLastError();
}

// The time-parallel form takes dstate 16 or 32 and conv width <= 4.
bool tp_supported(const M1Args &a) { return (a.N == 16 || a.N == 32) && a.K <= 4; }

template <typename T>
cudaError_t launch_tp(M1Args a, int nseqs, cudaStream_t st) {
    constexpr int E = 16 / sizeof(T);
    // B / C rows: 16-byte copies when dstate fills whole vectors (16 and 32 do)
    a.async_bc = a.async_bc && a.N % E == 0;
    // 8 channels per CTA (one warp per channel) when 16 would leave SMs without a CTA
    if ((int64_t)nseqs * ((a.Dn + 15) / 16) < sm_count())
        return a.N == 16 ? launch_tp_n<T, 16, 8>(a, nseqs, st) : launch_tp_n<T, 32, 8>(a, nseqs, st);
    return a.N == 16 ? launch_tp_n<T, 16, 16>(a, nseqs, st) : launch_tp_n<T, 32, 16>(a, nseqs, st);
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
    a.iv = inter_view(s);
    const int nseqs = s.cu_seqlens ? s.nseqs : (int)s.batch;
    if (nseqs == 0) return cudaSuccess;
    // The sequential form runs four warps per (sequence, 32 channels), each lane
    // walking every token of its channel; with fewer than about seven such warps
    // per SM its dependent chains leave the SM idle, and the time-parallel form
    // (whose lanes cover the tokens of a chunk) is faster.  Measured on B200,
    // bf16, dstate 16: 1536 sequential warps 0.31 vs 0.42 ms (sequential
    // wins), 768 warps 0.27 vs 0.24 ms, 192 warps 0.92 vs 0.41 ms.
    const int64_t seq_warps = (int64_t)nseqs * ((s.d_inner + 31) / 32) * 4;
    if (tp_supported(a) && seq_warps < 7 * (int64_t)sm_count())
        return s.dtype == SSM_BF16 ? launch_tp<__nv_bfloat16>(a, nseqs, st) : launch_tp<float>(a, nseqs, st);
    return s.dtype == SSM_BF16 ? launch_typed<__nv_bfloat16>(a, nseqs, st) : launch_typed<float>(a, nseqs, st);
}

// SM count of the current device (queried once per device; 148 when there is
// no device to ask, so host-only callers still get a deterministic answer).
int sm_count() {
    static int counts[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (counts[dev] == 0) {
        int n = 0;
        counts[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
    }
    return counts[dev];
}

}  // namespace ssm
