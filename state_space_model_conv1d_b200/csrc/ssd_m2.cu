// ssd_m2.cu -- Mamba-2 scan as the chunked state-space-dual (SSD) form on the
// sm_100a tensor cores (tcgen05 MMA, fp32 accumulators in tensor memory).
//
// The recurrence (scalar A per head, B / C shared by a contiguous group of
// heads; "Tensor-parallel SSM", Fast-LLM PR 333, repeat_interleave thread):
//   S_t = exp(delta_t A) S_{t-1} + delta_t x_t B_t^T,   y_t = S_t C_t + D x_t
// is evaluated exactly (up to rounding) chunk by chunk.  For a chunk of Q
// tokens with cs_i = sum_{j<=i} delta_j A (the running log-decay):
//   G     = C B^T                                             (Q x Q)
//   M     = G o L,  L[i, j] = exp(cs_i - cs_j) delta_j for j <= i, else 0
//   Y     = M X + diag(exp(cs)) (C S_prev^T)                  (Q x P)
//   S     = exp(cs_Q) S_prev + B^T X',  X'[j] = exp(cs_Q - cs_j) delta_j X[j]
// with S_prev = h0 for the first chunk ("Adding Initial Value Support to
// Selective Scan Forward Kernel", state-spaces/mamba issue 285: the carried
// state seeds the scan).  The kernel names in "Clean up SSM ops directory
// structure" (Megatron-LM PR 6444: ssd_bmm, ssd_chunk_state,
// ssd_state_passing, ssd_chunk_scan) are these four steps; here they are one
// kernel whose carried state never leaves the SM.
//
// Work: one CTA per (sequence, head), two CTAs per SM; sequences that leave
// the GPU short of CTAs are cut into token segments, one CTA per (segment,
// head), seeded by a state-only pass (the segment-states section below).
// Fixed-length rows are cut on the host; packed sequences, whose lengths only
// the device holds, by a segment table a one-CTA pre-pass writes.  The B / C causal conv + SiLU is shared by the heads of a group, so
// it runs once per group in a pre-pass that writes bf16 B, C into the
// workspace; the x conv + SiLU runs here.  Per chunk of Q = 64 tokens, four
// tensor-core products:
//   G   = C B^T     M=64  N=64 K=128  A K-major,  B K-major      -> TMEM 0..63
//   Yo  = C S^T     M=64  N=64 K=128  A K-major,  B MN-major     -> TMEM 128..191
//   Sc  = B^T X'    M=128 N=64 K=64   A MN-major, B MN-major     -> TMEM 192..255
//   Y   = M X       M=64  N=64 K=64   A K-major,  B MN-major     -> TMEM 64..127
// B and C are used as loaded (shared by every head of the group): the decay
// of the chunk-state product rides on X' (written by the x conv next to X),
// and the exp(cs_i) factor of the state read-out is applied to Yo in the
// epilogue, so no operand tile is rescaled in place.
//
// Warp roles.  Warps 0-7 compute; warp 8 is the control warp.  Its lane 0
// issues every TMA load and every MMA as soon as the inputs are ready
// (mbarriers), and the whole warp computes the per-chunk decay tables three
// chunks ahead, so no compute warp issues, waits to issue, or scans delta.
// Compute iteration k:
//   conv(k+1)   raw x -> X (double-buffered), X'             overlaps MMA Y(k)
//   epilogue(k) y = (Y + exp(cs) Yo) silu(z), written over z(k) in the z tile
//   S(k)        S = exp(cs_Q) S + Sc (fp32 registers) -> bf16 copy for Yo(k+1),
//               announced before the y tile's TMA store (which waits for every
//               warp), so Sc / Yo of k+1 do not wait for that barrier
//   mask(k+1)   G -> M
// and the control warp, for chunk k+1: G as soon as B / C have landed; the
// raw x of chunk k+3 once conv(k+1) has read its staging buffer (raw x is
// double-buffered, so a load has two chunks to land); z of chunk k+1 once the
// epilogue has read z(k); Sc and Yo once S(k) is written; Y once the mask is
// written; B / C of chunk k+2 once G, Sc and Yo have read them.  The serial
// chain across chunks is only the fp32 state update.
//
// Tensor memory: 256 columns.  Shared memory ~111 KB.  All mbarrier waits
// are bounded; a wait that runs out records SSM_DEVERR_TIMEOUT, raises a CTA
// abort flag that ends every other wait, and the CTA drains its in-flight
// copies and MMAs before it frees tensor memory and returns.
#include <stddef.h>
#include <cmath>
#include <string.h>

#include <type_traits>

#include "common.cuh"
#include "launch.h"
#include "tc05.cuh"

namespace ssm {
namespace {

constexpr int kQ = 64;                     // chunk length
constexpr int kP = 64;                     // headdim on this path
constexpr int kN = 128;                    // dstate on this path
constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 32;   // + the control warp
constexpr int kHx = 3;                     // raw x rows kept before each chunk (conv width <= 4)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t TM_G = 0, TM_Y = 64, TM_YO = 128, TM_SC = 192;

// Operand tiles (bf16, 128-byte swizzle, atoms of 8 rows x 64 elements), byte
// offsets from the 1024-aligned base of dynamic shared memory.
constexpr uint32_t OFF_C = 0;          // C rows i, K = n: two 8 KB K-atoms (n 0-63 | 64-127)
constexpr uint32_t OFF_B = 16384;      // B rows j, K = n (G); read as MN-major MN = n, K = j (Sc)
constexpr uint32_t OFF_S = 32768;      // bf16 S rows n, 64 p each: MN-major MN = p, K = n (Yo)
constexpr uint32_t OFF_M = 49152;      // M rows i, K = j (blocks above the diagonal stay zero)
constexpr uint32_t OFF_X = 57344;      // X rows j, 64 p: two buffers (chunk parity)
constexpr uint32_t OFF_XP = 73728;     // X' rows j, 64 p
constexpr uint32_t OFF_XR = 81920;     // raw x rows (row-major, 128 bytes each): two buffers
constexpr uint32_t OFF_Z = 98304;      // z rows i, 64 p (128-byte swizzle); y staged over it
constexpr uint32_t OFF_AUX = 106496;

// per-chunk decay tables (three slots: chunk c lives in slot c % 3 and is read
// in compute iterations c-1 and c; the control warp fills slot c % 3 with
// chunk c + 3 once S(c) is done)
struct alignas(16) Tables {            // 16-byte aligned: the x conv reads wj as float4
    float dlt[kQ];                   // delta
    float cs2[kQ];                   // running log2-decay
    float ecs[kQ];                   // exp(cs_i)
    float wj[kQ];                    // exp(cs_Q - cs_j) * delta_j
    float rf[kQ];                    // exp(cs_i - cs_{16*(i/16)}): row factor to the start of its block
    float cf[kQ];                    // exp(cs_{16*(j/16)+15} - cs_j) * delta_j: column factor to the end of its block
    float bf[4][4];                  // exp(cs_{16*I} - cs_{16*J+15}) for blocks J < I
    float dAc;                       // exp(cs_Q)
};
// mbarriers.  Raw x has one barrier per buffer (a buffer completes every
// other chunk); the tables one per slot.
enum {
    MB_X0, MB_X1, MB_BC, MB_Z, MB_G, MB_MMA, MB_BCFREE, MB_CONV, MB_ZFREE, MB_SREADY, MB_MREADY,
    MB_T0, MB_T1, MB_T2, MB_DRAIN, kNumMbar
};
struct Aux {
    float xh[2][kHx][kP];            // raw x rows before the chunk (double buffered)
    Tables tab[3];                   // at a 16-byte offset (xh is 1536 bytes)
    uint32_t tmem;
    int abort;
    uint64_t mb[kNumMbar];
};
static_assert(sizeof(Tables) % 16 == 0 && offsetof(Aux, tab) % 16 == 0, "table slots must be 16-byte aligned");
constexpr size_t kSmemBytes = OFF_AUX + sizeof(Aux) + 1024;   // + slack to align the base to 1024

constexpr uint32_t ID_G = tc::idesc_bf16(64, 64, 0, 0);
constexpr uint32_t ID_Y = tc::idesc_bf16(64, 64, 0, 1);
constexpr uint32_t ID_S = tc::idesc_bf16(128, 64, 1, 1);

struct SsdArgs {
    const __nv_bfloat16 *x, *z, *dt, *Bc, *Cc;
    __nv_bfloat16 *y;
    int64_t x_bs, x_ts, z_bs, z_ts, dt_bs, dt_ts, b_bs, b_ts, c_bs, c_ts, y_bs, y_ts;
    const float *A, *D, *dt_bias, *h0, *conv_w, *conv_b;
    float *h_final;
    const __nv_bfloat16 *conv_state_in;
    __nv_bfloat16 *conv_state_out;
    int64_t H, G, seqlen, cdim;
    int K, softplus;
    SeqView sv;
    int32_t *err;
    InterView iv;
    const __nv_bfloat16 *Braw, *Craw;   // the unconvolved B / C (intermediate conv history)
    int64_t braw_bs, braw_ts, craw_bs, craw_ts;
    // Segments of fixed-length rows (nseg = 1 otherwise): row s is cut into
    // nseg runs of seg_len tokens (whole chunks; the last one takes the rest).
    // sloc / slog hold, for every segment but the last, the state it leaves when
    // scanned from zero and its total log2-decay ([s][sg][H] rows of P x N, [s][sg][H];
    // for packed sequences [table entry][H]).
    int nseg;
    int64_t seg_len;
    float *sloc, *slog;
    // Packed sequences cut on the device: entry y of seg_tab is (sequence,
    // segment, segments of the sequence, sloc row of its segment 0); CTAs
    // from *seg_count on have no segment.  Null otherwise.
    const int4 *seg_tab;
    const int32_t *seg_count;
    int64_t nsloc;                      // rows of sloc / slog
};

SSM_DEVINL void st16(void *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }

// The segment a CTA row scans: its index within the sequence, whether it is
// the sequence's last, and the sloc / slog row of the sequence's segment 0.
SSM_DEVINL int seg_index(const SsdArgs &a) {
    if (a.seg_tab) return a.seg_tab[blockIdx.y].y;
    return a.sv.order ? 0 : (int)blockIdx.y % a.nseg;
}
SSM_DEVINL bool seg_is_last(const SsdArgs &a) {
    if (a.seg_tab) {
        const int4 e = a.seg_tab[blockIdx.y];
        return e.y == e.z - 1;
    }
    return a.sv.order || (int)blockIdx.y % a.nseg == a.nseg - 1;
}
SSM_DEVINL int64_t seg_row0(const SsdArgs &a, int s) {
    return a.seg_tab ? (int64_t)a.seg_tab[blockIdx.y].w : (int64_t)s * (a.nseg - 1);
}
SSM_DEVINL void bar_compute() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }
SSM_DEVINL void mb_arrive(uint64_t *mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(tc::smem_u32(mbar)) : "memory");
}

// Bounded wait on one mbarrier phase that also gives up as soon as another
// thread of the CTA has raised the abort flag.  The waiting thread is
// suspended inside try_wait (no time hint: the hardware wakes it when the
// phase completes; a hint made the waits about 3 % slower end to end); a wait
// that lasts longer than two seconds raises the flag itself and records the
// timeout in the device error word.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
SSM_DEVINL bool wait_bar(uint64_t *mb, int *abort, uint32_t parity, int32_t *err) {
    if (tc::mbar_try_wait(mb, parity)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    for (;;) {
        if (*reinterpret_cast<volatile int *>(abort)) return false;
        if (tc::mbar_try_wait(mb, parity)) return true;
        if (tc::globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
    *reinterpret_cast<volatile int *>(abort) = 1;
    if (err) atomicExch(err, SSM_DEVERR_TIMEOUT);
    return false;
}
SSM_DEVINL bool wait_mb(Aux &ax, int i, uint32_t parity, int32_t *err) { return wait_bar(&ax.mb[i], &ax.abort, parity, err); }
SSM_DEVINL bool aborted(Aux &ax) { return *reinterpret_cast<volatile int *>(&ax.abort) != 0; }

// Causal width-<=4 conv of one channel pair at one token plus SiLU: taps
// right-aligned (w3 multiplies the current token, w0 the one three back);
// silu(v) = h + h tanh(h), h = v / 2.
SSM_DEVINL float2 conv_silu2(float2 cur, float2 h2, float2 h1, float2 h0, float2 w3, float2 w2, float2 w1, float2 w0,
                             float2 bias) {
    float2 acc = __ffma2_rn(w3, cur, bias);
    acc = __ffma2_rn(w2, h2, acc);
    acc = __ffma2_rn(w1, h1, acc);
    acc = __ffma2_rn(w0, h0, acc);
    const float2 hv = __fmul2_rn(acc, make_float2(0.5f, 0.5f));
    return __ffma2_rn(hv, make_float2(tanh_approx(hv.x), tanh_approx(hv.y)), hv);
}

// Tensor maps (3-d: channel, token, batch row; bf16):
//   tm_x  raw x, box 64 x 64 rows, no swizzle    -> row-major staging rows of 128 bytes
//   tm_b, tm_c  conv'd B / C, box 64 x 64, 128-byte swizzle -> one K-atom of the operand tile
//   tm_z  z, box 64 x 64, 128-byte swizzle       -> the z tile the epilogue reads
//   tm_y  y, box 64 x 64, 128-byte swizzle       <- the z tile holding y (rows past the tensor are skipped)
__global__ void __launch_bounds__(kThreads, 2)
ssd_kernel(const SsdArgs a, const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
           const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_z,
           const __grid_constant__ CUtensorMap tm_y) {
    extern __shared__ unsigned char smem_raw[];
    // swizzle atoms need 1024-byte alignment: round the base up (1 KB of slack is allocated)
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    Aux &ax = *reinterpret_cast<Aux *>(smem + OFF_AUX);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hh = blockIdx.x;
    // sequence s, segment sg of it: from the segment table when packed
    // sequences are cut (rows past its count have none), else packed sequences
    // in schedule order and plain rows without segments have sg = 0 and the
    // segment is the whole sequence
    if (a.seg_tab && (int)blockIdx.y >= *a.seg_count) return;
    const int s = a.seg_tab ? a.seg_tab[blockIdx.y].x
                            : a.sv.order ? a.sv.order[blockIdx.y] : (int)blockIdx.y / a.nseg;
    const int sg = seg_index(a);
    int64_t seq_start = 0, seq_len = a.seqlen, row = s;
    if (a.sv.cu) {
        const int64_t c0 = min(max((int64_t)a.sv.cu[s], (int64_t)0), a.seqlen);
        const int64_t c1 = min(max((int64_t)a.sv.cu[s + 1], c0), a.seqlen);
        seq_start = c0; seq_len = c1 - c0; row = 0;
    }
    const int64_t start = seq_start + (int64_t)sg * a.seg_len;
    const int64_t len = max(min(a.seg_len, seq_len - (int64_t)sg * a.seg_len), (int64_t)0);
    // tokens of the sequence before the segment, recomputed where needed (keeps
    // it out of the registers the chunk loop holds)
    auto seg_off = [&]() -> int64_t { return (int64_t)seg_index(a) * a.seg_len; };
    const int64_t H = a.H, g = hh / (H / a.G);
    const int K = a.K;
    const int n = (int)((len + kQ - 1) / kQ);
    const int crow = (int)row, g0 = (int)(g * kN);
    const uint32_t sbase = tc::smem_u32(smem);
    // bounds-checked build: the CTA's ranges (uniform, so the whole CTA returns together)
    if (!SSM_BOUNDS(len > 0 ? start + len - 1 : 0, a.seqlen > 0 ? a.seqlen : 1, BS_SSD_SEQ) ||
        !SSM_BOUNDS((int64_t)hh * kP + kP - 1, a.H * kP, BS_SSD_HEAD) ||
        !SSM_BOUNDS((int64_t)g0 + kN - 1, a.G * kN, BS_SSD_GROUP) ||
        !SSM_BOUNDS((int64_t)s * H + hh, (int64_t)a.sv.nseqs * H, BS_SSD_STATE) ||
        !SSM_BOUNDS(((int64_t)s + 1) * a.cdim - 1, (int64_t)a.sv.nseqs * a.cdim, BS_SSD_CONV_STATE) ||
        !SSM_BOUNDS(sg, a.seg_tab ? a.nsloc : a.nseg, BS_SSD_SEGMENT) ||
        (sg > 0 && !SSM_BOUNDS(seg_row0(a, s) + sg - 1, a.nsloc, BS_SSD_SEGMENT)))
        return;
    const float A2 = a.A[hh] * kLog2e;

    if (tid == 0) {
        // one thread reads the error word, so every thread of the CTA takes the same branch below
        ax.abort = (a.sv.err && *a.sv.err != 0) ? 1 : 0;
        for (int i = 0; i < kNumMbar; ++i)
            tc::mbar_init(&ax.mb[i], (i == MB_CONV || i == MB_SREADY || i == MB_MREADY) ? kComputeWarps : 1);
        tc::mbar_init_fence();
        if (n > 0) {                       // a CTA with no chunk touches no tensor map
            tc::prefetch_map(&tm_x);
            tc::prefetch_map(&tm_b);
            tc::prefetch_map(&tm_c);
            if (a.z) tc::prefetch_map(&tm_z);
            tc::prefetch_map(&tm_y);
        }
    }
    if (warp == kComputeWarps) tc::tmem_alloc(&ax.tmem, kTmemCols);
    // the mask tile's blocks above the diagonal are zero for good
    for (int i = tid; i < 8192 / 16; i += kThreads) st16(smem + OFF_M + i * 16, make_uint4(0, 0, 0, 0));
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ax.tmem;
    if (ax.abort) {
        __syncthreads();
        if (warp == kComputeWarps) tc::tmem_dealloc(tmem, kTmemCols);
        return;
    }

    if (warp == kComputeWarps) {
        // ------------------------------------------------------------ control warp
        const bool lead = lane == 0;
        // shared-memory descriptors of the operand tiles; a K step adds its byte
        // offset / 16 to the start-address field (addresses stay below 256 KB)
        const uint64_t dCk = tc::desc_sw128(sbase + OFF_C, 16, 1024);     // K-major C (G, Yo)
        const uint64_t dBk = tc::desc_sw128(sbase + OFF_B, 16, 1024);     // K-major B (G)
        const uint64_t dBm = tc::desc_sw128(sbase + OFF_B, 8192, 1024);   // MN-major B^T (Sc)
        const uint64_t dXPm = tc::desc_sw128(sbase + OFF_XP, 8192, 1024); // MN-major X' (Sc)
        const uint64_t dSm = tc::desc_sw128(sbase + OFF_S, 8192, 1024);   // MN-major S^T (Yo)
        const uint64_t dMk = tc::desc_sw128(sbase + OFF_M, 16, 1024);     // K-major M (Y)
        const uint64_t dX0m = tc::desc_sw128(sbase + OFF_X, 8192, 1024);  // MN-major X, buffer 0 (Y)
        const float dtb = a.dt_bias ? a.dt_bias[hh] : 0.f;
        const __nv_bfloat16 *dtg = a.dt + row * a.dt_bs + start * a.dt_ts + hh;
        int last_x[2] = {-1, -1};
        int last_bc = -1, last_z = -1;
        auto load_x = [&](int cn) {
            const int b = cn & 1;
            tc::mbar_expect_tx(&ax.mb[MB_X0 + b], kQ * kP * 2);
            tc::tma_load_3d(smem + OFF_XR + b * 8192, &tm_x, (int)(hh * kP), (int)(start + (int64_t)cn * kQ), crow,
                            &ax.mb[MB_X0 + b]);
            last_x[b] = cn;
        };
        auto load_bc = [&](int cn) {
            const int tok = (int)(start + (int64_t)cn * kQ);
            tc::mbar_expect_tx(&ax.mb[MB_BC], 4 * kQ * 64 * 2);
            tc::tma_load_3d(smem + OFF_B, &tm_b, g0, tok, crow, &ax.mb[MB_BC]);
            tc::tma_load_3d(smem + OFF_B + 8192, &tm_b, g0 + 64, tok, crow, &ax.mb[MB_BC]);
            tc::tma_load_3d(smem + OFF_C, &tm_c, g0, tok, crow, &ax.mb[MB_BC]);
            tc::tma_load_3d(smem + OFF_C + 8192, &tm_c, g0 + 64, tok, crow, &ax.mb[MB_BC]);
            last_bc = cn;
        };
        auto load_z = [&](int cn) {
            tc::mbar_expect_tx(&ax.mb[MB_Z], kQ * kP * 2);
            tc::tma_load_3d(smem + OFF_Z, &tm_z, (int)(hh * kP), (int)(start + (int64_t)cn * kQ), crow, &ax.mb[MB_Z]);
            last_z = cn;
        };
        // raw dt of chunk cn: lane l holds tokens l and l + 32 (kept as bf16 until the tables need them)
        auto load_dt = [&](int cn, __nv_bfloat16 (&d)[2]) {
            const int64_t tn = (int64_t)cn * kQ;
            const int nvn = (int)min((int64_t)kQ, len - tn);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h;
                d[h] = j < nvn ? dtg[(tn + j) * a.dt_ts] : __float2bfloat16_rn(0.f);
            }
        };
        // delta, running log2-decay and the decay factor tables of chunk cn into
        // slot cn % 3 (lane l: tokens l and l + 32), then the slot's barrier
        auto tables = [&](int cn, const __nv_bfloat16 (&draw)[2]) {
            Tables &tw = ax.tab[cn % 3];
            const int nvn = (int)min((int64_t)kQ, len - (int64_t)cn * kQ);
            float d[2], sc[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h;
                const float u = __bfloat162float(draw[h]) + dtb;
                d[h] = j < nvn ? (a.softplus ? softplus(u) : u) : 0.f;
                sc[h] = d[h] * A2;
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v0 = __shfl_up_sync(0xffffffffu, sc[0], o);
                const float v1 = __shfl_up_sync(0xffffffffu, sc[1], o);
                if (lane >= o) { sc[0] += v0; sc[1] += v1; }
            }
            const float tot0 = __shfl_sync(0xffffffffu, sc[0], 31);
            sc[1] += tot0;
            const float last = __shfl_sync(0xffffffffu, sc[1], 31);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h;
                // block boundaries: token 16*(j/16) (start) and 16*(j/16)+15 (end)
                const float st = __shfl_sync(0xffffffffu, sc[h], lane & ~15);
                const float en = __shfl_sync(0xffffffffu, sc[h], lane | 15);
                tw.dlt[j] = d[h];
                tw.cs2[j] = sc[h];
                tw.ecs[j] = ex2(sc[h]);
                tw.wj[j] = ex2(last - sc[h]) * d[h];
                tw.rf[j] = ex2(sc[h] - st);
                tw.cf[j] = ex2(en - sc[h]) * d[h];
            }
            // block factor (I, J), J < I: exp(cs[16 I] - cs[16 J + 15]) (<= 1); lanes 0-15
            {
                const int I = (lane >> 2) & 3, J = lane & 3;
                const float s0 = __shfl_sync(0xffffffffu, sc[0], (I & 1) * 16);
                const float s1 = __shfl_sync(0xffffffffu, sc[1], (I & 1) * 16);
                const float e0 = __shfl_sync(0xffffffffu, sc[0], (J & 1) * 16 + 15);
                const float e1 = __shfl_sync(0xffffffffu, sc[1], (J & 1) * 16 + 15);
                const float bv = J < I ? ex2((I < 2 ? s0 : s1) - (J < 2 ? e0 : e1)) : 0.f;
                if (lane < 16) tw.bf[I][J] = bv;
            }
            if (lane == 0) tw.dAc = ex2(last);
            __syncwarp();
            if (lead) mb_arrive(&ax.mb[MB_T0 + cn % 3]);
        };
        if (n > 0) {
            if (lead) {
                load_x(0);
                if (n > 1) load_x(1);
                load_bc(0);
                if (a.z) load_z(0);
            }
            for (int cn = 0; cn < 3 && cn < n; ++cn) {
                __nv_bfloat16 dr[2];
                load_dt(cn, dr);
                tables(cn, dr);
            }
        }
        bool ok = true;
        for (int k = -1; k < n; ++k) {
            const int c1 = k + 1;
            __nv_bfloat16 dnext[2];
            if (k >= 0 && k + 3 < n) load_dt(k + 3, dnext);       // consumed after S(k)
            if (c1 < n) {
                // G(c1) = C B^T as soon as B / C have landed (mask(k) has read G(k))
                ok = wait_mb(ax, MB_BC, c1 & 1, a.err) && ok;
                tc::fence_after_sync();
                if (lead && ok) {
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint32_t ko = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
                        tc::mma_bf16(tmem + TM_G, dCk + ko, dBk + ko, ID_G, kk > 0);
                    }
                    tc::mma_commit(&ax.mb[MB_G]);
                }
                __syncwarp();
                // raw x of chunk c1 + 2 once conv(c1) has read its staging buffer
                ok = wait_mb(ax, MB_CONV, c1 & 1, a.err) && ok;
                if (lead && ok && c1 + 2 < n) load_x(c1 + 2);
                __syncwarp();
            }
            if (k >= 0) {
                // z of chunk c1 once the epilogue has read z(k)
                ok = wait_mb(ax, MB_ZFREE, k & 1, a.err) && ok;
                if (lead && ok && a.z && c1 < n) load_z(c1);
                __syncwarp();
            }
            // S(k) written (h0 for k = -1): Sc(c1) and Yo(c1)
            ok = wait_mb(ax, MB_SREADY, c1 & 1, a.err) && ok;
            tc::fence_after_sync();
            if (c1 < n) {
                if (lead && ok) {
#pragma unroll
                    for (int kk = 0; kk < kQ / 16; ++kk)
                        tc::mma_bf16(tmem + TM_SC, dBm + kk * 128, dXPm + kk * 128, ID_S, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk)
                        tc::mma_bf16(tmem + TM_YO, dCk + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), dSm + kk * 128, ID_Y,
                                     kk > 0);
                    tc::mma_commit(&ax.mb[MB_BCFREE]);
                }
                __syncwarp();
            }
            // the tables of chunk k + 3 into the slot S(k) has finished with
            if (k >= 0 && k + 3 < n) tables(k + 3, dnext);
            if (c1 < n) {
                // Y(c1) = M X once the mask is written
                ok = wait_mb(ax, MB_MREADY, c1 & 1, a.err) && ok;
                tc::fence_after_sync();
                const uint64_t dXm = dX0m + (uint64_t)((c1 & 1) * (8192 >> 4));
                if (lead && ok) {
#pragma unroll
                    for (int kk = 0; kk < kQ / 16; ++kk)
                        tc::mma_bf16(tmem + TM_Y, dMk + kk * 2, dXm + kk * 128, ID_Y, kk > 0);
                    tc::mma_commit(&ax.mb[MB_MMA]);
                }
                __syncwarp();
                // B / C of chunk c1 + 1 once G, Sc and Yo have read them
                if (c1 + 1 < n) {
                    ok = wait_mb(ax, MB_BCFREE, c1 & 1, a.err) && ok;
                    if (lead && ok) load_bc(c1 + 1);
                    __syncwarp();
                }
            }
        }
        if (lead && aborted(ax)) {
            // drain: every MMA this thread issued, and the last copies into each buffer
            tc::mma_commit(&ax.mb[MB_DRAIN]);
            tc::mbar_wait(&ax.mb[MB_DRAIN], 0, 1u << 22);
            for (int b = 0; b < 2; ++b)
                if (last_x[b] >= 0) tc::mbar_wait(&ax.mb[MB_X0 + b], (last_x[b] >> 1) & 1, 1u << 22);
            if (last_bc >= 0) tc::mbar_wait(&ax.mb[MB_BC], last_bc & 1, 1u << 22);
            if (last_z >= 0) tc::mbar_wait(&ax.mb[MB_Z], last_z & 1, 1u << 22);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ compute warps
        const int q4 = warp & 3;          // tensor-memory lane quarter of this warp
        const int half = warp >> 2;       // which 32 columns of a 64-column accumulator this warp reads
        const bool zg = a.z != nullptr;
        __nv_bfloat16 *yg = a.y + row * a.y_bs + start * a.y_ts + hh * kP;
        const float Dh = a.D ? a.D[hh] : 0.f;
        const uint32_t t_lane = (uint32_t)(q4 * 32) << 16;
        bool ok = true;

        // x conv role: channels 2 cq, 2 cq + 1 (one packed pair), tokens cr0 .. cr0+7;
        // taps right-aligned (cw3 multiplies the current token, cw0 the one 3 back)
        const int cq = lane, cr0 = warp * (kQ / 8);
        float2 cw0, cw1, cw2, cw3, cbias;
        {
            const int64_t ch = hh * kP + 2 * cq;
            auto tap = [&](int j) {
                const int k = K - 4 + j;
                return (K > 0 && k >= 0) ? make_float2(a.conv_w[ch * K + k], a.conv_w[(ch + 1) * K + k]) : make_float2(0.f, 0.f);
            };
            cw0 = tap(0); cw1 = tap(1); cw2 = tap(2); cw3 = tap(3);
            cbias = a.conv_b ? make_float2(a.conv_b[ch], a.conv_b[ch + 1]) : make_float2(0.f, 0.f);
        }
        // swizzled byte offset of (row cr0 + i, channel 2 cq) in an X tile:
        // row block = warp, row in block = i, 16-byte chunk (cq / 4) ^ i
        const uint32_t obase = (uint32_t)warp * 1024u + (uint32_t)(cq & 3) * 4u;

        // carried state: thread owns S[n][32*half .. 32*half+31] for n = 32*q4 + lane (fp32 pairs)
        const int sn = q4 * 32 + lane;
        float2 S[16];
        {
            const float *h0p = a.h0 ? a.h0 + ((int64_t)s * H + hh) * kP * kN : nullptr;
#pragma unroll
            for (int p = 0; p < 16; ++p)
                S[p] = h0p ? make_float2(h0p[(int64_t)(half * 32 + 2 * p) * kN + sn], h0p[(int64_t)(half * 32 + 2 * p + 1) * kN + sn])
                           : make_float2(0.f, 0.f);
            // the state entering segment sg: fold (exp(cs_end), S_loc) of every
            // segment before it onto h0, in order
            const int64_t q0 = sg > 0 ? seg_row0(a, s) : 0;
            for (int t = 0; t < sg; ++t) {
                const int64_t q = (q0 + t) * H + hh;
                const float e = ex2(a.slog[q]);
                const float2 e2 = make_float2(e, e);
                const float *lp = a.sloc + q * kP * kN;
#pragma unroll
                for (int p = 0; p < 16; ++p)
                    S[p] = __ffma2_rn(e2, S[p], make_float2(lp[(int64_t)(half * 32 + 2 * p) * kN + sn],
                                                            lp[(int64_t)(half * 32 + 2 * p + 1) * kN + sn]));
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                st16(smem + OFF_S + tc::off_sw128(sn, half * 32 + q * 8, 8192), tc::pack_bf16x8(reinterpret_cast<const float *>(&S[q * 4])));
        }
        // conv halo of chunk 0: the last K-1 raw inputs before the sequence (its
        // carried conv state), or the raw x rows before a later segment
        if (tid < kP) {
            const int p = tid;
#pragma unroll
            for (int j = 0; j < kHx; ++j) {
                const int q = j - (kHx - (K - 1));          // index into the carried conv state
                float v = 0.f;
                if (sg > 0)
                    v = __bfloat162float(a.x[row * a.x_bs + (start - kHx + j) * a.x_ts + hh * kP + p]);
                else if (K > 1 && q >= 0 && a.conv_state_in)
                    v = __bfloat162float(a.conv_state_in[((int64_t)s * a.cdim + hh * kP + p) * (K - 1) + q]);
                ax.xh[0][j][p] = v;
            }
        }

        // accumulator fragment of this thread (16-lane TMEM loads of an M = 64
        // accumulator): rows i0 = 16 q4 + lane / 4 and i1 = i0 + 8, columns
        // jc + 8 k and jc + 8 k + 1 for k = 0..3
        const int i0 = q4 * 16 + (lane >> 2), i1 = i0 + 8;
        const int jc = half * 32 + 2 * (lane & 3);
        // swizzled byte offset of (i0, jc + 8 k) in a 64 x 64 bf16 tile is
        // frag_off + (((4 half + k) ^ (lane / 4)) << 4); row i1 is 1024 bytes further
        const uint32_t frag_off = (uint32_t)q4 * 2048u + (uint32_t)(lane >> 2) * 128u + (uint32_t)(lane & 3) * 4u;

        bar_compute();                    // the chunk-0 halo and the initial state tile are written
        for (int k = -1; k < n; ++k) {
            const int c1 = k + 1;

            // ---- conv(c1): raw x rows -> X and X' (bf16, swizzled), halo of chunk c1 + 1
            if (c1 < n) {
                ok = wait_mb(ax, MB_T0 + c1 % 3, (c1 / 3) & 1, a.err) && ok;
                ok = wait_mb(ax, MB_X0 + (c1 & 1), (c1 >> 1) & 1, a.err) && ok;
                if (c1 > 0) ok = wait_mb(ax, MB_BCFREE, (c1 - 1) & 1, a.err) && ok;   // Sc(c1-1) has read X'
                const int nv = (int)min((int64_t)kQ, len - (int64_t)c1 * kQ);
                const int hb = c1 & 1;
                const Tables &tb = ax.tab[c1 % 3];
                const unsigned char *xraw = smem + OFF_XR + hb * 8192;
                unsigned char *xo = smem + OFF_X + hb * 8192;
                unsigned char *xpo = smem + OFF_XP;
                auto rawrow = [&](int v) -> float2 {
                    const uint32_t u = *reinterpret_cast<const uint32_t *>(xraw + v * (kP * 2) + cq * 4);
                    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
                };
                float2 h0v, h1v, h2v;                                   // raw rows t-3, t-2, t-1
                if (warp == 0) {
                    h0v = *reinterpret_cast<const float2 *>(&ax.xh[hb][0][2 * cq]);
                    h1v = *reinterpret_cast<const float2 *>(&ax.xh[hb][1][2 * cq]);
                    h2v = *reinterpret_cast<const float2 *>(&ax.xh[hb][2][2 * cq]);
                } else {
                    h0v = rawrow(cr0 - 3); h1v = rawrow(cr0 - 2); h2v = rawrow(cr0 - 1);
                }
                float wv[8];                                            // X' weights of the 8 tokens
                {
                    const float4 w0 = *reinterpret_cast<const float4 *>(&tb.wj[cr0]);
                    const float4 w1 = *reinterpret_cast<const float4 *>(&tb.wj[cr0 + 4]);
                    wv[0] = w0.x; wv[1] = w0.y; wv[2] = w0.z; wv[3] = w0.w;
                    wv[4] = w1.x; wv[5] = w1.y; wv[6] = w1.z; wv[7] = w1.w;
                }
                // full chunks take a copy of the loop without the end-of-sequence test
                auto conv_rows = [&](auto full_tag) {
                    constexpr bool kFull = decltype(full_tag)::value;
#pragma unroll
                    for (int i = 0; i < kQ / 8; ++i) {
                        const float2 cur = rawrow(cr0 + i);             // rows >= nv are zeroed below
                        float2 xc = cur;
                        if (K > 0) xc = conv_silu2(cur, h2v, h1v, h0v, cw3, cw2, cw1, cw0, cbias);
                        if (!kFull && cr0 + i >= nv) xc = make_float2(0.f, 0.f);
                        h0v = h1v; h1v = h2v; h2v = cur;
                        const float2 xw = __fmul2_rn(xc, make_float2(wv[i], wv[i]));
                        const uint32_t off = obase + (uint32_t)i * 128u + ((uint32_t)((cq >> 2) ^ i) << 4);
                        *reinterpret_cast<__nv_bfloat162 *>(xo + off) = __floats2bfloat162_rn(xc.x, xc.y);
                        *reinterpret_cast<__nv_bfloat162 *>(xpo + off) = __floats2bfloat162_rn(xw.x, xw.y);
                    }
                };
                if (nv == kQ) conv_rows(std::true_type{});
                else conv_rows(std::false_type{});
                // halo of the next chunk: raw rows nv-3 .. nv-1 (from the old halo when the chunk is shorter)
                if (tid < kP) {
                    const int p = tid;
#pragma unroll
                    for (int j = 0; j < kHx; ++j) {
                        const int v = nv - kHx + j;
                        ax.xh[hb ^ 1][j][p] = v >= 0 ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(
                                                           xraw + v * (kP * 2) + p * 2))
                                                     : ax.xh[hb][kHx + v][p];
                    }
                }
                tc::fence_proxy_async();
                __syncwarp();
                if (lane == 0) mb_arrive(&ax.mb[MB_CONV]);
            }

            // ---- epilogue(k): y = (Y + exp(cs_i) Yo) * silu(z); S(k) = exp(cs_Q) S + Sc
            if (k >= 0) {
                const int64_t t0 = (int64_t)k * kQ;
                const int nv = (int)min((int64_t)kQ, len - t0);
                const Tables &tb = ax.tab[k % 3];
                unsigned char *stg = smem + OFF_Z;     // y is staged over z, element by element
                // Whole chunks (and the tensor's last, clipped chunk) leave through a TMA
                // store of the staging tile; the partial last chunk of a packed sequence
                // is stored directly.
                const bool y_tma = nv == kQ || !a.sv.cu;
                ok = wait_mb(ax, MB_MMA, k & 1, a.err) && ok;
                if (zg) ok = wait_mb(ax, MB_Z, k & 1, a.err) && ok;
                tc::fence_after_sync();
                {
                    const float e0 = tb.ecs[i0], e1 = tb.ecs[i1];
                    const float2 e02 = make_float2(e0, e0), e12 = make_float2(e1, e1);
                    const float2 half2 = make_float2(0.5f, 0.5f);
                    // two passes of 16 columns keep the accumulator fragments at 16 registers;
                    // the staged (TMA) and the direct-store forms are separate copies
                    auto epi = [&](auto tma_tag) {
                        constexpr bool kTma = decltype(tma_tag)::value;
                        const bool st_ok = kTma || !aborted(ax);
#pragma unroll
                        for (int hp = 0; hp < 2; ++hp) {
                            uint32_t yr[8], yo[8];
                            tc::tmem_ld16x256b_x2(tmem + t_lane + TM_Y + half * 32 + hp * 16, yr);
                            tc::tmem_ld16x256b_x2(tmem + t_lane + TM_YO + half * 32 + hp * 16, yo);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int kq = 0; kq < 2; ++kq) {
                                const int kk = hp * 2 + kq;
                                const uint32_t off0 = frag_off + ((uint32_t)((half * 4 + kk) ^ (lane >> 2)) << 4);
#pragma unroll
                                for (int rr = 0; rr < 2; ++rr) {
                                    const uint32_t off = off0 + rr * 1024u;
                                    float2 o = __ffma2_rn(rr ? e12 : e02,
                                                          make_float2(__uint_as_float(yo[4 * kq + 2 * rr]), __uint_as_float(yo[4 * kq + 2 * rr + 1])),
                                                          make_float2(__uint_as_float(yr[4 * kq + 2 * rr]), __uint_as_float(yr[4 * kq + 2 * rr + 1])));
                                    if (zg) {
                                        // silu(z) = h + h tanh(h), h = z / 2
                                        const uint32_t zw = *reinterpret_cast<const uint32_t *>(smem + OFF_Z + off);
                                        const float2 hz = __fmul2_rn(make_float2(__uint_as_float(zw << 16), __uint_as_float(zw & 0xffff0000u)), half2);
                                        o = __fmul2_rn(o, __ffma2_rn(hz, make_float2(tanh_approx(hz.x), tanh_approx(hz.y)), hz));
                                    }
                                    const __nv_bfloat162 ob = __floats2bfloat162_rn(o.x, o.y);
                                    if (kTma) {
                                        *reinterpret_cast<__nv_bfloat162 *>(stg + off) = ob;
                                    } else {
                                        const int i = rr ? i1 : i0;
                                        if (i < nv && st_ok && SSM_BOUNDS(start + t0 + i, a.seqlen, BS_SSD_Y))
                                            *reinterpret_cast<__nv_bfloat162 *>(yg + (t0 + i) * a.y_ts + jc + 8 * kk) = ob;
                                    }
                                }
                            }
                        }
                    };
                    if (y_tma) epi(std::true_type{});
                    else epi(std::false_type{});
                }
                {
                    const float2 dA2 = make_float2(tb.dAc, tb.dAc);
                    float Sc[32];
                    tc::tmem_ld32(tmem + t_lane + TM_SC + half * 32, Sc);
#pragma unroll
                    for (int p = 0; p < 16; ++p) S[p] = __ffma2_rn(dA2, S[p], make_float2(Sc[2 * p], Sc[2 * p + 1]));
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st16(smem + OFF_S + tc::off_sw128(sn, half * 32 + q * 8, 8192),
                             tc::pack_bf16x8(reinterpret_cast<const float *>(&S[q * 4])));
                }
                // the state is ready before the y store's barrier, so the control warp
                // can issue Sc / Yo of the next chunk while the warps meet there
                tc::fence_proxy_async();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mb_arrive(&ax.mb[MB_SREADY]);
                // every warp has staged its y: store the tile, and once the store has read
                // it the z tile is free for the control warp to load z(k + 1)
                bar_compute();
                if (tid == 0) {
                    if (y_tma && !aborted(ax)) {
                        tc::tma_store_3d(&tm_y, (int)(hh * kP), (int)(start + t0), crow, stg);
                        tc::bulk_wait_read();
                    }
                    mb_arrive(&ax.mb[MB_ZFREE]);
                }
                // intermediate state after this chunk when it closes a state interval
                if (a.iv.interval > 0 && nv == kQ && !aborted(ax)) {
                    const int64_t slot = a.iv.slot_after(s, seg_off() + t0 + kQ);
                    if (slot >= 0 && SSM_BOUNDS(slot, a.iv.nslots, BS_SSD_POOL)) {
                        if (a.iv.states) {
                            float *dst = a.iv.states + (slot * H + hh) * kP * kN;
#pragma unroll
                            for (int p = 0; p < 16; ++p) {
                                dst[(int64_t)(half * 32 + 2 * p) * kN + sn] = S[p].x;
                                dst[(int64_t)(half * 32 + 2 * p + 1) * kN + sn] = S[p].y;
                            }
                        }
                        if (a.iv.conv && K > 1) {
                            // x channels of this head: the halo conv(k) left for chunk k + 1;
                            // B / C of the group (written by its first head): the raw inputs
                            // before the boundary
                            __nv_bfloat16 *cdst = static_cast<__nv_bfloat16 *>(a.iv.conv) + slot * a.cdim * (K - 1);
                            if (tid < kP)
                                for (int j = 0; j < K - 1; ++j)
                                    cdst[(hh * kP + tid) * (K - 1) + j] =
                                        __float2bfloat16_rn(ax.xh[(k + 1) & 1][kHx - (K - 1) + j][tid]);
                            if (hh % (H / a.G) == 0) {
                                const int64_t GN = a.G * kN;
                                for (int i = tid; i < 2 * kN * (K - 1); i += kComputeThreads) {
                                    const int which = i / (kN * (K - 1)), nn = (i / (K - 1)) % kN, j = i % (K - 1);
                                    const int64_t tok = start + t0 + kQ - (K - 1) + j;
                                    if (!SSM_BOUNDS(tok, a.seqlen, BS_SSD_RAW_BC)) continue;
                                    const __nv_bfloat16 v = which ? a.Craw[row * a.craw_bs + tok * a.craw_ts + g * kN + nn]
                                                                  : a.Braw[row * a.braw_bs + tok * a.braw_ts + g * kN + nn];
                                    cdst[(a.H * kP + which * GN + g * kN + nn) * (K - 1) + j] = v;
                                }
                            }
                        }
                    }
                }
            } else {
                // S(-1) = h0: its bf16 copy was written before the loop
                tc::fence_proxy_async();
                __syncwarp();
                if (lane == 0) mb_arrive(&ax.mb[MB_SREADY]);
            }

            // ---- mask(c1): G -> M (blocks on or below the diagonal)
            // Each warp reads its 16 accumulator rows (tokens i0, i1) for its 32 columns.
            // M[i, j] = G[i, j] exp(cs_i - cs_j) delta_j for j <= i, plus D on the diagonal
            // (the skip term D x rides along in M X).  Below the diagonal 16x16 block the
            // exponential factors as row x block x column terms, each <= 1.
            if (c1 < n) {
                ok = wait_mb(ax, MB_G, c1 & 1, a.err) && ok;
                tc::fence_after_sync();
                const Tables &tb = ax.tab[c1 % 3];
                const int I = q4;
                // The warp's two 16-column blocks J0 = 2 half (column groups k = 0, 1)
                // and J1 = 2 half + 1 (k = 2, 3) against its row block I = q4: J0 on the
                // diagonal and J1 above (I = 2 half), J0 below and J1 on the diagonal
                // (I = 2 half + 1), both below (I > 2 half + 1), or both above.
                if (I >= 2 * half) {
                    uint32_t gr[16];
                    tc::tmem_ld16x256b_x4(tmem + t_lane + TM_G + half * 32, gr);
                    const float ci0 = tb.cs2[i0], ci1 = tb.cs2[i1];
                    const float rf0 = tb.rf[i0], rf1 = tb.rf[i1];
                    tc::tmem_wait_ld();
                    auto put = [&](int kk, float m00, float m01, float m10, float m11) {
                        const uint32_t off = frag_off + ((uint32_t)((half * 4 + kk) ^ (lane >> 2)) << 4);
                        *reinterpret_cast<__nv_bfloat162 *>(smem + OFF_M + off) = __floats2bfloat162_rn(m00, m01);
                        *reinterpret_cast<__nv_bfloat162 *>(smem + OFF_M + off + 1024) = __floats2bfloat162_rn(m10, m11);
                    };
                    // below the diagonal: G exp(cs_i - cs_j) delta_j = G * row * block * column factors
                    auto below = [&](int kk) {
                        const int j = jc + 8 * kk;
                        const float bfac = tb.bf[I][half * 2 + (kk >> 1)];
                        const float2 cf = *reinterpret_cast<const float2 *>(&tb.cf[j]);
                        const float r0 = rf0 * bfac, r1 = rf1 * bfac;
                        put(kk, __uint_as_float(gr[4 * kk]) * (r0 * cf.x), __uint_as_float(gr[4 * kk + 1]) * (r0 * cf.y),
                            __uint_as_float(gr[4 * kk + 2]) * (r1 * cf.x), __uint_as_float(gr[4 * kk + 3]) * (r1 * cf.y));
                    };
                    // on the diagonal: direct exponentials, selected (not branched) at and below
                    // the diagonal, plus D on it (the skip term D x rides along in M X)
                    auto diag = [&](int kk) {
                        const int j = jc + 8 * kk;
                        const float2 cj = *reinterpret_cast<const float2 *>(&tb.cs2[j]);
                        const float2 dj = *reinterpret_cast<const float2 *>(&tb.dlt[j]);
                        const float v00 = __uint_as_float(gr[4 * kk]) * ex2(ci0 - cj.x) * dj.x;
                        const float v01 = __uint_as_float(gr[4 * kk + 1]) * ex2(ci0 - cj.y) * dj.y;
                        const float v10 = __uint_as_float(gr[4 * kk + 2]) * ex2(ci1 - cj.x) * dj.x;
                        const float v11 = __uint_as_float(gr[4 * kk + 3]) * ex2(ci1 - cj.y) * dj.y;
                        put(kk, j < i0 ? v00 : (j == i0 ? v00 + Dh : 0.f), j + 1 < i0 ? v01 : (j + 1 == i0 ? v01 + Dh : 0.f),
                            j < i1 ? v10 : (j == i1 ? v10 + Dh : 0.f), j + 1 < i1 ? v11 : (j + 1 == i1 ? v11 + Dh : 0.f));
                    };
                    if (I == 2 * half) {
                        diag(0); diag(1);
                    } else if (I == 2 * half + 1) {
                        below(0); below(1); diag(2); diag(3);
                    } else {
                        below(0); below(1); below(2); below(3);
                    }
                }
                tc::fence_proxy_async();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mb_arrive(&ax.mb[MB_MREADY]);
            }
        }
        if (tid == 0) tc::bulk_wait_all();
        if (!aborted(ax) && seg_is_last(a)) {   // the last segment
            if (a.h_final) {
                float *hf = a.h_final + ((int64_t)s * H + hh) * kP * kN;
#pragma unroll
                for (int p = 0; p < 16; ++p) {
                    hf[(int64_t)(half * 32 + 2 * p) * kN + sn] = S[p].x;
                    hf[(int64_t)(half * 32 + 2 * p + 1) * kN + sn] = S[p].y;
                }
            }
            if (K > 1 && a.conv_state_out && tid < kP) {
                const int p = tid, hbf = n & 1;
                for (int j = 0; j < K - 1; ++j)
                    a.conv_state_out[((int64_t)s * a.cdim + hh * kP + p) * (K - 1) + j] =
                        __float2bfloat16_rn(ax.xh[hbf][kHx - (K - 1) + j][p]);
            }
            if (K > 1 && a.conv_state_out && hh % (H / a.G) == 0) {
                // the group's B / C channels (first head of the group): the last K-1 raw
                // inputs of the sequence, from the carried state when it is shorter.  One
                // thread per channel reads all K-1 values before it writes, so the state
                // may be updated in place.
                const int which = tid / kN, nn = tid % kN;            // 256 threads: B then C
                const int64_t ch = a.H * kP + which * a.G * kN + g * kN + nn;
                const __nv_bfloat16 *raw = which ? a.Craw + row * a.craw_bs + g * kN + nn
                                                 : a.Braw + row * a.braw_bs + g * kN + nn;
                const int64_t rts = which ? a.craw_ts : a.braw_ts;
                __nv_bfloat16 v[kHx];
#pragma unroll
                for (int j = 0; j < kHx; ++j) {
                    const int64_t tau = seg_off() + len - (K - 1) + j;  // within the sequence
                    v[j] = __float2bfloat16_rn(0.f);
                    if (j < K - 1) {
                        if (tau >= 0) {
                            const int64_t tok = start - seg_off() + tau;
                            if (SSM_BOUNDS(tok, a.seqlen, BS_SSD_RAW_BC)) v[j] = raw[tok * rts];
                        }
                        else if (a.conv_state_in) v[j] = a.conv_state_in[((int64_t)s * a.cdim + ch) * (K - 1) + tau + (K - 1)];
                    }
                }
#pragma unroll
                for (int j = 0; j < kHx; ++j)
                    if (j < K - 1) a.conv_state_out[((int64_t)s * a.cdim + ch) * (K - 1) + j] = v[j];
            }
        }
        (void)ok;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kComputeWarps) tc::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ segment states
// A fixed-length batch with fewer (row, head) chains than the GPU holds CTAs
// is cut along its tokens: every row into nseg segments of whole chunks, one
// scan CTA per (segment, head).  The scan CTA of segment sg needs the state
// that enters it; the pair (exp(cs), S) of a segment composes associatively
// with seed (1, h0) ("Adding Initial Value Support to Selective Scan Forward
// Kernel", state-spaces/mamba issue 285), so this pass scans every segment but
// the last from a zero state and leaves
//   S_loc[p, n] = sum_j exp(cs_end - cs_j) delta_j X_j[p] B_j[n]
//   slog        = cs_end            (log2 units, cs over the segment's tokens)
// and the scan CTA folds h_in = exp(slog) h_in + S_loc over the segments before
// its own, starting from h0 (the ssd_chunk_state -> ssd_state_passing order of
// "Clean up SSM ops directory structure").  S_loc is one tensor-core
// accumulation over the segment: A = B^T (MN-major, M = 128 states), B = X'
// (MN-major, N = 64), K = the segment's tokens, X' = exp(cs_end - cs_j)
// delta_j X_j written by the fused x conv.
//
// Warp roles as in the scan kernel.  Before the chunk loop the compute warps
// sum delta A over every half chunk, then (after suffix sums over the chunks)
// write every token's X' weight into a shared table, so the loop itself reads
// no dt.  In the loop the control warp's lane 0 keeps three chunks of B and
// raw x in flight (TMA) and issues chunk c's four MMAs once the eight compute
// warps have written its X' (one of two buffers); the compute warps run the
// conv + SiLU + weight of chunk c as soon as its tiles have landed and the
// MMAs of chunk c - 2 have released the buffer.  The last conv warp hands the
// chunk's final raw rows (its rolling registers) to warp 0 as the next chunk's
// conv halo.  All waits are bounded as in the scan kernel.
constexpr int kStStages = 3;
constexpr int kMaxSegChunks = 64;
constexpr uint32_t ST_STAGE = 24576;                   // per stage: B tile (two 8 KB K-atoms), raw x rows (8 KB)
constexpr uint32_t ST_OFF_XP = kStStages * ST_STAGE;   // two X' buffers of 8 KB
constexpr uint32_t ST_OFF_W = ST_OFF_XP + 16384;       // fp32 X' weight of every token of the segment
constexpr uint32_t ST_OFF_AUX = ST_OFF_W + kMaxSegChunks * kQ * 4;
enum { SB_LD0 = 0, SB_MMA0 = kStStages, SB_CONV0 = kStStages + 2, SB_DRAIN = kStStages + 4, kNumStBar };
struct StAux {
    float xh[3][kHx][kP];                // conv halo of chunk c in slot c % 3
    float half[2 * kMaxSegChunks];       // sum of delta A (log2) over each half chunk
    float suf[kMaxSegChunks + 1];        // suf[c]: sum over chunks c .. n-1
    uint32_t tmem;
    int abort;
    uint64_t mb[kNumStBar];
};
constexpr size_t kStSmemBytes = ST_OFF_AUX + sizeof(StAux) + 1024;

__global__ void __launch_bounds__(kThreads, 2)
ssd_state_kernel(const SsdArgs a, const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    StAux &ax = *reinterpret_cast<StAux *>(smem + ST_OFF_AUX);
    float *wt = reinterpret_cast<float *>(smem + ST_OFF_W);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hh = blockIdx.x;
    // sequence s and segment sg (one with a successor): from the segment table
    // for packed sequences (the row of a last segment has nothing to do), else
    // nseg - 1 rows per fixed-length row
    int s, sg;
    int64_t start, row, qrow;
    if (a.seg_tab) {
        if ((int)blockIdx.y >= *a.seg_count) return;
        const int4 e = a.seg_tab[blockIdx.y];
        if (e.y >= e.z - 1) return;
        s = e.x; sg = e.y; row = 0; qrow = (int64_t)e.w + e.y;
        start = min(max((int64_t)a.sv.cu[s], (int64_t)0), a.seqlen) + (int64_t)sg * a.seg_len;
    } else {
        const int nsp = a.nseg - 1;                       // segments that have a successor
        s = (int)blockIdx.y / nsp; sg = (int)blockIdx.y % nsp;
        start = (int64_t)sg * a.seg_len; row = s; qrow = (int64_t)s * nsp + sg;
    }
    const int n = (int)(a.seg_len / kQ);                  // only whole segments come here
    const int64_t H = a.H, g = hh / (H / a.G);
    const int crow = (int)row, g0 = (int)(g * kN), K = a.K;
    const int64_t q = qrow * H + hh;                      // row of sloc / slog
    if (!SSM_BOUNDS(start + a.seg_len - 1, a.seqlen, BS_SSD_SEQ) || !SSM_BOUNDS(n - 1, kMaxSegChunks, BS_SSD_SEGMENT) ||
        !SSM_BOUNDS((int64_t)hh * kP + kP - 1, a.H * kP, BS_SSD_HEAD) ||
        !SSM_BOUNDS((int64_t)g0 + kN - 1, a.G * kN, BS_SSD_GROUP) ||
        !SSM_BOUNDS(q, a.nsloc * H, BS_SSD_STATE))
        return;
    const float A2 = a.A[hh] * kLog2e;
    const float dtb = a.dt_bias ? a.dt_bias[hh] : 0.f;
    const __nv_bfloat16 *dtg = a.dt + row * a.dt_bs + start * a.dt_ts + hh;
    // Warp w takes the half chunks hc = w + 8 k (k < kMaxHc; lane l: token
    // 32 hc + l): every dt load of the warp is issued first, then delta and its
    // inclusive prefix of delta A over the half chunk stay in registers for both
    // prologue passes.
    constexpr int kMaxHc = 2 * kMaxSegChunks / kComputeWarps;
    float dv[kMaxHc], sv[kMaxHc];

    if (tid == 0) {
        ax.abort = (a.err && *a.err != 0) ? 1 : 0;
        for (int i = 0; i < kNumStBar; ++i)
            tc::mbar_init(&ax.mb[i], (i == SB_CONV0 || i == SB_CONV0 + 1) ? kComputeWarps : 1);
        tc::mbar_init_fence();
        tc::prefetch_map(&tm_x);
        tc::prefetch_map(&tm_b);
    }
    if (warp == kComputeWarps) {
        tc::tmem_alloc(&ax.tmem, 64);
    } else {
#pragma unroll
        for (int k = 0; k < kMaxHc; ++k) {
            const int hc = warp + k * kComputeWarps;
            dv[k] = hc < 2 * n ? __bfloat162float(dtg[((int64_t)hc * 32 + lane) * a.dt_ts]) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kMaxHc; ++k) {
            const int hc = warp + k * kComputeWarps;
            if (hc < 2 * n) {                                 // uniform over the warp
                const float u = dv[k] + dtb;
                const float d = a.softplus ? softplus(u) : u;
                float sc = d * A2;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, sc, o);
                    if (lane >= o) sc += v;
                }
                dv[k] = d;
                sv[k] = sc;
                if (lane == 31) ax.half[hc] = sc;
            }
        }
        // conv halo of chunk 0: the row's carried conv state before its first
        // segment, else the raw x rows before the segment
        if (tid < kP) {
            const int p = tid;
#pragma unroll
            for (int j = 0; j < kHx; ++j) {
                const int qq = j - (kHx - (K - 1));
                float v = 0.f;
                if (sg > 0)
                    v = __bfloat162float(a.x[row * a.x_bs + (start - kHx + j) * a.x_ts + hh * kP + p]);
                else if (K > 1 && qq >= 0 && a.conv_state_in)
                    v = __bfloat162float(a.conv_state_in[((int64_t)s * a.cdim + hh * kP + p) * (K - 1) + qq]);
                ax.xh[0][j][p] = v;
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ax.tmem;
    if (ax.abort) {
        __syncthreads();
        if (warp == kComputeWarps) tc::tmem_dealloc(tmem, 64);
        return;
    }
    if (tid == 0) {
        ax.suf[n] = 0.f;
        for (int c = n - 1; c >= 0; --c) ax.suf[c] = (ax.half[2 * c] + ax.half[2 * c + 1]) + ax.suf[c + 1];
    }
    __syncthreads();
    if (warp < kComputeWarps) {
        // X' weight of every token: the decay left in its chunk after it, then
        // that of the later chunks, times its delta
#pragma unroll
        for (int k = 0; k < kMaxHc; ++k) {
            const int hc = warp + k * kComputeWarps;
            if (hc < 2 * n) {
                const int c = hc >> 1;
                const float pre = (hc & 1) ? ax.half[hc - 1] : 0.f;
                const float tot = ax.half[2 * c] + ax.half[2 * c + 1];
                wt[hc * 32 + lane] = ex2((tot - (pre + sv[k])) + ax.suf[c + 1]) * dv[k];
            }
        }
    }
    __syncthreads();

    const uint32_t sbase = tc::smem_u32(smem);
    if (warp == kComputeWarps) {
        // ------------------------------------------------------------ control warp
        if (lane == 0) {
            int last_ld[kStStages] = {-1, -1, -1};
            auto load = [&](int c) {
                const int st = c % kStStages;
                unsigned char *base = smem + st * ST_STAGE;
                const int tok = (int)(start + (int64_t)c * kQ);
                tc::mbar_expect_tx(&ax.mb[SB_LD0 + st], 2 * kQ * 64 * 2 + kQ * kP * 2);
                tc::tma_load_3d(base, &tm_b, g0, tok, crow, &ax.mb[SB_LD0 + st]);
                tc::tma_load_3d(base + 8192, &tm_b, g0 + 64, tok, crow, &ax.mb[SB_LD0 + st]);
                tc::tma_load_3d(base + 16384, &tm_x, (int)(hh * kP), tok, crow, &ax.mb[SB_LD0 + st]);
                last_ld[st] = c;
            };
            for (int c = 0; c < kStStages && c < n; ++c) load(c);
            for (int c = 0; c < n; ++c) {
                const int st = c % kStStages, xb = c & 1;
                if (!wait_bar(&ax.mb[SB_CONV0 + xb], &ax.abort, (c >> 1) & 1, a.err)) break;
                tc::fence_after_sync();
                const uint64_t dBm = tc::desc_sw128(sbase + st * ST_STAGE, 8192, 1024);          // MN-major B^T
                const uint64_t dXm = tc::desc_sw128(sbase + ST_OFF_XP + xb * 8192, 8192, 1024);  // MN-major X'
#pragma unroll
                for (int kk = 0; kk < kQ / 16; ++kk)
                    tc::mma_bf16(tmem, dBm + kk * 128, dXm + kk * 128, ID_S, (c > 0 || kk > 0) ? 1u : 0u);
                tc::mma_commit(&ax.mb[SB_MMA0 + xb]);
                // the stage of chunk c takes chunk c + 3 once MMA(c) has read its B
                // (every conv warp has read its raw x: conv(c) is complete)
                if (c + kStStages < n) {
                    if (!wait_bar(&ax.mb[SB_MMA0 + xb], &ax.abort, (c >> 1) & 1, a.err)) break;
                    load(c + kStStages);
                }
            }
            if (*reinterpret_cast<volatile int *>(&ax.abort)) {
                // drain: every MMA issued, and the last copy into each stage
                tc::mma_commit(&ax.mb[SB_DRAIN]);
                tc::mbar_wait(&ax.mb[SB_DRAIN], 0, 1u << 22);
                for (int b = 0; b < kStStages; ++b)
                    if (last_ld[b] >= 0) tc::mbar_wait(&ax.mb[SB_LD0 + b], (last_ld[b] / kStStages) & 1, 1u << 22);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ compute warps
        // x conv as in the scan kernel: channels 2 lane, 2 lane + 1; tokens 8 warp .. 8 warp + 7
        const int cq = lane, cr0 = warp * (kQ / 8);
        float2 cw0, cw1, cw2, cw3, cbias;
        {
            const int64_t ch = hh * kP + 2 * cq;
            auto tap = [&](int j) {
                const int k = K - 4 + j;
                return (K > 0 && k >= 0) ? make_float2(a.conv_w[ch * K + k], a.conv_w[(ch + 1) * K + k])
                                         : make_float2(0.f, 0.f);
            };
            cw0 = tap(0); cw1 = tap(1); cw2 = tap(2); cw3 = tap(3);
            cbias = a.conv_b ? make_float2(a.conv_b[ch], a.conv_b[ch + 1]) : make_float2(0.f, 0.f);
        }
        const uint32_t obase = (uint32_t)warp * 1024u + (uint32_t)(cq & 3) * 4u;
        bool ok = true;
        for (int c = 0; c < n; ++c) {
            const int st = c % kStStages, xb = c & 1;
            ok = wait_bar(&ax.mb[SB_LD0 + st], &ax.abort, (c / kStStages) & 1, a.err) && ok;
            if (c >= 2) ok = wait_bar(&ax.mb[SB_MMA0 + xb], &ax.abort, ((c - 2) >> 1) & 1, a.err) && ok;   // X' free
            // warp 0 reads the halo the last conv warp left with conv(c - 1)
            if (warp == 0 && c > 0) ok = wait_bar(&ax.mb[SB_CONV0 + ((c - 1) & 1)], &ax.abort, ((c - 1) >> 1) & 1, a.err) && ok;
            float wv[8];
            {
                const float4 w0 = *reinterpret_cast<const float4 *>(&wt[c * kQ + cr0]);
                const float4 w1 = *reinterpret_cast<const float4 *>(&wt[c * kQ + cr0 + 4]);
                wv[0] = w0.x; wv[1] = w0.y; wv[2] = w0.z; wv[3] = w0.w;
                wv[4] = w1.x; wv[5] = w1.y; wv[6] = w1.z; wv[7] = w1.w;
            }
            const unsigned char *xraw = smem + st * ST_STAGE + 16384;
            unsigned char *xpo = smem + ST_OFF_XP + xb * 8192;
            auto rawrow = [&](int v) -> float2 {
                const uint32_t u = *reinterpret_cast<const uint32_t *>(xraw + v * (kP * 2) + cq * 4);
                return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
            };
            float2 h0v, h1v, h2v;
            if (warp == 0) {
                const int hs = c % 3;
                h0v = *reinterpret_cast<const float2 *>(&ax.xh[hs][0][2 * cq]);
                h1v = *reinterpret_cast<const float2 *>(&ax.xh[hs][1][2 * cq]);
                h2v = *reinterpret_cast<const float2 *>(&ax.xh[hs][2][2 * cq]);
            } else {
                h0v = rawrow(cr0 - 3); h1v = rawrow(cr0 - 2); h2v = rawrow(cr0 - 1);
            }
#pragma unroll
            for (int i = 0; i < kQ / 8; ++i) {
                const float2 cur = rawrow(cr0 + i);
                const float2 xc = K > 0 ? conv_silu2(cur, h2v, h1v, h0v, cw3, cw2, cw1, cw0, cbias) : cur;
                h0v = h1v; h1v = h2v; h2v = cur;
                const float2 xw = __fmul2_rn(xc, make_float2(wv[i], wv[i]));
                const uint32_t off = obase + (uint32_t)i * 128u + ((uint32_t)((cq >> 2) ^ i) << 4);
                *reinterpret_cast<__nv_bfloat162 *>(xpo + off) = __floats2bfloat162_rn(xw.x, xw.y);
            }
            if (warp == kComputeWarps - 1) {
                // the chunk's last three raw rows: the halo of chunk c + 1
                const int hs = (c + 1) % 3;
                *reinterpret_cast<float2 *>(&ax.xh[hs][0][2 * cq]) = h0v;
                *reinterpret_cast<float2 *>(&ax.xh[hs][1][2 * cq]) = h1v;
                *reinterpret_cast<float2 *>(&ax.xh[hs][2][2 * cq]) = h2v;
            }
            tc::fence_proxy_async();
            __syncwarp();
            if (lane == 0) mb_arrive(&ax.mb[SB_CONV0 + xb]);
        }
        // the last accumulation
        ok = wait_bar(&ax.mb[SB_MMA0 + ((n - 1) & 1)], &ax.abort, ((n - 1) >> 1) & 1, a.err) && ok;
        (void)ok;
    }
    // No wait follows this barrier, so the abort flag (raised by any failed
    // wait) reads the same in every thread and the warp-wide loads stay converged.
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp < kComputeWarps && !*reinterpret_cast<volatile int *>(&ax.abort)) {
        const int q4 = warp & 3, hf = warp >> 2;
        float v[32];
        tc::tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + hf * 32, v);
        float *dst = a.sloc + q * kP * kN;
        const int nn = q4 * 32 + lane;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[(int64_t)(hf * 32 + i) * kN + nn] = v[i];
        if (tid == 0) a.slog[q] = ax.suf[0];
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kComputeWarps) tc::tmem_dealloc(tmem, 64);
}

// ------------------------------------------------------------------ B / C pre-pass
// Causal conv + SiLU of the B and C channels of x|B|C, once per group (every
// head of the group reads the result), into bf16 [tokens][G*N] workspace
// tiles.  One thread per (4 channels of B or C, 8 consecutive tokens): the
// K-1 rows before the run are loaded first (from the sequence's carried conv
// state before its first token), every row is one 8-byte load issued before
// any math, and a warp covers 32 consecutive channel vectors of one token
// row.  Four channels rather than eight keep a thread at 92 registers, so
// five CTAs (20 warps) fit per SM instead of three: the pass is bound by load
// latency.  Packed sequences restart the history at every sequence start.
struct BcArgs {
    const __nv_bfloat16 *B, *C;
    int64_t b_bs, b_ts, c_bs, c_ts;
    const float *w, *bias;            // full conv weight [conv_dim][K] and bias (or null)
    const __nv_bfloat16 *state_in;    // [nseq][conv_dim][K-1] or null
    __nv_bfloat16 *oB, *oC;           // [rows * seqlen][GN]
    const int32_t *cu;
    int nseqs;
    int64_t seqlen, GN, HP, cdim;
    bool w16, b16;                    // taps / bias of every 4-channel vector start 16-byte aligned
};

constexpr int kBcV = 4;               // channels per thread (one 8-byte row load)

SSM_DEVINL void unpack_bf16x4(uint2 r, float (&v)[kBcV]) {
    v[0] = __uint_as_float(r.x << 16); v[1] = __uint_as_float(r.x & 0xffff0000u);
    v[2] = __uint_as_float(r.y << 16); v[3] = __uint_as_float(r.y & 0xffff0000u);
}
SSM_DEVINL uint2 pack_bf16x4(const float (&v)[kBcV]) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
    return make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
}

// One thread per (4 channels of B or C, kBcR consecutive tokens); a warp
// covers 32 consecutive channel vectors of one token run.  Every load that
// does not depend on the sequence bounds (taps, bias, the K-1 rows before the
// run and its kBcR rows) is issued first, so their latency overlaps the
// search for the run's sequence in cu_seqlens (one thread per CTA, then each
// thread walks on from it); the conv history restarts at every sequence start.
constexpr int kBcR = 16;              // tokens per thread

template <int K>
__global__ void __launch_bounds__(128, 4) bc_conv_kernel(const BcArgs a) {
    constexpr int KH = K - 1;                             // rows before the run
    const int64_t nvec = 2 * a.GN / kBcV;                 // B and C vectors of one token row
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t vec = idx % nvec, run = idx / nvec;
    const int64_t t0 = run * kBcR;
    const int64_t row = blockIdx.y;
    const bool live = t0 < a.seqlen;
    const int which = vec >= nvec / 2;                    // 0: B, 1: C
    const int64_t c0 = (vec - which * (nvec / 2)) * kBcV; // channel within B (or C)
    const int64_t ts = which ? a.c_ts : a.b_ts;
    const __nv_bfloat16 *src = (which ? a.C + row * a.c_bs : a.B + row * a.b_bs) + c0;
    __nv_bfloat16 *dst = (which ? a.oC : a.oB) + row * a.seqlen * a.GN + c0;
    const int64_t cch = a.HP + which * a.GN + c0;         // conv channel of the first of the 4
    const bool in_range = SSM_BOUNDS(c0 + kBcV - 1, a.GN, BS_BC_CHANNEL) &&
                          (!live || SSM_BOUNDS(row * a.seqlen + t0, (int64_t)gridDim.y * a.seqlen, BS_BC_ROW));
    // taps and bias of the 4 channels: 16-byte loads when they are aligned (one
    // channel's 4 taps; 4 biases), scalar loads otherwise
    float wk[K][kBcV], bb[kBcV];
    if (K == 4 && a.w16) {
#pragma unroll
        for (int v = 0; v < kBcV; ++v) {
            const float4 q = *reinterpret_cast<const float4 *>(a.w + (cch + v) * 4);
            wk[0][v] = q.x; wk[1 % K][v] = q.y; wk[2 % K][v] = q.z; wk[3 % K][v] = q.w;
        }
    } else {
#pragma unroll
        for (int v = 0; v < kBcV; ++v)
#pragma unroll
            for (int k = 0; k < K; ++k) wk[k][v] = a.w[(cch + v) * K + k];
    }
    if (a.bias && a.b16) {
        const float4 b0 = *reinterpret_cast<const float4 *>(a.bias + cch);
        bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w;
    } else {
#pragma unroll
        for (int v = 0; v < kBcV; ++v) bb[v] = a.bias ? a.bias[cch + v] : 0.f;
    }
    // raw[j]: token t0 - (K-1) + j of the row (zero outside the tensor)
    uint2 raw[KH + kBcR];
#pragma unroll
    for (int j = 0; j < KH + kBcR; ++j) {
        const int64_t tau = t0 - KH + j;
        raw[j] = (live && in_range && tau >= 0 && tau < a.seqlen) ? *reinterpret_cast<const uint2 *>(src + tau * ts)
                                                                  : make_uint2(0u, 0u);
    }
    // packed sequences: one thread finds the sequence of the CTA's first token
    __shared__ int s_first;
    if (a.cu) {
        if (threadIdx.x == 0) {
            const int64_t tf = ((int64_t)blockIdx.x * blockDim.x / nvec) * kBcR;
            s_first = seq_of_token(a.cu, a.nseqs, min(tf, a.seqlen > 0 ? a.seqlen - 1 : (int64_t)0));
        }
        __syncthreads();
    }
    if (!live || !in_range) return;
    // sequence of the run's first token and its bounds (clamped: a malformed
    // cu_seqlens gives wrong values but no out-of-bounds access)
    int s = (int)row;
    if (a.cu) {
        s = s_first;
        while (s + 1 < a.nseqs && a.cu[s + 1] <= t0) ++s;
    }
    int64_t start = a.cu ? min(max((int64_t)a.cu[s], (int64_t)0), a.seqlen) : 0;
    int64_t end = a.cu ? min(max((int64_t)a.cu[s + 1], start), a.seqlen) : a.seqlen;
    // carried conv state of sequence s, tap q (0 .. K-2), or zero
    auto carried = [&](int q, float (&h)[kBcV]) {
        const bool in = a.state_in && SSM_BOUNDS(((int64_t)s * a.cdim + cch + kBcV - 1) * KH + q,
                                                 (int64_t)(a.cu ? a.nseqs : gridDim.y) * a.cdim * KH, BS_BC_STATE);
#pragma unroll
        for (int v = 0; v < kBcV; ++v)
            h[v] = in ? __bfloat162float(a.state_in[((int64_t)s * a.cdim + cch + v) * KH + q]) : 0.f;
    };
    float hist[KH > 0 ? KH : 1][kBcV];                    // hist[j] holds token t - (K-1) + j
#pragma unroll
    for (int j = 0; j < KH; ++j) {
        const int64_t tau = t0 - KH + j;
        if (tau >= start) unpack_bf16x4(raw[j], hist[j]);
        else carried((int)(tau - start + KH), hist[j]);   // tau >= t0 - (K-1) >= start - (K-1)
    }
    const int64_t t1 = min(t0 + kBcR, a.seqlen);
#pragma unroll
    for (int i = 0; i < kBcR; ++i) {
        const int64_t t = t0 + i;
        if (t >= t1) break;
        if (a.cu && t >= end) {                           // the next non-empty sequence starts here
            while (s + 1 < a.nseqs && a.cu[s + 1] <= t) ++s;
            start = min(max((int64_t)a.cu[s], (int64_t)0), a.seqlen);
            end = min(max((int64_t)a.cu[s + 1], start), a.seqlen);
            if (t < start || t >= end) return;
#pragma unroll
            for (int j = 0; j < KH; ++j) {                // taps before the sequence: its carried state
                const int64_t tau = t - KH + j;
                if (tau >= start) unpack_bf16x4(raw[i + j], hist[j]);
                else carried((int)(tau - start + KH), hist[j]);
            }
        }
        float cur[kBcV], o[kBcV];
        unpack_bf16x4(raw[KH + i], cur);
#pragma unroll
        for (int v = 0; v < kBcV; ++v) {
            float acc = bb[v];
#pragma unroll
            for (int k = 0; k < KH; ++k) acc = fmaf(wk[k][v], hist[k][v], acc);
            acc = fmaf(wk[K - 1][v], cur[v], acc);
            o[v] = silu_fast<__nv_bfloat16>(acc);
        }
        *reinterpret_cast<uint2 *>(dst + t * a.GN) = pack_bf16x4(o);
#pragma unroll
        for (int k = 0; k + 1 < KH; ++k)
#pragma unroll
            for (int v = 0; v < kBcV; ++v) hist[k][v] = hist[k + 1][v];
        if (KH > 0)
#pragma unroll
            for (int v = 0; v < kBcV; ++v) hist[KH > 0 ? KH - 1 : 0][v] = cur[v];
    }
}

// Segment table of packed sequences: in schedule order (longest first), each
// sequence of length len gets max(1, ceil(len / seg_len)) consecutive entries
// (sequence, segment, its segment count, the entry of its segment 0).  One
// CTA; a block-wide prefix sum over tiles of sequences.  Nothing is listed
// when the pre-pass found cu_seqlens malformed.
constexpr int kSegTabThreads = 1024;
__global__ void __launch_bounds__(kSegTabThreads)
seg_table_kernel(const int32_t *__restrict__ cu, const int32_t *__restrict__ order, const int32_t *err, int nseqs,
                 int64_t total, int64_t seg_len, int max_entries, int4 *__restrict__ tab, int32_t *count) {
    __shared__ int sh[kSegTabThreads];
    const int tid = threadIdx.x;
    if (err && *err != 0) {
        if (tid == 0) *count = 0;
        return;
    }
    int carry = 0;
    for (int p0 = 0; p0 < nseqs; p0 += kSegTabThreads) {
        const int p = p0 + tid;
        int sq = -1, ns = 0;
        if (p < nseqs) {
            sq = order ? order[p] : p;
            const int64_t c0 = min(max((int64_t)cu[sq], (int64_t)0), total);
            const int64_t c1 = min(max((int64_t)cu[sq + 1], c0), total);
            ns = (int)max((int64_t)1, (c1 - c0 + seg_len - 1) / seg_len);
        }
        sh[tid] = ns;
        __syncthreads();
        for (int o = 1; o < kSegTabThreads; o <<= 1) {        // inclusive scan
            const int v = tid >= o ? sh[tid - o] : 0;
            __syncthreads();
            sh[tid] += v;
            __syncthreads();
        }
        const int base = carry + sh[tid] - ns;
        for (int j = 0; j < ns; ++j)
            if (base + j < max_entries) tab[base + j] = make_int4(sq, j, ns, base);
        carry += sh[kSegTabThreads - 1];
        __syncthreads();
    }
    if (tid == 0) *count = min(carry, max_entries);
}

}  // namespace

bool ssd_shape_ok(const ssm_scan_args &s) {
    return s.mode == SSM_MAMBA2 && s.dtype == SSM_BF16 && s.headdim == kP && s.dstate == kN && s.d_conv >= 0 &&
           s.d_conv <= 4;
}

bool ssd_supported(const ssm_scan_args &s) {
    auto al16 = [](const void *p) { return p == nullptr || ((uintptr_t)p & 15) == 0; };
    auto st16ok = [](int64_t v) { return (v * 2) % 16 == 0; };
    return ssd_shape_ok(s) &&
           al16(s.x) && al16(s.z) && al16(s.y) && al16(s.B) && al16(s.C) && st16ok(s.x_token_stride) &&
           st16ok(s.x_batch_stride) && st16ok(s.y_token_stride) && st16ok(s.y_batch_stride) &&
           (s.z == nullptr || (st16ok(s.z_token_stride) && st16ok(s.z_batch_stride))) &&
           st16ok(s.B_token_stride) && st16ok(s.B_batch_stride) && st16ok(s.C_token_stride) &&
           st16ok(s.C_batch_stride);
}

namespace {
inline size_t round256(size_t v) { return (v + 255) / 256 * 256; }

// Segments of a fixed-length batch.  Requested (segments >= 2): about that
// many runs of whole chunks, at most kMaxSegChunks chunks per run.  Chosen
// (segments = 0): the count that minimises a model of the two launches in
// units of one chunk of one scan CTA, two CTAs per SM for both kernels, fitted
// to B200 timings of 4 x 4096 tokens x 80 heads at 1 to 8 segments:
//   scan   waves x (chunks per run + 1 + 0.15 (nseg - 1))  (pipeline fill, fold)
//   state  waves x (0.45 chunks per run + 2.5)               (prologue)
// A candidate must beat the whole-row plan by 3%.
struct SegPlan {
    int nseg;                           // fixed-length rows: segments per row
    int64_t seg_len;
    int64_t nslots = 0;                 // packed sequences: (segment) CTA rows launched, 0 = not cut
};
SegPlan plan_fixed(const ssm_scan_args &s) {
    SegPlan one{1, s.seqlen};
    if (s.batch <= 0 || s.seqlen <= kQ || s.segments == 1) return one;
    const int64_t nch = (s.seqlen + kQ - 1) / kQ;
    auto make = [&](int64_t k) {
        int64_t per = (nch + k - 1) / k;
        if (per > kMaxSegChunks) per = kMaxSegChunks;
        return SegPlan{(int)((nch + per - 1) / per), per * kQ};
    };
    auto fits = [&](const SegPlan &p) { return p.nseg >= 2 && s.batch * p.nseg <= 65535; };
    if (s.segments >= 2) {
        const SegPlan p = make(s.segments < nch ? s.segments : nch);
        return fits(p) ? p : one;
    }
    const double chains = (double)s.batch * (double)s.nheads, slots = 2.0 * sm_count();
    auto cost = [&](const SegPlan &p) {
        const double per = (double)(p.seg_len / kQ);
        double c = std::ceil(chains * p.nseg / slots) * (per + 1.0 + 0.15 * (p.nseg - 1));
        if (p.nseg > 1) c += std::ceil(chains * (p.nseg - 1) / slots) * (0.45 * per + 2.5);
        return c;
    };
    SegPlan best = one;
    double best_cost = std::ceil(chains / slots) * ((double)nch + 1.0);
    for (int64_t k = 2; k <= 8 && k <= nch; ++k) {
        const SegPlan p = make(k);
        if (!fits(p)) continue;
        const double c = cost(p);
        if (c < 0.97 * best_cost) { best = p; best_cost = c; }
    }
    return best;
}
// Packed sequences (lengths known on the device only): every sequence is cut
// into ceil(len / seg_len) segments of seg_len tokens (at least one), listed
// by a device pre-pass; nseqs + total / seg_len rows bound their count.  Cut
// when requested (segments >= 2: about that many runs for a sequence of the
// mean length) or, when chosen, if the sequences x heads give fewer chains
// than the GPU has CTA slots: then seg_len is the fixed-length choice for
// nseqs rows of the mean length.
SegPlan plan_packed(const ssm_scan_args &s) {
    SegPlan one{1, s.seqlen > 0 ? s.seqlen : 1};
    if (s.segments == 1 || s.nseqs <= 0 || s.seqlen <= kQ) return one;
    int64_t seg_len;
    if (s.segments >= 2) {
        const int64_t nch = (s.seqlen + kQ - 1) / kQ;
        int64_t per = (nch + (int64_t)s.nseqs * s.segments - 1) / ((int64_t)s.nseqs * s.segments);
        if (per < 1) per = 1;
        if (per > kMaxSegChunks) per = kMaxSegChunks;
        seg_len = per * kQ;
    } else {
        if ((double)s.nseqs * (double)s.nheads >= 2.0 * sm_count()) return one;
        ssm_scan_args m = s;
        m.cu_seqlens = nullptr;
        m.batch = s.nseqs;
        m.seqlen = (s.seqlen + s.nseqs - 1) / s.nseqs;
        const SegPlan f = plan_fixed(m);
        if (f.nseg < 2) return one;
        seg_len = f.seg_len;
    }
    const int64_t nslots = (int64_t)s.nseqs + (s.seqlen + seg_len - 1) / seg_len;
    if (nslots > 65535) return one;
    SegPlan p{1, seg_len, nslots};
    return p;
}
SegPlan plan_segments(const ssm_scan_args &s) { return s.cu_seqlens ? plan_packed(s) : plan_fixed(s); }
}  // namespace

int ssd_segments(const ssm_scan_args &s) {
    const SegPlan p = plan_segments(s);
    return p.nslots > 0 ? (int)p.nslots : p.nseg;
}

// Rows of segment states a plan keeps: fixed-length rows (nseg - 1) per row
// and head; packed sequences one per launched segment row and head.
size_t seg_state_rows(const ssm_scan_args &s, const SegPlan &p) {
    if (p.nslots > 0) return (size_t)p.nslots * (size_t)s.nheads;
    if (p.nseg > 1) return (size_t)s.batch * (size_t)(p.nseg - 1) * (size_t)s.nheads;
    return 0;
}

size_t ssd_workspace_bytes(const ssm_scan_args &s) {
    size_t total = 0;
    if (s.d_conv > 0) total += 2 * round256((size_t)s.batch * (size_t)s.seqlen * (size_t)(s.ngroups * s.dstate) * 2);
    const SegPlan sp = plan_segments(s);
    const size_t rows = seg_state_rows(s, sp);
    if (rows > 0) total += round256(rows * (size_t)(kP * kN) * 4) + round256(rows * 4);
    if (sp.nslots > 0) total += round256((size_t)sp.nslots * sizeof(int4) + 16);
    return total;
}

// cuTensorMapEncodeTiled from the driver, fetched once through the runtime
// (no link-time dependency on libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// A [batch][tokens][channels] bf16 tensor (element strides ts, bs) as a 3-d map
// with a 64-channel x 64-token box.
bool make_map_box(CUtensorMap *m, const void *base, int64_t channels, int64_t tokens, int64_t batch, int64_t ts,
                  int64_t bs, bool swizzle, int box_rows) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)channels, (cuuint64_t)tokens, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)ts * 2, (cuuint64_t)(batch > 1 ? bs : ts * tokens) * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool make_map(CUtensorMap *m, const void *base, int64_t channels, int64_t tokens, int64_t batch, int64_t ts, int64_t bs,
              bool swizzle) {
    return make_map_box(m, base, channels, tokens, batch, ts, bs, swizzle, kQ);
}

cudaError_t launch_ssd(const ssm_scan_args &s, const SeqView &sv, void *ws, cudaStream_t st) {
    const int nseqs = s.cu_seqlens ? s.nseqs : (int)s.batch;
    if (nseqs == 0) return cudaSuccess;
    const int64_t GN = s.ngroups * s.dstate;
    const int64_t cdim = s.d_inner + 2 * GN;
    const __nv_bfloat16 *Bc = static_cast<const __nv_bfloat16 *>(s.B), *Cc = static_cast<const __nv_bfloat16 *>(s.C);
    int64_t b_bs = s.B_batch_stride, b_ts = s.B_token_stride, c_bs = s.C_batch_stride, c_ts = s.C_token_stride;
    __nv_bfloat16 *wB = nullptr, *wC = nullptr;
    char *wp = static_cast<char *>(ws);
    if (s.d_conv > 0) {
        // the conv'd B and C live in the workspace
        const size_t one = round256((size_t)s.batch * (size_t)s.seqlen * (size_t)GN * 2);
        wB = reinterpret_cast<__nv_bfloat16 *>(wp);
        wC = reinterpret_cast<__nv_bfloat16 *>(wp + one);
        wp += 2 * one;
        Bc = wB; Cc = wC;
        b_bs = c_bs = s.seqlen * GN;
        b_ts = c_ts = GN;
    }
    // then the segment states (fixed-length rows cut into segments)
    const SegPlan sp = plan_segments(s);
    const bool packed_cut = sp.nslots > 0;
    const bool cut = sp.nseg > 1 || packed_cut;
    float *sloc = nullptr, *slog = nullptr;
    int4 *seg_tab = nullptr;
    int32_t *seg_count = nullptr;
    const size_t srows = seg_state_rows(s, sp);
    if (srows > 0) {
        sloc = reinterpret_cast<float *>(wp);
        slog = reinterpret_cast<float *>(wp + round256(srows * (size_t)(kP * kN) * 4));
        wp += round256(srows * (size_t)(kP * kN) * 4) + round256(srows * 4);
    }
    if (packed_cut) {
        seg_tab = reinterpret_cast<int4 *>(wp);
        seg_count = reinterpret_cast<int32_t *>(wp + (size_t)sp.nslots * sizeof(int4));
    }
    // Host work first (tensor maps over the whole packed / batched token range,
    // the kernel attribute), so nothing on the host separates the pre-pass
    // launches from the scan launch.
    const int64_t rows = s.cu_seqlens ? 1 : s.batch;
    CUtensorMap tm_x, tm_b, tm_c, tm_z, tm_y;
    memset(&tm_x, 0, sizeof(tm_x)); memset(&tm_b, 0, sizeof(tm_b)); memset(&tm_c, 0, sizeof(tm_c));
    memset(&tm_z, 0, sizeof(tm_z)); memset(&tm_y, 0, sizeof(tm_y));
    // With no tokens at all no CTA has a chunk, so no copy is issued and the
    // maps (which cannot describe an empty tensor) are left unset.
    if (s.seqlen > 0) {
        if (s.z && !make_map(&tm_z, s.z, s.d_inner, s.seqlen, rows, s.z_token_stride, s.z_batch_stride, true))
            return cudaErrorInvalidValue;
        if (!make_map(&tm_x, s.x, s.d_inner, s.seqlen, rows, s.x_token_stride, s.x_batch_stride, false) ||
            !make_map(&tm_b, Bc, GN, s.seqlen, rows, b_ts, b_bs, true) ||
            !make_map(&tm_c, Cc, GN, s.seqlen, rows, c_ts, c_bs, true) ||
            !make_map(&tm_y, s.y, s.d_inner, s.seqlen, rows, s.y_token_stride, s.y_batch_stride, true))
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(ssd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    if (cut) {
        e = cudaFuncSetAttribute(ssd_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStSmemBytes);
        if (e != cudaSuccess) return e;
    }
    if (packed_cut) {
        // the segment table of the packed sequences (their lengths live on the device)
        seg_table_kernel<<<1, kSegTabThreads, 0, st>>>(sv.cu, sv.order, sv.err, s.nseqs, s.seqlen, sp.seg_len,
                                                        (int)sp.nslots, seg_tab, seg_count);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (s.d_conv > 0) {
        // pre-pass: conv + SiLU of the B and C channels, once per group, into the workspace
        BcArgs b;
        b.B = static_cast<const __nv_bfloat16 *>(s.B); b.C = static_cast<const __nv_bfloat16 *>(s.C);
        b.b_bs = s.B_batch_stride; b.b_ts = s.B_token_stride; b.c_bs = s.C_batch_stride; b.c_ts = s.C_token_stride;
        b.w = s.conv_w; b.bias = s.conv_b;
        b.state_in = static_cast<const __nv_bfloat16 *>(s.conv_state_in);
        b.oB = wB; b.oC = wC;
        b.cu = s.cu_seqlens; b.nseqs = s.nseqs;
        b.seqlen = s.seqlen; b.GN = GN; b.HP = s.d_inner; b.cdim = cdim;
        // channel offsets are multiples of 8 (d_inner = H * 64, G * N = G * 128), so the
        // rows start 16-byte aligned whenever the arrays do
        b.w16 = ((uintptr_t)s.conv_w % 16) == 0;
        b.b16 = s.conv_b != nullptr && ((uintptr_t)s.conv_b % 16) == 0;
        const int64_t threads = (s.seqlen + kBcR - 1) / kBcR * (2 * GN / kBcV);
        const dim3 bgrid((unsigned)((threads + 127) / 128), (unsigned)rows);
        if (threads > 0) {
            switch (s.d_conv) {
                case 1: bc_conv_kernel<1><<<bgrid, 128, 0, st>>>(b); break;
                case 2: bc_conv_kernel<2><<<bgrid, 128, 0, st>>>(b); break;
                case 3: bc_conv_kernel<3><<<bgrid, 128, 0, st>>>(b); break;
                default: bc_conv_kernel<4><<<bgrid, 128, 0, st>>>(b); break;
            }
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }
    SsdArgs a;
    a.x = static_cast<const __nv_bfloat16 *>(s.x); a.z = static_cast<const __nv_bfloat16 *>(s.z);
    a.dt = static_cast<const __nv_bfloat16 *>(s.dt); a.Bc = Bc; a.Cc = Cc;
    a.y = static_cast<__nv_bfloat16 *>(s.y);
    a.x_bs = s.x_batch_stride; a.x_ts = s.x_token_stride; a.z_bs = s.z_batch_stride; a.z_ts = s.z_token_stride;
    a.dt_bs = s.dt_batch_stride; a.dt_ts = s.dt_token_stride;
    a.b_bs = b_bs; a.b_ts = b_ts; a.c_bs = c_bs; a.c_ts = c_ts;
    a.y_bs = s.y_batch_stride; a.y_ts = s.y_token_stride;
    a.A = s.A; a.D = s.D; a.dt_bias = s.dt_bias; a.h0 = s.h0; a.conv_w = s.conv_w; a.conv_b = s.conv_b;
    a.h_final = s.h_final;
    a.conv_state_in = static_cast<const __nv_bfloat16 *>(s.conv_state_in);
    a.conv_state_out = static_cast<__nv_bfloat16 *>(s.conv_state_out);
    a.H = s.nheads; a.G = s.ngroups; a.seqlen = s.seqlen; a.cdim = cdim;
    a.K = (int)s.d_conv; a.softplus = s.delta_softplus;
    a.sv = sv;
    a.err = sv.err;
    a.iv = inter_view(s);
    a.Braw = static_cast<const __nv_bfloat16 *>(s.B); a.Craw = static_cast<const __nv_bfloat16 *>(s.C);
    a.braw_bs = s.B_batch_stride; a.braw_ts = s.B_token_stride;
    a.craw_bs = s.C_batch_stride; a.craw_ts = s.C_token_stride;
    a.nseg = sp.nseg; a.seg_len = cut ? sp.seg_len : (s.seqlen > 0 ? s.seqlen : 1);
    a.sloc = sloc; a.slog = slog;
    a.seg_tab = seg_tab; a.seg_count = seg_count;
    a.nsloc = (int64_t)(srows / (size_t)s.nheads);
    // the timed region holds the state pass and the scan
    timing_begin(st);
    if (cut) {
        // the state each segment but the last leaves, from zero
        const dim3 sgrid((unsigned)s.nheads, (unsigned)(packed_cut ? sp.nslots : (int64_t)nseqs * (sp.nseg - 1)));
        ssd_state_kernel<<<sgrid, kThreads, kStSmemBytes, st>>>(a, tm_x, tm_b);
        e = cudaGetLastError();
        if (e != cudaSuccess) {
            timing_end(st);
            return e;
        }
    }
    dim3 grid((unsigned)s.nheads, (unsigned)(packed_cut ? sp.nslots : (int64_t)nseqs * sp.nseg));
    ssd_kernel<<<grid, kThreads, kSmemBytes, st>>>(a, tm_x, tm_b, tm_c, tm_z, tm_y);
    timing_end(st);
    return cudaGetLastError();
}

}  // namespace ssm
