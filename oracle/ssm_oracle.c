/*
 * ssm_oracle.c -- fp64 CPU oracle for the Mamba conv1d + selective-scan hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * loads this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA path.
 *
 * What it computes is the plain definition, sequential over tokens, in C
 * double precision (no fast-math, no SIMD intrinsics, no blocking or chunking):
 *
 *   conv (GGML_OP_SSM_CONV semantics):
 *     xc[t,c] = silu( b[c] + sum_{k<K} w[c,k] * u[t-K+1+k, c] )
 *     where u[<0] comes from the carried conv state (the last K-1 raw inputs
 *     of the previous call), and w[c,K-1] multiplies the current token.
 *     Source: "ggml : add GPU support for Mamba models" (llama.cpp issue
 *     6758), the test-backend-ops patch for SSM_CONV (state s of shape
 *     [d_conv-1, d_inner, n_seqs], weights c of shape [d_conv, d_inner]) and
 *     the reply on fusing the state concat into the op ("+1 on a pointer").
 *
 *   recurrence (GGML_OP_SSM_SCAN semantics, Mamba-1 and Mamba-2 forms):
 *     delta = softplus(dt + dt_bias)          (identity when softplus is off)
 *     h_t   = exp(delta_t * A) * h_{t-1} + delta_t * B_t * x_t
 *     y_t   = C_t . h_t + D * x_t,  then y_t *= silu(z_t) when z is given
 *     Source: "Adding Initial Value Support to Selective Scan Forward Kernel"
 *     (state-spaces/mamba issue 285): the opening post states the step
 *     h_t = A*h_{t-1} + Bx with h_0 = 0 by default, and the reply on the
 *     running prefix gives the scan element as the pair (exp(delta*A), h)
 *     seeded with (1, h0).  Mamba-2 grouping (contiguous groups of heads
 *     sharing B/C, as repeat_interleave does) follows "Tensor-parallel SSM"
 *     (Fast-LLM PR 333), review thread on repeat_kv / repeat_interleave.
 *
 *   The final state is returned as an output rather than written into an
 *   input, as the llama.cpp thread settles on (the op's output includes the
 *   final state so tests can compare it).
 *
 * Layouts (all contiguous, fp64, tokens packed across sequences):
 *   Mamba-1 (channels = d_inner = D_, states N):
 *     x,z,dt,y [tok][D_]; B,C [tok][N]; A [D_][N]; D,dt_bias [D_];
 *     h0,h_final [seq][D_][N]; conv channels = D_.
 *   Mamba-2 (H heads of P channels, G groups, N states):
 *     x,z,y [tok][H*P]; dt [tok][H]; B,C [tok][G][N]; A,D,dt_bias [H];
 *     h0,h_final [seq][H][P][N]; conv channels = H*P + 2*G*N in the order
 *     x | B | C (B and C are convolved too).
 *   conv_w [conv_dim][K]; conv_b [conv_dim]; conv_state [seq][conv_dim][K-1].
 *
 * Parity pins: closed forms, brute-force products, split invariance, conv
 * special cases and cross-mode reductions live in the test suite; this file
 * is the plain loop those pins check.
 *
 * SSM_ORACLE_MUTANT (compile-time, default 0) plants one deliberate mistake
 * so the test suite can show that its pins catch it.  A normal build has 0.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef SSM_ORACLE_MUTANT
#define SSM_ORACLE_MUTANT 0
#endif

#define ORACLE_M1 1
#define ORACLE_M2 2

typedef struct {
    int32_t mode;          /* ORACLE_M1 or ORACLE_M2 */
    int32_t delta_softplus;/* 1: delta = softplus(dt + dt_bias); 0: delta = dt + dt_bias */
    int32_t nthreads;      /* OpenMP threads over independent sequences (<=0: 1) */
    int32_t pad_;
    int64_t nseqs;         /* number of independent sequences */
    const int64_t *seq_start; /* [nseqs+1] token offsets into the packed axis */
    int64_t d_inner;       /* M1: channels; M2: H*P */
    int64_t nheads, headdim, ngroups, dstate;
    int64_t d_conv;        /* K; 0 = no conv (x, B, C used as given, no SiLU) */
    const double *x, *z, *dt, *B, *C;
    const double *A, *D, *dt_bias;
    const double *h0;      /* may be NULL (zeros) */
    const double *conv_w, *conv_b, *conv_state_in; /* conv_b / state_in may be NULL */
    double *y, *h_final, *conv_state_out;          /* conv_state_out may be NULL */
    /* Intermediate states for prefix caching ("Clean up SSM ops directory
     * structure", Megatron-LM PR 6444: intermediate_extraction, a conditional
     * scatter of flat state rows into slots).  When state_interval > 0, after
     * every state_interval tokens of a sequence (boundary k at token
     * (k+1)*state_interval from the sequence start, k < inter_stride) the
     * state and the conv history are copied to pool row
     * inter_slots[s*inter_stride + k] when that index lies in [0, inter_nslots);
     * other indices write nothing. */
    int64_t state_interval;
    const int32_t *inter_slots;    /* [nseqs][inter_stride] */
    int64_t inter_stride, inter_nslots;
    double *inter_states;          /* [inter_nslots][state size] */
    double *inter_conv;            /* [inter_nslots][conv_dim][K-1] or NULL */
} oracle_scan_args;

typedef struct {
    int32_t activation;    /* 0 none, 1 silu */
    int32_t pad_;
    int64_t nseqs;
    const int64_t *seq_start;
    int64_t channels, width;
    const double *x;       /* [tok][channels] */
    const double *w, *b;   /* [channels][width], [channels] or NULL */
    const double *state_in;/* [seq][channels][width-1] or NULL */
    double *out;           /* [tok][channels] */
    double *state_out;     /* [seq][channels][width-1] or NULL */
} oracle_conv_args;

typedef struct {
    int32_t mode, delta_softplus;
    int64_t batch, d_inner, nheads, headdim, ngroups, dstate;
    int64_t d_conv, conv_state_len;
    double *state;         /* in-out: M1 [b][D_][N]; M2 [b][H][P][N] */
    double *conv_state;    /* in-out: [b][conv_dim][conv_state_len] */
    const double *conv_w, *conv_b;
    const double *x, *z, *dt, *B, *C;  /* one token per row: layouts as above with tok = row */
    const double *A, *D, *dt_bias;
    double *y;
} oracle_update_args;

/* ---- scalar functions, written from their definitions ---- */

static double o_silu(double v) { return v / (1.0 + exp(-v)); }

/* softplus(u) = log(1 + e^u); the two branches are the same identity
 * (log(1+e^u) = u + log(1+e^-u)) and only avoid overflow of e^u. */
static double o_softplus(double u) {
    return u > 0.0 ? u + log1p(exp(-u)) : log1p(exp(u));
}

static double o_delta(double dt, double bias, int softplus_on) {
#if SSM_ORACLE_MUTANT == 7
    bias = 0.0;                              /* mutant: dt_bias dropped */
#endif
    double u = dt + bias;
#if SSM_ORACLE_MUTANT == 11
    softplus_on = !softplus_on;              /* mutant: softplus switch inverted */
#endif
    return softplus_on ? o_softplus(u) : u;
}

/* One causal depthwise conv output for channel c at the current token.
 * hist holds the previous K-1 raw inputs, oldest first; cur is the current raw
 * input.  Weight w[K-1] multiplies the current token, w[0] the oldest. */
static double o_conv_tap(const double *w, double bias, const double *hist, double cur, int64_t K) {
    double acc = bias;
    for (int64_t k = 0; k < K; ++k) {
        double u = (k == K - 1) ? cur : hist[k];
#if SSM_ORACLE_MUTANT == 4
        acc += w[K - 1 - k] * u;             /* mutant: taps reversed */
#else
        acc += w[k] * u;
#endif
    }
    return acc;
}

static void o_hist_push(double *hist, double cur, int64_t K) {
    for (int64_t k = 0; k + 1 < K - 1; ++k) hist[k] = hist[k + 1];
    if (K > 1) hist[K - 2] = cur;
}

static int64_t o_conv_dim(const oracle_scan_args *a) {
    if (a->mode == ORACLE_M1) return a->d_inner;
    return a->d_inner + 2 * a->ngroups * a->dstate;
}

/* ---- one sequence of the forward scan ---- */
static void scan_one_sequence(const oracle_scan_args *a, int64_t s) {
    const int64_t t0 = a->seq_start[s], t1 = a->seq_start[s + 1];
    const int64_t N = a->dstate, K = a->d_conv;
    const int64_t Dn = a->d_inner;
    const int64_t cdim = o_conv_dim(a);
    const int64_t H = (a->mode == ORACLE_M1) ? Dn : a->nheads;
    const int64_t P = (a->mode == ORACLE_M1) ? 1 : a->headdim;
    const int64_t G = (a->mode == ORACLE_M1) ? 1 : a->ngroups;
    const int64_t hsz = Dn * N; /* M1: D_*N ; M2: H*P*N */

    double *h = (double *)calloc((size_t)hsz, sizeof(double));
    double *hist = (K > 1) ? (double *)calloc((size_t)(cdim * (K - 1)), sizeof(double)) : NULL;
    double *u = (double *)malloc((size_t)cdim * sizeof(double));   /* conv outputs */

    /* initial state: the scan prefix is seeded with (1, h0) */
#if SSM_ORACLE_MUTANT != 1
    if (a->h0)
        for (int64_t i = 0; i < hsz; ++i) h[i] = a->h0[s * hsz + i];
#endif
    if (K > 1 && a->conv_state_in)
#if SSM_ORACLE_MUTANT != 10
        for (int64_t i = 0; i < cdim * (K - 1); ++i) hist[i] = a->conv_state_in[s * cdim * (K - 1) + i];
#else
        ;                                    /* mutant: conv state ignored */
#endif

    for (int64_t t = t0; t < t1; ++t) {
        /* raw channel values for this token, in conv channel order */
        for (int64_t c = 0; c < cdim; ++c) {
            double raw;
            if (c < Dn) raw = a->x[t * Dn + c];
            else if (c < Dn + G * N) raw = a->B[t * G * N + (c - Dn)];
            else raw = a->C[t * G * N + (c - Dn - G * N)];
            if (K > 0) {
                double pre = o_conv_tap(a->conv_w + c * K, a->conv_b ? a->conv_b[c] : 0.0,
                                        hist ? hist + c * (K - 1) : NULL, raw, K);
                u[c] = o_silu(pre);
                if (hist) o_hist_push(hist + c * (K - 1), raw, K);
            } else {
                u[c] = raw;
            }
        }
        /* B and C for this token: M1 takes them unconvolved (the conv covers x
         * only); M2 takes the convolved x|B|C channels. */
        const double *Bt, *Ct;
        if (a->mode == ORACLE_M1) {
            Bt = a->B + t * N;
            Ct = a->C + t * N;
        } else {
            Bt = u + Dn;
            Ct = u + Dn + G * N;
        }
#if SSM_ORACLE_MUTANT == 9
        { const double *tmp = Bt; Bt = Ct; Ct = tmp; }   /* mutant: B and C swapped */
#endif
        for (int64_t hh = 0; hh < H; ++hh) {
            int64_t g;
#if SSM_ORACLE_MUTANT == 5
            g = (a->mode == ORACLE_M1) ? 0 : hh % G;       /* mutant: strided group map */
#else
            g = (a->mode == ORACLE_M1) ? 0 : hh / (H / G); /* contiguous groups */
#endif
            const double dtv = (a->mode == ORACLE_M1) ? a->dt[t * Dn + hh] : a->dt[t * H + hh];
            const double delta = o_delta(dtv, a->dt_bias ? a->dt_bias[hh] : 0.0, a->delta_softplus);
            for (int64_t p = 0; p < P; ++p) {
                const int64_t ch = hh * P + p;             /* channel index into x / y */
                const double xv = u[ch];
                double *hs = h + ch * N;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double An = (a->mode == ORACLE_M1) ? a->A[hh * N + n] : a->A[hh];
#if SSM_ORACLE_MUTANT == 3
                    const double dA = exp(-delta * An);    /* mutant: sign flipped */
#else
                    const double dA = exp(delta * An);
#endif
#if SSM_ORACLE_MUTANT == 6
                    acc += Ct[g * N + n] * hs[n];          /* mutant: read-out before update */
                    hs[n] = dA * hs[n] + delta * Bt[g * N + n] * xv;
#else
                    hs[n] = dA * hs[n] + delta * Bt[g * N + n] * xv;
                    acc += Ct[g * N + n] * hs[n];
#endif
                }
                double yv = acc;
#if SSM_ORACLE_MUTANT == 12
                if (a->D) yv += a->D[hh] * (ch < Dn ? a->x[t * Dn + ch] : 0.0); /* mutant: pre-conv x */
#elif SSM_ORACLE_MUTANT != 2
                if (a->D) yv += a->D[(a->mode == ORACLE_M1) ? ch : hh] * xv;
#endif
#if SSM_ORACLE_MUTANT == 8
                if (a->z) yv *= o_silu(xv);                 /* mutant: gate on x */
#else
                if (a->z) yv *= o_silu(a->z[t * Dn + ch]);
#endif
                a->y[t * Dn + ch] = yv;
            }
        }
        /* intermediate state after this token, when it closes an interval */
#if SSM_ORACLE_MUTANT == 13
        const int64_t done = t - t0 + 2;             /* mutant: boundary one token early */
#else
        const int64_t done = t - t0 + 1;             /* tokens of this sequence processed so far */
#endif
        if (a->state_interval > 0 && a->inter_slots && done % a->state_interval == 0) {
            const int64_t k = done / a->state_interval - 1;
            if (k < a->inter_stride) {
                const int64_t slot = a->inter_slots[s * a->inter_stride + k];
                if (slot >= 0 && slot < a->inter_nslots) {
                    if (a->inter_states)
                        for (int64_t i = 0; i < hsz; ++i) a->inter_states[slot * hsz + i] = h[i];
                    if (a->inter_conv && K > 1)
                        for (int64_t i = 0; i < cdim * (K - 1); ++i) a->inter_conv[slot * cdim * (K - 1) + i] = hist[i];
                }
            }
        }
    }
    for (int64_t i = 0; i < hsz; ++i) a->h_final[s * hsz + i] = h[i];
    if (K > 1 && a->conv_state_out)
        for (int64_t i = 0; i < cdim * (K - 1); ++i) a->conv_state_out[s * cdim * (K - 1) + i] = hist[i];
    free(h);
    free(hist);
    free(u);
}

int oracle_scan_fwd(const oracle_scan_args *a) {
    if (!a || !a->seq_start || !a->x || !a->dt || !a->A || !a->B || !a->C || !a->y || !a->h_final) return -1;
    if (a->mode != ORACLE_M1 && a->mode != ORACLE_M2) return -1;
    if (a->mode == ORACLE_M2 && (a->nheads * a->headdim != a->d_inner || a->ngroups <= 0 ||
                                 a->nheads % a->ngroups != 0)) return -1;
    if (a->d_conv > 0 && !a->conv_w) return -1;
    const int64_t ns = a->nseqs;
#ifdef _OPENMP
    const int nt = a->nthreads > 0 ? a->nthreads : 1;
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
#endif
    for (int64_t s = 0; s < ns; ++s) scan_one_sequence(a, s);
    return 0;
}

/* ---- backward of the forward scan (reverse mode, plain loops) ----
 *
 * Gradients of L = sum(dy * y) + sum(dh_final * h_final) + sum(dconv_state_out
 * * conv_state_out) with respect to every input of oracle_scan_fwd, for the
 * same arguments.  The step h_t = a_t h_{t-1} + delta_t B_t x_t with
 * a_t = exp(delta_t A) is differentiated as it stands ("Adding Initial Value
 * Support to Selective Scan Forward Kernel", state-spaces/mamba issue 285: the
 * backward carries dh back through exp(delta A) down to the initial state,
 * whose gradient is the carried dh after the first token).  The forward
 * trajectory (every h_t, every conv output and pre-activation) is stored and
 * walked backwards; nothing is chunked.
 */
typedef struct {
    oracle_scan_args fwd;          /* the forward call (its y / h_final / conv_state_out are scratch) */
    const double *dy;              /* [tok][D_] */
    const double *dh_final;        /* [seq][state] or NULL */
    const double *dconv_state_out; /* [seq][conv_dim][K-1] or NULL */
    double *dx, *dz, *ddt, *dB, *dC;  /* like x, z, dt, B, C (raw, before the conv) */
    double *dA, *dD, *ddt_bias;       /* like A, D, dt_bias (dD / ddt_bias may be NULL) */
    double *dh0;                      /* [seq][state] */
    double *dconv_w, *dconv_b;        /* [conv_dim][K], [conv_dim] (may be NULL) */
    double *dconv_state_in;           /* [seq][conv_dim][K-1] (may be NULL) */
} oracle_scan_bwd_args;

static double o_sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }
static double o_dsilu(double v) { const double sg = o_sigmoid(v); return sg * (1.0 + v * (1.0 - sg)); }

static void bwd_one_sequence(const oracle_scan_bwd_args *b, int64_t s) {
    const oracle_scan_args *a = &b->fwd;
    const int64_t t0 = a->seq_start[s], t1 = a->seq_start[s + 1], T = t1 - t0;
    const int64_t N = a->dstate, K = a->d_conv, Dn = a->d_inner;
    const int64_t cdim = o_conv_dim(a);
    const int m1 = a->mode == ORACLE_M1;
    const int64_t H = m1 ? Dn : a->nheads, P = m1 ? 1 : a->headdim, G = m1 ? 1 : a->ngroups;
    const int64_t hsz = Dn * N, KW = K > 1 ? K - 1 : 0;

    /* forward trajectory: raw inputs r, pre-activations pre, conv outputs u, deltas, states */
    double *raw = (double *)calloc((size_t)((T + KW) * cdim + 1), sizeof(double)); /* KW history rows first */
    double *pre = (double *)calloc((size_t)(T * cdim + 1), sizeof(double));
    double *u = (double *)calloc((size_t)(T * cdim + 1), sizeof(double));
    double *dl = (double *)calloc((size_t)(T * H + 1), sizeof(double));
    double *hs = (double *)calloc((size_t)((T + 1) * hsz), sizeof(double));
    double *du = (double *)calloc((size_t)(T * cdim + 1), sizeof(double));
    double *g = (double *)calloc((size_t)hsz, sizeof(double));
    for (int64_t j = 0; j < KW; ++j)
        for (int64_t c = 0; c < cdim; ++c)
            raw[j * cdim + c] = a->conv_state_in ? a->conv_state_in[(s * cdim + c) * KW + j] : 0.0;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < cdim; ++c) {
            const int64_t tt = t0 + t;
            double r;
            if (c < Dn) r = a->x[tt * Dn + c];
            else if (c < Dn + G * N) r = a->B[tt * G * N + (c - Dn)];
            else r = a->C[tt * G * N + (c - Dn - G * N)];
            raw[(KW + t) * cdim + c] = r;
        }
    const int64_t ccov = m1 ? Dn : cdim;    /* channels that pass through the conv */
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < cdim; ++c) {
            const double r = raw[(KW + t) * cdim + c];
            if (K > 0 && c < ccov) {
                double acc = a->conv_b ? a->conv_b[c] : 0.0;
                for (int64_t k = 0; k < K; ++k) acc += a->conv_w[c * K + k] * raw[(KW + t - (K - 1) + k) * cdim + c];
                pre[t * cdim + c] = acc;
                u[t * cdim + c] = o_silu(acc);
            } else {
                u[t * cdim + c] = r;
            }
        }
    if (a->h0)
        for (int64_t i = 0; i < hsz; ++i) hs[i] = a->h0[s * hsz + i];
    for (int64_t t = 0; t < T; ++t) {
        const int64_t tt = t0 + t;
        for (int64_t hh = 0; hh < H; ++hh) {
            const double dtv = m1 ? a->dt[tt * Dn + hh] : a->dt[tt * H + hh];
            dl[t * H + hh] = o_delta(dtv, a->dt_bias ? a->dt_bias[hh] : 0.0, a->delta_softplus);
        }
        const double *Bt = m1 ? a->B + tt * N : u + t * cdim + Dn;
        for (int64_t hh = 0; hh < H; ++hh) {
            const int64_t gg = m1 ? 0 : hh / (H / G);
            const double delta = dl[t * H + hh];
            for (int64_t p = 0; p < P; ++p) {
                const int64_t ch = hh * P + p;
                for (int64_t n = 0; n < N; ++n) {
                    const double An = m1 ? a->A[hh * N + n] : a->A[hh];
                    hs[(t + 1) * hsz + ch * N + n] = exp(delta * An) * hs[t * hsz + ch * N + n] +
                                                     delta * Bt[gg * N + n] * u[t * cdim + ch];
                }
            }
        }
    }

    /* reverse sweep over the recurrence */
    for (int64_t i = 0; i < hsz; ++i) g[i] = b->dh_final ? b->dh_final[s * hsz + i] : 0.0;
    for (int64_t t = T - 1; t >= 0; --t) {
        const int64_t tt = t0 + t;
        const double *Bt = m1 ? a->B + tt * N : u + t * cdim + Dn;
        const double *Ct = m1 ? a->C + tt * N : u + t * cdim + Dn + G * N;
        for (int64_t hh = 0; hh < H; ++hh) {
            const int64_t gg = m1 ? 0 : hh / (H / G);
            const double delta = dl[t * H + hh];
            double ddelta = 0.0;
            for (int64_t p = 0; p < P; ++p) {
                const int64_t ch = hh * P + p;
                const double xv = u[t * cdim + ch];
                const double *ht = hs + (t + 1) * hsz + ch * N, *hp = hs + t * hsz + ch * N;
                double ybase = 0.0;
                for (int64_t n = 0; n < N; ++n) ybase += Ct[gg * N + n] * ht[n];
                const double Dv = a->D ? a->D[m1 ? ch : hh] : 0.0;
                ybase += Dv * xv;
                const double dyv = b->dy[tt * Dn + ch];
                double dyb = dyv;
                if (a->z) {
                    const double zv = a->z[tt * Dn + ch];
                    b->dz[tt * Dn + ch] = dyv * ybase * o_dsilu(zv);
                    dyb = dyv * o_silu(zv);
                }
                if (b->dD && a->D) b->dD[m1 ? ch : hh] += dyb * xv;
                du[t * cdim + ch] += dyb * Dv;
                for (int64_t n = 0; n < N; ++n) {
                    const double dCv = dyb * ht[n];
                    if (m1) b->dC[tt * N + n] += dCv;
                    else du[t * cdim + Dn + G * N + gg * N + n] += dCv;
                    g[ch * N + n] += dyb * Ct[gg * N + n];
                }
                for (int64_t n = 0; n < N; ++n) {
                    const double An = m1 ? a->A[hh * N + n] : a->A[hh];
                    const double av = exp(delta * An);
                    const double gn = g[ch * N + n];
                    const double dBv = gn * delta * xv;
                    if (m1) b->dB[tt * N + n] += dBv;
                    else du[t * cdim + Dn + gg * N + n] += dBv;
                    du[t * cdim + ch] += gn * delta * Bt[gg * N + n];
                    ddelta += gn * (hp[n] * av * An + Bt[gg * N + n] * xv);
                    if (m1) b->dA[hh * N + n] += gn * hp[n] * av * delta;
                    else b->dA[hh] += gn * hp[n] * av * delta;
#if SSM_ORACLE_MUTANT == 14
                    g[ch * N + n] = gn;                      /* mutant: dh not carried through exp(delta A) */
#else
                    g[ch * N + n] = gn * av;
#endif
                }
            }
            const double dtv = m1 ? a->dt[tt * Dn + hh] : a->dt[tt * H + hh];
            const double uarg = dtv + (a->dt_bias ? a->dt_bias[hh] : 0.0);
            const double dd = a->delta_softplus ? ddelta * o_sigmoid(uarg) : ddelta;
            b->ddt[m1 ? tt * Dn + hh : tt * H + hh] = dd;
            if (b->ddt_bias && a->dt_bias) b->ddt_bias[hh] += dd;
        }
    }
    for (int64_t i = 0; i < hsz; ++i) b->dh0[s * hsz + i] = g[i];

    /* reverse sweep over the conv: d(raw) over the sequence and its history */
    double *draw = (double *)calloc((size_t)((T + KW) * cdim + 1), sizeof(double));
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < cdim; ++c) {
            const double dv = du[t * cdim + c];
            if (K > 0 && c < ccov) {
                const double dp = dv * o_dsilu(pre[t * cdim + c]);
                if (b->dconv_b) b->dconv_b[c] += dp;
                for (int64_t k = 0; k < K; ++k) {
                    const int64_t r = KW + t - (K - 1) + k;
                    if (b->dconv_w) b->dconv_w[c * K + k] += dp * raw[r * cdim + c];
                    draw[r * cdim + c] += dp * a->conv_w[c * K + k];
                }
            } else {
                draw[(KW + t) * cdim + c] += dv;
            }
        }
    /* the carried conv state out is the last K-1 raw rows of history + sequence */
    if (b->dconv_state_out && KW > 0)
        for (int64_t j = 0; j < KW; ++j)
            for (int64_t c = 0; c < cdim; ++c) draw[(T + j) * cdim + c] += b->dconv_state_out[(s * cdim + c) * KW + j];
    for (int64_t j = 0; j < KW; ++j)
        for (int64_t c = 0; c < cdim; ++c)
            if (b->dconv_state_in) b->dconv_state_in[(s * cdim + c) * KW + j] = draw[j * cdim + c];
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < cdim; ++c) {
            const int64_t tt = t0 + t;
            const double v = draw[(KW + t) * cdim + c];
            if (c < Dn) b->dx[tt * Dn + c] = v;
            else if (c < Dn + G * N) b->dB[tt * G * N + (c - Dn)] += m1 ? 0.0 : v;
            else b->dC[tt * G * N + (c - Dn - G * N)] += m1 ? 0.0 : v;
        }
    free(draw); free(raw); free(pre); free(u); free(dl); free(hs); free(du); free(g);
}

int oracle_scan_bwd(const oracle_scan_bwd_args *b) {
    if (!b || !b->dy || !b->dx || !b->ddt || !b->dA || !b->dB || !b->dC || !b->dh0) return -1;
    const oracle_scan_args *a = &b->fwd;
    if (!a->seq_start || !a->x || !a->dt || !a->A || !a->B || !a->C) return -1;
    if (a->mode != ORACLE_M1 && a->mode != ORACLE_M2) return -1;
    if (a->mode == ORACLE_M2 && (a->nheads * a->headdim != a->d_inner || a->ngroups <= 0 ||
                                 a->nheads % a->ngroups != 0)) return -1;
    if (a->d_conv > 0 && !a->conv_w) return -1;
    if (a->z && !b->dz) return -1;
    /* accumulated outputs start at zero; sequences run one after another (shared dA, dB, ...) */
    for (int64_t s = 0; s < a->nseqs; ++s) bwd_one_sequence(b, s);
    return 0;
}

/* ---- standalone causal depthwise conv ---- */
int oracle_conv1d_fwd(const oracle_conv_args *a) {
    if (!a || !a->seq_start || !a->x || !a->w || !a->out || a->width < 1) return -1;
    const int64_t Cn = a->channels, K = a->width;
    for (int64_t s = 0; s < a->nseqs; ++s) {
        double *hist = (K > 1) ? (double *)calloc((size_t)(Cn * (K - 1)), sizeof(double)) : NULL;
        if (K > 1 && a->state_in)
            for (int64_t i = 0; i < Cn * (K - 1); ++i) hist[i] = a->state_in[s * Cn * (K - 1) + i];
        for (int64_t t = a->seq_start[s]; t < a->seq_start[s + 1]; ++t) {
            for (int64_t c = 0; c < Cn; ++c) {
                const double raw = a->x[t * Cn + c];
                double v = o_conv_tap(a->w + c * K, a->b ? a->b[c] : 0.0, hist ? hist + c * (K - 1) : NULL, raw, K);
                a->out[t * Cn + c] = a->activation ? o_silu(v) : v;
                if (hist) o_hist_push(hist + c * (K - 1), raw, K);
            }
        }
        if (K > 1 && a->state_out)
            for (int64_t i = 0; i < Cn * (K - 1); ++i) a->state_out[s * Cn * (K - 1) + i] = hist[i];
        free(hist);
    }
    return 0;
}

/* ---- single-token decode update, state and conv state in place ----
 * The conv state holds the last conv_state_len raw inputs (oldest first).  It
 * is rolled left by one and the new input appended; the conv then reads its
 * last K entries.  With conv_state_len = K-1 this is the llama.cpp layout;
 * with conv_state_len = K it is the rolling window of the decode kernels
 * ("causal_conv1d_update" / "selective_state_update" in the Megatron ops
 * directory clean-up, PR 6444). */
int oracle_state_update(const oracle_update_args *a) {
    if (!a || !a->state || !a->x || !a->dt || !a->A || !a->B || !a->C || !a->y) return -1;
    const int64_t N = a->dstate, K = a->d_conv, Ls = a->conv_state_len;
    const int64_t Dn = a->d_inner;
    const int is_m1 = (a->mode == ORACLE_M1);
    const int64_t H = is_m1 ? Dn : a->nheads;
    const int64_t P = is_m1 ? 1 : a->headdim;
    const int64_t G = is_m1 ? 1 : a->ngroups;
    const int64_t cdim = is_m1 ? Dn : Dn + 2 * G * N;
    if (K > 0 && (Ls < K - 1 || !a->conv_state || !a->conv_w)) return -1;
    double *u = (double *)malloc((size_t)cdim * sizeof(double));
    for (int64_t r = 0; r < a->batch; ++r) {
        for (int64_t c = 0; c < cdim; ++c) {
            double raw;
            if (c < Dn) raw = a->x[r * Dn + c];
            else if (c < Dn + G * N) raw = a->B[r * G * N + (c - Dn)];
            else raw = a->C[r * G * N + (c - Dn - G * N)];
            if (K > 0) {
                double *cs = a->conv_state + (r * cdim + c) * Ls;
                /* window = last K-1 stored inputs + the new input */
#if SSM_ORACLE_MUTANT == 16
                /* mutant: with a width-K state the window is read one position too old */
                double pre = o_conv_tap(a->conv_w + c * K, a->conv_b ? a->conv_b[c] : 0.0,
                                        cs + (Ls >= K ? Ls - K : Ls - (K - 1)), raw, K);
#else
                double pre = o_conv_tap(a->conv_w + c * K, a->conv_b ? a->conv_b[c] : 0.0,
                                        cs + (Ls - (K - 1)), raw, K);
#endif
#if SSM_ORACLE_MUTANT == 15
                /* mutant: the state rolled the wrong way (new input stored at the oldest end) */
                for (int64_t k = Ls - 1; k > 0; --k) cs[k] = cs[k - 1];
                if (Ls > 0) cs[0] = raw;
#else
                for (int64_t k = 0; k + 1 < Ls; ++k) cs[k] = cs[k + 1];
                if (Ls > 0) cs[Ls - 1] = raw;
#endif
                u[c] = o_silu(pre);
            } else {
                u[c] = raw;
            }
        }
        const double *Bt = is_m1 ? a->B + r * N : u + Dn;
        const double *Ct = is_m1 ? a->C + r * N : u + Dn + G * N;
        for (int64_t hh = 0; hh < H; ++hh) {
            const int64_t g = is_m1 ? 0 : hh / (H / G);
            const double dtv = is_m1 ? a->dt[r * Dn + hh] : a->dt[r * H + hh];
            const double delta = o_delta(dtv, a->dt_bias ? a->dt_bias[hh] : 0.0, a->delta_softplus);
            for (int64_t p = 0; p < P; ++p) {
                const int64_t ch = hh * P + p;
                const double xv = u[ch];
                double *hs = a->state + (r * Dn + ch) * N;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double An = is_m1 ? a->A[hh * N + n] : a->A[hh];
                    hs[n] = exp(delta * An) * hs[n] + delta * Bt[g * N + n] * xv;
                    acc += Ct[g * N + n] * hs[n];
                }
                double yv = acc;
                if (a->D) yv += a->D[is_m1 ? ch : hh] * xv;
                if (a->z) yv *= o_silu(a->z[r * Dn + ch]);
                a->y[r * Dn + ch] = yv;
            }
        }
    }
    free(u);
    return 0;
}

int oracle_mutant_id(void) { return SSM_ORACLE_MUTANT; }
