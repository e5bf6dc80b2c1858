/*
 * ssm.h -- C ABI of libssm.so: the Mamba short causal conv1d + SiLU and the
 * selective state-space scan on one B200 (sm_100a).
 *
 * Operations (what each computes, and the passage that defines it):
 *
 *   ssm_conv1d_fwd   Causal depthwise conv of width K over token-major input,
 *                    optional bias and SiLU, with a carried state of the last
 *                    K-1 raw inputs per sequence (in and out).
 *                    "ggml : add GPU support for Mamba models" (llama.cpp issue
 *                    6758): GGML_OP_SSM_CONV, test-backend-ops shapes
 *                    s [d_conv-1, d_inner, n_seqs], x [d_inner, n_tokens,
 *                    n_seqs], c [d_conv, d_inner]; the reply on concatenating
 *                    the state in front of the tokens.
 *
 *   ssm_scan_fwd     delta = softplus(dt + dt_bias);
 *                    h_t = exp(delta_t*A) h_{t-1} + delta_t B_t x_t;
 *                    y_t = C_t . h_t + D x_t, then y_t *= silu(z_t);
 *                    h_0 = h0 (zeros when absent), h_T returned in h_final.
 *                    Optionally the conv above runs in front (x for Mamba-1,
 *                    x|B|C for Mamba-2) inside the same kernel.
 *                    "Adding Initial Value Support to Selective Scan Forward
 *                    Kernel" (state-spaces/mamba issue 285): the step
 *                    h_t = A h_{t-1} + Bx, the scan element (exp(delta*A), h)
 *                    and its seed (1, h0); llama.cpp issue 6758: the scan op
 *                    returns the final state instead of overwriting an input;
 *                    "Tensor-parallel SSM" (Fast-LLM PR 333): Mamba-2 heads in
 *                    contiguous groups sharing B and C (repeat_interleave).
 *
 *   ssm_state_update One decode token per batch row: the conv state window is
 *                    rolled left by one and the new input appended, the conv +
 *                    SiLU read its last K entries, then one step of the
 *                    recurrence above updates the fp32 state in place.
 *                    "Clean up SSM ops directory structure" (Megatron-LM PR
 *                    6444): causal_conv1d_update and selective_state_update,
 *                    and slot-indexed state rows (intermediate_extraction).
 *
 * Conventions for every entry point:
 *   - Pointers are device pointers unless stated otherwise; the caller owns
 *     every buffer.  The library never allocates or frees memory, and only
 *     ssm_workspace_error synchronizes (it reads a device word back).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream).  A return of SSM_OK means the launch was enqueued.
 *   - Arguments are validated on the host before anything is launched; a
 *     rejected call launches nothing and returns a negative ssm_status.
 *     CUDA launch failures return SSM_ERR_CUDA; ssm_last_cuda_error() gives
 *     the underlying cudaError_t.
 *   - Tensors are token-major with the channel dimension contiguous (stride 1).
 *     Batch and token strides are in ELEMENTS, so x / z / B / C may be views
 *     into a wider projection output (e.g. x and z halves of one in_proj
 *     row).  Every pointer must be aligned to its element size, and the
 *     decode state to 16 bytes when dstate % 4 == 0 (else SSM_ERR_ALIGNMENT).
 *     16-byte aligned bases and strides whose byte size is a multiple of 16
 *     let the kernels use 16-byte vector loads; other layouts take a slower
 *     element-wise path with the same results.
 *   - Activations (x, z, dt, B, C, y, conv states) share one dtype, SSM_F32 or
 *     SSM_BF16.  Parameters (A, D, dt_bias, conv weight / bias) and the
 *     recurrent state (h0, h_final, decode state) are always fp32.  All
 *     arithmetic is fp32; y is rounded once to its dtype (nearest-even).
 *   - Optional pointers may be NULL: dt_bias (= 0), D (= 0), z (no gate),
 *     h0 (= 0), h_final (not written), conv_b (= 0), conv_state_in (= 0),
 *     conv_state_out (not written).
 *   - Outputs must not overlap inputs, except conv_state_out == conv_state_in
 *     (same layout), which is allowed: the state is read before it is
 *     written.
 */
#ifndef SSM_H_
#define SSM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSM_ABI_VERSION 3

#if defined(__GNUC__)
#define SSM_API __attribute__((visibility("default")))
#else
#define SSM_API
#endif

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = -1,   /* bad size, NULL required pointer, bad combination */
    SSM_ERR_UNSUPPORTED = -2,   /* valid but outside what the kernels implement (e.g. dstate too large) */
    SSM_ERR_ALIGNMENT = -3,     /* pointer not aligned to its element size (decode state: 16 bytes) */
    SSM_ERR_WORKSPACE = -4,     /* workspace missing or smaller than ssm_scan_workspace_size() */
    SSM_ERR_CUDA = -5,          /* a CUDA call failed; see ssm_last_cuda_error() */
    SSM_ERR_DEVICE = -6         /* the device rejected data it validated (e.g. cu_seqlens) */
} ssm_status;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;
typedef enum { SSM_MAMBA1 = 1, SSM_MAMBA2 = 2 } ssm_mode;

/* Device-side error codes written into the workspace error word. */
#define SSM_DEVERR_NONE 0
#define SSM_DEVERR_CU_SEQLENS 1   /* cu_seqlens not 0-based, decreasing, or not ending at seqlen */
#define SSM_DEVERR_TIMEOUT 2      /* a bounded wait for tensor-core completion ran out; outputs incomplete */
#define SSM_DEVERR_BOUNDS 3       /* bounds-checked build only: an index fell outside its tensor (see ssm_bounds_record) */

/* ------------------------------------------------------------------ conv */
typedef struct ssm_conv_args {
    int64_t batch;            /* rows; 1 when cu_seqlens is given */
    int64_t seqlen;           /* tokens per row (total packed tokens when varlen) */
    int64_t channels;         /* C */
    int64_t width;            /* K, 1..8 */
    int32_t dtype;            /* ssm_dtype of x, out, conv states */
    int32_t activation;       /* 0: none, 1: SiLU */
    int32_t nseqs;            /* number of sequences in cu_seqlens (varlen only) */
    int32_t reserved0;
    const void *x;            /* [batch][seqlen][channels], strides below */
    int64_t x_batch_stride, x_token_stride;
    const float *weight;      /* [channels][width]; weight[c][width-1] multiplies the current token */
    const float *bias;        /* [channels] or NULL */
    const void *state_in;     /* [batch or nseqs][channels][width-1], oldest first, or NULL */
    void *state_out;          /* same layout, or NULL */
    const int32_t *cu_seqlens;/* [nseqs+1] device int32 offsets (0 .. seqlen), or NULL */
    void *out;                /* [batch][seqlen][channels] */
    int64_t out_batch_stride, out_token_stride;
} ssm_conv_args;

/* ------------------------------------------------------------------ scan */
typedef struct ssm_scan_args {
    int32_t mode;             /* SSM_MAMBA1 or SSM_MAMBA2 */
    int32_t dtype;            /* ssm_dtype of x, z, dt, B, C, y, conv states */
    int32_t delta_softplus;   /* 1: delta = softplus(dt + dt_bias); 0: delta = dt + dt_bias */
    int32_t nseqs;            /* number of sequences when cu_seqlens != NULL */
    int64_t batch;            /* 1 when cu_seqlens != NULL */
    int64_t seqlen;           /* tokens per row, or total packed tokens */
    int64_t d_inner;          /* Mamba-1: channels D; Mamba-2: nheads*headdim */
    int64_t nheads, headdim;  /* Mamba-2 only (ignored for Mamba-1) */
    int64_t ngroups;          /* Mamba-2: groups of B/C (nheads % ngroups == 0); Mamba-1: 1 */
    int64_t dstate;           /* N */
    int64_t d_conv;           /* K of the fused conv (0 = no conv; x, B, C used as given) */
    /* activations (dtype): Mamba-1 x,z,dt,y [b][T][D]; B,C [b][T][N].
     *                      Mamba-2 x,z,y [b][T][H*P]; dt [b][T][H]; B,C [b][T][G*N]. */
    const void *x;  int64_t x_batch_stride, x_token_stride;
    const void *z;  int64_t z_batch_stride, z_token_stride;
    const void *dt; int64_t dt_batch_stride, dt_token_stride;
    const void *B;  int64_t B_batch_stride, B_token_stride;
    const void *C;  int64_t C_batch_stride, C_token_stride;
    void *y;        int64_t y_batch_stride, y_token_stride;
    /* fp32 parameters: Mamba-1 A [D][N], D, dt_bias [D]; Mamba-2 A, D, dt_bias [H] */
    const float *A, *D, *dt_bias;
    /* fp32 states, contiguous: Mamba-1 [nseq][D][N]; Mamba-2 [nseq][H][P][N] */
    const float *h0;
    float *h_final;
    const int32_t *cu_seqlens;/* [nseqs+1] device int32, or NULL */
    /* fused conv: weight [conv_dim][K] fp32, bias [conv_dim]; states
     * [nseq][conv_dim][K-1] in dtype.  conv_dim = D (Mamba-1, x only) or
     * H*P + 2*G*N (Mamba-2, channels ordered x | B | C). */
    const float *conv_w, *conv_b;
    const void *conv_state_in;
    void *conv_state_out;
    int64_t chunk;            /* Mamba-2 chunk length hint (0 = kernel default); results do not depend on it */
    /* Intermediate states for prefix caching (optional): the conditional
     * scatter of flat state rows into slots that "Clean up SSM ops directory
     * structure" (Megatron-LM PR 6444) names intermediate_extraction
     * (scatter_intermediate_ssm / scatter_intermediate_conv).  With
     * state_interval > 0, after every state_interval tokens of a sequence
     * (boundary k at token (k+1)*state_interval from the sequence's start,
     * k < inter_stride) the fp32 state and the conv history (the last K-1 raw
     * conv inputs) are written to row inter_slots[s*inter_stride + k] of the
     * pools when that index lies in [0, inter_nslots); any other index writes
     * nothing, and pool rows nobody names keep their contents.
     * state_interval must be a positive multiple of 64 (0 disables). */
    int64_t state_interval;
    const int32_t *inter_slots;   /* device int32 [nseqs][inter_stride] */
    int64_t inter_stride;         /* slot entries per sequence (>= 0) */
    int64_t inter_nslots;         /* pool rows (>= 0) */
    float *inter_states;          /* [inter_nslots][state size] fp32, rows laid out as h_final's; may be NULL */
    void *inter_conv;             /* [inter_nslots][conv_dim][K-1] in dtype; may be NULL */
    /* Token segments of the Mamba-2 tensor-core path (ignored elsewhere): 0
     * lets the library choose, 1 keeps one CTA per (sequence, head), n >= 2
     * cuts every row into about n runs of whole 64-token chunks that separate
     * CTAs scan at the same time.  Packed sequences (cu_seqlens) are cut into
     * runs of one length for all of them, chosen from the total: about n runs
     * for a sequence of the mean length; the library cuts them only when the
     * sequences x heads leave the GPU short of CTAs, with the run length it
     * would choose for nseqs rows of the mean length.  Each run's
     * entering state comes from a state-only pass over the runs before it (the
     * pair (exp(delta A), h) composes associatively, seed (1, h0): "Adding
     * Initial Value Support to Selective Scan Forward Kernel"), so results
     * agree with the unsegmented scan up to fp32 rounding.  The workspace size
     * depends on it. */
    int64_t segments;
} ssm_scan_args;

/* ---------------------------------------------------------------- decode */
typedef struct ssm_update_args {
    int32_t mode, dtype, delta_softplus, reserved0;
    int64_t batch;            /* rows, one new token each */
    int64_t d_inner, nheads, headdim, ngroups, dstate;   /* as in ssm_scan_args */
    int64_t d_conv;           /* K (0 = no conv) */
    int64_t conv_state_len;   /* columns kept per channel, >= K-1 (K-1 or K typical) */
    float *state;             /* in-out fp32, per slot: Mamba-1 [D][N]; Mamba-2 [H][P][N]; slots contiguous */
    void *conv_state;         /* in-out dtype, per slot [conv_dim][conv_state_len], oldest first */
    const float *conv_w, *conv_b;
    const void *x;  int64_t x_batch_stride;   /* Mamba-1 [b][D]; Mamba-2 [b][H*P] */
    const void *z;  int64_t z_batch_stride;
    const void *dt; int64_t dt_batch_stride;  /* Mamba-1 [b][D]; Mamba-2 [b][H] */
    const void *B;  int64_t B_batch_stride;   /* Mamba-1 [b][N]; Mamba-2 [b][G*N] */
    const void *C;  int64_t C_batch_stride;
    void *y;        int64_t y_batch_stride;
    const float *A, *D, *dt_bias;
    const int32_t *state_batch_indices;  /* [batch]: slot of row r (NULL = r); a negative
                                            slot marks a padding row: nothing is read or
                                            written for it except y, which is set to 0 */
    int64_t nslots;           /* number of state / conv-state slots (>= batch when indices are NULL) */
} ssm_update_args;

/* Backward of ssm_scan_fwd: gradients of
 *   L = sum(dy * y) + sum(dh_final * h_final) + sum(dconv_state_out * conv_state_out)
 * with respect to every input of the forward call described by `fwd` (its
 * y, h_final, conv_state_out and intermediate-state fields are ignored).
 * The step h_t = exp(delta_t A) h_{t-1} + delta_t B_t x_t is differentiated
 * as it stands, carrying dh back through exp(delta A) to the initial state
 * ("Adding Initial Value Support to Selective Scan Forward Kernel",
 * state-spaces/mamba issue 285, on the backward pass and dh0).
 *
 * Every gradient is fp32 and contiguous:
 *   dx, dz [b][T][d_inner]; ddt [b][T][D or H]; dB, dC [b][T][G*N] (the raw,
 *   pre-conv B / C); dA, dD, ddt_bias like A, D, dt_bias; dh0 [nseq][state];
 *   dconv_w [conv_dim][K], dconv_b [conv_dim]; dconv_state_in [nseq][conv_dim][K-1].
 * dx, dB, dC, ddt, dA, dh0 are required; dz is required when z is given; the
 * others may be NULL when not wanted (dD needs D, ddt_bias needs dt_bias,
 * dconv_* need the conv).  Every requested output is overwritten. */
typedef struct ssm_scan_bwd_args {
    ssm_scan_args fwd;
    const void *dy; int64_t dy_batch_stride, dy_token_stride;   /* like y (dtype) */
    const float *dh_final;          /* [nseq][state] or NULL */
    const void *dconv_state_out;    /* [nseq][conv_dim][K-1] dtype, or NULL */
    float *dx, *dz, *ddt, *dB, *dC;
    float *dA, *dD, *ddt_bias;
    float *dh0;
    float *dconv_w, *dconv_b;
    float *dconv_state_in;
} ssm_scan_bwd_args;

/* Library version and status text. */
SSM_API int32_t ssm_abi_version(void);
SSM_API const char *ssm_status_string(ssm_status s);
/* The cudaError_t of the last failing CUDA call made by this thread (0 if none). */
SSM_API int32_t ssm_last_cuda_error(void);

/* Standalone conv (bias, activation).  No workspace. */
SSM_API ssm_status ssm_conv1d_fwd(const ssm_conv_args *args, void *stream);

/* Bytes of device workspace ssm_scan_fwd needs for these arguments (0 when
 * none is needed; the packed varlen path needs one).  Launches nothing; it
 * reads the current device's SM count (148 when no device answers), which
 * the choice of token segments depends on. */
SSM_API size_t ssm_scan_workspace_size(const ssm_scan_args *args);
/* Token segments ssm_scan_fwd cuts every row into for these arguments: 1 when
 * rows stay whole (Mamba-1, the SIMT Mamba-2 path, rows of one chunk), 0 for
 * arguments ssm_scan_fwd would reject.  For packed sequences, which are cut on
 * the device, it is 1 or, when they are cut, the bound nseqs + ceil(total /
 * run length) on the runs of all sequences together (the CTA rows launched).
 * Launches nothing. */
SSM_API int64_t ssm_scan_segments(const ssm_scan_args *args);

/* Forward scan.  `workspace` (device, 256-byte aligned, ws_bytes long) may be
 * NULL when ssm_scan_workspace_size() is 0.  The workspace holds the device
 * error word (read it with ssm_workspace_error) and the varlen schedule. */
SSM_API ssm_status ssm_scan_fwd(const ssm_scan_args *args, void *workspace, size_t ws_bytes, void *stream);

/* Backward scan (see ssm_scan_bwd_args).  Needs a workspace of
 * ssm_scan_bwd_workspace_size() bytes (device, 256-byte aligned): chunk-start
 * state checkpoints of a recomputed forward pass and the fp32 accumulators of
 * the grouped B / C gradients.  Supports dstate <= 256. */
SSM_API size_t ssm_scan_bwd_workspace_size(const ssm_scan_bwd_args *args);
SSM_API ssm_status ssm_scan_bwd(const ssm_scan_bwd_args *args, void *workspace, size_t ws_bytes, void *stream);

/* Decode update, in place on state and conv_state.  No workspace. */
SSM_API ssm_status ssm_state_update(const ssm_update_args *args, void *stream);

/* Per-kernel device timing of the dominant kernel of each call (the scan
 * kernel of ssm_scan_fwd, the update kernel of ssm_state_update, the backward
 * kernel of ssm_scan_bwd, the fix-up kernel of ssm_split_fixup), for
 * roofline measurements.  The papers have no counterpart.  While enabled
 * (process-wide, off by default), every such launch is bracketed by a CUDA
 * event pair recorded on the call's own stream (events are created on first
 * use and reused).  ssm_kernel_time_ms synchronizes on the recorded events,
 * returns the summed elapsed time and the number of launches since the last
 * read, and starts a new tally.  Not for use inside stream capture. */
SSM_API ssm_status ssm_kernel_timing(int32_t enable);
SSM_API ssm_status ssm_kernel_time_ms(float *total_ms, int32_t *launches);

/* ssm_scan_fwd without a caller-supplied workspace, for callers that cannot
 * allocate device memory (code inside a CUDA-graph capture that must not
 * allocate, a runtime whose memory pool belongs to another component, a
 * plugin handed buffers but no allocator).  The paper has no counterpart:
 * this is an interface convenience of this library, not a step of the method.
 *
 * The workspace comes from a file-scope device array of
 * SSM_NOALLOC_SCRATCH_BYTES bytes (one per GPU that loads the library, held
 * until the process exits).  Calls whose ssm_scan_workspace_size() exceeds
 * that return SSM_ERR_WORKSPACE and launch nothing; use ssm_scan_fwd then.
 * Nothing here allocates or frees memory.  The first call on a device looks
 * up the array's device address (cudaGetSymbolAddress, with that device
 * current) and caches it: make that first call before any stream capture.
 * The cached address belongs to the device's primary context: it does not
 * survive cudaDeviceReset() (the module may come back at another address),
 * so a process that resets a device must not call this entry point on that
 * device again.  Every call shares the one array and the scan initialises
 * what it reads (the error word, the varlen schedule) on each call; calls
 * that may overlap on the GPU (different streams, or different host threads
 * on one device) race on it, so serialise them.  The error word can be read
 * back with ssm_workspace_error() only by code that knows the array's
 * address.  A malformed cu_seqlens leaves every output (y, h_final,
 * conv_state_out) unwritten, as in ssm_scan_fwd; a bounded wait that runs
 * out (SSM_DEVERR_TIMEOUT) can leave them partly written. */
/* With segments = 0, a call that would fit the scratch only with its rows
 * kept whole runs them whole. */
#define SSM_NOALLOC_SCRATCH_BYTES (4u << 20)
SSM_API ssm_status ssm_scan_fwd_noalloc(const ssm_scan_args *args, void *stream);

/* Bounds-checked build (libssm_checked.so, compiled with SSM_CHECK_BOUNDS).
 * The paper has no counterpart: this is a debugging aid of the library.  In
 * that build every kernel tests the element indices it derives (sequence
 * ranges from cu_seqlens, head / channel / group ranges, state and conv-state
 * rows, pool slots, store positions) against the extent the call's shapes
 * give the tensor.  A failing test does not trap: it records the first
 * failure of the process on that device (code SSM_DEVERR_BOUNDS, the check
 * site, the index and the extent) and the access is skipped (a CTA whose
 * ranges fail returns before touching memory), so the context stays usable.
 *
 * ssm_check_bounds_enabled: 1 in the checked build, 0 in libssm.so.
 * ssm_bounds_record: waits for the device, then reads the record into the
 * non-NULL pointers (code 0 when no check failed) and clears it when `clear`
 * is nonzero.  Returns SSM_ERR_UNSUPPORTED in the normal build. */
SSM_API int32_t ssm_check_bounds_enabled(void);
SSM_API ssm_status ssm_bounds_record(int32_t *code, int32_t *site, int64_t *index, int64_t *extent, int32_t clear);

/* Waits for `stream`, then reads the device error word of a workspace last
 * used by ssm_scan_fwd: SSM_OK, or SSM_ERR_DEVICE with *code set to an
 * SSM_DEVERR_* value.  `code` may be NULL. */
SSM_API ssm_status ssm_workspace_error(const void *workspace, int32_t *code, void *stream);

/* ------------------------------------------------------- sequence split */
/* One batch of sequences split along its tokens across R ranks: rank r holds
 * the contiguous segment r of every batch row (batch mode; no cu_seqlens).
 * The scan's element (exp(delta*A), h) composes associatively, with seed
 * (1, h0) ("Adding Initial Value Support to Selective Scan Forward Kernel",
 * state-spaces/mamba issue 285), so each rank scans its own segment from a
 * zero state and one exchange of per-segment pairs joins the segments.  Per
 * rank, in this order:
 *
 *   1. ssm_split_conv_tail: the segment's last K-1 raw conv inputs.  Rank r
 *      passes rank r-1's tail as conv_state_in of its scan (exchange 1).
 *   2. ssm_scan_fwd on the segment, with the caller's h0 on rank 0 and
 *      h0 = NULL elsewhere: y_loc and h_loc (its h_final).
 *   3. ssm_split_cum_delta: cs_t = sum of delta over the segment's tokens up
 *      to and including t, per batch row and delta unit (channel for
 *      Mamba-1, head for Mamba-2), and the segment total sum_delta; the
 *      segment multiplies an incoming state by exp(A * sum_delta).
 *   4. all ranks exchange (sum_delta, h_loc) (exchange 2, an all-gather).
 *   5. ssm_split_combine: H_0 = h_loc_0, H_k = exp(A sum_delta_k) H_{k-1}
 *      + h_loc_k; h_in = H_{r-1} (zero on rank 0) is the state entering the
 *      segment and h_out = H_r the state leaving it.
 *   6. ssm_split_fixup (ranks r > 0): y_t += silu(z_t) * C_t . (exp(A cs_t) h_in)
 *      for every token of the segment (C_t after the conv for Mamba-2).
 *
 * y and h_out then equal an unsplit scan of the whole sequence up to
 * rounding (y is rounded to its dtype twice on ranks r > 0), and the last
 * rank's h_out and conv_state_out are the sequence's final states.
 * Every segment must hold at least K-1 tokens so that a tail does not depend
 * on the segments before it. */
typedef struct ssm_split_args {
    int32_t mode;             /* SSM_MAMBA1 or SSM_MAMBA2 */
    int32_t rank, nranks;     /* 0 <= rank < nranks */
    int32_t reserved0;
    int64_t batch, d_inner, nheads, headdim, dstate;   /* as in ssm_scan_args */
    const float *A;           /* as in ssm_scan_args */
    const float *sum_delta;   /* [nranks][batch][U] fp32, every rank's step-3 output (U = D or H) */
    const float *h_local;     /* [nranks][batch][state] fp32, every rank's h_loc */
    float *h_in;              /* [batch][state] out, or NULL */
    float *h_out;             /* [batch][state] out, or NULL */
    /* Elements from one rank's sum_delta (h_local) to the next rank's; 0 for
     * the dense [nranks][batch][...] layout, else at least batch x U (batch x
     * state) and a multiple of 4, so the gathered (sum_delta, h_loc) pairs of
     * one buffer per rank can be read in place.  Added with ABI version 3. */
    int64_t sum_delta_rank_stride, h_local_rank_stride;
} ssm_split_args;

/* Step 1.  `tail` is [batch][conv_dim][K-1] in the activation dtype, oldest
 * first, in the layout of conv_state_out; positions before the segment's
 * first token come from conv_state_in (zeros when NULL).  Needs d_conv > 1.
 * On ranks r > 0 the tail is built before the previous rank's tail arrives,
 * so it is only right when the segment holds at least K-1 tokens: a caller
 * must not split a sequence into shorter segments (this call cannot see the
 * rank and does not check it). */
SSM_API ssm_status ssm_split_conv_tail(const ssm_scan_args *args, void *tail, void *stream);
/* Step 3.  cum_delta [batch][seqlen][U] fp32 (may be NULL), sum_delta
 * [batch][U] fp32.  delta as in ssm_scan_fwd (dt + dt_bias, then softplus
 * when delta_softplus). */
SSM_API ssm_status ssm_split_cum_delta(const ssm_scan_args *args, float *cum_delta, float *sum_delta,
                                       void *stream);
/* Step 5.  No workspace. */
SSM_API ssm_status ssm_split_combine(const ssm_split_args *args, void *stream);
/* Step 6.  `args` describes the segment's ssm_scan_fwd call; its y is
 * updated in place, its h0 / h_final / conv_state_out fields are ignored.
 * cum_delta is step 3's output, h_in step 5's.  A segment with no tokens
 * returns SSM_OK without touching anything (the pointers may be NULL).
 * Mamba-2 in bf16 with headdim 64, dstate 128 and 16-byte aligned C, y, z
 * rows runs the correction as a tensor-core product per head (h_in rounded
 * to bf16 as the operand, fp32 accumulation); its device waits are bounded,
 * and one that runs out (not expected) leaves that tile's y as NaN, since
 * this call has no workspace for an error word. */
SSM_API ssm_status ssm_split_fixup(const ssm_scan_args *args, const float *cum_delta, const float *h_in,
                                   void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SSM_H_ */
