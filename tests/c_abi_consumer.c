/* A plain C consumer of libssm.so, built against include/ssm.h alone (no
 * Python, no PyTorch).  It exercises the host side of the contract that
 * holds without a GPU: the version and status strings, the workspace sizes
 * (shapes only), and the rejection of bad arguments before any launch.
 * Device pointers are fake, aligned addresses that no call dereferences.
 * Prints "ok" and exits 0 when every check holds; otherwise names the first
 * failed check and exits 1. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ssm.h"

#define FAKE ((void *)(uintptr_t)0x10000000u)
#define CHECK(cond)                                             \
    do {                                                        \
        if (!(cond)) {                                          \
            printf("failed: %s (line %d)\n", #cond, __LINE__);  \
            return 1;                                           \
        }                                                       \
    } while (0)

/* A Mamba-2 scan over 2 rows of 16 tokens, 4 heads of 2 channels, 2 groups
 * of dstate 16, bf16 activations, contiguous token-major layouts. */
static ssm_scan_args mamba2_args(void) {
    ssm_scan_args a;
    memset(&a, 0, sizeof(a));
    a.mode = SSM_MAMBA2;
    a.dtype = SSM_BF16;
    a.delta_softplus = 1;
    a.batch = 2;
    a.seqlen = 16;
    a.d_inner = 8;
    a.nheads = 4;
    a.headdim = 2;
    a.ngroups = 2;
    a.dstate = 16;
    a.x = FAKE; a.x_token_stride = 8; a.x_batch_stride = 128;
    a.y = FAKE; a.y_token_stride = 8; a.y_batch_stride = 128;
    a.dt = FAKE; a.dt_token_stride = 4; a.dt_batch_stride = 64;
    a.B = FAKE; a.B_token_stride = 32; a.B_batch_stride = 512;
    a.C = FAKE; a.C_token_stride = 32; a.C_batch_stride = 512;
    a.A = (const float *)FAKE;
    return a;
}

int main(void) {
    CHECK(ssm_abi_version() == SSM_ABI_VERSION);
    CHECK(strcmp(ssm_status_string(SSM_OK), "ok") == 0);
    CHECK(strcmp(ssm_status_string((ssm_status)-99), "unknown status") == 0);

    /* workspace sizes depend on shapes only */
    ssm_scan_args a = mamba2_args();
    CHECK(ssm_scan_workspace_size(&a) == 0);              /* off the tensor-core path, no varlen */
    a.nheads = 4; a.headdim = 64; a.d_inner = 256; a.dstate = 128; a.d_conv = 4; a.conv_w = (const float *)FAKE;
    CHECK(ssm_scan_workspace_size(&a) == 256 + 2 * (2 * 16 * 2 * 128 * 2));   /* error word + conv'd B, C */

    /* rejected before any launch */
    a = mamba2_args();
    a.nheads = 3;                                          /* nheads * headdim != d_inner */
    CHECK(ssm_scan_fwd(&a, NULL, 0, NULL) == SSM_ERR_INVALID_ARG);
    a = mamba2_args();
    a.x = (const void *)((uintptr_t)FAKE + 1);             /* bf16 needs 2-byte alignment */
    CHECK(ssm_scan_fwd(&a, NULL, 0, NULL) == SSM_ERR_ALIGNMENT);
    a = mamba2_args();
    a.cu_seqlens = (const int32_t *)FAKE; a.nseqs = 2; a.batch = 1;   /* varlen needs a workspace */
    CHECK(ssm_scan_fwd(&a, NULL, 0, NULL) == SSM_ERR_WORKSPACE);
    CHECK(ssm_scan_fwd(NULL, NULL, 0, NULL) == SSM_ERR_INVALID_ARG);
    CHECK(ssm_conv1d_fwd(NULL, NULL) == SSM_ERR_INVALID_ARG);
    CHECK(ssm_state_update(NULL, NULL) == SSM_ERR_INVALID_ARG);

    /* sequence split: batch mode only, and the combine checks its rank */
    a = mamba2_args();
    a.d_conv = 4; a.conv_w = (const float *)FAKE;
    CHECK(ssm_split_conv_tail(&a, NULL, NULL) == SSM_ERR_INVALID_ARG);
    a.cu_seqlens = (const int32_t *)FAKE; a.nseqs = 2; a.batch = 1;
    CHECK(ssm_split_cum_delta(&a, NULL, (float *)FAKE, NULL) == SSM_ERR_UNSUPPORTED);
    ssm_split_args s;
    memset(&s, 0, sizeof(s));
    s.mode = SSM_MAMBA2; s.rank = 2; s.nranks = 2;
    s.batch = 2; s.d_inner = 8; s.nheads = 4; s.headdim = 2; s.dstate = 16;
    s.A = (const float *)FAKE; s.sum_delta = (const float *)FAKE; s.h_local = (const float *)FAKE;
    CHECK(ssm_split_combine(&s, NULL) == SSM_ERR_INVALID_ARG);

    printf("ok\n");
    return 0;
}
