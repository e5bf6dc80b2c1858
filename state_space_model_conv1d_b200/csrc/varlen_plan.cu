// varlen_plan.cu -- device pre-pass for packed variable-length batches.
//
// Checks cu_seqlens on the device (0-based, non-decreasing, ending at the
// packed token count) and writes the outcome into the workspace error word,
// then writes a schedule that lists sequences longest first, so the scan
// kernels start the long chains first and short ones fill in behind them.
// No host synchronisation: the scan kernels read the error word and return
// at once when it is set.
#include "common.cuh"
#include "launch.h"

namespace ssm {
namespace {

constexpr int kThreads = 1024;
constexpr int kMaxSortedSeqs = 16384;   // above this the schedule is the identity

__global__ void __launch_bounds__(kThreads)
varlen_plan_kernel(const int32_t *__restrict__ cu, int nseqs, int64_t total, int32_t *err, int32_t *order) {
    int bad = 0;
    for (int i = threadIdx.x; i < nseqs; i += kThreads)
        if (cu[i + 1] < cu[i]) bad = 1;
    if (threadIdx.x == 0 && (cu[0] != 0 || (int64_t)cu[nseqs] != total)) bad = 1;
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) *err = bad ? SSM_DEVERR_CU_SEQLENS : SSM_DEVERR_NONE;
    if (bad) return;
    if (nseqs > kMaxSortedSeqs) {
        for (int i = threadIdx.x; i < nseqs; i += kThreads) order[i] = i;
        return;
    }
    // rank = number of sequences that go before i: longer ones, then equal
    // length with a smaller index (a stable descending order)
    for (int i = threadIdx.x; i < nseqs; i += kThreads) {
        const int li = cu[i + 1] - cu[i];
        int rank = 0;
        for (int j = 0; j < nseqs; ++j) {
            const int lj = cu[j + 1] - cu[j];
            rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
    }
}

}  // namespace

cudaError_t launch_varlen_plan(const int32_t *cu, int nseqs, int64_t total, int32_t *err, int32_t *order,
                               cudaStream_t st) {
    varlen_plan_kernel<<<1, kThreads, 0, st>>>(cu, nseqs, total, err, order);
    return cudaGetLastError();
}

}  // namespace ssm
