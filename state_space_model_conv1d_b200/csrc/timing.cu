// timing.cu -- optional device timing of the dominant kernel of each call.
//
// While enabled, the launchers bracket their main kernel with an event pair
// on the launching stream; ssm_kernel_time_ms() waits for the recorded pairs
// and reports their summed duration.  Events are pooled and reused.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/ssm.h"
#include "launch.h"

namespace ssm {
namespace {

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<cudaEvent_t> g_free;                              // spare events
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_done;      // recorded pairs
cudaEvent_t g_open = nullptr;                                 // begin event awaiting its end

cudaEvent_t take_event() {
    if (!g_free.empty()) {
        cudaEvent_t e = g_free.back();
        g_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

void timing_begin(cudaStream_t st) {
    if (!g_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_mu);
    cudaEvent_t e = take_event();
    if (e && cudaEventRecord(e, st) == cudaSuccess) g_open = e;
}

void timing_end(cudaStream_t st) {
    if (!g_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_open) return;
    cudaEvent_t e = take_event();
    if (e && cudaEventRecord(e, st) == cudaSuccess) g_done.emplace_back(g_open, e);
    else if (e) g_free.push_back(e);
    g_open = nullptr;
}

}  // namespace ssm

extern "C" {

ssm_status ssm_kernel_timing(int32_t enable) {
    if (enable != 0 && enable != 1) return SSM_ERR_INVALID_ARG;
    ssm::g_on.store(enable != 0);
    return SSM_OK;
}

ssm_status ssm_kernel_time_ms(float *total_ms, int32_t *launches) {
    if (!total_ms || !launches) return SSM_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(ssm::g_mu);
    float sum = 0.f;
    int32_t n = 0;
    ssm_status st = SSM_OK;
    for (auto &pr : ssm::g_done) {
        float ms = 0.f;
        if (cudaEventSynchronize(pr.second) != cudaSuccess || cudaEventElapsedTime(&ms, pr.first, pr.second) != cudaSuccess)
            st = SSM_ERR_CUDA;
        else {
            sum += ms;
            ++n;
        }
        ssm::g_free.push_back(pr.first);
        ssm::g_free.push_back(pr.second);
    }
    ssm::g_done.clear();
    *total_ms = sum;
    *launches = n;
    return st;
}

}  // extern "C"
