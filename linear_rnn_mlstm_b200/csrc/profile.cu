// Per-kernel timing with CUDA events (see xlstm_profile_begin in the header).
#include <mutex>
#include <string.h>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/xlstm_mlstm.h"
#include "profile.h"

namespace xlstm {

CallRange::CallRange(const char *name) { nvtxRangePushA(name); }
CallRange::~CallRange() { nvtxRangePop(); }

namespace {
struct Record {
    const char *name;
    cudaEvent_t start, stop;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Record> g_records;
}  // namespace

bool profiling_enabled() {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_on;
}

KernelTimer::KernelTimer(const char *name, cudaStream_t st) : name_(name), st_(st) {
    if (!profiling_enabled()) return;
    if (cudaEventCreate(&start_) != cudaSuccess) { start_ = nullptr; return; }
    if (cudaEventRecord(start_, st_) != cudaSuccess) {
        cudaEventDestroy(start_);
        start_ = nullptr;
    }
}

KernelTimer::~KernelTimer() {
    if (!start_) return;
    cudaEvent_t stop = nullptr;
    if (cudaEventCreate(&stop) != cudaSuccess || cudaEventRecord(stop, st_) != cudaSuccess) {
        if (stop) cudaEventDestroy(stop);
        cudaEventDestroy(start_);
        return;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    g_records.push_back({name_, start_, stop});
}

}  // namespace xlstm

using namespace xlstm;

extern "C" {

xlstm_status xlstm_profile_begin(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto &r : g_records) { cudaEventDestroy(r.start); cudaEventDestroy(r.stop); }
    g_records.clear();
    g_on = true;
    return XLSTM_OK;
}

xlstm_status xlstm_profile_end(xlstm_kernel_time *out, int max, int *count) {
    std::vector<Record> recs;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        g_on = false;
        recs.swap(g_records);
    }
    std::vector<xlstm_kernel_time> agg;
    xlstm_status st = XLSTM_OK;
    for (auto &r : recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess ||
            cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
            st = XLSTM_ERR_CUDA;
        size_t i = 0;
        for (; i < agg.size(); ++i)
            if (strncmp(agg[i].name, r.name, sizeof(agg[i].name) - 1) == 0) break;
        if (i == agg.size()) {
            xlstm_kernel_time t;
            memset(&t, 0, sizeof(t));
            strncpy(t.name, r.name, sizeof(t.name) - 1);
            agg.push_back(t);
        }
        agg[i].launches += 1;
        agg[i].total_ms += ms;
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
    }
    if (count) *count = (int)agg.size();
    for (int i = 0; out && i < max && i < (int)agg.size(); ++i) out[i] = agg[i];
    return st;
}

}  // extern "C"
