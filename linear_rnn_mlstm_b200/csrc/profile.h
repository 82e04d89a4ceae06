// Per-kernel CUDA-event timing behind xlstm_profile_begin / xlstm_profile_end.
#pragma once

#include <cuda_runtime.h>

namespace xlstm {

bool profiling_enabled();
// Records a start event on `st` (when profiling is on) and, on destruction,
// the matching stop event.  Wrap each kernel launch in one.
class KernelTimer {
  public:
    KernelTimer(const char *name, cudaStream_t st);
    ~KernelTimer();
    KernelTimer(const KernelTimer &) = delete;
    KernelTimer &operator=(const KernelTimer &) = delete;

  private:
    const char *name_;
    cudaStream_t st_;
    cudaEvent_t start_ = nullptr;
};

// Marks one C-ABI call as a named range on the host timeline (NVTX), so a
// profiler's timeline shows which library call issued which kernels.  Without
// a profiler attached the NVTX calls do nothing.
class CallRange {
  public:
    explicit CallRange(const char *name);
    ~CallRange();
    CallRange(const CallRange &) = delete;
    CallRange &operator=(const CallRange &) = delete;
};

}  // namespace xlstm
