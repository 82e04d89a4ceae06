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

}  // namespace xlstm
