// Self-test of the bounded-wait failure path: a barrier nothing completes.
#include "../../include/xlstm_mlstm.h"
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace {

__global__ void wait_timeout_kernel(unsigned int *status, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        xlstm::tc::mbar_init(&bar, 1);
        abort_flag = 0;
        xlstm::tc::fence_mbar_init();
    }
    __syncthreads();
    // nothing arrives on `bar`: the wait runs out, latches `status` and returns false
    const bool done = xlstm::tc::mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    if (done && threadIdx.x == 0) atomicOr(status, 2u);    // never expected
}

}  // namespace

extern "C" xlstm_status xlstm_selftest_wait_timeout(int limit_us, void *cuda_stream) {
    if (limit_us < 1 || limit_us > 1000000) return XLSTM_ERR_SHAPE;
    unsigned int *status = xlstm::device_status_ptr();
    if (!status) return XLSTM_ERR_CUDA;
    wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)cuda_stream>>>(status, 1000ull * (unsigned long long)limit_us);
    return cudaGetLastError() == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}
