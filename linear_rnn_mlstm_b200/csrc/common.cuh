// Device helpers shared by the mLSTM kernels: element loads, gate activations,
// warp reductions, and the forward's launch plan.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/xlstm_mlstm.h"

namespace xlstm {

// ---------------------------------------------------------------- elements
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// ------------------------------------------------------------------- gates
// log sigmoid(x) without overflow in either tail (CUDA's expf / log1pf).
__device__ __forceinline__ float log_sigmoid(float x) {
    return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}
__device__ __forceinline__ float sigmoid(float x) {
    if (x >= 0.f) return 1.f / (1.f + expf(-x));
    const float e = expf(x);
    return e / (1.f + e);
}
// log f_t from the forget pre-activation: log sigmoid, or identity for the
// exponential forget gate ("xLSTM" section 2.2 allows either activation).
__device__ __forceinline__ float log_forget(float f_pre, int fgate_exp) {
    return fgate_exp ? f_pre : log_sigmoid(f_pre);
}

// ---------------------------------------------------------- warp reductions
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// ------------------------------------------------ programmatic dependent launch
// The forward's kernels after the first are launched with the programmatic
// stream-serialisation attribute, so each may be scheduled while its
// predecessor on the stream drains.  pdl_wait() returns once the predecessor
// grid has completed and its writes are visible; every thread calls it before
// touching memory the predecessor writes (or reads).  pdl_launch_dependents(),
// issued near the end of a kernel, lets the next kernel be scheduled while this
// one drains (issued at the start instead, the waiting CTAs of the next kernel
// were measured to slow the forward down).  Both are no-ops for a kernel
// launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Bits of the device status word (see xlstm_device_status); kernels that can
// give up a bounded wait get its address as an argument.
constexpr unsigned int kStatusTimeout = 1u;

}  // namespace xlstm
