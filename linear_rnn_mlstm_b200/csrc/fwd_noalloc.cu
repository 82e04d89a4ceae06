// xlstm_mlstm_fwd_noalloc: the chunkwise forward with its scratch memory built
// into the library, for callers that cannot allocate device memory.
//
// Who needs it: a caller that reaches this library only through its C ABI and
// owns no device allocator of its own (for example a plugin running inside a
// host runtime that owns all device memory), or one that must not call
// cudaMalloc from its serving loop, where an allocation can synchronise the
// device, fail under memory pressure, or stall the loop for an unbounded time.
// Such a caller still passes its inputs and outputs, but not a workspace.
//
// The scratch is one file-scope device array of a fixed size.  Every GPU that
// loads this library holds it until the process exits.  Host code cannot use
// the array's name as a device address (in host code it names a host-side
// stand-in), so every call fetches the device address with
// cudaGetSymbolAddress, with the call's device current.  The address is not
// cached: after a cudaDeviceReset, or under another context, the module is
// loaded afresh and an address kept from before would be stale.
#include "../../include/xlstm_mlstm.h"
#include <cuda_runtime.h>

namespace {

static __device__ __align__(256) unsigned char g_fwd_noalloc_scratch[XLSTM_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device.
xlstm_status scratch_for_current_device(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_noalloc_scratch) != cudaSuccess || !p) return XLSTM_ERR_CUDA;
    *out = p;
    return XLSTM_OK;
}

}  // namespace

extern "C" xlstm_status xlstm_mlstm_fwd_noalloc(
    const void *q, const void *k, const void *v,
    const float *i_pre, const float *f_pre, const float *o_pre, void *h,
    const float *C0, const float *n0, const float *m0,
    float *C_out, float *n_out, float *m_out,
    int B, int NH, int S, int DH, int chunk, xlstm_dtype dt, xlstm_fgate fg,
    void *cuda_stream) {
    size_t need = 0;
    xlstm_status st = xlstm_mlstm_fwd_workspace_size(B, NH, S, DH, chunk, dt, &need);
    if (st != XLSTM_OK) return st;
    if (need > (size_t)XLSTM_NOALLOC_SCRATCH_BYTES) return XLSTM_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0) {
        st = scratch_for_current_device(&scratch);
        if (st != XLSTM_OK) return st;
    }
    // The forward overwrites every scratch word it later reads (prefix sums,
    // chunk and segment statistics, segment summaries), so what an earlier call
    // left in the array does not matter and nothing needs clearing.
    return xlstm_mlstm_fwd(q, k, v, i_pre, f_pre, o_pre, h, C0, n0, m0, C_out, n_out, m_out,
                           B, NH, S, DH, chunk, dt, fg, scratch, (size_t)XLSTM_NOALLOC_SCRATCH_BYTES,
                           cuda_stream);
}
