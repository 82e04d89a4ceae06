// Internal launch interface between the C ABI (abi.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "plan.h"

namespace xlstm {

struct FwdArgs {
    const void *q, *k, *v;
    const float *i_pre, *f_pre, *o_pre;
    void *h;
    const float *C0, *n0, *m0;
    float *C_out, *n_out, *m_out;
    void *workspace;
    unsigned int *status;     // device status word of the current device
    int bf16;
    int fgate_exp;
};

// Address of the device status word on the current device (nullptr on failure).
unsigned int *device_status_ptr();

// SM count of the current device (148 when it cannot be queried).
int num_sms_current_device();

struct StepArgs {
    const void *q, *k, *v;
    const float *i_pre, *f_pre, *o_pre;
    void *h;
    float *C, *n, *m;
    int BH, DH;
    int bf16;
    int fgate_exp;
    unsigned int *status;     // device status word of the current device
};

// Launches `kern` with the programmatic stream-serialisation attribute: it may
// be scheduled while the previous kernel on `st` finishes, and waits for it in
// pdl_wait() (common.cuh).  Used for the forward's kernels after the first.
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                           Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Where the fold of seqpar.cu finds run g of head bh: its (C' | n') summary at
// C + g*cg + bh*cbh (DH*DH floats) and n + g*ng + bh*nbh (DH floats), and its
// total log forget and own stabiliser at F / m + g*sg + bh*sbh.  Every C/n
// offset is a multiple of 4 floats and the bases are 16-byte aligned.
struct FoldSource {
    const float *C, *n, *F, *m;
    size_t cg, cbh, ng, nbh, sg, sbh;
};
// Folds `count` runs into (C_out, n_out, m_out) from (C0, n0, m0) (NULL: zeros,
// and m = 0, or -inf when start_neg_inf); F_out (nullable) gets the summed log
// forget.  scanned != 0: the runs were already folded in place by the segment
// scan from the same start, so only the last one is read.
cudaError_t launch_state_fold(const FoldSource &src, int count, int scanned, const float *C0, const float *n0,
                              const float *m0, int start_neg_inf, float *C_out, float *n_out, float *m_out,
                              float *F_out, int BH, int D, cudaStream_t st);

cudaError_t launch_gate_prologue(const FwdArgs &a, const FwdPlan &p, cudaStream_t st);
// Segment summaries + segment scan of the two-level chunk-state scan, on the
// tensor cores (bf16, DH 64, 128 or 256); nothing when the plan has one segment.
cudaError_t launch_segment_summaries(const FwdArgs &a, const FwdPlan &p, cudaStream_t st);
// Segment summaries only (no scan), fp32 arithmetic, any DH and chunk: the raw
// per-segment (dC, dn) and (total log forget, stabiliser) of segments 0..P-2.
cudaError_t launch_segment_summaries_simt(const FwdArgs &a, const FwdPlan &p, cudaStream_t st);
cudaError_t launch_fwd_simt(const FwdArgs &a, const FwdPlan &p, cudaStream_t st);
cudaError_t launch_fwd_tensor(const FwdArgs &a, const FwdPlan &p, cudaStream_t st);
bool tensor_path_supports(int DH, int L);
// Register-state tensor-core forward (fwd_rs.cu): bf16, DH 64 / 128 / 256 / 512,
// chunk 64 / 128 / 256 (DH 512: 64 / 128); rs_key_splits = CTAs sharing one
// value tile's key columns (their partial outputs are combined afterwards).
bool rs_path_supports(int DH, int L);
int rs_key_splits(int DH, int L);
cudaError_t launch_fwd_rs(const FwdArgs &a, const FwdPlan &p, cudaStream_t st);
int tensor_path_max_chunks_per_segment();
cudaError_t launch_state_passthrough(const FwdArgs &a, int BH, int DH, cudaStream_t st);
cudaError_t launch_step(const StepArgs &a, cudaStream_t st);

// TMA descriptors over a [BH, S, D] tensor: bf16 with 64-column boxes of
// `box_rows` rows (128-byte swizzle or none), or fp32 with box_cols x box_rows
// boxes and no swizzle.  False if the driver refuses the encoding.
bool make_map_bf16(CUtensorMap *m, const void *base, int BH, int S, int D, bool swizzle = true,
                   int box_rows = 64);
// A 3-D tensor map without swizzle: dims innermost first, strides in bytes of
// dimensions 1 and 2 (multiples of 16), box sizes (box[0] * elem_bytes a
// multiple of 16, each at most 256).  elem_bytes 2 (bf16) or 4 (fp32).
bool make_tensor_map_3d(CUtensorMap *m, const void *base, int elem_bytes, const unsigned long long dims[3],
                        const unsigned long long strides_bytes[2], const unsigned box[3]);
bool make_map_f32_rows(CUtensorMap *m, const void *base, int BH, int S, int D, int box_cols = 128,
                       int box_rows = 64);

size_t simt_summary_smem(int DH, int rows);
size_t simt_output_smem(int DH, int rows, int L);

}  // namespace xlstm
