// Sequence parallelism: the state a run of tokens leaves behind, and the fold
// that joins such states.
//
// Unrolling the mLSTM recurrence ("xLSTM: Extended Long Short-Term Memory",
// section 2.3: C_t = f_t C_{t-1} + i_t v_t k_t^T, n_t likewise) over a run j of
// tokens that starts from the zero state gives, in raw units,
//   C_end = e^{F_j} C_start + sum_s e^{log i_s + F_j - F_{j,s}} v_s khat_s^T,
// with F_j the run's total log forget and F_{j,s} its prefix up to token s.
// In stabilised units (section 2.2's stabiliser, applied to mLSTM in 2.3) the
// run is summarised by X_j = (C'_j, n'_j) under its own stabiliser
//   mloc_j = max_s (log i_s + F_j - F_{j,s})        (no initial-state term),
// and consecutive runs fold exactly as the recurrence does:
//   M_j = max(F_j + M_{j-1}, mloc_j),
//   X   = e^{F_j + M_{j-1} - M_j} X_{j-1} + e^{mloc_j - M_j} X_j.
// Starting from the caller's (C'_0, n'_0, m_0) this reproduces the (C', n', m)
// the token-by-token recurrence reaches at the end of the last run; starting
// from M = -inf it yields the summary of the concatenated runs, again in the
// same (X, mloc, F) form.  The same fold joins the segments of one head inside
// the chunkwise forward; here the runs are also the slices of a sequence held
// by different GPUs.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace xlstm {

// One thread per 4 consecutive floats of a head's (C' | n'); every thread
// walks the runs in order (the per-run scalars are recomputed by each thread:
// they are a few flops and come from L1).
__global__ void __launch_bounds__(256)
state_fold_kernel(FoldSource src, int count, int scanned, const float *__restrict__ C0,
                  const float *__restrict__ n0, const float *__restrict__ m0, int start_neg_inf,
                  float *__restrict__ C_out, float *__restrict__ n_out, float *__restrict__ m_out,
                  float *__restrict__ F_out, int D) {
    const int bh = blockIdx.y;
    const size_t DD = (size_t)D * D;
    const size_t e4 = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (e4 >= DD + D) return;
    const bool in_c = e4 < DD;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (in_c ? C0 != nullptr : n0 != nullptr)
        x = in_c ? *reinterpret_cast<const float4 *>(C0 + bh * DD + e4)
                 : *reinterpret_cast<const float4 *>(n0 + (size_t)bh * D + (e4 - DD));
    float mc = m0 ? m0[bh] : (start_neg_inf ? -INFINITY : 0.f);
    float ftot = 0.f;
    // unrolled so that several runs' loads are in flight at once (they do not
    // depend on the running state)
#pragma unroll 8
    for (int g = 0; g < count; ++g) {
        const float F = src.F[g * src.sg + bh * src.sbh];
        const float ml = src.m[g * src.sg + bh * src.sbh];
        const float mn = fmaxf(F + mc, ml);
        ftot += F;
        if (!scanned) {
            // mn = -inf only while every run so far was empty (and the start is
            // -inf): the state is still zero
            const float al = mn == -INFINITY ? 0.f : expf(F + mc - mn);
            const float be = mn == -INFINITY ? 0.f : expf(ml - mn);
            const float4 d = in_c ? *reinterpret_cast<const float4 *>(src.C + g * src.cg + bh * src.cbh + e4)
                                  : *reinterpret_cast<const float4 *>(src.n + g * src.ng + bh * src.nbh + (e4 - DD));
            x.x = al * x.x + be * d.x;
            x.y = al * x.y + be * d.y;
            x.z = al * x.z + be * d.z;
            x.w = al * x.w + be * d.w;
        }
        mc = mn;
    }
    if (scanned && count > 0) {
        // the runs were already folded in place (from the same starting M); the
        // last slot holds the result
        const size_t g = (size_t)count - 1;
        x = in_c ? *reinterpret_cast<const float4 *>(src.C + g * src.cg + bh * src.cbh + e4)
                 : *reinterpret_cast<const float4 *>(src.n + g * src.ng + bh * src.nbh + (e4 - DD));
    }
    if (in_c)
        *reinterpret_cast<float4 *>(C_out + bh * DD + e4) = x;
    else
        *reinterpret_cast<float4 *>(n_out + (size_t)bh * D + (e4 - DD)) = x;
    if (e4 == 0) {
        m_out[bh] = mc;
        if (F_out) F_out[bh] = ftot;
    }
}

cudaError_t launch_state_fold(const FoldSource &src, int count, int scanned, const float *C0, const float *n0,
                              const float *m0, int start_neg_inf, float *C_out, float *n_out, float *m_out,
                              float *F_out, int BH, int D, cudaStream_t st) {
    if (BH == 0) return cudaSuccess;
    const size_t per4 = ((size_t)D * D + D) / 4;
    KernelTimer timer("state_fold", st);
    state_fold_kernel<<<dim3((unsigned)((per4 + 255) / 256), BH), 256, 0, st>>>(
        src, count, scanned, C0, n0, m0, start_neg_inf, C_out, n_out, m_out, F_out, D);
    return cudaGetLastError();
}

}  // namespace xlstm
