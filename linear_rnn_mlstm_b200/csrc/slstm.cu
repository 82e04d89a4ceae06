// sLSTM forward ("xLSTM: Extended Long Short-Term Memory" section 2.2): one
// CTA per (batch, head), one thread per unit, fp32.  The recurrence mixes the
// units of a head through h_{t-1} at every step, so the sequence is walked in
// order; h_{t-1} lives in one of two shared arrays while h_t is written to the
// other, one barrier per step.  The recurrent matrices are read from global
// memory (each head's 4 DH x DH block stays in L2).  This is the
// correctness-first form, kept for the head sizes the cluster kernel
// (slstm_cluster.cu: DH 64, 128, 256) does not take; the per-unit step is in
// slstm_body.cuh.
#include <math.h>
#include <stdint.h>

#include "../../include/xlstm_mlstm.h"
#include "common.cuh"
#include "profile.h"
#include "slstm_body.cuh"

namespace xlstm {
namespace {

using slstm::SlstmPtrs;

__global__ void __launch_bounds__(512) slstm_fwd_kernel(SlstmPtrs p) {
    extern __shared__ float hbuf[];        // [2][DH]
    const int bh = blockIdx.x, j = threadIdx.x, DH = p.DH;
    float c, n, m;
    slstm::unit_init(p, bh, j, c, n, m, hbuf);
    __syncthreads();
    for (int t = 0; t < p.S; ++t) {
        slstm::unit_step(p, bh, j, t, hbuf + (t & 1) * DH, hbuf + ((t + 1) & 1) * DH, c, n, m);
        __syncthreads();
    }
    slstm::unit_final(p, bh, j, c, n, m, hbuf + (p.S & 1) * DH);
}

bool misaligned16(const void *ptr) { return ((uintptr_t)ptr & 15u) != 0; }

}  // namespace

// The cluster kernel for DH 64, 128 and 256 (slstm_cluster.cu).
bool slstm_cluster_supports(int DH);
cudaError_t launch_slstm_cluster(const slstm::SlstmPtrs &p, cudaStream_t st);

}  // namespace xlstm

using namespace xlstm;

extern "C" xlstm_status xlstm_slstm_fwd(const float *zx, const float *ix, const float *fx,
                                        const float *ox, const float *R, float *h,
                                        const float *c0, const float *n0, const float *m0,
                                        const float *h0, float *c_out, float *n_out,
                                        float *m_out, float *h_out, int B, int NH, int S,
                                        int DH, xlstm_fgate fg, void *cuda_stream) {
    CallRange range("xlstm_slstm_fwd");
    if (fg != XLSTM_FGATE_SIGMOID && fg != XLSTM_FGATE_EXP) return XLSTM_ERR_DTYPE;
    if (B < 0 || NH < 0 || S < 0 || DH < 1 || DH > 512) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH * S * DH > (1LL << 40) || (long long)B * NH > 0x7fffffffLL)
        return XLSTM_ERR_SHAPE;
    const long long BH = (long long)B * NH;
    if (BH == 0) return XLSTM_OK;
    if (S > 0 && (!zx || !ix || !fx || !ox || !R || !h)) return XLSTM_ERR_NULL;
    if (S == 0 && !c_out && !n_out && !m_out && !h_out) return XLSTM_OK;
    const void *inputs[] = {zx, ix, fx, ox, R, c0, n0, m0, h0};
    const void *outputs[] = {h, c_out, n_out, m_out, h_out};
    for (const void *ptr : inputs)
        if (misaligned16(ptr)) return XLSTM_ERR_ALIGN;
    for (const void *ptr : outputs)
        if (misaligned16(ptr)) return XLSTM_ERR_ALIGN;
    for (int a = 0; a < 5; ++a) {
        if (!outputs[a]) continue;
        for (const void *in : inputs)
            if (outputs[a] == in) return XLSTM_ERR_UNSUPPORTED;
        for (int b = a + 1; b < 5; ++b)
            if (outputs[a] == outputs[b]) return XLSTM_ERR_UNSUPPORTED;
    }
    slstm::SlstmPtrs p;
    p.zx = zx; p.ix = ix; p.fx = fx; p.ox = ox; p.R = R; p.h = h;
    p.c0 = c0; p.n0 = n0; p.m0 = m0; p.h0 = h0;
    p.c_out = c_out; p.n_out = n_out; p.m_out = m_out; p.h_out = h_out;
    p.BH = (int)BH; p.NH = NH; p.S = S; p.DH = DH;
    p.fgate_exp = fg == XLSTM_FGATE_EXP;
    cudaStream_t st = (cudaStream_t)cuda_stream;
    if (slstm_cluster_supports(DH)) {
        KernelTimer timer("slstm_cluster", st);
        return launch_slstm_cluster(p, st) == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
    }
    KernelTimer timer("slstm_fwd", st);
    slstm_fwd_kernel<<<(unsigned)BH, DH, 2 * DH * sizeof(float), st>>>(p);
    return cudaGetLastError() == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}
