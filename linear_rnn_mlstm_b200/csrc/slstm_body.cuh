// Per-unit bodies of the sLSTM forward kernel (slstm.cu).
//
// The sLSTM cell of "xLSTM: Extended Long Short-Term Memory" section 2.2: a
// scalar memory cell per unit with exponential input gating, a sigmoid or
// exponential forget gate, a normaliser state, the stabiliser m_t, and memory
// mixing through recurrent connections from h_{t-1} to the cell input and the
// gates, within each head.  Per unit j of a head, step t:
//
//   zt = zx_t + R_z h_{t-1},  it = ix_t + R_i h_{t-1},  ft = fx_t + R_f h_{t-1},
//   ot = ox_t + R_o h_{t-1}   (R_g: the head's DH x DH block, row = unit j)
//   z = tanh(zt), log i = it, log f = log sigmoid(ft) | ft, o = sigmoid(ot)
//   m_t = max(log f + m_{t-1}, log i)
//   c_t = e^{log f + m_{t-1} - m_t} c_{t-1} + e^{log i - m_t} z
//   n_t = e^{log f + m_{t-1} - m_t} n_{t-1} + e^{log i - m_t}
//   h_t = o c_t / n_t
//
// A CTA runs one head: thread j keeps (c, n, m) of unit j in registers and
// h_{t-1} of all units is read from one of two shared arrays while h_t is
// written to the other, with one barrier per step.  Written as per-unit
// functions with the barrier left to the caller, the same code runs on the
// host, one unit after another between the "barriers", which the tests use to
// check it against the float64 sLSTM oracle.
#pragma once

#include <math.h>
#include <stddef.h>

#if defined(__CUDACC__)
#define XLSTM_HD __host__ __device__ __forceinline__
#else
#define XLSTM_HD inline
#endif

namespace xlstm {
namespace slstm {

struct SlstmPtrs {
    const float *zx, *ix, *fx, *ox;     // [BH, S, DH] input pre-activations
    const float *R;                     // [NH, 4, DH, DH] gate order z, i, f, o
    float *h;                           // [BH, S, DH] output
    const float *c0, *n0, *m0, *h0;     // [BH, DH] initial state; nullable (zeros)
    float *c_out, *n_out, *m_out, *h_out;   // [BH, DH] final state; nullable
    int BH, NH, S, DH, fgate_exp;
};

XLSTM_HD float log_sigmoid_hd(float x) {
    return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}
XLSTM_HD float sigmoid_hd(float x) {
    if (x >= 0.f) return 1.f / (1.f + expf(-x));
    const float e = expf(x);
    return e / (1.f + e);
}

// Unit j of head bh before the first step: its state, and h_0[j] into hbuf0.
XLSTM_HD void unit_init(const SlstmPtrs &p, int bh, int j, float &c, float &n, float &m,
                        float *hbuf0) {
    const size_t s = (size_t)bh * p.DH + j;
    c = p.c0 ? p.c0[s] : 0.f;
    n = p.n0 ? p.n0[s] : 0.f;
    m = p.m0 ? p.m0[s] : 0.f;
    hbuf0[j] = p.h0 ? p.h0[s] : 0.f;
}

// Step t of unit j: reads h_{t-1} of every unit from hprev, writes h_t[j] to
// hnext and to the output.
XLSTM_HD void unit_step(const SlstmPtrs &p, int bh, int j, int t, const float *hprev,
                        float *hnext, float &c, float &n, float &m) {
    const int DH = p.DH;
    const int head = bh % p.NH;
    const size_t x = ((size_t)bh * p.S + t) * DH + j;
    const size_t DD = (size_t)DH * DH;
    const float *Rz = p.R + ((size_t)head * 4 + 0) * DD + (size_t)j * DH;
    const float *Ri = Rz + DD;
    const float *Rf = Ri + DD;
    const float *Ro = Rf + DD;
    float zt = p.zx[x], it = p.ix[x], ft = p.fx[x], ot = p.ox[x];
    for (int l = 0; l < DH; ++l) {
        const float hl = hprev[l];
        zt += Rz[l] * hl;
        it += Ri[l] * hl;
        ft += Rf[l] * hl;
        ot += Ro[l] * hl;
    }
    const float z = tanhf(zt);
    const float log_f = p.fgate_exp ? ft : log_sigmoid_hd(ft);
    const float o = sigmoid_hd(ot);
    const float m_new = fmaxf(log_f + m, it);
    const float fg = expf(log_f + m - m_new);
    const float ig = expf(it - m_new);
    m = m_new;
    c = fg * c + ig * z;
    n = fg * n + ig;
    const float h = o * c / n;
    p.h[x] = h;
    hnext[j] = h;
}

// After the last step: the final state of unit j (hlast holds h_S).
XLSTM_HD void unit_final(const SlstmPtrs &p, int bh, int j, float c, float n, float m,
                         const float *hlast) {
    const size_t s = (size_t)bh * p.DH + j;
    if (p.c_out) p.c_out[s] = c;
    if (p.n_out) p.n_out[s] = n;
    if (p.m_out) p.m_out[s] = m;
    if (p.h_out) p.h_out[s] = hlast[j];
}

}  // namespace slstm
}  // namespace xlstm
