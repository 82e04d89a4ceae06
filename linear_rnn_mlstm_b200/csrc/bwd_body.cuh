// Per-thread bodies of the mLSTM backward kernels (bwd.cu).
//
// The gradient of L = sum(dh h) + sum(dC C'_T) + sum(dn n'_T) through the cell
// of "xLSTM: Extended Long Short-Term Memory" section 2.3, in the blocked form:
// the stabiliser m_t is held fixed (section 2.2: the stabilised gates change
// neither the output nor the loss's derivatives), the chunk-start states and a
// reverse state are carried across chunks, and every token's gradients are
// formed from its own chunk.  Per head, chunk c = tokens [cL, cL+L):
//
//   b_t   chunk-local cumulative log forget, m_t stabiliser, B_c = b at chunk end
//   num'_t = g_t C'_c q_t + sum_{s<=t} W_ts S_ts v_s,  g_t = e^{b_t + m_{c-1} - m_t}
//   nq'_t  = g_t n'_c . q_t + sum_{s<=t} W_ts S_ts,    W_ts = e^{b_t - b_s + i_s - m_t},
//   den'_t = max(|nq'_t|, e^{-m_t}),                    S_ts = q_t . khat_s
//   dnum'_t = dh_t o_t / den'_t,  dnq'_t = -(dh_t o_t . h~_t) / den'_t sign(nq'_t)
//            where |nq'_t| > e^{-m_t} (the floor passes no gradient), else 0
//   reverse state at the end of chunk c (stabilised at m_c):
//   dC~_{c-1} = e^{B_c + m_{c-1} - m_c} dC~_c + sum_{t in c} g_t dnum'_t q_t^T
//   dq_t  = sum_{s<=t} W_ts dP_ts khat_s + g_t (C'_c^T dnum'_t + dnq'_t n'_c)
//   dkhat_s = sum_{t>=s} W_ts dP_ts q_t + wk_s (dC~_c^T v_s + dn~_c),
//   dv_s  = sum_{t>=s} W_ts S_ts dnum'_t + wk_s dC~_c khat_s,
//            dP_ts = dnum'_t . v_s + dnq'_t,  wk_s = e^{B_c - b_s + i_s - m_c}
//   ditilde_s = khat_s . dkhat_s;  d log f_j = sum_{t>=j} (A_t - ditilde_t),
//            A_t = dnum'_t . num'_t + dnq'_t nq'_t
//   and, for final-state cotangents, the returned state's m_T = F_T +
//   max(0, max_s(i_s - F_s)) moves A_final = sum dC C'_T + sum dn n'_T from
//   ditilde to F at the maximising key.
//
// Each body works on one head (K1, K6), one state row (K2, K4) or one token
// (K3, K5) and touches no shared memory, so the same code also runs on the
// host, one "thread" after another, which the tests use to check it against
// the float64 gradient oracle before it ever runs on a GPU.
#pragma once

#include <math.h>
#include <stddef.h>

#include <cuda_bf16.h>

#if defined(__CUDACC__)
#define XLSTM_HD __host__ __device__ __forceinline__
#else
#define XLSTM_HD inline
#endif

namespace xlstm {
namespace bwd {

constexpr int kMaxChunk = 64;      // tokens per chunk held in a thread's local arrays

template <typename T> XLSTM_HD float ld(const T *p, size_t i);
template <> XLSTM_HD float ld<float>(const float *p, size_t i) { return p[i]; }
template <> XLSTM_HD float ld<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
template <typename T> XLSTM_HD void st(T *p, size_t i, float x);
template <> XLSTM_HD void st<float>(float *p, size_t i, float x) { p[i] = x; }
template <> XLSTM_HD void st<__nv_bfloat16>(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

XLSTM_HD float log_sigmoid_hd(float x) {
    return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}
XLSTM_HD float sigmoid_hd(float x) {
    if (x >= 0.f) return 1.f / (1.f + expf(-x));
    const float e = expf(x);
    return e / (1.f + e);
}
XLSTM_HD int imin(int a, int b) { return a < b ? a : b; }

// Inputs, outputs and workspace of one backward call.
struct BwdPtrs {
    const void *q, *k, *v;            // [BH, S, DH] dtype T
    const float *ip, *fp, *op;        // itilde, ftilde [BH, S]; otilde [BH, S, DH]
    const void *dh;                   // [BH, S, DH] dtype T
    const float *dC, *dn;             // final-state cotangents [BH, DH, DH], [BH, DH]; nullable
    void *dq, *dk, *dv;               // [BH, S, DH] dtype T
    float *di, *df, *dO;              // [BH, S], [BH, S], [BH, S, DH]
    // workspace
    float *logf, *b, *mt, *den, *nq, *A, *dF, *dnq;   // [BH, S]
    float *mprev, *mend, *Bsum;                         // [BH, NC]
    float *Cst;                       // [BH, NC + 1, DH, DH] chunk-start C' (slot NC: final)
    float *nst;                       // [BH, NC + 1, DH]
    float *num, *dnum;                // [BH, S, DH]; dnum on the fp32 kernels only
    float *dCb;                       // [BH, NC, DH, DH] reverse state at the end of chunk c
    float *dnb;                       // [BH, NC, DH]
    int BH, S, DH, L, NC, fgate_exp;
    // Tensor-core products with the states (bf16, DH 128 / 256): tc != 0 stores
    // every C' and dC~ slot as two bf16 planes (high part, then low part, each
    // DH*DH, in the 128-byte-swizzled tile order the MMAs read) instead of
    // fp32, and the per-token kernels take the state products from:
    void *dnhl;                       // [2][BH, S, DH] bf16: dnum' high, then low part
    float *dki, *dvi;                 // [BH, S, DH]: v_s^T dC~ and dC~ k_s per token
    float *wrec, *decay;              // [BH, NC, 128] token weights of the state walks, [BH, NC] decays
    int tc;
};

// K1, one head: log f, chunk-local cumulative log forget, the stabiliser per
// token (the recurrence m_t = max(log f_t + m_{t-1}, itilde_t), m_0 = 0) and
// the per-chunk m at start and end and sum of log f.
XLSTM_HD void gates_head(const BwdPtrs &p, int bh) {
    const size_t base = (size_t)bh * p.S;
    const size_t cbase = (size_t)bh * p.NC;
    float m = 0.f, bcum = 0.f;
    for (int t = 0; t < p.S; ++t) {
        const int c = t / p.L;
        if (t % p.L == 0) {
            p.mprev[cbase + c] = m;
            bcum = 0.f;
        }
        const float fpre = p.fp[base + t];
        const float lf = p.fgate_exp ? fpre : log_sigmoid_hd(fpre);
        bcum += lf;
        const float mn = fmaxf(lf + m, p.ip[base + t]);
        p.logf[base + t] = lf;
        p.b[base + t] = bcum;
        p.mt[base + t] = mn;
        m = mn;
        if (t % p.L == p.L - 1 || t == p.S - 1) {
            p.mend[cbase + c] = m;
            p.Bsum[cbase + c] = bcum;
        }
    }
}

// K2, one state row r of one head (r == DH: the normaliser n'): the chunk-start
// states C'_c[r, :] for c = 0..NC (slot NC is the final state).
template <typename T>
XLSTM_HD void states_row(const BwdPtrs &p, int bh, int r) {
    const int S = p.S, DH = p.DH, L = p.L, NC = p.NC;
    const size_t DD = (size_t)DH * DH;
    const float inv_sqrt = 1.f / sqrtf((float)DH);
    const bool nrow = r == DH;
    float *slot0 = nrow ? p.nst + (size_t)bh * (NC + 1) * DH
                        : p.Cst + (size_t)bh * (NC + 1) * DD + (size_t)r * DH;
    const size_t stride = nrow ? (size_t)DH : DD;
    const T *k = (const T *)p.k;
    const T *v = (const T *)p.v;
    for (int j = 0; j < DH; ++j) slot0[j] = 0.f;
    for (int c = 0; c < NC; ++c) {
        const float *prev = slot0 + (size_t)c * stride;
        float *next = slot0 + (size_t)(c + 1) * stride;
        const size_t hc = (size_t)bh * NC + c;
        const float mend = p.mend[hc];
        const float decay = expf(p.Bsum[hc] + p.mprev[hc] - mend);
        for (int j = 0; j < DH; ++j) next[j] = decay * prev[j];
        const int a = c * L, e = imin(S, a + L);
        for (int s = a; s < e; ++s) {
            const size_t ts = (size_t)bh * S + s;
            const float wk = expf(p.Bsum[hc] - p.b[ts] + p.ip[ts] - mend);
            const float coef = wk * inv_sqrt * (nrow ? 1.f : ld(v, ts * DH + r));
            for (int j = 0; j < DH; ++j) next[j] += coef * ld(k, ts * DH + j);
        }
    }
}

// K3, one token: recompute num', nq', den' and form the token's own
// gradient quantities dotilde, dnum', dnq' and A.
template <typename T>
XLSTM_HD void token_fwd(const BwdPtrs &p, int bh, int t) {
    const int S = p.S, DH = p.DH, L = p.L, NC = p.NC;
    const size_t DD = (size_t)DH * DH;
    const float inv_sqrt = 1.f / sqrtf((float)DH);
    const T *q = (const T *)p.q;
    const T *k = (const T *)p.k;
    const T *v = (const T *)p.v;
    const T *dh = (const T *)p.dh;
    const size_t ts = (size_t)bh * S + t;
    const int c = t / L, a = c * L;
    const size_t hc = (size_t)bh * NC + c;
    const float m_t = p.mt[ts], b_t = p.b[ts];
    const float g = expf(b_t + p.mprev[hc] - m_t);
    const float *Cc = p.Cst + ((size_t)bh * (NC + 1) + c) * DD;
    const float *nc = p.nst + ((size_t)bh * (NC + 1) + c) * DH;
    float ws[kMaxChunk];
    float nq = 0.f;
    for (int s = a; s <= t; ++s) {
        const size_t ss = (size_t)bh * S + s;
        float dot = 0.f;
        for (int j = 0; j < DH; ++j) dot += ld(q, ts * DH + j) * ld(k, ss * DH + j);
        const float w = expf(b_t - p.b[ss] + p.ip[ss] - m_t);
        ws[s - a] = w * dot * inv_sqrt;
        nq += ws[s - a];
    }
    float nq_inter = 0.f;
    for (int j = 0; j < DH; ++j) nq_inter += nc[j] * ld(q, ts * DH + j);
    nq += g * nq_inter;
    float *num = p.num + ts * DH;
    for (int r = 0; r < DH; ++r) {
        float acc = 0.f;
        for (int j = 0; j < DH; ++j) acc += Cc[(size_t)r * DH + j] * ld(q, ts * DH + j);
        acc *= g;
        for (int s = a; s <= t; ++s) acc += ws[s - a] * ld(v, ((size_t)bh * S + s) * DH + r);
        num[r] = acc;
    }
    const float floor_ = expf(-m_t);
    const float den = fmaxf(fabsf(nq), floor_);
    float *dnum = p.dnum + ts * DH;
    float sdot = 0.f, A = 0.f;
    for (int r = 0; r < DH; ++r) {
        const float o = sigmoid_hd(p.op[ts * DH + r]);
        const float hv = num[r] / den;
        const float dhr = ld(dh, ts * DH + r);
        const float dht = dhr * o;
        p.dO[ts * DH + r] = dhr * hv * o * (1.f - o);
        dnum[r] = dht / den;
        sdot += dht * hv;
        A += dnum[r] * num[r];
    }
    const float dnq = fabsf(nq) > floor_ ? -sdot / den * (nq > 0.f ? 1.f : -1.f) : 0.f;
    p.dnq[ts] = dnq;
    p.nq[ts] = nq;
    p.den[ts] = den;
    p.A[ts] = A + dnq * nq;
}

// K4, one row r of the reverse state (r == DH: dn~), from the last chunk to the
// first; slot c holds the state at the end of chunk c.
template <typename T>
XLSTM_HD void reverse_row(const BwdPtrs &p, int bh, int r) {
    const int S = p.S, DH = p.DH, L = p.L, NC = p.NC;
    const size_t DD = (size_t)DH * DH;
    const bool nrow = r == DH;
    const T *q = (const T *)p.q;
    float *slot0 = nrow ? p.dnb + (size_t)bh * NC * DH : p.dCb + (size_t)bh * NC * DD + (size_t)r * DH;
    const size_t stride = nrow ? (size_t)DH : DD;
    float *last = slot0 + (size_t)(NC - 1) * stride;
    for (int j = 0; j < DH; ++j) {
        if (nrow)
            last[j] = p.dn ? p.dn[(size_t)bh * DH + j] : 0.f;
        else
            last[j] = p.dC ? p.dC[(size_t)bh * DD + (size_t)r * DH + j] : 0.f;
    }
    for (int c = NC - 1; c >= 1; --c) {
        const float *cur = slot0 + (size_t)c * stride;
        float *prv = slot0 + (size_t)(c - 1) * stride;
        const size_t hc = (size_t)bh * NC + c;
        const float decay = expf(p.Bsum[hc] + p.mprev[hc] - p.mend[hc]);
        for (int j = 0; j < DH; ++j) prv[j] = decay * cur[j];
        const int a = c * L, e = imin(S, a + L);
        for (int t = a; t < e; ++t) {
            const size_t tt = (size_t)bh * S + t;
            const float g = expf(p.b[tt] + p.mprev[hc] - p.mt[tt]);
            const float coef = g * (nrow ? p.dnq[tt] : p.dnum[tt * DH + r]);
            for (int j = 0; j < DH; ++j) prv[j] += coef * ld(q, tt * DH + j);
        }
    }
}

// K5, one token s: dq_s, dk_s, dv_s, ditilde_s and the token's term of d log f.
template <typename T>
XLSTM_HD void token_grad(const BwdPtrs &p, int bh, int s) {
    const int S = p.S, DH = p.DH, L = p.L, NC = p.NC;
    const size_t DD = (size_t)DH * DH;
    const float inv_sqrt = 1.f / sqrtf((float)DH);
    const T *q = (const T *)p.q;
    const T *k = (const T *)p.k;
    const T *v = (const T *)p.v;
    T *dq = (T *)p.dq;
    T *dk = (T *)p.dk;
    T *dv = (T *)p.dv;
    const size_t ss = (size_t)bh * S + s;
    const int c = s / L, a = c * L, e = imin(S, a + L);
    const size_t hc = (size_t)bh * NC + c;
    const float m_s = p.mt[ss], b_s = p.b[ss], i_s = p.ip[ss];
    const float *dnum_s = p.dnum + ss * DH;
    float wdp_a[kMaxChunk];    // u in [a, s]:  W_su dP_su
    float wdp_b[kMaxChunk];    // t in [s, e):  W_ts dP_ts
    float wsc_b[kMaxChunk];    // t in [s, e):  W_ts S_ts
    for (int u = a; u <= s; ++u) {
        const size_t us = (size_t)bh * S + u;
        float dot = 0.f;
        for (int j = 0; j < DH; ++j) dot += dnum_s[j] * ld(v, us * DH + j);
        const float w = expf(b_s - p.b[us] + p.ip[us] - m_s);
        wdp_a[u - a] = w * (dot + p.dnq[ss]);
    }
    for (int t = s; t < e; ++t) {
        const size_t tt = (size_t)bh * S + t;
        const float w = expf(p.b[tt] - b_s + i_s - p.mt[tt]);
        float dot = 0.f, sc = 0.f;
        for (int j = 0; j < DH; ++j) {
            dot += p.dnum[tt * DH + j] * ld(v, ss * DH + j);
            sc += ld(q, tt * DH + j) * ld(k, ss * DH + j);
        }
        wdp_b[t - s] = w * (dot + p.dnq[tt]);
        wsc_b[t - s] = w * sc * inv_sqrt;
    }
    const float g = expf(b_s + p.mprev[hc] - m_s);
    const float wk = expf(p.Bsum[hc] - b_s + i_s - p.mend[hc]);
    const float *Cc = p.Cst + ((size_t)bh * (NC + 1) + c) * DD;
    const float *ncs = p.nst + ((size_t)bh * (NC + 1) + c) * DH;
    const float *dCc = p.dCb + ((size_t)bh * NC + c) * DD;
    const float *dnc = p.dnb + ((size_t)bh * NC + c) * DH;
    float di = 0.f;
    for (int j = 0; j < DH; ++j) {
        float acc = 0.f;
        for (int u = a; u <= s; ++u) acc += wdp_a[u - a] * ld(k, ((size_t)bh * S + u) * DH + j);
        acc *= inv_sqrt;
        float inter = 0.f;
        for (int r = 0; r < DH; ++r) inter += Cc[(size_t)r * DH + j] * dnum_s[r];
        acc += g * (inter + p.dnq[ss] * ncs[j]);
        st(dq, ss * DH + j, acc);
        float dkh = 0.f;
        for (int t = s; t < e; ++t) dkh += wdp_b[t - s] * ld(q, ((size_t)bh * S + t) * DH + j);
        float rv = 0.f;
        for (int r = 0; r < DH; ++r) rv += dCc[(size_t)r * DH + j] * ld(v, ss * DH + r);
        dkh += wk * (rv + dnc[j]);
        di += dkh * ld(k, ss * DH + j) * inv_sqrt;
        st(dk, ss * DH + j, dkh * inv_sqrt);
    }
    for (int r = 0; r < DH; ++r) {
        float acc = 0.f;
        for (int t = s; t < e; ++t) acc += wsc_b[t - s] * p.dnum[((size_t)bh * S + t) * DH + r];
        float rk = 0.f;
        for (int j = 0; j < DH; ++j) rk += dCc[(size_t)r * DH + j] * ld(k, ss * DH + j);
        acc += wk * rk * inv_sqrt;
        st(dv, ss * DH + r, acc);
    }
    p.di[ss] = di;
    p.dF[ss] = p.A[ss] - di;
}

// K6, one head: the final state's m_T term, then d log f as the reverse
// cumulative sum of dF, and dftilde.
XLSTM_HD void forget_head(const BwdPtrs &p, int bh) {
    const int S = p.S, DH = p.DH, NC = p.NC;
    const size_t base = (size_t)bh * S;
    const size_t DD = (size_t)DH * DH;
    if (p.dC || p.dn) {
        float a_final = 0.f;
        const float *CT = p.Cst + ((size_t)bh * (NC + 1) + NC) * DD;
        const float *nT = p.nst + ((size_t)bh * (NC + 1) + NC) * DH;
        if (p.dC)
            for (size_t i = 0; i < DD; ++i) a_final += p.dC[(size_t)bh * DD + i] * CT[i];
        if (p.dn)
            for (int j = 0; j < DH; ++j) a_final += p.dn[(size_t)bh * DH + j] * nT[j];
        float F = 0.f, best = 0.f;
        int sstar = -1;
        for (int t = 0; t < S; ++t) {
            F += p.logf[base + t];
            const float cand = p.ip[base + t] - F;
            if (cand > best) {
                best = cand;
                sstar = t;
            }
        }
        if (sstar >= 0) {
            p.di[base + sstar] -= a_final;
            p.dF[base + sstar] += a_final;
        }
    }
    float acc = 0.f;
    for (int t = S - 1; t >= 0; --t) {
        acc += p.dF[base + t];
        p.df[base + t] = p.fgate_exp ? acc : acc * sigmoid_hd(-p.fp[base + t]);
    }
}

}  // namespace bwd
}  // namespace xlstm
