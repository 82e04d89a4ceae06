/*
 * mLSTM cell forward -- float64 CPU oracle (test infrastructure only).
 *
 * This file is the slow, obviously-correct reference that the CUDA path is
 * checked against.  Only the tests, the smoke entry point and the CPU-baseline
 * leg of the benchmark may load it; the product library never links it and
 * shares no code with it.
 *
 * What it computes: the mLSTM recurrence of "xLSTM: Extended Long Short-Term
 * Memory", section 2.3 (matrix memory, covariance rule eq. (18)), with the
 * exponential input gate and forget gate of section 2.2, the normaliser state
 * of section 2.3 with its lower bound of 1.0 on |n^T q|, and the log-space
 * stabiliser state m_t of section 2.2 (the Milakov & Gimelshein running max),
 * which section 2.3 applies unchanged to mLSTM.  The pages print none of the
 * displayed equations except eq. (18); the exact per-token recurrence below is
 * the plain reading that agrees with every sentence they do print:
 *
 *   log i_t = itilde_t                        (exponential input gate)
 *   log f_t = log sigmoid(ftilde_t)           (sigmoid forget gate)
 *           | ftilde_t                        (exponential forget gate)
 *   o_t     = sigmoid(otilde_t)               (per element of DH)
 *   khat_t  = k_t / sqrt(DH)
 *   m_t     = max(log f_t + m_{t-1}, log i_t)
 *   f'_t    = exp(log f_t + m_{t-1} - m_t),   i'_t = exp(log i_t - m_t)
 *   C'_t    = f'_t C'_{t-1} + i'_t v_t khat_t^T      (C' is [value, key])
 *   n'_t    = f'_t n'_{t-1} + i'_t khat_t
 *   h_t     = o_t * (C'_t q_t) / max(|n'_t^T q_t|, exp(-m_t))
 *
 * The last line is the section 2.3 bound max(|n_t^T q_t|, 1) written in the
 * stabilised units C' = C exp(-m), n' = n exp(-m): the bound scales with the
 * state, which is what keeps the output independent of the stabiliser, as
 * section 2.2 (and appendix A.2) claims for f -> f', i -> i'.
 *
 * The raw mode (stabilised == 0) runs the unstabilised recurrence
 * C_t = f_t C_{t-1} + i_t v_t khat_t^T, n_t likewise, h = o * C q / max(|n^T q|, 1)
 * on the same inputs; it exists only so that the tests can check the
 * invariance claim.  Raw-mode state in and out is in raw units.
 *
 * Plain C, double precision, one token at a time; OpenMP runs independent
 * (batch, head) pairs in parallel, which section 2.3 allows because heads
 * have no memory mixing.  No blocking, no reordering of the sums.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* log sigmoid(x), written so that neither branch overflows. */
static double log_sigmoid(double x)
{
    if (x >= 0.0)
        return -log1p(exp(-x));
    return x - log1p(exp(x));
}

static double sigmoid(double x)
{
    if (x >= 0.0)
        return 1.0 / (1.0 + exp(-x));
    double e = exp(x);
    return e / (1.0 + e);
}

int mlstm_oracle_abi_version(void) { return 1; }

int mlstm_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Forward over S tokens for BH = B*NH independent heads.
 *   q, k, v, o_pre : [BH, S, DH]      i_pre, f_pre : [BH, S]
 *   h              : [BH, S, DH] out
 *   C0 [BH, DH, DH], n0 [BH, DH], m0 [BH] : initial state, each may be NULL (zeros)
 *   C_out, n_out, m_out : final state, each may be NULL
 * fgate_exp: 0 = sigmoid forget gate, 1 = exponential forget gate.
 * stabilised: 1 = stabilised recurrence (state in C', n', m units),
 *             0 = raw recurrence (state in raw units, m ignored / returned 0).
 * Returns 0, or -1 if a work buffer cannot be allocated.
 */
int mlstm_oracle_fwd(const double *q, const double *k, const double *v,
                     const double *i_pre, const double *f_pre, const double *o_pre,
                     double *h,
                     const double *C0, const double *n0, const double *m0,
                     double *C_out, double *n_out, double *m_out,
                     long BH, long S, long DH, int fgate_exp, int stabilised)
{
    int failed = 0;
    const double inv_sqrt_d = 1.0 / sqrt((double)DH);

#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        double *C = (double *)malloc(sizeof(double) * DH * DH);
        double *n = (double *)malloc(sizeof(double) * DH);
        double *khat = (double *)malloc(sizeof(double) * DH);
        if (!C || !n || !khat) {
            free(C); free(n); free(khat);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        if (C0) memcpy(C, C0 + bh * DH * DH, sizeof(double) * DH * DH);
        else    memset(C, 0, sizeof(double) * DH * DH);
        if (n0) memcpy(n, n0 + bh * DH, sizeof(double) * DH);
        else    memset(n, 0, sizeof(double) * DH);
        double m = (m0 && stabilised) ? m0[bh] : 0.0;

        for (long t = 0; t < S; ++t) {
            const long tok = bh * S + t;
            const double *qt = q + tok * DH;
            const double *kt = k + tok * DH;
            const double *vt = v + tok * DH;
            const double *ot = o_pre + tok * DH;
            double *ht = h + tok * DH;

            const double log_i = i_pre[tok];
            const double log_f = fgate_exp ? f_pre[tok] : log_sigmoid(f_pre[tok]);
            double fg, ig, floor_;
            if (stabilised) {
                const double m_new = fmax(log_f + m, log_i);
                fg = exp(log_f + m - m_new);
                ig = exp(log_i - m_new);
                m = m_new;
                floor_ = exp(-m_new);
            } else {
                fg = exp(log_f);
                ig = exp(log_i);
                floor_ = 1.0;
            }
            for (long j = 0; j < DH; ++j)
                khat[j] = kt[j] * inv_sqrt_d;

            /* state and normaliser update */
            for (long i = 0; i < DH; ++i) {
                double *row = C + i * DH;
                const double a = ig * vt[i];
                for (long j = 0; j < DH; ++j)
                    row[j] = fg * row[j] + a * khat[j];
            }
            for (long j = 0; j < DH; ++j)
                n[j] = fg * n[j] + ig * khat[j];

            /* retrieval, normalisation and output gate */
            double den = 0.0;
            for (long j = 0; j < DH; ++j)
                den += n[j] * qt[j];
            const double denom = fmax(fabs(den), floor_);
            for (long i = 0; i < DH; ++i) {
                const double *row = C + i * DH;
                double num = 0.0;
                for (long j = 0; j < DH; ++j)
                    num += row[j] * qt[j];
                ht[i] = sigmoid(ot[i]) * num / denom;
            }
        }
        if (C_out) memcpy(C_out + bh * DH * DH, C, sizeof(double) * DH * DH);
        if (n_out) memcpy(n_out + bh * DH, n, sizeof(double) * DH);
        if (m_out) m_out[bh] = stabilised ? m : 0.0;
        free(C); free(n); free(khat);
    }
    return failed ? -1 : 0;
}
