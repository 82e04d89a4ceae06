/*
 * sLSTM cell forward -- float64 CPU oracle (test infrastructure only).
 *
 * Only the tests, the smoke entry point and the CPU-baseline leg of the
 * benchmark may load it; the product library never links it.
 *
 * What it computes: the sLSTM of "xLSTM: Extended Long Short-Term Memory",
 * section 2.2: a scalar memory cell per unit with exponential input gating and
 * an optionally exponential forget gate, a normaliser state that sums the input
 * gate times all following forget gates, the stabiliser state m_t (Milakov &
 * Gimelshein), and memory mixing through recurrent connections R_z, R_i, R_f,
 * R_o from the hidden state h_{t-1} to the cell input z and the gates i, f, o,
 * within each head but not across heads.  The pages lost the displayed
 * equations; the recurrence below is the plain reading of that prose (the LSTM
 * cell with these changes), per batch b, head hd, unit j of DH:
 *
 *   zt_t = zx_t + R_z h_{t-1}       it_t = ix_t + R_i h_{t-1}
 *   ft_t = fx_t + R_f h_{t-1}       ot_t = ox_t + R_o h_{t-1}
 *       (R_g is the head's DH x DH block: row = receiving unit, column = h unit;
 *        the *x inputs carry the input projection and bias)
 *   z_t = tanh(zt_t);  log i_t = it_t;  log f_t = log sigmoid(ft_t) | ft_t;
 *   o_t = sigmoid(ot_t)
 *   m_t = max(log f_t + m_{t-1}, log i_t)
 *   i'_t = exp(log i_t - m_t),  f'_t = exp(log f_t + m_{t-1} - m_t)
 *   c_t = f'_t c_{t-1} + i'_t z_t,   n_t = f'_t n_{t-1} + i'_t
 *   h_t = o_t * c_t / n_t
 *
 * c and n are held in stabilised units (c' = c exp(-m)); their ratio, and so
 * h, does not depend on the stabiliser, as section 2.2 (appendix A.2) states.
 * The raw mode (stabilised == 0) runs c_t = f_t c_{t-1} + i_t z_t,
 * n_t = f_t n_{t-1} + i_t so that the tests can check that claim.
 *
 * Plain C, double precision, one token at a time; OpenMP over independent
 * (batch, head) pairs (no mixing across heads).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

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

/*
 * Layouts (row-major):
 *   zx, ix, fx, ox, h   [BH, S, DH]      (BH = B * NH, head-major)
 *   R                   [NH, 4, DH, DH]  gate order z, i, f, o; R[hd][g][row][col]
 *   state c, n, m, h0   [BH, DH]         (in: initial, NULL = zeros;
 *                                          out: final, NULL = not written)
 * Returns 0, or 1 if scratch could not be allocated.
 */
int slstm_oracle_fwd(const double *zx, const double *ix, const double *fx, const double *ox,
                     const double *R, double *h,
                     const double *c0, const double *n0, const double *m0, const double *h0,
                     double *c_out, double *n_out, double *m_out, double *h_out,
                     long B, long NH, long S, long DH, int fgate_exp, int stabilised)
{
    const long BH = B * NH;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (long bh = 0; bh < BH; ++bh) {
        const long hd = bh % NH;
        double *c = malloc(sizeof(double) * DH);
        double *n = malloc(sizeof(double) * DH);
        double *m = malloc(sizeof(double) * DH);
        double *hp = malloc(sizeof(double) * DH);   /* h_{t-1} */
        double *hn = malloc(sizeof(double) * DH);   /* h_t */
        if (!c || !n || !m || !hp || !hn) {
            free(c); free(n); free(m); free(hp); free(hn);
            failed |= 1;
            continue;
        }
        for (long j = 0; j < DH; ++j) {
            c[j] = c0 ? c0[bh * DH + j] : 0.0;
            n[j] = n0 ? n0[bh * DH + j] : 0.0;
            m[j] = m0 ? m0[bh * DH + j] : 0.0;
            hp[j] = h0 ? h0[bh * DH + j] : 0.0;
        }
        const double *Rz = R + ((hd * 4 + 0) * DH) * DH;
        const double *Ri = R + ((hd * 4 + 1) * DH) * DH;
        const double *Rf = R + ((hd * 4 + 2) * DH) * DH;
        const double *Ro = R + ((hd * 4 + 3) * DH) * DH;
        for (long t = 0; t < S; ++t) {
            const long row = (bh * S + t) * DH;
            for (long j = 0; j < DH; ++j) {
                double zt = zx[row + j], it = ix[row + j], ft = fx[row + j], ot = ox[row + j];
                for (long l = 0; l < DH; ++l) {
                    zt += Rz[j * DH + l] * hp[l];
                    it += Ri[j * DH + l] * hp[l];
                    ft += Rf[j * DH + l] * hp[l];
                    ot += Ro[j * DH + l] * hp[l];
                }
                const double z = tanh(zt);
                const double log_i = it;
                const double log_f = fgate_exp ? ft : log_sigmoid(ft);
                const double o = sigmoid(ot);
                double fg, ig;
                if (stabilised) {
                    const double m_new = fmax(log_f + m[j], log_i);
                    fg = exp(log_f + m[j] - m_new);
                    ig = exp(log_i - m_new);
                    m[j] = m_new;
                } else {
                    fg = exp(log_f);
                    ig = exp(log_i);
                }
                c[j] = fg * c[j] + ig * z;
                n[j] = fg * n[j] + ig;
                hn[j] = o * c[j] / n[j];
            }
            for (long j = 0; j < DH; ++j) {
                h[row + j] = hn[j];
                hp[j] = hn[j];
            }
        }
        for (long j = 0; j < DH; ++j) {
            if (c_out) c_out[bh * DH + j] = c[j];
            if (n_out) n_out[bh * DH + j] = n[j];
            if (m_out) m_out[bh * DH + j] = m[j];
            if (h_out) h_out[bh * DH + j] = hp[j];
        }
        free(c); free(n); free(m); free(hp); free(hn);
    }
    return failed ? 1 : 0;
}
