// Chunkwise mLSTM forward, fp32-arithmetic SIMT kernels.
//
// These kernels compute the chunkwise-parallel form of the mLSTM recurrence
// ("xLSTM: Extended Long Short-Term Memory" section 2.3: matrix memory with the
// gated covariance rule, normaliser floored at 1.0; section 2.2: exponential
// input gate with the stabiliser m) in fp32 CUDA-core arithmetic.  They are the
// forward for fp32 inputs and an independent second path for bf16 inputs.
//
// Notation per head, chunk c covering tokens [cL, cL + L):
//   lf_t = log f_t,  li_t = itilde_t,  b_t = sum_{j = cL..t} lf_j  (chunk-local)
//   u_t  = li_t - b_t
//   m_t  = b_t + max(m_prev, max_{s <= t in chunk} u_s)     (exact unrolling of
//          m_t = max(lf_t + m_{t-1}, li_t))
//   h_t  = o_t * [g_t C'_prev q_t + sum_{s<=t} e^{u_s + b_t - m_t} (q_t.khat_s) v_s]
//               / max(|g_t n'_prev.q_t + sum_{s<=t} e^{u_s + b_t - m_t} q_t.khat_s|, e^{-m_t})
//          with g_t = e^{b_t + m_prev - m_t}
//   chunk end: C'_next = e^{b_L + m_prev - m_next} C'_prev + sum_s e^{u_s + b_L - m_next} v_s khat_s^T
// Every exponent above is <= 0 by construction of m.
#include "common.cuh"
#include "plan.h"
#include "kernels.h"
#include "profile.h"

namespace xlstm {

// ------------------------------------------------------------------ phase 0
// One warp per (head, chunk): lf, the chunk-local inclusive prefix sum b, the
// chunk-local inclusive prefix maximum of u = li - b, the chunk total and the
// chunk maximum of u; u, b and the prefix maximum also go to copies whose rows
// are padded to 64 tokens, so that 64-token tiles of them can be fetched by
// bulk copies.
__global__ void __launch_bounds__(256)
gate_prologue_kernel(const float *__restrict__ i_pre, const float *__restrict__ f_pre,
                     float *__restrict__ bcum, float *__restrict__ pmx, float2 *__restrict__ cstat,
                     float *__restrict__ upad, float *__restrict__ bpad, float *__restrict__ xpad,
                     int BH, int S, int Spad, int L, int nchunks, int fgate_exp) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= BH * nchunks) return;
    const int bh = warp / nchunks, c = warp - bh * nchunks;
    const int t0 = c * L, t1 = min(S, t0 + L);
    const size_t base = (size_t)bh * S;
    float carry = 0.f, umax = -INFINITY;
    // the next 32 tokens' gates are loaded while this group is scanned
    float nf = t0 + lane < t1 ? f_pre[base + t0 + lane] : 0.f;
    float ni = t0 + lane < t1 ? i_pre[base + t0 + lane] : 0.f;
    for (int t = t0; t < t1; t += 32) {
        const int tt = t + lane;
        const bool ok = tt < t1;
        const float fcur = nf, icur = ni;
        if (t + 32 < t1) {
            nf = tt + 32 < t1 ? f_pre[base + tt + 32] : 0.f;
            ni = tt + 32 < t1 ? i_pre[base + tt + 32] : 0.f;
        }
        float lf = ok ? log_forget(fcur, fgate_exp) : 0.f;
        // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, lf, o);
            if (lane >= o) lf += y;
        }
        const float b = carry + lf;
        const float u_raw = ok ? icur - b : 0.f;
        float u = ok ? u_raw : -INFINITY;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {          // inclusive prefix max of u
            const float y = __shfl_up_sync(0xffffffffu, u, o);
            if (lane >= o) u = fmaxf(u, y);
        }
        u = fmaxf(u, umax);
        if (ok) {
            bcum[base + tt] = b;
            pmx[base + tt] = u;
            upad[(size_t)bh * Spad + tt] = u_raw;
            bpad[(size_t)bh * Spad + tt] = b;
            xpad[(size_t)bh * Spad + tt] = u;
        }
        carry = __shfl_sync(0xffffffffu, b, 31);
        umax = __shfl_sync(0xffffffffu, u, 31);
    }
    if (lane == 0) cstat[(size_t)bh * nchunks + c] = make_float2(carry, umax);
    pdl_launch_dependents();      // the next kernel may be scheduled; it waits for this one
}

// ------------------------------------------------------------------ phase 1
// Segment summary, one CTA per (value-row tile, segment g < P-1, head):
//   E_c   = sum_{c' >= c, c' in segment} btot_c'        (decay from chunk c's end... to segment end, incl. c)
//   mloc  = max_c (cmax_c + E_c)
//   dC[i,j] = sum_s exp(u_s + E_c(s) - mloc) v_s[i] khat_s[j],   dn[j] likewise with khat_s
// Raw units: the segment adds e^{mloc} dC to the state at its end.
template <typename T>
__global__ void __launch_bounds__(256)
segment_summary_simt_kernel(const T *__restrict__ k, const T *__restrict__ v,
                            const float *__restrict__ i_pre, const float *__restrict__ bcum,
                            const float2 *__restrict__ cstat, float2 *__restrict__ sstat,
                            float *__restrict__ summ, int S, int DH, int L, int nchunks,
                            int P, int cps, int rows) {
    extern __shared__ float smem[];
    const int tile = blockIdx.x, g = blockIdx.y, bh = blockIdx.z;
    const int tid = threadIdx.x;
    const int i0 = tile * rows;
    const int nrows = min(rows, DH - i0);
    const int c0 = g * cps, c1 = min(nchunks, c0 + cps);
    const float inv_sqrt_d = rsqrtf((float)DH);
    const int KS = DH + 1;                      // padded row stride of the K block
    float *kb = smem;                           // [16][DH+1]
    float *vb = kb + 16 * KS;                   // [16][rows]
    float *wt = vb + 16 * rows;                 // [16]
    float *acc = wt + 16;                       // [rows][DH] accumulators
    float *nacc = acc + rows * DH;              // [DH]
    __shared__ float s_E[2];

    // segment totals and stabiliser (sequential over this segment's chunks)
    if (tid == 0) {
        float E = 0.f, mloc = -INFINITY;
        for (int c = c1 - 1; c >= c0; --c) {
            const float2 cs = cstat[(size_t)bh * nchunks + c];
            E += cs.x;
            mloc = fmaxf(mloc, cs.y + E);
        }
        s_E[0] = E;       // segment total of log f
        s_E[1] = mloc;
        if (tile == 0) sstat[(size_t)bh * P + g] = make_float2(E, mloc);
    }
    for (int e = tid; e < rows * DH; e += blockDim.x) acc[e] = 0.f;
    for (int e = tid; e < DH; e += blockDim.x) nacc[e] = 0.f;
    __syncthreads();
    const float mloc = s_E[1];

    // suffix sum of chunk totals, walked forward: E_c = Etot - sum_{c' < c} btot_c'
    float Ebefore = 0.f;
    const size_t tok_base = (size_t)bh * S;
    for (int c = c0; c < c1; ++c) {
        const float2 cs = cstat[(size_t)bh * nchunks + c];
        const float Ec = s_E[0] - Ebefore;       // sum over chunks c..c1-1
        Ebefore += cs.x;
        const int t0 = c * L, t1 = min(S, t0 + L);
        for (int tb = t0; tb < t1; tb += 16) {
            const int nt = min(16, t1 - tb);
            __syncthreads();
            for (int e = tid; e < 16 * DH; e += blockDim.x) {
                const int s = e / DH, j = e - s * DH;
                kb[s * KS + j] = s < nt ? to_f32(k[(tok_base + tb + s) * DH + j]) * inv_sqrt_d : 0.f;
            }
            for (int e = tid; e < 16 * rows; e += blockDim.x) {
                const int s = e / rows, i = e - s * rows;
                vb[e] = (s < nt && i < nrows) ? to_f32(v[(tok_base + tb + s) * DH + i0 + i]) : 0.f;
            }
            if (tid < 16) {
                const int s = tid;
                wt[s] = s < nt ? expf(i_pre[tok_base + tb + s] - bcum[tok_base + tb + s] + Ec - mloc) : 0.f;
            }
            __syncthreads();
            for (int e = tid; e < nrows * DH; e += blockDim.x) {
                const int i = e / DH, j = e - i * DH;
                float a = acc[e];
#pragma unroll
                for (int s = 0; s < 16; ++s) a += wt[s] * vb[s * rows + i] * kb[s * KS + j];
                acc[e] = a;
            }
            if (tile == 0) {
                for (int j = tid; j < DH; j += blockDim.x) {
                    float a = nacc[j];
#pragma unroll
                    for (int s = 0; s < 16; ++s) a += wt[s] * kb[s * KS + j];
                    nacc[j] = a;
                }
            }
        }
    }
    __syncthreads();
    float *out = summ + ((size_t)bh * (P - 1) + g) * ((size_t)DH * DH + DH);
    for (int e = tid; e < nrows * DH; e += blockDim.x) out[(size_t)i0 * DH + e] = acc[e];
    if (tile == 0)
        for (int j = tid; j < DH; j += blockDim.x) out[(size_t)DH * DH + j] = nacc[j];
}

// ------------------------------------------------------------------ phase 3
// Outputs, one CTA per (value-row tile, segment, head).  The CTA keeps its
// rows of C' (fp32) and all of n' in shared memory and walks its chunks.
template <typename T>
__global__ void __launch_bounds__(256)
segment_output_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                           const float *__restrict__ i_pre, const float *__restrict__ o_pre,
                           T *__restrict__ h,
                           const float *__restrict__ C0, const float *__restrict__ n0,
                           const float *__restrict__ m0,
                           float *__restrict__ C_out, float *__restrict__ n_out, float *__restrict__ m_out,
                           const float *__restrict__ bcum, const float2 *__restrict__ cstat,
                           const float2 *__restrict__ sstat, const float *__restrict__ summ,
                           int S, int DH, int L, int nchunks, int P, int cps, int rows) {
    extern __shared__ float smem[];
    const int tile = blockIdx.x, g = blockIdx.y, bh = blockIdx.z;
    const int tid = threadIdx.x;
    const int i0 = tile * rows;
    const int nrows = min(rows, DH - i0);
    const float inv_sqrt_d = rsqrtf((float)DH);
    const int KS = DH + 1;
    float *Cs = smem;                       // [rows][DH+1]   C' rows of this tile
    float *ns = Cs + rows * KS;             // [DH]           n'
    float *qb = ns + DH;                    // [16][DH+1]     query block
    float *kb = qb + 16 * KS;               // [16][DH+1]     key block (scaled by 1/sqrt(d))
    float *vb = kb + 16 * KS;               // [16][rows]     value block (tile rows)
    float *pb = vb + 16 * rows;             // [16][16]       decayed scores
    float *num = pb + 256;                  // [16][rows]     intra numerators
    float *inum = num + 16 * rows;          // [16][rows]     inter numerators
    float *den = inum + 16 * rows;          // [16]  intra denominators
    float *iden = den + 16;                 // [16]  inter denominators
    float *gb = iden + 16;                  // [L]   b_t
    float *gu = gb + L;                     // [L]   u_t = li - b
    float *gm = gu + L;                     // [L]   m_t

    const size_t tok_base = (size_t)bh * S;
    // ---- incoming state: initial state folded with the summaries of segments < g
    for (int e = tid; e < nrows * DH; e += blockDim.x) {
        const int i = e / DH, j = e - i * DH;
        Cs[i * KS + j] = C0 ? C0[((size_t)bh * DH + i0 + i) * DH + j] : 0.f;
    }
    for (int j = tid; j < DH; j += blockDim.x) ns[j] = n0 ? n0[(size_t)bh * DH + j] : 0.f;
    float m_cur = m0 ? m0[bh] : 0.f;
    for (int gp = 0; gp < g; ++gp) {
        const float2 st = sstat[(size_t)bh * P + gp];
        const float m_new = fmaxf(st.x + m_cur, st.y);
        const float alpha = expf(st.x + m_cur - m_new), beta = expf(st.y - m_new);
        const float *sm = summ + ((size_t)bh * (P - 1) + gp) * ((size_t)DH * DH + DH);
        __syncthreads();
        for (int e = tid; e < nrows * DH; e += blockDim.x) {
            const int i = e / DH, j = e - i * DH;
            Cs[i * KS + j] = alpha * Cs[i * KS + j] + beta * sm[(size_t)(i0 + i) * DH + j];
        }
        for (int j = tid; j < DH; j += blockDim.x) ns[j] = alpha * ns[j] + beta * sm[(size_t)DH * DH + j];
        m_cur = m_new;
    }
    __syncthreads();

    const int c0 = g * cps, c1 = min(nchunks, c0 + cps);
    for (int c = c0; c < c1; ++c) {
        const int t0 = c * L, t1 = min(S, t0 + L), Lc = t1 - t0;
        // chunk gates: b, u, m_t (prefix max, one warp)
        for (int t = tid; t < Lc; t += blockDim.x) {
            const float b = bcum[tok_base + t0 + t];
            gb[t] = b;
            gu[t] = i_pre[tok_base + t0 + t] - b;
        }
        __syncthreads();
        if (tid < 32) {
            float run = m_cur;
            for (int t = 0; t < Lc; t += 32) {
                const int tt = t + tid;
                float x = tt < Lc ? gu[tt] : -INFINITY;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, o);
                    if (tid >= o) x = fmaxf(x, y);
                }
                x = fmaxf(x, run);
                if (tt < Lc) gm[tt] = gb[tt] + x;
                run = __shfl_sync(0xffffffffu, x, 31);
            }
        }
        __syncthreads();
        const float m_prev = m_cur;

        for (int tq = 0; tq < Lc; tq += 16) {
            const int nq = min(16, Lc - tq);
            for (int e = tid; e < 16 * DH; e += blockDim.x) {
                const int t = e / DH, j = e - t * DH;
                qb[t * KS + j] = t < nq ? to_f32(q[(tok_base + t0 + tq + t) * DH + j]) : 0.f;
            }
            __syncthreads();
            // inter-chunk retrieval from the state at the chunk start
            for (int e = tid; e < 16 * rows; e += blockDim.x) {
                const int t = e / rows, i = e - t * rows;
                float a = 0.f;
                if (i < nrows) {
                    const float *cr = Cs + i * KS, *qr = qb + t * KS;
                    for (int j = 0; j < DH; ++j) a += cr[j] * qr[j];
                }
                inum[e] = a;
                num[e] = 0.f;
            }
            if (tid < 16) {
                float a = 0.f;
                const float *qr = qb + tid * KS;
                for (int j = 0; j < DH; ++j) a += ns[j] * qr[j];
                iden[tid] = a;
                den[tid] = 0.f;
            }
            // intra-chunk: key blocks up to and including the query block
            for (int tk = 0; tk <= tq; tk += 16) {
                const int nk = min(16, Lc - tk);
                __syncthreads();
                for (int e = tid; e < 16 * DH; e += blockDim.x) {
                    const int s = e / DH, j = e - s * DH;
                    kb[s * KS + j] = s < nk ? to_f32(k[(tok_base + t0 + tk + s) * DH + j]) * inv_sqrt_d : 0.f;
                }
                for (int e = tid; e < 16 * rows; e += blockDim.x) {
                    const int s = e / rows, i = e - s * rows;
                    vb[e] = (s < nk && i < nrows) ? to_f32(v[(tok_base + t0 + tk + s) * DH + i0 + i]) : 0.f;
                }
                __syncthreads();
                {
                    const int t = tid >> 4, s = tid & 15;
                    const int tg = tq + t, sg = tk + s;
                    float a = 0.f;
                    if (t < nq && s < nk && sg <= tg) {
                        const float *qr = qb + t * KS, *kr = kb + s * KS;
                        for (int j = 0; j < DH; ++j) a += qr[j] * kr[j];
                        a *= expf(gu[sg] + gb[tg] - gm[tg]);
                    }
                    pb[tid] = a;
                }
                __syncthreads();
                for (int e = tid; e < 16 * rows; e += blockDim.x) {
                    const int t = e / rows, i = e - t * rows;
                    float a = num[e];
#pragma unroll
                    for (int s = 0; s < 16; ++s) a += pb[t * 16 + s] * vb[s * rows + i];
                    num[e] = a;
                }
                if (tid < 16) {
                    float a = den[tid];
#pragma unroll
                    for (int s = 0; s < 16; ++s) a += pb[tid * 16 + s];
                    den[tid] = a;
                }
            }
            __syncthreads();
            // combine, normalise, output gate
            for (int e = tid; e < 16 * rows; e += blockDim.x) {
                const int t = e / rows, i = e - t * rows;
                if (t < nq && i < nrows) {
                    const int tg = tq + t;
                    const float gt = expf(gb[tg] + m_prev - gm[tg]);
                    const float dd = fmaxf(fabsf(gt * iden[t] + den[t]), expf(-gm[tg]));
                    const size_t idx = (tok_base + t0 + tg) * DH + i0 + i;
                    h[idx] = from_f32<T>(sigmoid(o_pre[idx]) * (gt * inum[e] + num[e]) / dd);
                }
            }
            __syncthreads();
        }

        // state update at the chunk end
        const float m_next = gm[Lc - 1];
        const float bL = gb[Lc - 1];
        const float a_decay = expf(bL + m_prev - m_next);
        for (int e = tid; e < nrows * DH; e += blockDim.x) {
            const int i = e / DH, j = e - i * DH;
            Cs[i * KS + j] *= a_decay;
        }
        for (int j = tid; j < DH; j += blockDim.x) ns[j] *= a_decay;
        for (int tk = 0; tk < Lc; tk += 16) {
            const int nk = min(16, Lc - tk);
            __syncthreads();
            for (int e = tid; e < 16 * DH; e += blockDim.x) {
                const int s = e / DH, j = e - s * DH;
                kb[s * KS + j] = s < nk ? to_f32(k[(tok_base + t0 + tk + s) * DH + j]) * inv_sqrt_d : 0.f;
            }
            for (int e = tid; e < 16 * rows; e += blockDim.x) {
                const int s = e / rows, i = e - s * rows;
                vb[e] = (s < nk && i < nrows) ? to_f32(v[(tok_base + t0 + tk + s) * DH + i0 + i]) : 0.f;
            }
            if (tid < 16) pb[tid] = tid < nk ? expf(gu[tk + tid] + bL - m_next) : 0.f;
            __syncthreads();
            for (int e = tid; e < nrows * DH; e += blockDim.x) {
                const int i = e / DH, j = e - i * DH;
                float a = Cs[i * KS + j];
#pragma unroll
                for (int s = 0; s < 16; ++s) a += pb[s] * vb[s * rows + i] * kb[s * KS + j];
                Cs[i * KS + j] = a;
            }
            for (int j = tid; j < DH; j += blockDim.x) {
                float a = ns[j];
#pragma unroll
                for (int s = 0; s < 16; ++s) a += pb[s] * kb[s * KS + j];
                ns[j] = a;
            }
        }
        m_cur = m_next;
        __syncthreads();
    }

    if (g == P - 1) {
        if (C_out)
            for (int e = tid; e < nrows * DH; e += blockDim.x) {
                const int i = e / DH, j = e - i * DH;
                C_out[((size_t)bh * DH + i0 + i) * DH + j] = Cs[i * KS + j];
            }
        if (tile == 0) {
            if (n_out) for (int j = tid; j < DH; j += blockDim.x) n_out[(size_t)bh * DH + j] = ns[j];
            if (m_out && tid == 0) m_out[bh] = m_cur;
        }
    }
}

// --------------------------------------------------------------- launchers
size_t simt_summary_smem(int DH, int rows) {
    return sizeof(float) * (16 * (DH + 1) + 16 * rows + 16 + (size_t)rows * DH + DH);
}
size_t simt_output_smem(int DH, int rows, int L) {
    return sizeof(float) * ((size_t)rows * (DH + 1) + DH + 2 * 16 * (DH + 1) + 16 * rows + 256 +
                            2 * 16 * rows + 32 + 3 * (size_t)L);
}

cudaError_t launch_gate_prologue(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    float *ws = (float *)a.workspace;
    const int warps = p.BH * p.nchunks;
    const int blocks = (warps + 7) / 8;
    KernelTimer timer("gate_prologue", st);
    gate_prologue_kernel<<<blocks, 256, 0, st>>>(a.i_pre, a.f_pre, ws + p.off_bcum, ws + p.off_pmax,
                                                 (float2 *)(ws + p.off_cstat), ws + p.off_upad,
                                                 ws + p.off_bpad, ws + p.off_xpad, p.BH, p.S,
                                                 p.Spad, p.L, p.nchunks, a.fgate_exp);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_simt_t(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    float *ws = (float *)a.workspace;
    const float *bcum = ws + p.off_bcum;
    const float2 *cstat = (const float2 *)(ws + p.off_cstat);
    float2 *sstat = (float2 *)(ws + p.off_sstat);
    float *summ = ws + p.off_summ;
    cudaError_t e;
    if (p.P > 1) {
        const size_t sm1 = simt_summary_smem(p.DH, p.rows);
        e = cudaFuncSetAttribute(segment_summary_simt_kernel<T>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
        if (e != cudaSuccess) return e;
        dim3 g1(p.ntiles, p.P - 1, p.BH);
        KernelTimer timer("segment_summary_simt", st);
        segment_summary_simt_kernel<T><<<g1, 256, sm1, st>>>(
            (const T *)a.k, (const T *)a.v, a.i_pre, bcum, cstat, sstat, summ,
            p.S, p.DH, p.L, p.nchunks, p.P, p.cps, p.rows);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t sm3 = simt_output_smem(p.DH, p.rows, p.L);
    e = cudaFuncSetAttribute(segment_output_simt_kernel<T>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3);
    if (e != cudaSuccess) return e;
    dim3 g3(p.ntiles, p.P, p.BH);
    KernelTimer timer("segment_output_simt", st);
    segment_output_simt_kernel<T><<<g3, 256, sm3, st>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, a.i_pre, a.o_pre, (T *)a.h,
        a.C0, a.n0, a.m0, a.C_out, a.n_out, a.m_out, bcum, cstat, sstat, summ,
        p.S, p.DH, p.L, p.nchunks, p.P, p.cps, p.rows);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_summaries_simt_t(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    float *ws = (float *)a.workspace;
    const size_t sm1 = simt_summary_smem(p.DH, p.rows);
    cudaError_t e = cudaFuncSetAttribute(segment_summary_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    if (e != cudaSuccess) return e;
    KernelTimer timer("segment_summary_simt", st);
    segment_summary_simt_kernel<T><<<dim3(p.ntiles, p.P - 1, p.BH), 256, sm1, st>>>(
        (const T *)a.k, (const T *)a.v, a.i_pre, ws + p.off_bcum, (const float2 *)(ws + p.off_cstat),
        (float2 *)(ws + p.off_sstat), ws + p.off_summ, p.S, p.DH, p.L, p.nchunks, p.P, p.cps, p.rows);
    return cudaGetLastError();
}

cudaError_t launch_segment_summaries_simt(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    if (p.P <= 1) return cudaSuccess;
    if (a.bf16) return launch_summaries_simt_t<__nv_bfloat16>(a, p, st);
    return launch_summaries_simt_t<float>(a, p, st);
}

cudaError_t launch_fwd_simt(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    cudaError_t e = launch_gate_prologue(a, p, st);
    if (e != cudaSuccess) return e;
    if (a.bf16) return launch_simt_t<__nv_bfloat16>(a, p, st);
    return launch_simt_t<float>(a, p, st);
}

}  // namespace xlstm
