// One-token mLSTM decode step: an HBM stream over the resident fp32 state.
//
// Per (b, h), with the recurrence of "xLSTM: Extended Long Short-Term Memory"
// section 2.3 (gated covariance rule, normaliser floored at 1.0) stabilised as
// in section 2.2:
//   m  = max(log f + m_prev, itilde);  f' = e^{log f + m_prev - m};  i' = e^{itilde - m}
//   C' <- f' C' + i' v khat^T          (in place, fp32, [value row, key column])
//   n' <- f' n' + i' khat
//   h  = sigmoid(otilde) * (C' q) / max(|n'.q|, e^{-m})
// The state is 4 * DH^2 bytes per head and is read and written exactly once;
// everything else is O(DH).  Section 2.5 of the paper: constant memory in the
// sequence length, so a decode step is a pure stream of the state.
//
// Two launches per step: step_rows_kernel splits each head's rows over several
// CTAs (so the grid has many more CTAs than SMs and the tail wave is short)
// and reads the OLD n' and m to form the shared denominator
//   n'_new . q = f' (n'_old . q) + i' (khat . q);
// step_state_kernel then overwrites n' and m.  Keeping the two apart avoids
// any CTA reading n'/m after another CTA wrote them.
#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace xlstm {

constexpr int kStepThreads = 256;          // 8 warps
constexpr int kStepRowsPerWarp = 8;
constexpr int kStepRowsPerCta = kStepRowsPerWarp * (kStepThreads / 32);
constexpr int kStepRowGroup = 4;           // rows in flight per warp

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ void load(const float *p, float (&x)[4]) {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&x)[4]) {
        const uint2 t = __ldg(reinterpret_cast<const uint2 *>(p));
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&t.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&t.y);
        const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
    }
};

__device__ __forceinline__ void step_gates(float i_pre, float f_pre, float m_old, int fgate_exp,
                                           float &m_new, float &fp, float &ip) {
    const float lf = log_forget(f_pre, fgate_exp);
    m_new = fmaxf(lf + m_old, i_pre);
    fp = expf(lf + m_old - m_new);
    ip = expf(i_pre - m_new);
}

// NV = number of 128-column groups a lane covers (ceil(DH / 128)).
template <typename T, int NV>
__global__ void __launch_bounds__(kStepThreads)
step_rows_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const float *__restrict__ i_pre, const float *__restrict__ f_pre,
                 const float *__restrict__ o_pre, T *__restrict__ h,
                 float *__restrict__ C, const float *__restrict__ n, const float *__restrict__ m,
                 int DH, int fgate_exp) {
    const int bh = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float inv_sqrt_d = rsqrtf((float)DH);

    float m_new, fp, ip;
    step_gates(i_pre[bh], f_pre[bh], m[bh], fgate_exp, m_new, fp, ip);

    // this lane's columns: j = 4*lane + 128*u
    float kh[NV][4], qv[NV][4];
    float nq = 0.f, kq = 0.f;
    const size_t vec = (size_t)bh * DH;
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int j = 4 * lane + 128 * u;
        if (j < DH) {
            Vec4<T>::load(k + vec + j, kh[u]);
            Vec4<T>::load(q + vec + j, qv[u]);
            float nn[4];
            Vec4<float>::load(n + vec + j, nn);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                kh[u][e] *= inv_sqrt_d;
                nq += nn[e] * qv[u][e];
                kq += kh[u][e] * qv[u][e];
            }
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) { kh[u][e] = 0.f; qv[u][e] = 0.f; }
        }
    }
    nq = warp_sum(nq);
    kq = warp_sum(kq);
    const float denom = fmaxf(fabsf(fp * nq + ip * kq), expf(-m_new));
    const float inv_denom = 1.f / denom;

    const int row0 = blockIdx.x * kStepRowsPerCta + warp * kStepRowsPerWarp;
    float *Cb = C + (size_t)bh * DH * DH;
#pragma unroll 1
    for (int rg = 0; rg < kStepRowsPerWarp; rg += kStepRowGroup) {
        float4 c[kStepRowGroup][NV];
        float vr[kStepRowGroup];
#pragma unroll
        for (int r = 0; r < kStepRowGroup; ++r) {
            const int row = row0 + rg + r;
            const bool okr = row < DH;
            vr[r] = okr ? to_f32(v[vec + row]) * ip : 0.f;
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const int j = 4 * lane + 128 * u;
                if (okr && j < DH)
                    c[r][u] = __ldcs(reinterpret_cast<const float4 *>(Cb + (size_t)row * DH + j));
                else
                    c[r][u] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        float part[kStepRowGroup];
#pragma unroll
        for (int r = 0; r < kStepRowGroup; ++r) {
            const int row = row0 + rg + r;
            float acc = 0.f;
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                float4 x = c[r][u];
                x.x = fp * x.x + vr[r] * kh[u][0];
                x.y = fp * x.y + vr[r] * kh[u][1];
                x.z = fp * x.z + vr[r] * kh[u][2];
                x.w = fp * x.w + vr[r] * kh[u][3];
                acc += x.x * qv[u][0] + x.y * qv[u][1] + x.z * qv[u][2] + x.w * qv[u][3];
                const int j = 4 * lane + 128 * u;
                if (row < DH && j < DH)
                    __stcs(reinterpret_cast<float4 *>(Cb + (size_t)row * DH + j), x);
            }
            part[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < kStepRowGroup; ++r) part[r] = warp_sum(part[r]);
        if (lane < kStepRowGroup) {
            float mine = part[0];
#pragma unroll
            for (int r = 1; r < kStepRowGroup; ++r) if (lane == r) mine = part[r];
            const int row = row0 + rg + lane;
            if (row < DH)
                h[vec + row] = from_f32<T>(sigmoid(o_pre[vec + row]) * mine * inv_denom);
        }
    }
}

// n' <- f' n' + i' khat and m <- m_new, after step_rows_kernel has read them.
template <typename T>
__global__ void __launch_bounds__(128)
step_state_kernel(const T *__restrict__ k, const float *__restrict__ i_pre,
                  const float *__restrict__ f_pre, float *__restrict__ n, float *__restrict__ m,
                  int DH, int fgate_exp) {
    const int bh = blockIdx.x;
    float m_new, fp, ip;
    step_gates(i_pre[bh], f_pre[bh], m[bh], fgate_exp, m_new, fp, ip);
    const float inv_sqrt_d = rsqrtf((float)DH);
    const size_t vec = (size_t)bh * DH;
    for (int j = threadIdx.x; j < DH; j += blockDim.x)
        n[vec + j] = fp * n[vec + j] + ip * to_f32(k[vec + j]) * inv_sqrt_d;
    __syncthreads();                       // every thread has read m[bh] before it changes
    if (threadIdx.x == 0) m[bh] = m_new;
}

template <typename T, int NV>
static cudaError_t launch_rows(const StepArgs &a, cudaStream_t st) {
    dim3 grid((a.DH + kStepRowsPerCta - 1) / kStepRowsPerCta, a.BH);
    KernelTimer timer("step_rows", st);
    step_rows_kernel<T, NV><<<grid, kStepThreads, 0, st>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, a.i_pre, a.f_pre, a.o_pre, (T *)a.h,
        a.C, a.n, a.m, a.DH, a.fgate_exp);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_step_t(const StepArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int nv = (a.DH + 127) / 128;
    switch (nv) {
        case 1: e = launch_rows<T, 1>(a, st); break;
        case 2: e = launch_rows<T, 2>(a, st); break;
        case 3: e = launch_rows<T, 3>(a, st); break;
        default: e = launch_rows<T, 4>(a, st); break;
    }
    if (e != cudaSuccess) return e;
    KernelTimer timer("step_state", st);
    step_state_kernel<T><<<a.BH, 128, 0, st>>>((const T *)a.k, a.i_pre, a.f_pre, a.n, a.m, a.DH,
                                               a.fgate_exp);
    return cudaGetLastError();
}

cudaError_t launch_step(const StepArgs &a, cudaStream_t st) {
    if (a.bf16) return launch_step_t<__nv_bfloat16>(a, st);
    return launch_step_t<float>(a, st);
}

}  // namespace xlstm
