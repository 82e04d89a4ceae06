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
// Two launches per step.  The row update reads the OLD n' and m to form the
// shared denominator
//   n'_new . q = f' (n'_old . q) + i' (khat . q);
// for DH a multiple of 128 it is step_stream_kernel (the state streamed through
// shared memory by bulk copies), else step_rows_kernel (rows split over CTAs,
// staged in registers).  step_state_kernel then overwrites n' and m.  Keeping
// the two apart avoids any CTA reading n'/m after another CTA wrote them.
#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "tc_ptx.cuh"

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

// The same row update for DH a multiple of 128, with the state streamed through
// shared memory by bulk copies: each CTA owns 128 consecutive rows of one head
// and moves them in 8 KB stages (4, 8 or 16 rows) through a ring of kRing
// stages.  One thread issues the bulk loads (and, after the update, the bulk
// stores of the same stage); the CTA's 256 threads each update 8 consecutive
// floats of one row per stage.  Bytes in flight per SM are set by the ring, not
// by registers.  Every wait is bounded and latches the device status word.
namespace ts = xlstm::tc;
constexpr int kStreamRows = 128;           // rows of a head per CTA
constexpr int kStageBytes = 8192;          // one bulk copy
constexpr int kRing = 6;                   // stages in flight

template <typename T>
__global__ void __launch_bounds__(256)
step_stream_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const float *__restrict__ i_pre, const float *__restrict__ f_pre,
                   const float *__restrict__ o_pre, T *__restrict__ h,
                   float *__restrict__ C, const float *__restrict__ n, const float *__restrict__ m,
                   int DH, int fgate_exp, unsigned int *status) {
    extern __shared__ __align__(128) uint8_t st_smem[];
    float *ring = reinterpret_cast<float *>(st_smem);                           // kRing x 2048 floats
    uint64_t *full = reinterpret_cast<uint64_t *>(st_smem + kRing * kStageBytes);
    float *part = reinterpret_cast<float *>(full + kRing);                        // [256] row partial sums
    __shared__ int abort_flag;
    __shared__ float s_red[2];

    const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
    const int rows_per_stage = kStageBytes / (4 * DH);       // 4, 8 or 16
    const int tpr = DH / 8;                                   // threads per row: 64, 32 or 16
    const int nstage = kStreamRows / rows_per_stage;
    const int row_base = blockIdx.x * kStreamRows;
    float *Cb = C + ((size_t)bh * DH + row_base) * DH;        // this CTA's 128 rows, contiguous
    const size_t vec = (size_t)bh * DH;
    const float inv_sqrt_d = rsqrtf((float)DH);

    if (tid == 0) {
        for (int s = 0; s < kRing; ++s) ts::mbar_init(&full[s], 1);
        abort_flag = 0;
        ts::fence_mbar_init();
    }
    __syncthreads();
    int issued = 0;                           // bulk loads issued (thread 0)
    auto load_stage = [&](int s) {            // thread 0 only
        ++issued;
        float *dst = ring + (s % kRing) * (kStageBytes / 4);
        ts::mbar_arrive_expect_tx(&full[s % kRing], kStageBytes);
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     ::"r"(ts::smem_u32(dst)), "l"(Cb + (size_t)s * (kStageBytes / 4)), "r"(kStageBytes),
                     "r"(ts::smem_u32(&full[s % kRing])) : "memory");
    };
    if (tid == 0)
        for (int s = 0; s < min(kRing - 1, nstage); ++s) load_stage(s);

    float m_new, fp, ip;
    step_gates(i_pre[bh], f_pre[bh], m[bh], fgate_exp, m_new, fp, ip);
    // this thread's 8 columns (the same in every stage) and its row inside a stage
    const int col = 8 * (tid % tpr), rin = tid / tpr;
    float kh[8], qv[8];
    float nq = 0.f, kq = 0.f;
    {
        float a[4], b[4];
        Vec4<T>::load(k + vec + col, a); Vec4<T>::load(k + vec + col + 4, b);
        float c4[4], d4[4];
        Vec4<T>::load(q + vec + col, c4); Vec4<T>::load(q + vec + col + 4, d4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            kh[e] = a[e] * inv_sqrt_d; kh[e + 4] = b[e] * inv_sqrt_d;
            qv[e] = c4[e]; qv[e + 4] = d4[e];
        }
        if (rin == 0) {                      // the first row's threads cover every column once
            float nn[4], nm[4];
            Vec4<float>::load(n + vec + col, nn); Vec4<float>::load(n + vec + col + 4, nm);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                nq += nn[e] * qv[e] + nm[e] * qv[e + 4];
                kq += kh[e] * qv[e] + kh[e + 4] * qv[e + 4];
            }
        }
    }
    nq = warp_sum(nq);
    kq = warp_sum(kq);
    if (tid < tpr && lane == 0) { part[tid >> 5] = nq; part[8 + (tid >> 5)] = kq; }
    __syncthreads();
    if (tid == 0) {
        float a = 0.f, b = 0.f;
        for (int w = 0; w < (tpr + 31) / 32; ++w) { a += part[w]; b += part[8 + w]; }
        s_red[0] = a; s_red[1] = b;
    }
    __syncthreads();
    const float inv_denom = 1.f / fmaxf(fabsf(fp * s_red[0] + ip * s_red[1]), expf(-m_new));
    __syncthreads();                          // part[] is reused below

    bool ok = true;
    for (int s = 0; s < nstage; ++s) {
        if (tid == 0 && s + kRing - 1 < nstage) {
            // the slot refilled here held stage s - 1, whose bulk store (the latest
            // group) must have finished reading it
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            load_stage(s + kRing - 1);
        }
        const bool got = ts::mbar_wait(&full[s % kRing], (s / kRing) & 1, &abort_flag, status);
        if (!__syncthreads_and(got)) { ok = false; break; }
        float *st = ring + (s % kRing) * (kStageBytes / 4);
        const int row = row_base + s * rows_per_stage + rin;          // row of the head
        const float vr = to_f32(v[vec + row]) * ip;
        float4 *cp = reinterpret_cast<float4 *>(st + rin * DH + col);
        float4 x0 = cp[0], x1 = cp[1];
        x0.x = fp * x0.x + vr * kh[0]; x0.y = fp * x0.y + vr * kh[1];
        x0.z = fp * x0.z + vr * kh[2]; x0.w = fp * x0.w + vr * kh[3];
        x1.x = fp * x1.x + vr * kh[4]; x1.y = fp * x1.y + vr * kh[5];
        x1.z = fp * x1.z + vr * kh[6]; x1.w = fp * x1.w + vr * kh[7];
        cp[0] = x0; cp[1] = x1;
        float acc = x0.x * qv[0] + x0.y * qv[1] + x0.z * qv[2] + x0.w * qv[3] +
                    x1.x * qv[4] + x1.y * qv[5] + x1.z * qv[6] + x1.w * qv[7];
        // row sums over the row's tpr threads: two warps, one warp, or a half warp
        if (tpr >= 32) {
            acc = warp_sum(acc);
            if (lane == 0) part[tid >> 5] = acc;
        } else {
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if ((lane & 15) == 0) part[tid >> 4] = acc;
        }
        ts::fence_async_smem();               // the updated stage leaves by bulk store
        __syncthreads();
        if (tid == 0) {
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                         ::"l"(Cb + (size_t)s * (kStageBytes / 4)), "r"(ts::smem_u32(st)), "r"(kStageBytes)
                         : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        if (tid < rows_per_stage) {           // h for this stage's rows
            const int r = row_base + s * rows_per_stage + tid;
            const float dot = tpr == 64 ? part[2 * tid] + part[2 * tid + 1] : part[tid];
            h[vec + r] = from_f32<T>(sigmoid(o_pre[vec + r]) * dot * inv_denom);
        }
        __syncthreads();                      // part[] is rewritten by the next stage
    }
    if (tid == 0) {                           // nothing in flight at exit
        if (!ok) {
            // Loads issued but maybe not consumed.  One deadline (200 ms) covers
            // the whole drain rather than a full wait per stage; the status word
            // is already latched, and the call's outputs are undefined.
            const uint64_t deadline = ts::globaltimer_ns() + 200000000ull;
            for (int t = max(0, issued - kRing); t < issued; ++t) {
                const uint64_t now = ts::globaltimer_ns();
                const uint64_t left = now < deadline ? deadline - now : 0ull;
                ts::mbar_wait(&full[t % kRing], (t / kRing) & 1, nullptr, status, left);
            }
        }
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
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
static cudaError_t launch_stream(const StepArgs &a, cudaStream_t st) {
    const int sm = kRing * kStageBytes + kRing * 8 + 256 * 4;
    cudaError_t e = cudaFuncSetAttribute(step_stream_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    KernelTimer timer("step_rows", st);
    step_stream_kernel<T><<<dim3(a.DH / kStreamRows, a.BH), 256, sm, st>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, a.i_pre, a.f_pre, a.o_pre, (T *)a.h,
        a.C, a.n, a.m, a.DH, a.fgate_exp, a.status);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_step_t(const StepArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int nv = (a.DH + 127) / 128;
    if (a.DH % kStreamRows == 0) {
        e = launch_stream<T>(a, st);          // DH 128, 256, 512: bulk-copy stream
    } else {
        switch (nv) {
            case 1: e = launch_rows<T, 1>(a, st); break;
            case 2: e = launch_rows<T, 2>(a, st); break;
            case 3: e = launch_rows<T, 3>(a, st); break;
            default: e = launch_rows<T, 4>(a, st); break;
        }
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
