// Block epilogue of the mLSTM cell: per-head GroupNorm, learnable skip and the
// external output gate ("xLSTM: Extended Long Short-Term Memory" section 2.4,
// Figure 10), in one pass over HBM that also turns the cell's [B, NH, S, DH]
// layout into the block's [B, S, NH*DH].
//
// Per token and head (a "row" of DH channels, channel c = head*DH + j):
//   mean, biased variance over the row (GroupNorm with one group per head,
//   Wu & He), xn = (h - mean) * rsqrt(var + eps),
//   y = (xn * gamma[c] + beta[c] + skip_w[c] * x_skip[c]) * act(z[c]),
//   act = z*sigmoid(z) (SiLU) or sigmoid(z).
//
// The op moves 4 * DH elements per row (h, x_skip, z in; y out) and does O(DH)
// arithmetic, so it is bound by HBM bandwidth.  Each row is one contiguous run
// of DH elements in every tensor; a group of LPR lanes (a power of two, up to
// a warp) covers a row with 16-byte vectors, so a warp handles 32 / LPR rows
// and every access is a full 16-byte load or store.  The row statistics are
// two butterfly sums over the lane group (mean first, then the centred squares,
// from values held in registers).  Streaming loads and stores keep the
// per-row tensors from displacing the per-channel parameters in L2.
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace xlstm {
namespace {

constexpr int kThreads = 256;
constexpr int kNumSms = 148;           // B200

// Elements per 16-byte vector, and the most vectors one lane holds (DH <= 512).
template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; static constexpr int kMax = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; static constexpr int kMax = 2; };

template <typename T> __device__ __forceinline__ void unpack(const uint4 &u, float *f);
template <> __device__ __forceinline__ void unpack<float>(const uint4 &u, float *f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
// bf16 pairs: the element with the lower index sits in the low half of each word
template <> __device__ __forceinline__ void unpack<__nv_bfloat16>(const uint4 &u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

template <typename T> __device__ __forceinline__ uint4 pack(const float *f);
template <> __device__ __forceinline__ uint4 pack<float>(const float *f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}
template <> __device__ __forceinline__ uint4 pack<__nv_bfloat16>(const float *f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(f[2 * i]));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(f[2 * i + 1]));
        w[i] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Sum over the aligned group of LPR lanes this lane belongs to.
template <int LPR> __device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float external_gate(float z, int silu) {
    const float s = sigmoid(z);
    return silu ? z * s : s;
}

template <typename T, int LPR>
__global__ void __launch_bounds__(kThreads)
headnorm_gate_kernel(const T *__restrict__ h, const float *__restrict__ gamma,
                     const float *__restrict__ beta, const float *__restrict__ skip_w,
                     const T *__restrict__ x_skip, const T *__restrict__ z, T *__restrict__ y,
                     long long rows, int S, int NH, int DH, float eps, int silu) {
    constexpr int VN = Vec<T>::N;
    constexpr int kMaxV = Vec<T>::kMax;
    constexpr int kRowsPerWarp = 32 / LPR;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPR;
    const int slot = lane / LPR;
    const int nvec = DH / VN;
    const long long warp = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * kThreads) >> 5;

    // `base` is the same for every lane of the warp, so the shuffles below
    // always run with the whole warp.
    for (long long base = warp * kRowsPerWarp; base < rows; base += nwarps * kRowsPerWarp) {
        const long long r = base + slot;          // r = (b * S + t) * NH + head
        const bool valid = r < rows;
        const long long bt = valid ? r / NH : 0;
        const int head = valid ? (int)(r - bt * NH) : 0;
        const long long b = bt / S, t = bt - b * S;
        const T *hrow = h + (((size_t)b * NH + head) * S + t) * DH;
        const size_t yoff = (size_t)(valid ? r : 0) * DH;

        float hv[kMaxV][VN];
        uint4 zr[kMaxV], xr[kMaxV];
        float sum = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxV; ++k) {
            const int v = sub + k * LPR;
            zr[k] = make_uint4(0, 0, 0, 0);
            xr[k] = make_uint4(0, 0, 0, 0);
            if (valid && v < nvec) {
                unpack<T>(__ldcs(reinterpret_cast<const uint4 *>(hrow) + v), hv[k]);
                zr[k] = __ldcs(reinterpret_cast<const uint4 *>(z + yoff) + v);
                if (x_skip) xr[k] = __ldcs(reinterpret_cast<const uint4 *>(x_skip + yoff) + v);
            } else {
#pragma unroll
                for (int e = 0; e < VN; ++e) hv[k][e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < VN; ++e) sum += hv[k][e];
        }
        // true divisions: a constant row gives exactly its value as the mean
        const float mean = group_sum<LPR>(sum) / (float)DH;
        float sq = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxV; ++k) {
            if (valid && sub + k * LPR < nvec) {
#pragma unroll
                for (int e = 0; e < VN; ++e) {
                    const float d = hv[k][e] - mean;
                    sq += d * d;
                }
            }
        }
        const float rstd = rsqrtf(group_sum<LPR>(sq) / (float)DH + eps);

#pragma unroll
        for (int k = 0; k < kMaxV; ++k) {
            const int v = sub + k * LPR;
            if (!valid || v >= nvec) continue;
            const int c0 = head * DH + v * VN;
            float zf[VN], xf[VN], out[VN];
            unpack<T>(zr[k], zf);
            unpack<T>(xr[k], xf);
#pragma unroll
            for (int e = 0; e < VN; e += 4) {
                const float4 g = __ldg(reinterpret_cast<const float4 *>(gamma + c0 + e));
                const float4 bb = __ldg(reinterpret_cast<const float4 *>(beta + c0 + e));
                float4 sw = make_float4(0.f, 0.f, 0.f, 0.f);
                if (x_skip) sw = __ldg(reinterpret_cast<const float4 *>(skip_w + c0 + e));
                const float gs[4] = {g.x, g.y, g.z, g.w}, bs[4] = {bb.x, bb.y, bb.z, bb.w},
                            ss[4] = {sw.x, sw.y, sw.z, sw.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float xn = (hv[k][e + i] - mean) * rstd;
                    out[e + i] = (xn * gs[i] + bs[i] + ss[i] * xf[e + i]) *
                                 external_gate(zf[e + i], silu);
                }
            }
            __stcs(reinterpret_cast<uint4 *>(y + yoff) + v, pack<T>(out));
        }
    }
}

int lanes_per_row(int nvec) {
    int l = 1;
    while (l < nvec && l < 32) l <<= 1;
    return l;
}

// CTAs of one instantiation resident per SM (registers decide it); the grid is
// one full wave of them and each warp strides over the rows.
template <typename T, int LPR> int resident_blocks() {
    static int n = 0;
    if (n == 0) {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, headnorm_gate_kernel<T, LPR>,
                                                          kThreads, 0) != cudaSuccess || b < 1)
            b = 1;
        n = b;
    }
    return n;
}

template <typename T>
cudaError_t launch_typed(const T *h, const float *gamma, const float *beta, const float *skip_w,
                         const T *x_skip, const T *z, T *y, long long rows, int S, int NH, int DH,
                         float eps, int silu, cudaStream_t st) {
    const int lpr = lanes_per_row(DH / Vec<T>::N);
    const long long rows_per_block = (long long)(kThreads / 32) * (32 / lpr);
    const long long needed = (rows + rows_per_block - 1) / rows_per_block;
    KernelTimer timer("headnorm_gate", st);
#define XLSTM_HN_CASE(L)                                                                       \
    case L: {                                                                                  \
        const long long wave = (long long)kNumSms * resident_blocks<T, L>();                  \
        const dim3 grid((unsigned)(needed < wave ? needed : wave));                            \
        headnorm_gate_kernel<T, L><<<grid, kThreads, 0, st>>>(h, gamma, beta, skip_w, x_skip, \
                                                              z, y, rows, S, NH, DH, eps, silu); \
        break;                                                                                 \
    }
    switch (lpr) {
        XLSTM_HN_CASE(2)
        XLSTM_HN_CASE(4)
        XLSTM_HN_CASE(8)
        XLSTM_HN_CASE(16)
        XLSTM_HN_CASE(32)
        default: return cudaErrorInvalidValue;
    }
#undef XLSTM_HN_CASE
    return cudaGetLastError();
}

bool misaligned16(const void *p) { return ((uintptr_t)p & 15u) != 0; }

}  // namespace
}  // namespace xlstm

extern "C" xlstm_status xlstm_mlstm_headnorm_gate(const void *h, const float *gamma,
                                                  const float *beta, const float *skip_w,
                                                  const void *x_skip, const void *z, void *y,
                                                  int B, int NH, int S, int DH, float eps,
                                                  xlstm_dtype dt, xlstm_ogate og,
                                                  void *cuda_stream) {
    using namespace xlstm;
    if (dt != XLSTM_F32 && dt != XLSTM_BF16) return XLSTM_ERR_DTYPE;
    if (og != XLSTM_OGATE_SILU && og != XLSTM_OGATE_SIGMOID) return XLSTM_ERR_DTYPE;
    if (B < 0 || NH < 0 || S < 0) return XLSTM_ERR_SHAPE;
    if (DH < 16 || DH > 512 || DH % 16 != 0) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH * S * DH > (1LL << 40)) return XLSTM_ERR_SHAPE;
    if (!(eps > 0.f) || !(eps < INFINITY)) return XLSTM_ERR_UNSUPPORTED;
    const long long rows = (long long)B * S * NH;
    if (rows == 0) return XLSTM_OK;
    if (!h || !gamma || !beta || !z || !y) return XLSTM_ERR_NULL;
    if ((skip_w == nullptr) != (x_skip == nullptr)) return XLSTM_ERR_NULL;
    const void *ptrs[] = {h, gamma, beta, skip_w, x_skip, z, y};
    for (const void *p : ptrs)
        if (misaligned16(p)) return XLSTM_ERR_ALIGN;
    if (y == h || y == z || y == x_skip || y == (const void *)gamma || y == (const void *)beta ||
        (skip_w && y == (const void *)skip_w))
        return XLSTM_ERR_UNSUPPORTED;
    const int silu = og == XLSTM_OGATE_SILU;
    cudaStream_t st = (cudaStream_t)cuda_stream;
    cudaError_t e;
    if (dt == XLSTM_BF16) {
        using T = __nv_bfloat16;
        e = launch_typed<T>((const T *)h, gamma, beta, skip_w, (const T *)x_skip, (const T *)z,
                            (T *)y, rows, S, NH, DH, eps, silu, st);
    } else {
        e = launch_typed<float>((const float *)h, gamma, beta, skip_w, (const float *)x_skip,
                                (const float *)z, (float *)y, rows, S, NH, DH, eps, silu, st);
    }
    return e == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}
