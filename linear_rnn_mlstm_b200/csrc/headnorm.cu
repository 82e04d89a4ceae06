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
// and every access is a full 16-byte load or store.  A lane group issues the
// loads of its next rows before it reduces any of them.  The row statistics
// are two butterfly sums over the lane group (mean first, then the centred
// squares, from values held in registers).  Streaming loads and stores keep
// the per-row tensors from displacing the per-channel parameters in L2.  The
// grid is one resident wave of CTAs; each warp strides over the rows.
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace xlstm {
namespace {

constexpr int kThreads = 256;

// Elements per 16-byte vector.
template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };

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

// The gate's logistic function without branches, from CUDA's fast exponential
// and division intrinsics: relative error ~1e-6 for |z| < 10 (far below the
// bf16 output rounding and the fp32 tolerance), exactly 1 at +inf and 0 at
// -inf.  An accurate expf with an IEEE division on each side of a sign branch
// made the gate, not HBM, the limit of this kernel.
__device__ __forceinline__ float external_gate(float z, int silu) {
    const float s = __fdividef(1.f, 1.f + __expf(-z));
    return silu ? z * s : s;
}

// Row r = (b * S + t) * NH + head -> (b, t, head); 32-bit division when the
// row count allows it (the branch is uniform over the grid).
__device__ __forceinline__ void split_row(long long r, int S, int NH, bool narrow, long long &b,
                                          long long &t, int &head) {
    if (narrow) {
        const unsigned ur = (unsigned)r, bt = ur / (unsigned)NH, ub = bt / (unsigned)S;
        head = (int)(ur - bt * (unsigned)NH);
        b = ub;
        t = bt - ub * (unsigned)S;
    } else {
        const long long bt = r / NH;
        head = (int)(r - bt * NH);
        b = bt / S;
        t = bt - b * S;
    }
}

// Rows a lane group takes per pass when each lane holds V 16-byte vectors of a
// row: two vectors of each of h, z and x_skip in flight per lane.  (Four, with
// ~120 registers and two CTAs per SM, measured slower than two with ~66
// registers and three CTAs per SM.)
__host__ __device__ constexpr int rows_per_pass(int V) { return V >= 2 ? 1 : 2 / V; }

// LPR lanes per row, V 16-byte vectors per lane and row (LPR * V * VN >= DH),
// R rows per lane group per pass: every load of a pass is issued before the
// first row's statistics wait on them.
template <typename T, int LPR, int V>
__global__ void __launch_bounds__(kThreads)
headnorm_gate_kernel(const T *__restrict__ h, const float *__restrict__ gamma,
                     const float *__restrict__ beta, const float *__restrict__ skip_w,
                     const T *__restrict__ x_skip, const T *__restrict__ z, T *__restrict__ y,
                     long long rows, int S, int NH, int DH, float eps, int silu) {
    constexpr int VN = Vec<T>::N;
    constexpr int R = rows_per_pass(V);
    constexpr int kRowsPerWarp = 32 / LPR;
    constexpr int kRowsPerPass = kRowsPerWarp * R;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPR;
    const int slot = lane / LPR;
    const int nvec = DH / VN;
    const bool narrow = rows < (1LL << 31);
    const long long warp = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * kThreads) >> 5;

    // `base` is the same for every lane of the warp, so the shuffles below
    // always run with the whole warp.
    for (long long base = warp * kRowsPerPass; base < rows; base += nwarps * kRowsPerPass) {
        uint4 hr[R][V], zr[R][V], xr[R][V];
        size_t yoff[R];
        int head[R];
        bool valid[R];
#pragma unroll
        for (int j = 0; j < R; ++j) {
            const long long r = base + j * kRowsPerWarp + slot;
            valid[j] = r < rows;
            long long b = 0, t = 0;
            head[j] = 0;
            if (valid[j]) split_row(r, S, NH, narrow, b, t, head[j]);
            const T *hrow = h + (((size_t)b * NH + head[j]) * S + t) * DH;
            yoff[j] = (size_t)(valid[j] ? r : 0) * DH;
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const int v = sub + k * LPR;
                hr[j][k] = zr[j][k] = xr[j][k] = make_uint4(0, 0, 0, 0);
                if (valid[j] && v < nvec) {
                    hr[j][k] = __ldcs(reinterpret_cast<const uint4 *>(hrow) + v);
                    zr[j][k] = __ldcs(reinterpret_cast<const uint4 *>(z + yoff[j]) + v);
                    if (x_skip)
                        xr[j][k] = __ldcs(reinterpret_cast<const uint4 *>(x_skip + yoff[j]) + v);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < R; ++j) {
            // vectors that were not loaded are zero and add nothing to the sum
            float hv[V][VN];
            float sum = 0.f;
#pragma unroll
            for (int k = 0; k < V; ++k) {
                unpack<T>(hr[j][k], hv[k]);
#pragma unroll
                for (int e = 0; e < VN; ++e) sum += hv[k][e];
            }
            // true divisions: a constant row gives exactly its value as the mean
            const float mean = group_sum<LPR>(sum) / (float)DH;
            float sq = 0.f;
#pragma unroll
            for (int k = 0; k < V; ++k) {
                if (sub + k * LPR < nvec) {
#pragma unroll
                    for (int e = 0; e < VN; ++e) {
                        const float d = hv[k][e] - mean;
                        sq += d * d;
                    }
                }
            }
            const float rstd = rsqrtf(group_sum<LPR>(sq) / (float)DH + eps);

#pragma unroll
            for (int k = 0; k < V; ++k) {
                const int v = sub + k * LPR;
                if (!valid[j] || v >= nvec) continue;
                const int c0 = head[j] * DH + v * VN;
                float zf[VN], xf[VN], out[VN];
                unpack<T>(zr[j][k], zf);
                unpack<T>(xr[j][k], xf);
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
                __stcs(reinterpret_cast<uint4 *>(y + yoff[j]) + v, pack<T>(out));
            }
        }
    }
}

int lanes_per_row(int nvec) {
    int l = 1;
    while (l < nvec && l < 32) l <<= 1;
    return l;
}

// CTAs of one instantiation resident per SM (registers decide it); the grid is
// one full wave of them and each warp strides over the rows.  Cached after the
// first query; host threads that race on the cache all store the same value.
template <typename T, int LPR, int V> int resident_blocks() {
    static int n = 0;
    if (n == 0) {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, headnorm_gate_kernel<T, LPR, V>,
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
    const int nvec = DH / Vec<T>::N;
    const int lpr = lanes_per_row(nvec);
    int vpl = (nvec + lpr - 1) / lpr;                 // vectors per lane: 1, 2, 3 or 4
    if (vpl == 3) vpl = 4;
    const int num_sms = num_sms_current_device();
    KernelTimer timer("headnorm_gate", st);
#define XLSTM_HN_CASE(L, V)                                                                    \
    if (lpr == L && vpl == V) {                                                                \
        const long long per_block = (long long)(kThreads / 32) * (32 / L) * rows_per_pass(V);  \
        const long long needed = (rows + per_block - 1) / per_block;                           \
        const long long wave = (long long)num_sms * resident_blocks<T, L, V>();               \
        const dim3 grid((unsigned)(needed < wave ? needed : wave));                            \
        headnorm_gate_kernel<T, L, V><<<grid, kThreads, 0, st>>>(h, gamma, beta, skip_w,       \
                                                                 x_skip, z, y, rows, S, NH, DH, \
                                                                 eps, silu);                   \
        return cudaGetLastError();                                                             \
    }
    XLSTM_HN_CASE(2, 1)
    XLSTM_HN_CASE(4, 1)
    XLSTM_HN_CASE(8, 1)
    XLSTM_HN_CASE(16, 1)
    XLSTM_HN_CASE(32, 1)
    XLSTM_HN_CASE(32, 2)
    XLSTM_HN_CASE(32, 4)
    return cudaErrorInvalidValue;
#undef XLSTM_HN_CASE
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
    CallRange range("xlstm_mlstm_headnorm_gate");
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
