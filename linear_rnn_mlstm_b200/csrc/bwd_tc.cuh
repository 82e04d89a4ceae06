// Tensor-core products of the backward with the chunk states (included by
// bwd.cu; bf16 inputs, DH 128 or 256).
//
// The chunkwise backward of "xLSTM: Extended Long Short-Term Memory" (section
// 2.3's recurrence, stabiliser held fixed per section 2.2) multiplies every
// chunk's tokens by two DH x DH states: the forward state C'_c at the chunk's
// start and the reverse state dC~_c at its end.  Per chunk c these are four
// [tokens x DH] x [DH x DH] products:
//   num'_inter[t] = C'_c q_t         dq_inter[t] = C'_c^T dnum'_t
//   dk_inter[s]   = dC~_c^T v_s      dv_inter[s] = dC~_c k_s
// Each runs here as tcgen05 MMAs with an fp32 accumulator in tensor memory:
// one CTA per (chunk, 128 output columns, head) forms out^T[m][t] = sum_k
// A[m][k] B[t][k] with M = 128, N = 64 tokens, K = DH.  The state is A, stored
// by the state kernels as two bf16 planes (x = high + low, 16 significant bits)
// in 128 x 64 blocks with 128-byte swizzle, and read by bulk copies: as a
// K-major operand for C'_c q and dC~_c k, as an MN-major one (the same bytes)
// for C'_c^T dnum' and dC~_c^T v.  B is the chunk's 64 token rows of q, k, v
// (exact in bf16) or of dnum' as high and low bf16 planes, fetched by TMA with
// the same swizzle.  Products: A_hi B + A_lo B (+ A_hi B_lo for dnum'), fp32
// accumulation.  Token rows past the chunk (the next chunk's, or zeros past
// the sequence) are computed and not stored.
#pragma once

#include "tc_ptx.cuh"

namespace xlstm {
namespace bwdtc {

// Byte offset of element (r, j) of a DH x DH state inside one of its bf16
// planes: 128-row x 64-column blocks of 16 KB, block (r / 128, j / 64) at
// index (r / 128) * (DH / 64) + j / 64, rows 128 bytes apart, the 16-byte
// piece p of row rr stored at p ^ (rr & 7) (the order of a 64-column TMA box
// with 128-byte swizzle).
__host__ __device__ inline uint32_t plane_offset(int r, int j, int DH) {
    const int rr = r & 127;
    const uint32_t blk = (uint32_t)((r >> 7) * (DH >> 6) + (j >> 6));
    return blk * 16384u + (uint32_t)rr * 128u + ((uint32_t)(((j & 63) >> 3) ^ (rr & 7)) << 4) +
           ((uint32_t)(j & 7) << 1);
}

constexpr int kMmaThreads = 128;

template <int D, bool B_SPLIT>
struct MmaLay {
    static constexpr int kAtoms = D / 64;               // 64-wide K blocks
    static constexpr int kAPlane = kAtoms * 16384;      // one plane of this CTA's 128 A rows
    static constexpr int kBPlane = kAtoms * 8192;       // 64 token rows x D, bf16
    static constexpr int kA = 0;
    static constexpr int kB = 2 * kAPlane;
    static constexpr int kBar = kB + (B_SPLIT ? 2 : 1) * kBPlane;
    static constexpr int kBytes = kBar + 64 + 1024;     // barriers, TMEM slot, flag; 1 KB alignment slack
};

__device__ __forceinline__ uint8_t *align1k(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// A_T: A = X^T (MN-major view of the stored planes); else A = X (K-major).
// grid (chunks x heads, D / 128).
template <int D, bool A_T, bool B_SPLIT>
__global__ void __launch_bounds__(kMmaThreads, 1)
state_mma_kernel(const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_b2,
                 const uint8_t *__restrict__ states, size_t head_stride, size_t chunk_stride,
                 float *__restrict__ out, int S, int L, int NC, unsigned int *status) {
    using Lay = MmaLay<D, B_SPLIT>;
    using namespace tc;
    extern __shared__ uint8_t mma_smem_raw[];
    uint8_t *smem = align1k(mma_smem_raw);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + Lay::kBar);     // [0] operands in, [1] products done
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + Lay::kBar + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kBar + 20);
    const int c = (int)(blockIdx.x % (unsigned)NC), bh = (int)(blockIdx.x / (unsigned)NC), mt = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int a0 = c * L, n = min(S, a0 + L) - a0;
    const uint8_t *slot = states + (size_t)bh * head_stride + (size_t)c * chunk_stride;
    constexpr uint32_t kPlaneBytes = (uint32_t)D * D * 2;

    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tslot, 64);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = *tslot;

    bool loaded = true;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar[0], 2 * Lay::kAPlane + (B_SPLIT ? 2 : 1) * Lay::kBPlane);
        for (int pl = 0; pl < 2; ++pl)
            for (int a = 0; a < Lay::kAtoms; ++a) {
                // K-major: this CTA's row tile mt, column blocks a.  MN-major: column
                // blocks 2 mt and 2 mt + 1 of every row tile (a / 2).
                const uint32_t gblk = A_T ? (uint32_t)((a >> 1) * (D / 64) + 2 * mt + (a & 1))
                                          : (uint32_t)(mt * Lay::kAtoms + a);
                bulk_load(smem + Lay::kA + pl * Lay::kAPlane + a * 16384, slot + pl * kPlaneBytes + gblk * 16384u,
                          16384u, &bar[0]);
            }
        for (int a = 0; a < Lay::kAtoms; ++a) {
            tma_load_3d(smem + Lay::kB + a * 8192, &map_b, &bar[0], 64 * a, a0, bh);
            if (B_SPLIT) tma_load_3d(smem + Lay::kB + Lay::kBPlane + a * 8192, &map_b2, &bar[0], 64 * a, a0, bh);
        }
        loaded = mbar_wait(&bar[0], 0, abort_flag, status);
        if (loaded) {
            tc_fence_after();
            const uint32_t idesc = idesc_f32acc(kFmtBF16, kFmtBF16, A_T, false, 128, 64);
            const uint32_t sa = smem_u32(smem + Lay::kA), sb = smem_u32(smem + Lay::kB);
#pragma unroll 1
            for (int ks = 0; ks < D / 16; ++ks) {
                const int atom = ks >> 2, sub = ks & 3;
                // K-major A: 32 bytes per 16-element K step inside a 64-wide block.
                // MN-major A: K runs down the rows (16 rows = 2 KB); the two 64-wide
                // M blocks of a row tile are 16 KB apart.
                const uint32_t aoff = A_T ? (uint32_t)(((16 * ks) >> 7) * 32768 + ((16 * ks) & 127) * 128)
                                          : (uint32_t)(atom * 16384 + sub * 32);
                const uint32_t albo = A_T ? 16384u : 16u;
                const uint32_t boff = (uint32_t)(atom * 8192 + sub * 32);
                const uint64_t ahi = sdesc_sw128(sa + aoff, albo, 1024);
                const uint64_t alo = sdesc_sw128(sa + Lay::kAPlane + aoff, albo, 1024);
                const uint64_t bhi = sdesc_sw128(sb + boff, 16, 1024);
                mma_bf16_ss(tacc, ahi, bhi, idesc, ks > 0 ? 1u : 0u);
                mma_bf16_ss(tacc, alo, bhi, idesc, 1u);
                if (B_SPLIT) mma_bf16_ss(tacc, ahi, sdesc_sw128(sb + Lay::kBPlane + boff, 16, 1024), idesc, 1u);
            }
            mma_commit(&bar[1]);
        } else {
            // never leave the copies in flight into this CTA's shared memory
            mbar_wait(&bar[0], 0, nullptr, nullptr);
        }
    }
    // one poller per warp; the warp then reads its 32 TMEM lanes converged
    __syncwarp();
    int ok = 0;
    if (lane == 0) ok = mbar_wait(&bar[1], 0, abort_flag, status) ? 1 : 0;
    const bool done = __shfl_sync(0xffffffffu, ok, 0) != 0;
    if (done) {
        tc_fence_after();
        uint32_t v[4][16];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld16(tacc + ((uint32_t)(32 * warp) << 16) + 16 * q, v[q]);
        tmem_wait_ld();
        float *dst = out + ((size_t)bh * S + a0) * D + 128 * mt + 32 * warp + lane;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int t = 16 * q + e;
                if (t < n) dst[(size_t)t * D] = __uint_as_float(v[q][e]);
            }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tacc, 64);
    }
}

}  // namespace bwdtc
}  // namespace xlstm
