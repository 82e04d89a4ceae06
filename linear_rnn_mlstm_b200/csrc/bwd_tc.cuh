// The backward's tensor-core kernels (included by bwd.cu; bf16 inputs, DH 64,
// 128 or 256): the walks that form the chunk states, the products with the
// states, and the two per-token passes.
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
// by the state walks as two bf16 planes (x = high + low, 16 significant bits)
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

// 128-row tiles along a DH-long dimension (DH 64: one tile, rows 64-127 of its
// MMAs are padding, computed and never stored), and the bytes of one 128 x 64
// plane block in global memory (DH 64: 64 rows).
template <int D> constexpr int kTiles = D >= 128 ? D / 128 : 1;
template <int D> constexpr uint32_t kBlkBytes = D >= 128 ? 16384u : (uint32_t)D * 128u;

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
    __syncwarp();
    if (warp == 0) tmem_alloc(tslot, 64);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = *tslot;

    bool loaded = true;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar[0], 2 * Lay::kAtoms * kBlkBytes<D> + (B_SPLIT ? 2 : 1) * Lay::kBPlane);
        for (int pl = 0; pl < 2; ++pl)
            for (int a = 0; a < Lay::kAtoms; ++a) {
                // K-major: this CTA's row tile mt, column blocks a.  MN-major: column
                // blocks 2 mt and 2 mt + 1 of every row tile (a / 2).
                const uint32_t gblk = A_T ? (uint32_t)((a >> 1) * (D / 64) + 2 * mt + (a & 1))
                                          : (uint32_t)(mt * Lay::kAtoms + a);
                bulk_load(smem + Lay::kA + pl * Lay::kAPlane + a * 16384, slot + pl * kPlaneBytes + gblk * 16384u,
                          kBlkBytes<D>, &bar[0]);
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
    __syncwarp();
    const bool done = __shfl_sync(0xffffffffu, ok, 0) != 0;
    if (done) {
        tc_fence_after();
        uint32_t v[4][16];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld16(tacc + ((uint32_t)(32 * warp) << 16) + 16 * q, v[q]);
        tmem_wait_ld();
        const int row = 128 * mt + 32 * warp + lane;
        float *dst = out + ((size_t)bh * S + a0) * D + row;
        if (row < D)
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

// ------------------------------------------------------------ bulk store
__device__ __forceinline__ void bulk_store(void *gdst, const void *ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(tc::smem_u32(ssrc)), "r"(bytes)
                 : "memory");
}

// ------------------------------------------------------------ state walk
// The chunk recurrences of the states, C'_{c+1} = decay_c C'_c + dC_c (forward)
// and dC~_{c-1} = decay_c dC~_c + ddC_c (reverse), walked chunk by chunk with
// the running state in fp32 registers, so that every slot is written once and
// no increment leaves the chip: one CTA per (head, 128-row tile, 64-column
// block).  Per chunk the
// increment is one M = 128 (rows r), N = 64 (columns j), K = 64 (tokens)
// product on the tensor cores with the token weight moved onto B:
//   dC_c[r][j]  = sum_{s in c} v_s[r] (w_s k_s[j])
//   ddC_c[r][j] = sum_{t in c} dnum'_t[r] (g_t q_t[j])
// A = v (or dnum' as its high and low planes) as loaded by TMA, MN-major; B =
// the weighted k (or q) tile, split in place into bf16 high and low parts.
// The token weights (w_s or g_t, and the normaliser's: 1 or dnq'_t) arrive
// with the tiles as the chunk's 512-byte record, written beforehand by
// walk_weights_kernel with the chunk decays.  Four warp roles, a ring of
// stages apart:
//   warp 13 (loads): refills a stage with a later chunk's tiles and record
//     once the MMAs that read it completed;
//   warps 9-12 (transform): form B as soon as a chunk's tiles land and, in
//     row tile 0, the normaliser's 64 column sums and its walk;
//   warp 8 (MMA): issues the chunk's MMAs into one of four tensor-memory
//     buffers;
//   warps 0-7 (consumers): read the increment out of tensor memory, update
//     their 32 state elements (row 32 (warp & 3) + lane, columns
//     32 (warp >> 2) ...) and stage them as bf16 high / low rows; each pair of
//     warps sharing 32 rows stores them with two 4 KB bulk copies.
// Walk step i holds the state after i increments: forward slot i (slot 0 =
// 0), reverse slot NC - 1 - i (slot NC - 1 = the final-state cotangent, or 0).
template <int D, bool REVERSE>
struct WalkLay {
    static constexpr int kStages = REVERSE ? 3 : 4;
    static constexpr int kBufs = 4;                                  // tensor-memory buffers, 64 columns each
    static constexpr int kRawA = REVERSE ? 32768 : 16384;            // v: 2 boxes; dnum': 2 planes x 2 boxes
    static constexpr int kRec = kRawA + 16384;                       // after the B box (high in place) + low part
    static constexpr int kStage = kRec + 1024;                       // + the chunk's weight record (512 B)
    static constexpr int kOut = kStages * kStage;                    // 2 x (high 16 KB + low 16 KB) staging
    static constexpr int kRed = kOut + 65536;                        // column partial sums [2][16][64]
    static constexpr int kBar = kRed + 8192;
    static constexpr int kBytes = kBar + 256 + 1024;
    static constexpr uint32_t kTx = (uint32_t)kRawA + 8192u + 512u;
};
constexpr int kWalkThreads = 448;
static_assert(WalkLay<256, true>::kBytes <= 232448 && WalkLay<256, false>::kBytes <= 232448,
              "state walk shared memory (227 KB per CTA)");

// The walk's inputs per chunk c of head bh: record [bh, c] = w[64], wn[64]
// (0 past the chunk's tokens) and decay[bh, c] = e^{B_c + m_prev,c - m_end,c}.
// Forward: w_s = e^{B_c - b_s + itilde_s - m_end,c} / sqrt(d), wn_s = 1;
// reverse: g_t = e^{b_t + m_prev,c - m_t}, wn_t = dnq'_t (B_c: the chunk's
// sum of log f, b: its cumulative sum up to the token).
// One thread per (chunk, token slot).
template <bool REVERSE>
__global__ void __launch_bounds__(256) walk_weights_kernel(bwd::BwdPtrs p) {
    const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t rc = g >> 6;                                        // bh * NC + c
    if (rc >= (size_t)p.BH * p.NC) return;
    const int t = (int)(g & 63), c = (int)(rc % (size_t)p.NC), bh = (int)(rc / (size_t)p.NC);
    const int a0 = c * p.L, n = min(p.S, a0 + p.L) - a0;
    float w = 0.f, wn = 0.f;
    if (t < n) {
        const size_t ts = (size_t)bh * p.S + a0 + t;
        if (REVERSE) {
            w = expf(p.b[ts] + p.mprev[rc] - p.mt[ts]);
            wn = p.dnq[ts];
        } else {
            w = expf(p.Bsum[rc] - p.b[ts] + p.ip[ts] - p.mend[rc]) * rsqrtf((float)p.DH);
            wn = 1.f;
        }
    }
    p.wrec[rc * 128 + t] = w;
    p.wrec[rc * 128 + 64 + t] = wn;
    if (t == 0) p.decay[rc] = expf(p.Bsum[rc] + p.mprev[rc] - p.mend[rc]);
}

template <int D, bool REVERSE>
__global__ void __launch_bounds__(kWalkThreads, 1)
state_walk_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_a2,
                  const __grid_constant__ CUtensorMap map_b, bwd::BwdPtrs p, unsigned int *status) {
    using Lay = WalkLay<D, REVERSE>;
    using namespace tc;
    constexpr int NS = Lay::kStages, NB = Lay::kBufs;
    extern __shared__ uint8_t walk_smem_raw[];
    uint8_t *smem = align1k(walk_smem_raw);
    float *red = reinterpret_cast<float *>(smem + Lay::kRed);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Lay::kBar);   // [NS] tiles landed
    uint64_t *bready = full + 4;                                       // [NS] B formed
    uint64_t *mma_done = full + 8, *tmem_free = full + 12;             // [NB] each
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + Lay::kBar + 128);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kBar + 132);
    const int bh = blockIdx.x, mt = blockIdx.y, kb = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = p.L, NC = p.NC;
    const int steps = REVERSE ? NC - 1 : NC;                         // increments walked
    const size_t DD = (size_t)D * D, hbase = (size_t)bh * NC;
    uint8_t *slots = reinterpret_cast<uint8_t *>(REVERSE ? p.dCb + hbase * DD : p.Cst + (size_t)bh * (NC + 1) * DD);
    float *nslots = REVERSE ? p.dnb + hbase * D : p.nst + (size_t)bh * (NC + 1) * D;
    auto chunk_of = [&](int i) { return REVERSE ? NC - 1 - i : i; };
    auto slot_of = [&](int i) { return REVERSE ? NC - 1 - i : i; };
    // the chunk decays, 32 steps to a warp register (lane l: step 32 k + l), the
    // next block in flight a block ahead
    auto decay_block = [&](int blk) {
        const int i = 32 * blk + lane;
        return i < steps ? p.decay[hbase + chunk_of(i)] : 0.f;
    };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&bready[s], 4);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&mma_done[b], 1);
            mbar_init(&tmem_free[b], 8);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (warp == 0) tmem_alloc(tslot, 64 * NB);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;

    if (warp < 8) {
        // ------------------------------------------------ consumers
        constexpr int kRows = D >= 128 ? 128 : D;                    // rows of a plane block in global memory
        const int rr = 32 * (warp & 3) + lane, cg = warp >> 2;
        const int r = 128 * mt + rr, j0 = 64 * kb + 32 * cg;
        float x[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = 0.f;
        if (REVERSE && p.dC && r < D) {
            const float4 *src = reinterpret_cast<const float4 *>(p.dC + (size_t)bh * DD + (size_t)r * D + j0);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float4 f = src[e];
                x[4 * e] = f.x; x[4 * e + 1] = f.y; x[4 * e + 2] = f.z; x[4 * e + 3] = f.w;
            }
        }
        // the 32 rows of this warp pair: staged at row rr, stored from the pair's
        // first warp by two bulk copies of (up to) 4 KB
        const int q = warp & 3, nrows = min(32, kRows - 32 * q);
        const bool issuer = cg == 0 && lane == 0 && nrows > 0;
        const size_t blk_off = (size_t)(mt * (D / 64) + kb) * kBlkBytes<D> + (size_t)(32 * q) * 128u;
        auto stage = [&](int buf) {
            uint8_t *hi = smem + Lay::kOut + buf * 32768;
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                uint32_t h[4], l[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float x0 = x[8 * pp + 2 * k], x1 = x[8 * pp + 2 * k + 1];
                    h[k] = cvt_bf16x2(x0, x1);
                    const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&h[k]);
                    l[k] = cvt_bf16x2(x0 - __low2float(h2), x1 - __high2float(h2));
                }
                const uint32_t off = (uint32_t)rr * 128u + ((uint32_t)((4 * cg + pp) ^ (rr & 7)) << 4);
                *reinterpret_cast<uint4 *>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4 *>(hi + 16384 + off) = make_uint4(l[0], l[1], l[2], l[3]);
            }
            fence_async_smem();
        };
        auto put = [&](int i) {                      // the pair's issuer: walk step i from buffer i & 1
            uint8_t *dst = slots + (size_t)slot_of(i) * DD * 4 + blk_off;
            const uint8_t *src = smem + Lay::kOut + (i & 1) * 32768 + (32 * q) * 128;
            bulk_store(dst, src, (uint32_t)nrows * 128u);
            bulk_store(dst + DD * 2, src + 16384, (uint32_t)nrows * 128u);
            bulk_commit();
        };
        // named barrier 2 + q: the 64 threads of warps q and q + 4
        auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(2 + q) : "memory"); };
        stage(0);
        pair_sync();
        if (issuer) put(0);
        float dcur = decay_block(0), dnxt = decay_block(1);
#pragma unroll 1
        for (int i = 0; i < steps; ++i) {
            const float dec = __shfl_sync(0xffffffffu, dcur, i & 31);
            if ((i & 31) == 31) {
                dcur = dnxt;
                dnxt = decay_block((i >> 5) + 2);
            }
            const int b = i % NB;
            int got = 0;
            if (lane == 0) got = mbar_wait(&mma_done[b], (uint32_t)((i / NB) & 1), abort_flag, status) ? 1 : 0;
            __syncwarp();
            got = __shfl_sync(0xffffffffu, got, 0);
            if (got) {
                tc_fence_after();
                uint32_t v0[16], v1[16];
                const uint32_t ta = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(64 * b + 32 * cg);
                tmem_ld16(ta, v0);
                tmem_ld16(ta + 16, v1);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tmem_free[b]);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    x[e] = fmaf(x[e], dec, __uint_as_float(v0[e]));
                    x[16 + e] = fmaf(x[16 + e], dec, __uint_as_float(v1[e]));
                }
                stage((i + 1) & 1);
            }
            if (issuer) bulk_wait_read_all();        // step i's copies have read their buffer
            __syncwarp();
            // both warps' verdicts: a pair leaves together
            int both;
            asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                         "bar.red.and.pred q, %2, 64, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                         : "=r"(both) : "r"(got), "r"(2 + q) : "memory");
            if (!both) break;
            if (issuer) put(i + 1);
        }
        if (issuer) bulk_wait_all();
    } else if (warp == 8) {
        // ------------------------------------------------ MMA issue
        if (lane == 0) {
            int mmas = 0;
            const uint32_t idesc = idesc_f32acc(kFmtBF16, kFmtBF16, true, true, 128, 64);
#pragma unroll 1
            for (int i = 0; i < steps; ++i) {
                const int s = i % NS, b = i % NB;
                if (!mbar_wait(&bready[s], (uint32_t)((i / NS) & 1), abort_flag, status)) break;
                if (i >= NB && !mbar_wait(&tmem_free[b], (uint32_t)((i / NB - 1) & 1), abort_flag, status)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * Lay::kStage), sb = sa + (uint32_t)Lay::kRawA;
                const uint32_t td = tbase + (uint32_t)(64 * b);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ahi = sdesc_sw128(sa + ks * 2048, 8192, 1024);
                    const uint64_t bhi = sdesc_sw128(sb + ks * 2048, 8192, 1024);
                    mma_bf16_ss(td, ahi, bhi, idesc, ks > 0 ? 1u : 0u);
                    mma_bf16_ss(td, ahi, sdesc_sw128(sb + 8192 + ks * 2048, 8192, 1024), idesc, 1u);
                    if (REVERSE) mma_bf16_ss(td, sdesc_sw128(sa + 16384 + ks * 2048, 8192, 1024), bhi, idesc, 1u);
                }
                mma_commit(&mma_done[b]);
                ++mmas;
            }
            // no MMA left in flight (a short bound: this only runs after a timeout)
            if (mmas > 0)
                mbar_wait(&mma_done[(mmas - 1) % NB], (uint32_t)(((mmas - 1) / NB) & 1), nullptr, nullptr, 200000000ull);
        }
        __syncwarp();
    } else if (warp == 13) {
        // ------------------------------------------------ loads
        if (lane == 0) {
            int issued = 0;
            auto issue = [&](int k) {                // the tiles and weights of walk step k's chunk
                const int s = k % NS, c = chunk_of(k), a0 = c * L;
                uint8_t *st = smem + s * Lay::kStage;
                mbar_arrive_expect_tx(&full[s], Lay::kTx);
                for (int h = 0; h < 2; ++h) {
                    tma_load_3d(st + h * 8192, &map_a, &full[s], 128 * mt + 64 * h, a0, bh);
                    if (REVERSE) tma_load_3d(st + 16384 + h * 8192, &map_a2, &full[s], 128 * mt + 64 * h, a0, bh);
                }
                tma_load_3d(st + Lay::kRawA, &map_b, &full[s], 64 * kb, a0, bh);
                bulk_load(st + Lay::kRec, p.wrec + (hbase + c) * 128, 512, &full[s]);
            };
            for (; issued < min(NS, steps); ++issued) issue(issued);
            // the stage of step k is free once step k's MMAs completed
#pragma unroll 1
            for (int k = 0; issued < steps; ++k) {
                if (!mbar_wait(&mma_done[k % NB], (uint32_t)((k / NB) & 1), abort_flag, status)) break;
                issue(issued++);
            }
            // no copy left in flight (the last copy into each stage); one 200 ms
            // deadline for the whole drain, which only waits after a timeout
            const uint64_t deadline = globaltimer_ns() + 200000000ull;
            for (int k = max(0, issued - NS); k < issued; ++k) {
                const uint64_t now = globaltimer_ns();
                mbar_wait(&full[k % NS], (uint32_t)((k / NS) & 1), nullptr, nullptr, now < deadline ? deadline - now : 0ull);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ transform
        // Thread tt forms the pieces 8 t + pp of the B box for the tokens
        // t = t0 + 16 m (m = 0..3); with the 128-byte swizzle those four pieces
        // hold the same 8 columns, 8 lp ... 8 lp + 7.
        const int tt = tid - 288;
        const bool norm = mt == 0;
        const int pp = tt & 7, t0 = tt >> 3, lp = pp ^ (t0 & 7);
        float n_run = 0.f;
        float dcur = decay_block(0), dnxt = decay_block(1);
        if (norm && tt < 64) {
            if (REVERSE && p.dn) n_run = p.dn[(size_t)bh * D + 64 * kb + tt];
            nslots[(size_t)slot_of(0) * D + 64 * kb + tt] = n_run;
        }
#pragma unroll 1
        for (int i = 0; i < steps; ++i) {
            const int s = i % NS;
            uint8_t *bt = smem + s * Lay::kStage + Lay::kRawA;
            const float *rec = reinterpret_cast<const float *>(smem + s * Lay::kStage + Lay::kRec);
            const float dec = __shfl_sync(0xffffffffu, dcur, i & 31);
            if ((i & 31) == 31) {
                dcur = dnxt;
                dnxt = decay_block((i >> 5) + 2);
            }
            int got = 0;
            if (lane == 0) got = mbar_wait(&full[s], (uint32_t)((i / NS) & 1), abort_flag, status) ? 1 : 0;
            __syncwarp();
            got = __shfl_sync(0xffffffffu, got, 0);
            float acc[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = 0.f;
            if (got) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int t = t0 + 16 * m, e = 8 * t + pp;
                    const float wt = rec[t], wn = rec[64 + t];
                    const uint4 raw = reinterpret_cast<const uint4 *>(bt)[e];
                    const __nv_bfloat16 *rb = reinterpret_cast<const __nv_bfloat16 *>(&raw);
                    uint32_t h[4], l[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float x0 = wt * __bfloat162float(rb[2 * k]), x1 = wt * __bfloat162float(rb[2 * k + 1]);
                        acc[2 * k] = fmaf(wn, x0, acc[2 * k]);
                        acc[2 * k + 1] = fmaf(wn, x1, acc[2 * k + 1]);
                        h[k] = cvt_bf16x2(x0, x1);
                        const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&h[k]);
                        l[k] = cvt_bf16x2(x0 - __low2float(h2), x1 - __high2float(h2));
                    }
                    reinterpret_cast<uint4 *>(bt)[e] = make_uint4(h[0], h[1], h[2], h[3]);
                    reinterpret_cast<uint4 *>(bt + 8192)[e] = make_uint4(l[0], l[1], l[2], l[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bready[s]);
            }
            if (norm) {                              // the normaliser: column sums over the 16 token groups
                float *rd = red + (i & 1) * 1024 + t0 * 64 + lp * 8;
                reinterpret_cast<float4 *>(rd)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                reinterpret_cast<float4 *>(rd)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
                if (!group_all<1, 128>(got != 0)) break;
                if (tt < 64) {
                    const float *rs = red + (i & 1) * 1024 + tt;
                    float dn = 0.f;
#pragma unroll
                    for (int g = 0; g < 16; ++g) dn += rs[g * 64];
                    n_run = fmaf(n_run, dec, dn);
                    nslots[(size_t)slot_of(i + 1) * D + 64 * kb + tt] = n_run;
                }
            } else if (!got) {
                break;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 64 * NB);
    }
}

// ------------------------------------------------------------ per-token pass
// K3 on the tensor cores, one CTA per (chunk, head): the forward quantities of
// every token of the chunk and the first gradients.
//   S   = Q K^T                       M = 64 tokens t, N = 64 keys s, K = DH
//   W_ts = e^{b_t - b_s + itilde_s - m_t} S_ts / sqrt(d)  (s <= t), rowsum_t = sum_s W_ts
//   num_intra^T = V^T W^T              M = 128 value rows per tile, N = 64 tokens, K = 64
// (W as bf16 high + low parts), then per (value row i, token t), with
// C'_c q_t from the state product kernel (p.num):
//   num' = g_t C'q + num_intra,  nq' = g_t n'_c.q_t + rowsum_t,  den' = max(|nq'|, e^{-m_t}),
//   h~ = num'/den', dh~ = dh o, d o~ = dh h~ o (1 - o), dnum' = dh~ / den',
//   dnq' = -(dh~ . h~)/den' sign(nq') where |nq'| > e^{-m_t}, A = dnum'.num' + dnq' nq'.
// 16 warps: in the epilogue warp w owns TMEM lane quadrant w % 4 (32 value
// rows of each 128-row tile, coalesced per token) and tokens 16 (w / 4) to
// 16 (w / 4) + 15; the per-token sums over the value rows go through warp
// shuffles and shared memory.
constexpr int kTokThreads = 512;

template <int D>
struct TokLay {
    static constexpr int kTile = D / 64 * 8192;          // 64 token rows x D, bf16, 128-byte swizzle
    static constexpr int kQ = 0, kK = kTile, kV = 2 * kTile;
    static constexpr int kWhi = 3 * kTile, kWlo = kWhi + 8192;
    static constexpr int kF = kWlo + 8192;                // floats: b ip mt g den nq nqi rs [64 each], red [2][4][64], n' [D]
    static constexpr int kFloats = 8 * 64 + 2 * 8 * 64 + D;
    static constexpr int kBar = kF + kFloats * 4;
    static constexpr int kBytes = kBar + 64 + 1024;
    static constexpr int kCols = D == 256 ? 256 : 128;    // TMEM: S in 0-63, num_intra^T tiles from 64
};

template <int D>
__global__ void __launch_bounds__(kTokThreads, 1)
token_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, bwd::BwdPtrs p, unsigned int *status) {
    using Lay = TokLay<D>;
    using namespace tc;
    extern __shared__ uint8_t tok_smem_raw[];
    uint8_t *smem = align1k(tok_smem_raw);
    float *fb = reinterpret_cast<float *>(smem + Lay::kF);
    float *sb = fb, *sip = fb + 64, *smt = fb + 128, *sg = fb + 192, *sden = fb + 256, *snq = fb + 320,
          *red = fb + 512, *snp = fb + 512 + 1024;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + Lay::kBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + Lay::kBar + 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kBar + 36);
    const int NC = p.NC, S = p.S, L = p.L;
    const int c = (int)(blockIdx.x % (unsigned)NC), bh = (int)(blockIdx.x / (unsigned)NC);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int a0 = c * L, n = min(S, a0 + L) - a0;
    const size_t row0 = (size_t)bh * S + a0, hc = (size_t)bh * NC + c;
    const float inv_sqrt = rsqrtf((float)D);

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar[0], 3 * Lay::kTile);
        for (int a = 0; a < D / 64; ++a) {
            tma_load_3d(smem + Lay::kQ + a * 8192, &map_q, &bar[0], 64 * a, a0, bh);
            tma_load_3d(smem + Lay::kK + a * 8192, &map_k, &bar[0], 64 * a, a0, bh);
            tma_load_3d(smem + Lay::kV + a * 8192, &map_v, &bar[0], 64 * a, a0, bh);
        }
    }
    __syncwarp();
    if (warp == 0) tmem_alloc(tslot, Lay::kCols);
    if (tid < 64) {
        const int t = tid;
        float b = 0.f, ip = -INFINITY, mt = 0.f, g = 0.f;
        if (t < n) {
            b = p.b[row0 + t];
            ip = p.ip[row0 + t];
            mt = p.mt[row0 + t];
            g = expf(b + p.mprev[hc] - mt);
        }
        sb[t] = b; sip[t] = ip; smt[t] = mt; sg[t] = g;
    }
    for (int j = tid; j < D; j += kTokThreads) snp[j] = p.nst[((size_t)bh * (NC + 1) + c) * D + j];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = *tslot;
    const int quad = warp & 3;
    const uint32_t lane_addr = ((uint32_t)(32 * quad)) << 16;
    int ok = 0;
    if (lane == 0) ok = mbar_wait(&bar[0], 0, abort_flag, status) ? 1 : 0;
    __syncwarp();
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f32acc(kFmtBF16, kFmtBF16, false, false, 64, 64);
        const uint32_t sq = smem_u32(smem + Lay::kQ), sk = smem_u32(smem + Lay::kK);
#pragma unroll 1
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (uint32_t)((ks >> 2) * 8192 + (ks & 3) * 32);
            mma_bf16_ss(tacc, sdesc_sw128(sq + off, 16, 1024), sdesc_sw128(sk + off, 16, 1024), idesc,
                        ks > 0 ? 1u : 0u);
        }
        mma_commit(&bar[1]);
    }
    if (ok) {                                         // n'_c . q_t, eight threads per token
        const int t = tid >> 3, h = tid & 7;
        float acc = 0.f;
        for (int pc = h * (D / 64); pc < (h + 1) * (D / 64); ++pc) {      // 16-byte pieces of the row
            const int j0 = pc * 8;
            const uint4 raw = *reinterpret_cast<const uint4 *>(
                smem + Lay::kQ + (j0 >> 6) * 8192 + t * 128 + ((((j0 & 63) >> 3) ^ (t & 7)) << 4));
            const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(&raw);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc += snp[j0 + e] * __bfloat162float(qb[e]);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if (h == 0) red[t] = acc;
    }
    // ---- scores -> W (bf16 high / low tiles), row sums
    int done1 = 0;
    if (ok && lane == 0) done1 = mbar_wait(&bar[1], 0, abort_flag, status) ? 1 : 0;
    __syncwarp();
    done1 = __shfl_sync(0xffffffffu, done1, 0);
    if (done1) {
        tc_fence_after();
        // all 16 warps: warp w reads TMEM lane quadrant w % 4 (M = 64 layout: rows
        // t = 16 (w % 4) + (lane & 15) in the quadrant's lanes 0-15) at columns
        // 16 (w / 4) .. + 15; lanes 16-31 take their row's upper 8 of those columns
        const int cg = warp >> 2, t = 16 * quad + (lane & 15), hh = lane >> 4;
        uint32_t sa[16];
        tmem_ld16(tacc + lane_addr + 16 * cg, sa);
        tmem_wait_ld();
        const float bt = sb[t], mtt = smt[t];
        float rs = 0.f;
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float w2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t up = __shfl_sync(0xffffffffu, sa[8 + e + u], lane & 15);
                const float sv = __uint_as_float(hh ? up : sa[e + u]);
                const int s_ = 16 * cg + 8 * hh + e + u;
                w2[u] = (t < n && s_ <= t) ? expf(bt - sb[s_] + sip[s_] - mtt) * sv * inv_sqrt : 0.f;
                rs += w2[u];
            }
            hi[e / 2] = cvt_bf16x2(w2[0], w2[1]);
            const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&hi[e / 2]);
            lo[e / 2] = cvt_bf16x2(w2[0] - __low2float(h2), w2[1] - __high2float(h2));
        }
        rs += __shfl_xor_sync(0xffffffffu, rs, 16);
        if (hh == 0) red[256 + cg * 64 + t] = rs;     // this warp's 16 columns of row t's sum
        const uint32_t off = (uint32_t)t * 128u + ((uint32_t)((2 * cg + hh) ^ (t & 7)) << 4);
        *reinterpret_cast<uint4 *>(smem + Lay::kWhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(smem + Lay::kWlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (done1 && tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f32acc(kFmtBF16, kFmtBF16, true, false, 128, 64);
        const uint32_t svv = smem_u32(smem + Lay::kV), wh = smem_u32(smem + Lay::kWhi), wl = smem_u32(smem + Lay::kWlo);
#pragma unroll
        for (int mt = 0; mt < kTiles<D>; ++mt)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sdesc_sw128(svv + 2 * mt * 8192 + ks * 2048, 8192, 1024);
                mma_bf16_ss(tacc + 64 + 64 * mt, ad, sdesc_sw128(wh + ks * 32, 16, 1024), idesc, ks > 0 ? 1u : 0u);
                mma_bf16_ss(tacc + 64 + 64 * mt, ad, sdesc_sw128(wl + ks * 32, 16, 1024), idesc, 1u);
            }
        mma_commit(&bar[2]);
    }
    if (done1 && tid < 64) {                          // normaliser and floor per token
        const int t = tid;
        const float rsum = red[256 + t] + red[320 + t] + red[384 + t] + red[448 + t];
        const float nq = sg[t] * red[t] + rsum;
        snq[t] = nq;
        sden[t] = t < n ? fmaxf(fabsf(nq), expf(-smt[t])) : 1.f;
    }
    __syncthreads();
    int done2 = 0;
    if (done1 && lane == 0) done2 = mbar_wait(&bar[2], 0, abort_flag, status) ? 1 : 0;
    __syncwarp();
    done2 = __shfl_sync(0xffffffffu, done2, 0);
    if (done2) {
        tc_fence_after();
        __nv_bfloat16 *hl = reinterpret_cast<__nv_bfloat16 *>(p.dnhl);
        const size_t plane = (size_t)p.BH * S * D;
        {
            const int tg = warp >> 2;
            // eight tokens at a time: every load of the batch is issued before
            // the first store (the stores could alias them otherwise)
#pragma unroll
            for (int e0 = 0; e0 < 16; e0 += 8) {
                uint32_t v[kTiles<D>][8];
#pragma unroll
                for (int mt = 0; mt < kTiles<D>; ++mt) tmem_ld8(tacc + lane_addr + 64 + 64 * mt + 16 * tg + e0, v[mt]);
                tmem_wait_ld();
                float xn[8][kTiles<D>], xo[8][kTiles<D>], xd[8][kTiles<D>];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = 16 * tg + e0 + e;
                    const size_t rowoff = (row0 + (t < n ? t : 0)) * D;
#pragma unroll
                    for (int mt = 0; mt < kTiles<D>; ++mt) {
                        const int i = 128 * mt + 32 * quad + lane;
                        const bool in = t < n && i < D;
                        xn[e][mt] = in ? p.num[rowoff + i] : 0.f;
                        xo[e][mt] = in ? p.op[rowoff + i] : 0.f;
                        xd[e][mt] = in ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p.dh)[rowoff + i]) : 0.f;
                    }
                }
                float sd[8], aa[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = 16 * tg + e0 + e;
                    sd[e] = 0.f;
                    aa[e] = 0.f;
                    if (t >= n) continue;
                    const float g = sg[t], den = sden[t];
                    const size_t rowoff = (row0 + t) * D;
#pragma unroll
                    for (int mt = 0; mt < kTiles<D>; ++mt) {
                        const int i = 128 * mt + 32 * quad + lane;
                        if (i >= D) continue;                // padding rows of a 64-row head
                        const float num = g * xn[e][mt] + __uint_as_float(v[mt][e]);
                        const float ht = num / den;
                        const float o = bwd::sigmoid_hd(xo[e][mt]);
                        const float dhr = xd[e][mt];
                        const float dht = dhr * o;
                        p.dO[rowoff + i] = dhr * ht * o * (1.f - o);
                        const float dn = dht / den;      // kept as its high / low planes only
                        const __nv_bfloat16 h16 = __float2bfloat16_rn(dn);
                        hl[rowoff + i] = h16;
                        hl[plane + rowoff + i] = __float2bfloat16_rn(dn - __bfloat162float(h16));
                        sd[e] += dht * ht;
                        aa[e] += dn * num;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        sd[e] += __shfl_xor_sync(0xffffffffu, sd[e], o);
                        aa[e] += __shfl_xor_sync(0xffffffffu, aa[e], o);
                    }
                if (lane == 0)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = 16 * tg + e0 + e;
                        red[quad * 64 + t] = sd[e];
                        red[256 + quad * 64 + t] = aa[e];
                    }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (done2 && tid < n) {
        const int t = tid;
        float sdot = 0.f, A = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            sdot += red[w * 64 + t];
            A += red[256 + w * 64 + t];
        }
        const float nq = snq[t], den = sden[t];
        const float dnq = fabsf(nq) > expf(-smt[t]) ? -sdot / den * (nq > 0.f ? 1.f : -1.f) : 0.f;
        p.dnq[row0 + t] = dnq;
        p.nq[row0 + t] = nq;
        p.den[row0 + t] = den;
        p.A[row0 + t] = A + dnq * nq;
    }
    if (tid == 0 && !ok) mbar_wait(&bar[0], 0, nullptr, nullptr);     // no copy left in flight
    __syncwarp();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tacc, Lay::kCols);
    }
}

// ------------------------------------------------------------ gradient pass
// K5 on the tensor cores, one CTA per (chunk, head), 16 warps:
//   S = Q K^T, dP0 = dnum' V^T                      M = 64 tokens, N = 64 keys, K = DH
//   W~_ts = e^{b_t - b_s + itilde_s - m_t} (s <= t), M2 = W~ S / sqrt(d), M1 = W~ (dP0 + dnq'_t)
//   dq^T = K^T M1^T,  dk^T = Q^T M1,  dv^T = dnum'^T M2    M = 128 rows per tile, N = 64, K = 64
// (M1, M2 as bf16 high + low tiles, dnum' from its high / low planes); then,
// with the state products of the tensor-core kernels (p.num: C'^T dnum',
// p.dki: dC~^T v, p.dvi: dC~ k):
//   dq_t = dq^T_t / sqrt(d) + g_t (C'^T dnum'_t + dnq'_t n'_c)
//   dkhat_s = dk^T_s + wk_s (dC~^T v_s + dn~_c),  dk = dkhat / sqrt(d),  ditilde_s = khat_s . dkhat_s
//   dv_s = dv^T_s + wk_s / sqrt(d) dC~ k_s,   d log f term dF_s = A_s - ditilde_s.
template <int D>
struct GradLay {
    static constexpr int kTile = D / 64 * 8192;
    static constexpr int kQ = 0, kK = kTile, kV = 2 * kTile, kDh = 3 * kTile, kDl = 4 * kTile;
    static constexpr int kM1h = 5 * kTile, kM1l = kM1h + 8192, kM2h = kM1l + 8192, kM2l = kM2h + 8192;
    static constexpr int kF = kM2l + 8192;        // floats: b ip mt dnq A g wk [64 each], red [4][64], n', dn~ [D]
    static constexpr int kFloats = 7 * 64 + 4 * 64 + 2 * D;
    static constexpr int kBar = kF + kFloats * 4;
    static constexpr int kBytes = kBar + 64 + 1024;
    static constexpr int cS = 0, cP = 64, cDq = 128, cDk = 128 + 64 * (kTiles<D>), cDv = 128 + 128 * (kTiles<D>);
};

// Persistent: one CTA per SM walks (chunk, head) items; the next item's tiles
// are loaded while this item's epilogue runs (all but k at its start, k, which
// the epilogue still reads, after it).
template <int D>
__global__ void __launch_bounds__(kTokThreads, 1)
token_grad_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_dh,
                     const __grid_constant__ CUtensorMap map_dl, bwd::BwdPtrs p, unsigned int *status) {
    using Lay = GradLay<D>;
    using namespace tc;
    extern __shared__ uint8_t grad_smem_raw[];
    uint8_t *smem = align1k(grad_smem_raw);
    float *fb = reinterpret_cast<float *>(smem + Lay::kF);
    float *sb = fb, *sip = fb + 64, *smt = fb + 128, *sdnq = fb + 192, *sA = fb + 256, *sg = fb + 320,
          *swk = fb + 384, *red = fb + 448, *snp = fb + 704, *sdnb = snp + D;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + Lay::kBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + Lay::kBar + 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kBar + 36);
    const int NC = p.NC, S = p.S, L = p.L;
    const long long items = (long long)NC * p.BH;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, quad = warp & 3;
    const float inv_sqrt = rsqrtf((float)D);
    // the tiles of item `item` (all five, or all but k / only k)
    auto load_tiles = [&](long long item, bool arm, bool k_tile, bool others) {
        const int ci = (int)(item % NC), bhi = (int)(item / NC), ai = ci * L;
        if (arm) mbar_arrive_expect_tx(&bar[0], 5 * Lay::kTile);
        for (int a = 0; a < D / 64; ++a) {
            if (others) {
                tma_load_3d(smem + Lay::kQ + a * 8192, &map_q, &bar[0], 64 * a, ai, bhi);
                tma_load_3d(smem + Lay::kV + a * 8192, &map_v, &bar[0], 64 * a, ai, bhi);
                tma_load_3d(smem + Lay::kDh + a * 8192, &map_dh, &bar[0], 64 * a, ai, bhi);
                tma_load_3d(smem + Lay::kDl + a * 8192, &map_dl, &bar[0], 64 * a, ai, bhi);
            }
            if (k_tile) tma_load_3d(smem + Lay::kK + a * 8192, &map_k, &bar[0], 64 * a, ai, bhi);
        }
    };
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        if ((long long)blockIdx.x < items) load_tiles(blockIdx.x, true, true, true);
    }
    __syncwarp();
    if (warp == 0) tmem_alloc(tslot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = *tslot;
    const uint32_t lane_addr = ((uint32_t)(32 * quad)) << 16;
    // thread 0: a fill of the tiles armed and not yet waited for, and its parity
    bool loads_pending = (long long)blockIdx.x < items;
    uint32_t pend_par = 0;
    int it = 0;
    for (long long item = blockIdx.x; item < items; item += gridDim.x, ++it) {
    const int c = (int)(item % NC), bh = (int)(item / NC);
    const int a0 = c * L, n = min(S, a0 + L) - a0;
    const size_t row0 = (size_t)bh * S + a0, hc = (size_t)bh * NC + c;
    const uint32_t par = (uint32_t)it & 1u;
    if (tid < 64) {
        const int t = tid;
        float b = 0.f, ip = -INFINITY, mt = 0.f, dnq = 0.f, A = 0.f, g = 0.f, wk = 0.f;
        if (t < n) {
            b = p.b[row0 + t];
            ip = p.ip[row0 + t];
            mt = p.mt[row0 + t];
            dnq = p.dnq[row0 + t];
            A = p.A[row0 + t];
            g = expf(b + p.mprev[hc] - mt);
            wk = expf(p.Bsum[hc] - b + ip - p.mend[hc]);
        }
        sb[t] = b; sip[t] = ip; smt[t] = mt; sdnq[t] = dnq; sA[t] = A; sg[t] = g; swk[t] = wk;
    }
    for (int j = tid; j < D; j += kTokThreads) {
        snp[j] = p.nst[((size_t)bh * (NC + 1) + c) * D + j];
        sdnb[j] = p.dnb[hc * D + j];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    int ok = 0;
    if (lane == 0) ok = mbar_wait(&bar[0], par, abort_flag, status) ? 1 : 0;
    if (tid == 0 && ok) loads_pending = false;
    __syncwarp();
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f32acc(kFmtBF16, kFmtBF16, false, false, 64, 64);
        const uint32_t sq = smem_u32(smem + Lay::kQ), sk = smem_u32(smem + Lay::kK), sv = smem_u32(smem + Lay::kV),
                       sdh = smem_u32(smem + Lay::kDh), sdl = smem_u32(smem + Lay::kDl);
#pragma unroll 1
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (uint32_t)((ks >> 2) * 8192 + (ks & 3) * 32);
            const uint32_t acc = ks > 0 ? 1u : 0u;
            mma_bf16_ss(tacc + Lay::cS, sdesc_sw128(sq + off, 16, 1024), sdesc_sw128(sk + off, 16, 1024), idesc, acc);
            const uint64_t bv = sdesc_sw128(sv + off, 16, 1024);
            mma_bf16_ss(tacc + Lay::cP, sdesc_sw128(sdh + off, 16, 1024), bv, idesc, acc);
            mma_bf16_ss(tacc + Lay::cP, sdesc_sw128(sdl + off, 16, 1024), bv, idesc, 1u);
        }
        mma_commit(&bar[1]);
    }
    // ---- M1, M2 tiles (warps 0-3: M = 64 layout, row t = 16 quad + (lane & 15))
    int done1 = 0;
    if (ok && lane == 0) done1 = mbar_wait(&bar[1], par, abort_flag, status) ? 1 : 0;
    __syncwarp();
    done1 = __shfl_sync(0xffffffffu, done1, 0);
    if (done1) {
        tc_fence_after();
        // all 16 warps: warp w reads TMEM lane quadrant w % 4 (M = 64 layout: rows
        // t = 16 (w % 4) + (lane & 15) in the quadrant's lanes 0-15) at columns
        // 16 (w / 4) .. + 15 of S and dP0; lanes 16-31 take their row's upper 8
        const int cg = warp >> 2, t = 16 * quad + (lane & 15), hh = lane >> 4;
        const float bt = sb[t], mtt = smt[t], dnqt = sdnq[t];
        uint32_t ss[16], sp[16];
        tmem_ld16(tacc + Lay::cS + lane_addr + 16 * cg, ss);
        tmem_ld16(tacc + Lay::cP + lane_addr + 16 * cg, sp);
        tmem_wait_ld();
        uint32_t h1[4], l1[4], h2_[4], l2_[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float m1[2], m2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t us = __shfl_sync(0xffffffffu, ss[8 + e + u], lane & 15);
                const uint32_t up = __shfl_sync(0xffffffffu, sp[8 + e + u], lane & 15);
                const float sv = __uint_as_float(hh ? us : ss[e + u]);
                const float dp = __uint_as_float(hh ? up : sp[e + u]);
                const int s_ = 16 * cg + 8 * hh + e + u;
                const float w = (t < n && s_ <= t) ? expf(bt - sb[s_] + sip[s_] - mtt) : 0.f;
                m2[u] = w * sv * inv_sqrt;
                m1[u] = w * (dp + dnqt);
            }
            h1[e / 2] = cvt_bf16x2(m1[0], m1[1]);
            const __nv_bfloat162 a1 = *reinterpret_cast<const __nv_bfloat162 *>(&h1[e / 2]);
            l1[e / 2] = cvt_bf16x2(m1[0] - __low2float(a1), m1[1] - __high2float(a1));
            h2_[e / 2] = cvt_bf16x2(m2[0], m2[1]);
            const __nv_bfloat162 a2 = *reinterpret_cast<const __nv_bfloat162 *>(&h2_[e / 2]);
            l2_[e / 2] = cvt_bf16x2(m2[0] - __low2float(a2), m2[1] - __high2float(a2));
        }
        const uint32_t off = (uint32_t)t * 128u + ((uint32_t)((2 * cg + hh) ^ (t & 7)) << 4);
        *reinterpret_cast<uint4 *>(smem + Lay::kM1h + off) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
        *reinterpret_cast<uint4 *>(smem + Lay::kM1l + off) = make_uint4(l1[0], l1[1], l1[2], l1[3]);
        *reinterpret_cast<uint4 *>(smem + Lay::kM2h + off) = make_uint4(h2_[0], h2_[1], h2_[2], h2_[3]);
        *reinterpret_cast<uint4 *>(smem + Lay::kM2l + off) = make_uint4(l2_[0], l2_[1], l2_[2], l2_[3]);
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (done1 && tid == 0) {
        tc_fence_after();
        const uint32_t i_kt = idesc_f32acc(kFmtBF16, kFmtBF16, true, false, 128, 64);   // A^T, B K-major
        const uint32_t i_tt = idesc_f32acc(kFmtBF16, kFmtBF16, true, true, 128, 64);    // A^T, B^T
        const uint32_t sq = smem_u32(smem + Lay::kQ), sk = smem_u32(smem + Lay::kK), sdh = smem_u32(smem + Lay::kDh),
                       sdl = smem_u32(smem + Lay::kDl), m1h = smem_u32(smem + Lay::kM1h), m1l = smem_u32(smem + Lay::kM1l),
                       m2h = smem_u32(smem + Lay::kM2h), m2l = smem_u32(smem + Lay::kM2l);
#pragma unroll
        for (int mt = 0; mt < kTiles<D>; ++mt)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint32_t ta = 2 * mt * 8192 + ks * 2048;          // 16 token rows of a 128-row tile's two boxes
                const uint32_t acc = ks > 0 ? 1u : 0u;
                // dq^T = K^T M1^T: B = M1 rows t, K = s (K-major)
                const uint64_t ak = sdesc_sw128(sk + ta, 8192, 1024);
                mma_bf16_ss(tacc + Lay::cDq + 64 * mt, ak, sdesc_sw128(m1h + ks * 32, 16, 1024), i_kt, acc);
                mma_bf16_ss(tacc + Lay::cDq + 64 * mt, ak, sdesc_sw128(m1l + ks * 32, 16, 1024), i_kt, 1u);
                // dk^T = Q^T M1: B = M1 read as (N = s contiguous, K = t rows)
                const uint64_t aq = sdesc_sw128(sq + ta, 8192, 1024);
                mma_bf16_ss(tacc + Lay::cDk + 64 * mt, aq, sdesc_sw128(m1h + ks * 2048, 8192, 1024), i_tt, acc);
                mma_bf16_ss(tacc + Lay::cDk + 64 * mt, aq, sdesc_sw128(m1l + ks * 2048, 8192, 1024), i_tt, 1u);
                // dv^T = dnum'^T M2
                const uint64_t adh = sdesc_sw128(sdh + ta, 8192, 1024), adl = sdesc_sw128(sdl + ta, 8192, 1024);
                const uint64_t bm2h = sdesc_sw128(m2h + ks * 2048, 8192, 1024);
                mma_bf16_ss(tacc + Lay::cDv + 64 * mt, adh, bm2h, i_tt, acc);
                mma_bf16_ss(tacc + Lay::cDv + 64 * mt, adl, bm2h, i_tt, 1u);
                mma_bf16_ss(tacc + Lay::cDv + 64 * mt, adh, sdesc_sw128(m2l + ks * 2048, 8192, 1024), i_tt, 1u);
            }
        mma_commit(&bar[2]);
    }
    int done2 = 0;
    if (done1 && lane == 0) done2 = mbar_wait(&bar[2], par, abort_flag, status) ? 1 : 0;
    __syncwarp();
    done2 = __shfl_sync(0xffffffffu, done2, 0);
    const long long next = item + gridDim.x;
    if (done2 && tid == 0 && next < items) {     // the MMAs are done with the tiles: next item's, but k
        load_tiles(next, true, false, true);
        loads_pending = true;
        pend_par = par ^ 1u;
    }
    if (done2) {
        tc_fence_after();
        const int tg = warp >> 2;
        uint32_t v[kTiles<D>][16];
        __nv_bfloat16 *dq = reinterpret_cast<__nv_bfloat16 *>(p.dq), *dk = reinterpret_cast<__nv_bfloat16 *>(p.dk),
                      *dv = reinterpret_cast<__nv_bfloat16 *>(p.dv);
        // the state products of the 16 tokens are loaded before the first store
        // (the stores could alias them otherwise)
        float x[16][kTiles<D>];
        auto preload = [&](const float *src) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int t = 16 * tg + e;
#pragma unroll
                for (int mt = 0; mt < kTiles<D>; ++mt) {
                    const int r = 128 * mt + 32 * quad + lane;
                    x[e][mt] = t < n && r < D ? src[(row0 + t) * D + r] : 0.f;
                }
            }
        };
        // dq
        preload(p.num);
#pragma unroll
        for (int mt = 0; mt < kTiles<D>; ++mt) tmem_ld16(tacc + Lay::cDq + 64 * mt + lane_addr + 16 * tg, v[mt]);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int t = 16 * tg + e;
            if (t >= n) continue;
            const size_t ro = (row0 + t) * D;
#pragma unroll
            for (int mt = 0; mt < kTiles<D>; ++mt) {
                const int j = 128 * mt + 32 * quad + lane;
                if (j >= D) continue;
                dq[ro + j] = __float2bfloat16_rn(__uint_as_float(v[mt][e]) * inv_sqrt +
                                                 sg[t] * (x[e][mt] + sdnq[t] * snp[j]));
            }
        }
        // dk, ditilde
        preload(p.dki);
#pragma unroll
        for (int mt = 0; mt < kTiles<D>; ++mt) tmem_ld16(tacc + Lay::cDk + 64 * mt + lane_addr + 16 * tg, v[mt]);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int s_ = 16 * tg + e;
            if (s_ >= n) continue;
            const size_t ro = (row0 + s_) * D;
            float di = 0.f;
#pragma unroll
            for (int mt = 0; mt < kTiles<D>; ++mt) {
                const int j = 128 * mt + 32 * quad + lane;
                if (j >= D) continue;
                const float dkh = __uint_as_float(v[mt][e]) + swk[s_] * (x[e][mt] + sdnb[j]);
                const float kv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(
                    smem + Lay::kK + (j >> 6) * 8192 + s_ * 128 + ((((j & 63) >> 3) ^ (s_ & 7)) << 4) + ((j & 7) << 1)));
                di += dkh * kv * inv_sqrt;
                dk[ro + j] = __float2bfloat16_rn(dkh * inv_sqrt);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) di += __shfl_xor_sync(0xffffffffu, di, o);
            if (lane == 0) red[quad * 64 + s_] = di;
        }
        // dv
        preload(p.dvi);
#pragma unroll
        for (int mt = 0; mt < kTiles<D>; ++mt) tmem_ld16(tacc + Lay::cDv + 64 * mt + lane_addr + 16 * tg, v[mt]);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int s_ = 16 * tg + e;
            if (s_ >= n) continue;
            const size_t ro = (row0 + s_) * D;
#pragma unroll
            for (int mt = 0; mt < kTiles<D>; ++mt) {
                const int i = 128 * mt + 32 * quad + lane;
                if (i >= D) continue;
                dv[ro + i] = __float2bfloat16_rn(__uint_as_float(v[mt][e]) + swk[s_] * inv_sqrt * x[e][mt]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (done2 && tid == 0 && next < items) load_tiles(next, false, true, false);   // k, read by the epilogue until here
    if (done2 && tid < n) {
        const int s_ = tid;
        const float di = red[s_] + red[64 + s_] + red[128 + s_] + red[192 + s_];
        p.di[row0 + s_] = di;
        p.dF[row0 + s_] = sA[s_] - di;
    }
    __syncthreads();
    if (*abort_flag) break;                          // every thread reads the flag after the barrier
    }
    // no copy left in flight into shared memory
    if (tid == 0 && loads_pending) mbar_wait(&bar[0], pend_par, nullptr, nullptr);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tacc, 512);
    }
}

}  // namespace bwdtc
}  // namespace xlstm
