// Chunkwise mLSTM forward on the 5th-generation tensor cores with the matrix
// memory held in registers ("xLSTM: Extended Long Short-Term Memory" section
// 2.3: retrieval by matrix multiplication, covariance update of the matrix
// memory; section 2.2: exponential gating with the stabiliser m).
//
// One CTA owns RV = min(DH, 128) value rows and KC key columns of one head's
// state over one segment of the sequence (the segments combine through the
// two-level scan of fwd_tc.cu).  The CTA's part of the stabilised state C'
// stays in fp32 registers of eight "state" warps for the whole segment; at
// each chunk boundary those warps fold the chunk's update into it and write
// it into tensor memory as two bf16 parts, C' = Chi + Clo (15 to 16
// significant bits), the A operand of the retrieval.
//
// A chunk of L = 64 NSUB tokens is processed as NSUB sub-blocks of 64 tokens.
// The state is carried across chunks only; inside a chunk the outputs are the
// causal quadratic form over all L tokens, taken tile by tile.  Per chunk,
// with Q_j, K_i, V_i the bf16 tiles of sub-blocks j, i (staged by TMA):
//
//   S_ji  = Q_j [K_i; n'hi; n'mid; n'lo]^T        M=64,  N=72, K=KC  (i <= j)
//   H_j^T = sum_{i<=j} (w V_i)^T P_ji^T            M=128, N=64, K=64
//           P_ji = rho * S_ji (masked s <= t when i = j)
//   H_j^T += (Chi + Clo) Q_j^T                     M=128, N=64, K=KC (A in TMEM)
//   U     = sum_i (w V_i)^T K_i                    M=128, N=KC, K=64
//   C'   <- a C' + U                               (fp32, in the state warps)
//
// with u_s = itilde_s - b_s (b = within-chunk cumulative log f), Mc = max_s
// u_s over the chunk, m_prev the stabiliser before the chunk, M = max(m_prev,
// Mc) and
//   w_s = e^{u_s - M} / sqrt(d),  rho = e^{M - m_prev},  a = e^{m_prev - M},
//   g_t = e^{m_prev - max(m_prev, pmax_t)},  m_t = b_t + max(m_prev, pmax_t),
// so the state after the chunk is exactly a C' + U (all exponents <= 0), the
// exact intra-chunk weight e^{b_t - b_s + itilde_s - m_t} / sqrt(d) equals
// g_t rho w_s, and
//   h_t = o_t * g_t H_t / max(|g_t (n'.q_t + rho sum_s w_s S_ts)|, e^{-m_t}).
// n'.q_t rides in the scores product: the normaliser n' (of the chunk start),
// as three bf16 parts (about 24 significant bits), fills key rows 64-66 of
// every key tile, so S has 72 columns.
// A chunk is "wide" when Mc > m_prev + 40 (rho would leave the fp32 range):
// then P carries exact per-row weights against V as loaded (rows whose own
// stabiliser moved by more than e^40 have the old state's share below fp32
// resolution; their retrieval term is dropped by zeroing those query rows
// after the scores have read them), and V is scaled by w only after the
// intra-chunk products have read it.
//
// DH 512 (and DH 256 at chunk 256) split the key columns over KS = 2 CTAs:
// the cell is linear in the scores and the state until the final division, so
// each CTA writes its share of the numerator and the denominator (its scores
// carried as bf16 hi + lo parts, since the halves' partial scores can cancel)
// and combine_keysplit_kernel forms h.
//
// Warp roles (16 warps): 0 TMA (q, k, v), 1 MMA issue and TMEM owner, 2 gates
// and the normaliser chain n', 3 TMA (output gates); 4-11 state (C' rows, the
// fold, the bf16 parts, w V, and h from H, stored straight to global memory);
// 12-15 scores (masked weighted scores and the denominators).  Every wait is
// bounded (tc_ptx.cuh): on a timeout the kernel raises the device status word
// and unwinds.
#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "tc_ptx.cuh"

namespace xlstm {

using namespace tc;

namespace {

constexpr int kRsThreads = 512;
constexpr float kWideGap = 40.f;   // ln of the largest factor rho may take

template <int D, int NSUB>
struct RsCfg {
    static constexpr int L = 64 * NSUB;                // chunk (tokens)
    static constexpr int KC = (NSUB == 4 && D >= 256) ? 128 : (D > 256 ? 256 : D);   // key columns per CTA
    static constexpr int KS = D / KC;                  // key splits (CTAs per value tile)
    static constexpr int RV = D < 128 ? D : 128;       // value rows (MMAs keep M = 128)
    static constexpr int VB = RV / 64;                 // 64-column blocks of the value tile
    static constexpr int KPT = KC / 2;                 // keys per state thread (two warps per lane quadrant)
    static constexpr int NKV = NSUB >= 2 ? NSUB : 2;   // key / value slots (one chunk, or a ring of two)
    static constexpr int TPC = NSUB * (NSUB + 1) / 2;  // score tiles per chunk
    static constexpr bool kSharedRU = 2 * KC + 72 + 128 > 512;
    static constexpr uint32_t R0 = 0;                  // bf16 parts: hi [0, KC/2), lo [KC/2, KC)
    static constexpr uint32_t U0 = kSharedRU ? 0 : KC; // fp32 chunk update
    static constexpr uint32_t S0 = kSharedRU ? KC : 2 * KC;
    static constexpr uint32_t H0 = S0 + 72;            // two 64-column buffers
    static_assert(H0 + 128 <= 512, "tensor memory");
    // shared memory (bytes; 1024-aligned operand tiles first)
    static constexpr int kQbytes = (KC / 64) * 8192;   // [64 tokens][KC] bf16, 64-key blocks, 128 B swizzle
    static constexpr int kKBlock = 72 * 128;           // key block: 64 key rows + n' hi/mid/lo + 5 zero rows
    static constexpr int kKbytes = (KC / 64) * kKBlock;
    static constexpr int kVbytes = 16384;              // [64 tokens][128 values] bf16, two blocks
    static constexpr int kObytes = KS == 1 ? 64 * RV * 4 : 0;   // [64 tokens][RV] fp32 output-gate pre-activations
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + 2 * kQbytes;
    static constexpr int kV = kK + NKV * kKbytes;
    static constexpr int kO = kV + NKV * kVbytes;
    // [64][64] bf16 masked scores, 128 B swizzle; with split keys also a low part
    // (each CTA's partial scores are rounded on their own, so where the halves
    // cancel one bf16 rounding would be amplified)
    static constexpr int kPparts = KS > 1 ? 2 : 1;
    static constexpr int kP = kO + kObytes;
    static constexpr int kGB = NSUB >= 4 ? 2 : 3;      // gate buffers (ring)
    static constexpr int kNG = 8;
    static constexpr int kG = kP + kPparts * 8192;     // per-token gate arrays [kGB][kNG][L]
    static constexpr int kGs = kG + kGB * kNG * L * 4; // per-chunk gate scalars [kGB][8]
    static constexpr int kBar = kGs + kGB * 8 * 4;
    static constexpr int kNumBars = 56;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 64 + 1024;   // + slack for 1024-byte alignment
    static_assert(kBytes <= 232448, "shared memory");
};

// per-token gate arrays
enum { G_W = 0, G_G, G_FL, G_U, G_REF, G_OF, G_INV, G_LATE };
// per-chunk scalars
enum { GS_RHO = 0, GS_A, GS_WIDE, GS_LC };

// barriers; the K / V ones have one slot per key/value buffer (up to 4)
enum {
    B_QF = 0, B_QE = 2, B_KF = 4, B_KE = 8, B_VF = 12, B_VE = 16, B_VH = 20,
    B_OF = 24, B_OE, B_SF, B_SE, B_PR, B_PE, B_HF, B_HE = B_HF + 2, B_RR = B_HE + 2, B_RD, B_UF, B_ID,
    B_SQ, B_QZ, B_GR, B_GE = B_GR + 3, B_NR = B_GE + 3, B_INV, B_DONE = B_INV + 2, B_NUM
};
static_assert(B_NUM <= 56, "barrier slots");

#ifdef XLSTM_RS_TRACE
// Timing trace of the pipeline steps (diagnostic builds only): 32 clock64()
// stamps per (CTA, chunk) for the first kRsTraceChunks chunks.
__device__ unsigned long long *g_rs_trace = nullptr;
constexpr int kRsTraceChunks = 64;
#define RS_TRACE(cond, c, slot)                                                                    \
    do {                                                                                           \
        if (g_rs_trace && (cond) && (c) < kRsTraceChunks) {                                        \
            const size_t cta_ = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x; \
            g_rs_trace[(cta_ * kRsTraceChunks + (c)) * 32 + (slot)] = clock64();                   \
        }                                                                                          \
    } while (0)
#else
#define RS_TRACE(cond, c, slot) do { } while (0)
#endif

// Waits of this kernel: hardware-suspending by default (a spinning poller
// costs the co-scheduled warps issue slots); XLSTM_RS_SPIN_WAITS selects the
// spinning variant for comparison.
__device__ __forceinline__ bool rs_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, unsigned int *status) {
#ifdef XLSTM_RS_SPIN_WAITS
    return mbar_wait(bar, parity, abort_flag, status);
#else
    return mbar_wait_sleep(bar, parity, abort_flag, status);
#endif
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// named barriers: 1 = state group (256 threads), 2 = score group (128)
__device__ __forceinline__ void sync_state() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void sync_so() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

// The thread's KPT state values (keys kbase ...) as two bf16 parts, hi + lo,
// into the retrieval operand in tensor memory: hi at columns [0, KC/2) and lo
// at [KC/2, KC) of `t_row` (two keys per 32-bit column, even key low).  Both
// parts are truncations (hi = the upper 16 bits of x, lo = those of x - hi,
// which is exact in fp32), so x - (hi + lo) < 2^-14 |x|; byte permutes pack
// them without conversion instructions.
template <int KPT, int KC>
__device__ __forceinline__ void write_parts(const float (&Cs)[KPT], uint32_t t_row, int kbase) {
#pragma unroll
    for (int pc = 0; pc < KPT / 16; ++pc) {
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t x0 = __float_as_uint(Cs[16 * pc + 2 * e]), x1 = __float_as_uint(Cs[16 * pc + 2 * e + 1]);
            hi[e] = __byte_perm(x0, x1, 0x7632);
            const float r0 = __uint_as_float(x0) - __uint_as_float(x0 & 0xFFFF0000u);
            const float r1 = __uint_as_float(x1) - __uint_as_float(x1 & 0xFFFF0000u);
            lo[e] = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
        }
        const uint32_t col = (uint32_t)((kbase + 16 * pc) / 2);
        tmem_st8(t_row + col, hi);
        tmem_st8(t_row + KC / 2 + col, lo);
    }
    tmem_wait_st();
}

// Score tile t of a chunk (0 <= t < NSUB (NSUB + 1) / 2) in issue order
// (0,0), (1,0), (1,1), (2,0), ...: query sub-block j, key sub-block i <= j.
__device__ __forceinline__ void tile_ji(int t, int &j, int &i) {
    j = 0;
    while ((j + 1) * (j + 2) / 2 <= t) ++j;
    i = t - j * (j + 1) / 2;
}

template <int D, int NSUB>
__global__ void __launch_bounds__(kRsThreads, 1)
segment_output_rs_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                         __nv_bfloat16 *__restrict__ h_out, const float *__restrict__ i_pre,
                         const float *__restrict__ C0, const float *__restrict__ n0, const float *__restrict__ m0,
                         float *__restrict__ C_out, float *__restrict__ n_out, float *__restrict__ m_out,
                         const float *__restrict__ bcum, const float *__restrict__ pmx,
                         const float2 *__restrict__ cstat, const float2 *__restrict__ sstat,
                         const float *__restrict__ summ, float *__restrict__ part, float *__restrict__ dpart,
                         float2 *__restrict__ tokrec, unsigned int *status, int S, int nchunks, int P, int cps) {
    using Cfg = RsCfg<D, NSUB>;
    constexpr int L = Cfg::L, KC = Cfg::KC, KS = Cfg::KS, RV = Cfg::RV, VB = Cfg::VB, KPT = Cfg::KPT;
    constexpr int GB = Cfg::kGB, KB = Cfg::kKBlock, NKV = Cfg::NKV, TPC = Cfg::TPC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sQ = smem + Cfg::kQ;
    uint8_t *sK = smem + Cfg::kK;
    uint8_t *sV = smem + Cfg::kV;
    float *sO = reinterpret_cast<float *>(smem + Cfg::kO);
    uint8_t *sP = smem + Cfg::kP;
    float *gA = reinterpret_cast<float *>(smem + Cfg::kG);      // [GB][kNG][L]
    float *gS = reinterpret_cast<float *>(smem + Cfg::kGs);     // [GB][8]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Cfg::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kMisc + 4);
    auto garr = [&](int gb, int which) { return gA + (gb * Cfg::kNG + which) * L; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x / KS, kh = blockIdx.x % KS, g = blockIdx.y, bh = blockIdx.z;
    const int i0 = tile * RV, k0 = kh * KC;        // value rows and key columns of this CTA
    const int c0 = g * cps;                        // first chunk of this segment
    const int nch = max(0, min(nchunks, c0 + cps) - c0);
    const int nsb = nch * NSUB;                    // sub-blocks of this segment
    const int tseg = c0 * L;                       // first token of this segment
    const size_t tok0 = (size_t)bh * S;
    const float inv_sqrt_d = rsqrtf((float)D);
    const int q4 = warp & 3;
    const uint32_t lane_addr = ((uint32_t)(32 * q4)) << 16;

    if (tid == 0) {
        for (int i = 0; i < B_NUM; ++i) {
            const bool two = (i >= B_KE && i < B_KE + 4) || (i >= B_GE && i < B_GE + 3);
            mbar_init(&bars[i], two ? 2 : 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    // rows 64-71 of every key block start at zero (TMA writes rows 0-63 only;
    // the normaliser parts go to rows 64-66), and so does an unloaded value block
    for (int e = tid; e < NKV * (KC / 64) * 64; e += kRsThreads) {     // (slot, block, row 64-71, chunk)
        const int ch = e & 7, row = 64 + ((e >> 3) & 7), blk = (e >> 6) % (KC / 64), sl = e / (64 * (KC / 64));
        *reinterpret_cast<uint4 *>(sK + sl * Cfg::kKbytes + blk * KB + sw128_offset(row, ch)) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (VB == 1) {
        for (int e = tid; e < NKV * 512; e += kRsThreads)
            *reinterpret_cast<uint4 *>(sV + (e >> 9) * Cfg::kVbytes + 8192 + (e & 511) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    pdl_wait();                                    // the segment scan's states and the gate statistics
    const uint32_t tbase = *tmem_slot;
    const uint32_t tR = tbase + Cfg::R0, tU = tbase + Cfg::U0, tS = tbase + Cfg::S0, tH = tbase + Cfg::H0;

    // Register budget per warpgroup (KC = 256: the state warps hold 128 floats of
    // C' per thread): 128 x 64 + 256 x 168 + 128 x 104 = 64512 <= 512 x 128.
    if (warp < 4) {
        if (KC == 256) regs_dec<64>();
        if (warp == 0) {
            // ------------------------------------------------ TMA: q, k, v per sub-block
            if (lane == 0 && nch > 0) {
                tma_prefetch_desc(&map_q);
                tma_prefetch_desc(&map_k);
                tma_prefetch_desc(&map_v);
                int issued[3][4] = {};
                for (int b = 0; b < nsb; ++b) {
                    const int t0 = tseg + 64 * b, qs = b & 1, ks = b % NKV;
                    if (b + 2 < nsb) {
                        for (int jb = 0; jb < KC / 64; ++jb) {
                            tma_prefetch_l2_3d(&map_q, k0 + jb * 64, t0 + 128, bh);
                            tma_prefetch_l2_3d(&map_k, k0 + jb * 64, t0 + 128, bh);
                        }
                        for (int vb = 0; vb < VB; ++vb) tma_prefetch_l2_3d(&map_v, i0 + 64 * vb, t0 + 128, bh);
                    }
                    if (b >= 2 && !rs_wait(&bars[B_QE + qs], ((b >> 1) - 1) & 1, abort_flag, status)) break;
                    mbar_arrive_expect_tx(&bars[B_QF + qs], 64 * KC * 2);
                    for (int jb = 0; jb < KC / 64; ++jb)
                        tma_load_3d(sQ + qs * Cfg::kQbytes + jb * 8192, &map_q, &bars[B_QF + qs], k0 + jb * 64, t0, bh);
                    ++issued[0][qs];
                    if (b >= NKV && !rs_wait(&bars[B_KE + ks], ((b / NKV) - 1) & 1, abort_flag, status)) break;
                    mbar_arrive_expect_tx(&bars[B_KF + ks], 64 * KC * 2);
                    for (int jb = 0; jb < KC / 64; ++jb)
                        tma_load_3d(sK + ks * Cfg::kKbytes + jb * KB, &map_k, &bars[B_KF + ks], k0 + jb * 64, t0, bh);
                    ++issued[1][ks];
                    if (b >= NKV && !rs_wait(&bars[B_VE + ks], ((b / NKV) - 1) & 1, abort_flag, status)) break;
                    mbar_arrive_expect_tx(&bars[B_VF + ks], 64 * VB * 64 * 2);
                    for (int vb = 0; vb < VB; ++vb)
                        tma_load_3d(sV + ks * Cfg::kVbytes + vb * 8192, &map_v, &bars[B_VF + ks], i0 + 64 * vb, t0, bh);
                    ++issued[2][ks];
                }
                // never leave a load in flight into shared memory
                for (int s = 0; s < 4; ++s) {
                    if (s < 2 && issued[0][s]) mbar_wait(&bars[B_QF + s], (issued[0][s] - 1) & 1, nullptr, status);
                    if (s < NKV && issued[1][s]) mbar_wait(&bars[B_KF + s], (issued[1][s] - 1) & 1, nullptr, status);
                    if (s < NKV && issued[2][s]) mbar_wait(&bars[B_VF + s], (issued[2][s] - 1) & 1, nullptr, status);
                }
            }
        } else if (warp == 3) {
            // ------------------------------------------ TMA: output gates per sub-block
            if (KS == 1 && lane == 0 && nch > 0) {
                tma_prefetch_desc(&map_o);
                int issued = 0;
                for (int b = 0; b < nsb; ++b) {
                    const int t0 = tseg + 64 * b;
                    if (b + 1 < nsb) tma_prefetch_l2_3d(&map_o, i0, t0 + 64, bh);
                    if (b >= 1 && !rs_wait(&bars[B_OE], (b - 1) & 1, abort_flag, status)) break;
                    mbar_arrive_expect_tx(&bars[B_OF], 64 * RV * 4);
                    tma_load_3d(sO, &map_o, &bars[B_OF], i0, t0, bh);
                    ++issued;
                }
                if (issued) mbar_wait(&bars[B_OF], (issued - 1) & 1, nullptr, status);
            }
        } else if (warp == 2) {
            // ------------------------------------------- gates and normaliser chain
            // Gates run two chunks ahead of the normaliser.  Stabiliser entering
            // this segment: the initial m, folded through the statistics (total
            // log f, own stabiliser) of the segments before it.
            float mc = m0 ? m0[bh] : 0.f;
            for (int gp = 0; gp < g; ++gp) {
                const float2 st = sstat[(size_t)bh * P + gp];
                mc = fmaxf(st.x + mc, st.y);
            }
            constexpr int TPL = L / 32;                      // tokens per lane
            float pb_[TPL], px_[TPL], pi_[TPL];
            auto fetch = [&](int c) {
                const int t0 = tseg + c * L;
#pragma unroll
                for (int h2 = 0; h2 < TPL; ++h2) {
                    const int t = t0 + lane + 32 * h2;
                    const bool ok = t < S;
                    pb_[h2] = ok ? bcum[tok0 + t] : 0.f;
                    px_[h2] = ok ? pmx[tok0 + t] : 0.f;
                    pi_[h2] = ok ? i_pre[tok0 + t] : 0.f;
                }
            };
            auto gates = [&](int c) -> bool {
                const int gb = c % GB, t0 = tseg + c * L, Lc = min(L, S - t0);
                if (c >= GB && !rs_wait(&bars[B_GE + gb], ((c / GB) - 1) & 1, abort_flag, status)) return false;
                const float2 cs = cstat[(size_t)bh * nchunks + c0 + c];   // (sum of log f, max of u)
                const float Mc = cs.y;
                const bool wide = Mc > mc + kWideGap;
                const float big = fmaxf(mc, Mc);
                float b_[TPL], x_[TPL], ii_[TPL];
#pragma unroll
                for (int h2 = 0; h2 < TPL; ++h2) { b_[h2] = pb_[h2]; x_[h2] = px_[h2]; ii_[h2] = pi_[h2]; }
                if (c + 1 < nch) fetch(c + 1);
#pragma unroll
                for (int h2 = 0; h2 < TPL; ++h2) {
                    const int t = lane + 32 * h2;
                    const bool valid = t < Lc;
                    const float u = ii_[h2] - b_[h2];
                    const float pm = x_[h2];
                    const float run = fmaxf(mc, pm);
                    const bool late = wide && pm > mc + kWideGap;
                    const float gt = valid ? expf(mc - run) : 0.f;
                    garr(gb, G_W)[t] = valid ? expf(u - big) * inv_sqrt_d : 0.f;
                    garr(gb, G_G)[t] = gt;
                    garr(gb, G_FL)[t] = valid ? expf(-(b_[h2] + run)) : 1.f;
                    garr(gb, G_U)[t] = valid ? u : -INFINITY;
                    garr(gb, G_REF)[t] = late ? pm : mc;
                    garr(gb, G_OF)[t] = late ? 1.f : gt;
                    garr(gb, G_LATE)[t] = late ? 1.f : 0.f;
                }
                if (lane == 0) {
                    float *gs = gS + gb * 8;
                    gs[GS_RHO] = wide ? 0.f : expf(big - mc);
                    gs[GS_A] = expf(mc - big);
                    gs[GS_WIDE] = wide ? 1.f : 0.f;
                    gs[GS_LC] = (float)Lc;
                }
                mc = cs.x + big;
                __syncwarp();
                RS_TRACE(lane == 0, c, 24);
                if (lane == 0) mbar_arrive(&bars[B_GR + gb]);
                return true;
            };
            // normaliser n': lane holds keys [KPL lane, KPL lane + KPL) of this CTA's columns
            constexpr int KPL = KC / 32;
            float nr[KPL];
            const float *nsrc = g == 0 ? (n0 ? n0 + (size_t)bh * D : nullptr)
                                       : summ + ((size_t)bh * (P - 1) + g - 1) * ((size_t)D * D + D) + (size_t)D * D;
#pragma unroll
            for (int e = 0; e < KPL; ++e) nr[e] = nsrc ? nsrc[k0 + KPL * lane + e] : 0.f;
            const int kblk = (KPL * lane) / 64;                     // key block of this lane's keys
            const int kbyte = (KPL * lane * 2) % 128;               // byte offset within a 128-byte row
            // n' as bf16 hi / mid / lo parts into rows 64-66 of key slot sl
            auto write_nparts = [&](int sl) {
                uint8_t *blk = sK + sl * Cfg::kKbytes + kblk * KB;
                uint32_t ph[KPL / 2], pmid[KPL / 2], plo[KPL / 2];
#pragma unroll
                for (int e = 0; e < KPL / 2; ++e) {
                    const float x0 = nr[2 * e], x1 = nr[2 * e + 1];
                    const uint32_t h2 = cvt_bf16x2(x0, x1);
                    const float r0 = x0 - bf_lo(h2), r1 = x1 - bf_hi(h2);
                    const uint32_t m2 = cvt_bf16x2(r0, r1);
                    ph[e] = h2;
                    pmid[e] = m2;
                    plo[e] = cvt_bf16x2(r0 - bf_lo(m2), r1 - bf_hi(m2));
                }
#pragma unroll
                for (int e = 0; e < KPL / 2; ++e) {
                    const int byte = kbyte + 4 * e;
                    const int cc = byte >> 4, within = byte & 15;
                    *reinterpret_cast<uint32_t *>(blk + sw128_offset(64, cc) + within) = ph[e];
                    *reinterpret_cast<uint32_t *>(blk + sw128_offset(65, cc) + within) = pmid[e];
                    *reinterpret_cast<uint32_t *>(blk + sw128_offset(66, cc) + within) = plo[e];
                }
            };
            // the parts of chunk c go to the key slots of its sub-blocks
            auto publish_n = [&](int c) {
                for (int j = 0; j < NSUB; ++j) write_nparts((c * NSUB + j) % NKV);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_NR]);
            };
            bool ok = true;
            if (nch > 0) {
                fetch(0);
                ok = gates(0) && (nch < 2 || gates(1));
                if (ok) publish_n(0);
            }
            for (int c = 0; ok && c < nch; ++c) {
                const int gb = c % GB;
                // n'(c+1) = a n'(c) + sum_s w_s k_s over this chunk's keys, fp32
                const float *w = garr(gb, G_W);
                const float a = gS[gb * 8 + GS_A];
                float acc[KPL];
#pragma unroll
                for (int e = 0; e < KPL; ++e) acc[e] = 0.f;
                for (int j = 0; j < NSUB && ok; ++j) {
                    const int b = c * NSUB + j, ks = b % NKV;
                    if (!rs_wait(&bars[B_KF + ks], (b / NKV) & 1, abort_flag, status)) { ok = false; break; }
                    const uint8_t *kt = sK + ks * Cfg::kKbytes + kblk * KB;
#pragma unroll 4
                    for (int s = 0; s < 64; ++s) {
                        const float ws = w[64 * j + s];
                        const uint8_t *rp = kt + sw128_offset(s, kbyte >> 4) + (kbyte & 15);
                        if (KPL == 8) {
                            const uint4 kv = *reinterpret_cast<const uint4 *>(rp);
                            acc[0] += ws * bf_lo(kv.x); acc[1] += ws * bf_hi(kv.x);
                            acc[2] += ws * bf_lo(kv.y); acc[3] += ws * bf_hi(kv.y);
                            acc[4 % KPL] += ws * bf_lo(kv.z); acc[5 % KPL] += ws * bf_hi(kv.z);
                            acc[6 % KPL] += ws * bf_lo(kv.w); acc[7 % KPL] += ws * bf_hi(kv.w);
                        } else if (KPL == 4) {
                            const uint2 kv = *reinterpret_cast<const uint2 *>(rp);
                            acc[0] += ws * bf_lo(kv.x); acc[1] += ws * bf_hi(kv.x);
                            acc[2 % KPL] += ws * bf_lo(kv.y); acc[3 % KPL] += ws * bf_hi(kv.y);
                        } else {
                            const uint32_t kv = *reinterpret_cast<const uint32_t *>(rp);
                            acc[0] += ws * bf_lo(kv); acc[1 % KPL] += ws * bf_hi(kv);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[B_KE + ks]);
                }
                if (!ok) break;
#pragma unroll
                for (int e = 0; e < KPL; ++e) nr[e] = fmaf(a, nr[e], acc[e]);
                if (c + 1 < nch) {
                    // the slots chunk c+1 uses were last read by the scores of chunk
                    // c + 1 - NKV / NSUB; that chunk's update completing implies they are done
                    const int cp = c + 1 - NKV / NSUB;
                    if (cp >= 0 && !rs_wait(&bars[B_UF], cp & 1, abort_flag, status)) { ok = false; break; }
                    publish_n(c + 1);
                }
                if (c + 2 < nch && !gates(c + 2)) { ok = false; break; }
            }
            if (ok && g == P - 1 && tile == 0 && nch > 0 && !*abort_flag) {
                if (lane == 0 && kh == 0 && m_out) m_out[bh] = mc;
                if (n_out) {
#pragma unroll
                    for (int e = 0; e < KPL; ++e) n_out[(size_t)bh * D + k0 + KPL * lane + e] = nr[e];
                }
            }
        } else {
            // ------------------------------------------------------- MMA issue
            if (lane == 0 && nch > 0) {
                const uint32_t idesc_S = idesc_f32acc(kFmtBF16, kFmtBF16, false, false, 64, 72);
                const uint32_t idesc_R = idesc_f32acc(kFmtBF16, kFmtBF16, false, false, 128, 64);
                const uint32_t idesc_I = idesc_f32acc(kFmtBF16, kFmtBF16, true, false, 128, 64);
                const uint32_t idesc_U = idesc_f32acc(kFmtBF16, kFmtBF16, true, true, 128, KC);
                bool ok = true;
                int nw = 0;                  // wide sub-blocks seen
                // scores of global tile gt (chunk gt / TPC): wait for its operands and a free S
                auto issue_scores = [&](int gt_) -> bool {
                    const int c = gt_ / TPC;
                    int j, i;
                    tile_ji(gt_ % TPC, j, i);
                    const int bq = c * NSUB + j, bk = c * NSUB + i;
                    const int qs = bq & 1, ks = bk % NKV;
                    if (!rs_wait(&bars[B_QF + qs], (bq >> 1) & 1, abort_flag, status) ||
                        !rs_wait(&bars[B_KF + ks], (bk / NKV) & 1, abort_flag, status) ||
                        !rs_wait(&bars[B_NR], c & 1, abort_flag, status) ||
                        (gt_ >= 1 && !rs_wait(&bars[B_SE], (gt_ - 1) & 1, abort_flag, status)))
                        return false;
                    tc_fence_after();
                    uint64_t dq = sdesc_sw128(smem_u32(sQ + qs * Cfg::kQbytes), 16, 1024);
                    uint64_t dk = sdesc_sw128(smem_u32(sK + ks * Cfg::kKbytes), 16, 1024);
#pragma unroll 1
                    for (int jb = 0; jb < KC / 64; ++jb) {
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) mma_bf16_ss(tS, dq + 2 * k4, dk + 2 * k4, idesc_S, (jb | k4) != 0);
                        dq += 8192 >> 4;
                        dk += KB >> 4;
                    }
                    mma_commit(&bars[B_SF]);
                    return true;
                };
                const int ntiles = nch * TPC;
                int issued_s = 0;            // score tiles issued so far (global order)
                ok = issue_scores(0);
                if (ok) issued_s = 1;
                for (int c = 0; ok && c < nch; ++c) {
                    const int gb = c % GB;
                    if (!rs_wait(&bars[B_GR + gb], (c / GB) & 1, abort_flag, status)) { ok = false; break; }
                    const bool wide = gS[gb * 8 + GS_WIDE] != 0.f;
                    for (int tt = 0; ok && tt < TPC; ++tt) {
                        const int gt_ = c * TPC + tt;
                        int j, i;
                        tile_ji(tt, j, i);
                        const int bq = c * NSUB + j, bk = c * NSUB + i;
                        const int hb = bq & 1, ks = bk % NKV;
                        const uint32_t tHb = tH + 64 * hb;
                        RS_TRACE(tt == 0, c, 0);
                        // the next score tile into S as soon as this one has been read
                        // (across chunks only when the key slots allow it)
                        if (gt_ + 1 < ntiles && issued_s == gt_ + 1 && (NKV > NSUB || tt + 1 < TPC)) {
                            if (!issue_scores(gt_ + 1)) { ok = false; break; }
                            issued_s = gt_ + 2;
                        }
                        if (i == 0 && bq >= 2 && !rs_wait(&bars[B_HE + hb], ((bq >> 1) - 1) & 1, abort_flag, status)) { ok = false; break; }
                        if ((!wide && !rs_wait(&bars[B_VH + ks], (bk / NKV) & 1, abort_flag, status)) ||
                            !rs_wait(&bars[B_VF + ks], (bk / NKV) & 1, abort_flag, status) ||
                            !rs_wait(&bars[B_PR], gt_ & 1, abort_flag, status)) { ok = false; break; }
                        tc_fence_after();
                        {   // intra-chunk term: H_j^T (+)= (w V_i)^T P_ji^T (wide chunks: V as loaded)
                            const uint32_t va = smem_u32(sV + ks * Cfg::kVbytes), pa = smem_u32(sP);
#pragma unroll
                            for (int pp = 0; pp < Cfg::kPparts; ++pp)
#pragma unroll
                                for (int k4 = 0; k4 < 4; ++k4)
                                    mma_bf16_ss(tHb, sdesc_sw128(va + k4 * 2048, 8192, 1024),
                                                sdesc_sw128(pa + pp * 8192 + k4 * 32, 16, 1024), idesc_I,
                                                (i | pp | k4) != 0);
                            mma_commit(&bars[B_PE]);
                        }
                        RS_TRACE(tt == 0, c, 2);
                        if (i == j) {
                            // the sub-block's scores are all issued: a wide chunk zeroes the
                            // query rows whose retrieval term is dropped before the retrieval
                            if (wide) {
                                mma_commit(&bars[B_SQ]);
                                if (!rs_wait(&bars[B_QZ], nw & 1, abort_flag, status)) { ok = false; break; }
                                ++nw;
                            }
                            if (j == 0 && !rs_wait(&bars[B_RR], c & 1, abort_flag, status)) { ok = false; break; }
                            tc_fence_after();
                            // retrieval: H_j^T += (Chi + Clo) Q_j^T, the parts of C' from TMEM
                            uint64_t dq = sdesc_sw128(smem_u32(sQ + (bq & 1) * Cfg::kQbytes), 16, 1024);
#pragma unroll 1
                            for (int jb = 0; jb < KC / 64; ++jb) {
#pragma unroll
                                for (int k4 = 0; k4 < 4; ++k4) {
                                    const uint32_t col = (uint32_t)(jb * 32 + 8 * k4);
                                    mma_bf16_ts(tHb, tR + col, dq + 2 * k4, idesc_R, 1u);
                                    mma_bf16_ts(tHb, tR + KC / 2 + col, dq + 2 * k4, idesc_R, 1u);
                                }
                                dq += 8192 >> 4;
                            }
                            mma_commit(&bars[B_HF + hb]);
                            mma_commit(&bars[B_QE + (bq & 1)]);
                            if (Cfg::kSharedRU && j == NSUB - 1) mma_commit(&bars[B_RD]);
                            RS_TRACE(j == 0, c, 1);
                        }
                    }
                    if (!ok) break;
                    // the chunk's update: U = sum_i (w V_i)^T K_i, after every retrieval has read the parts
                    if (wide) mma_commit(&bars[B_ID]);
                    if (Cfg::kSharedRU && !rs_wait(&bars[B_RD], c & 1, abort_flag, status)) { ok = false; break; }
                    for (int i = 0; ok && i < NSUB; ++i) {
                        const int bk = c * NSUB + i, ks = bk % NKV;
                        if (wide && !rs_wait(&bars[B_VH + ks], (bk / NKV) & 1, abort_flag, status)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t va = smem_u32(sV + ks * Cfg::kVbytes), ka = smem_u32(sK + ks * Cfg::kKbytes);
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4)
                            mma_bf16_ss(tU, sdesc_sw128(va + k4 * 2048, 8192, 1024), sdesc_sw128(ka + k4 * 2048, KB, 1024),
                                        idesc_U, (i | k4) != 0);
                    }
                    if (!ok) break;
                    mma_commit(&bars[B_UF]);
                    for (int i = 0; i < NSUB; ++i) {
                        const int ks = (c * NSUB + i) % NKV;
                        mma_commit(&bars[B_VE + ks]);
                        mma_commit(&bars[B_KE + ks]);
                    }
                    RS_TRACE(true, c, 4);
                    // the first score tile of the next chunk, when it could not go early
                    if (c + 1 < nch && issued_s == (c + 1) * TPC) {
                        if (!issue_scores((c + 1) * TPC)) { ok = false; break; }
                        issued_s = (c + 1) * TPC + 1;
                    }
                }
                mma_commit(&bars[B_DONE]);
                mbar_wait(&bars[B_DONE], 0, nullptr, status);   // every MMA has completed before TMEM is freed
            }
        }
    } else if (warp < 12) {
        if (KC == 256) regs_inc<168>();
        // ------------------------------------------------------------ state group
        const int sw = warp - 4;                 // 0..7
        const int half = sw >> 2;                // key half (fold) and token half (outputs) of this thread
        const int i = 32 * q4 + lane;            // value row within the tile
        const bool has_row = i < RV;
        const int kbase = half * KPT;            // first key column of this thread (within the CTA's KC)
        const bool leader = sw == 0 && lane == 0;
        float Cs[KPT];
        bool ok = true;
        auto swait = [&](uint64_t *bar, uint32_t parity) -> bool {
            const bool r = leader ? rs_wait(bar, parity, abort_flag, status) : true;
            return group_all<1, 256>(r);
        };
        // V of sub-block b scaled in place by w (the operand of the intra and update products)
        auto scale_v = [&](int b, int gb) {
            const int ks = b % NKV;
            const float *w = garr(gb, G_W) + 64 * (b % NSUB);
            uint8_t *vb = sV + ks * Cfg::kVbytes;
            for (int e = sw * 32 + lane; e < VB * 64 * 8; e += 256) {       // (block, row s, 16 B chunk)
                const int blk = e / (64 * 8), s = (e / 8) % 64, cc = e & 7;
                uint4 *pv = reinterpret_cast<uint4 *>(vb + blk * 8192 + sw128_offset(s, cc));
                const uint4 src = *pv;
                const float ws = w[s];
                uint4 dst;
                dst.x = cvt_bf16x2(bf_lo(src.x) * ws, bf_hi(src.x) * ws);
                dst.y = cvt_bf16x2(bf_lo(src.y) * ws, bf_hi(src.y) * ws);
                dst.z = cvt_bf16x2(bf_lo(src.z) * ws, bf_hi(src.z) * ws);
                dst.w = cvt_bf16x2(bf_lo(src.w) * ws, bf_hi(src.w) * ws);
                *pv = dst;
            }
            fence_async_smem();
            sync_state();
            if (leader) mbar_arrive(&bars[B_VH + ks]);
        };
        // h of sub-block b from H: this thread takes value row i, tokens 32 half ... + 31
        // of the sub-block, and stores straight to global memory (a warp writes 64
        // contiguous bytes per token); with split keys, this CTA's numerator share
        auto out_pass = [&](int b, int gb) -> bool {
            const int hb = b & 1;
            if (!swait(&bars[B_HF + hb], (b >> 1) & 1) || !swait(&bars[B_INV + hb], (b >> 1) & 1) ||
                (KS == 1 && !swait(&bars[B_OF], b & 1)))
                return false;
            RS_TRACE(leader, b / NSUB, 20);
            tc_fence_after();
            const float *inv = garr(gb, G_INV) + 64 * (b % NSUB);
            const int t0 = tseg + 64 * b;
            __nv_bfloat16 *hrow = h_out + (tok0 + t0) * D + i0 + i;
            float *prow = part + (((size_t)kh * gridDim.z + bh) * S + t0) * D + i0 + i;
#pragma unroll 1
            for (int pc = 0; pc < 2; ++pc) {
                const int tb = 32 * half + 16 * pc;
                uint32_t r[16];
                tmem_ld16(tH + 64 * hb + lane_addr + tb, r);
                tmem_wait_ld();
                const int lim = min(16, S - t0 - tb);            // tokens of this piece inside the sequence
                if (KS > 1) {
                    if (has_row) {
#pragma unroll
                        for (int kk = 0; kk < 16; ++kk)
                            if (lim >= 16 || kk < lim) prow[(size_t)(tb + kk) * D] = __uint_as_float(r[kk]);
                    }
                } else if (has_row) {
#pragma unroll
                    for (int kk = 0; kk < 16; ++kk) {
                        const int tt = tb + kk;
                        const float hv = __uint_as_float(r[kk]) * inv[tt];
                        const float o = sO[tt * RV + i];
                        const __nv_bfloat16 hb16 = __float2bfloat16_rn(fmaf(hv, tanh_approx(0.5f * o), hv));
                        if (lim >= 16 || kk < lim) hrow[(size_t)tt * D] = hb16;
                    }
                }
            }
            tc_fence_before();
            sync_state();
            if (leader) {
                mbar_arrive(&bars[B_HE + hb]);
                mbar_arrive(&bars[B_OE]);
            }
            RS_TRACE(leader, b / NSUB, 21);
            return true;
        };
        // wide chunk: zero the query rows of sub-block b whose retrieval term is dropped
        auto zero_late_rows = [&](int b, int gb) {
            const float *lt = garr(gb, G_LATE) + 64 * (b % NSUB);
            uint8_t *qt = sQ + (b & 1) * Cfg::kQbytes;
            for (int e = sw * 32 + lane; e < (KC / 64) * 64 * 8; e += 256) {
                const int blk = e / (64 * 8), t = (e / 8) % 64, ch = e & 7;
                if (lt[t] != 0.f)
                    *reinterpret_cast<uint4 *>(qt + blk * 8192 + sw128_offset(t, ch)) = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_async_smem();
        };
        // incoming state: the initial state for segment 0, else the state at the
        // end of segment g - 1, which segment_scan_kernel left in summary slot g - 1
        {
            const float *src = g == 0 ? (C0 ? C0 + (size_t)bh * D * D : nullptr)
                                      : summ + ((size_t)bh * (P - 1) + g - 1) * ((size_t)D * D + D);
            if (src && has_row) {
                const float4 *row = reinterpret_cast<const float4 *>(src + (size_t)(i0 + i) * D + k0 + kbase);
#pragma unroll
                for (int e = 0; e < KPT / 4; ++e) {
                    const float4 x = row[e];
                    Cs[4 * e] = x.x; Cs[4 * e + 1] = x.y; Cs[4 * e + 2] = x.z; Cs[4 * e + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < KPT; ++e) Cs[e] = 0.f;
            }
        }
        if (nch > 0) {
            write_parts<KPT, KC>(Cs, tR + lane_addr, kbase);
            tc_fence_before();
            sync_state();
            if (leader) mbar_arrive(&bars[B_RR]);
            ok = swait(&bars[B_GR], 0);
        }
        int nw = 0, nwc = 0;
        for (int c = 0; ok && c < nch; ++c) {
            const int gb = c % GB;
            const float a = gS[gb * 8 + GS_A];
            const bool wide = gS[gb * 8 + GS_WIDE] != 0.f;
            // (1) w V for the chunk's sub-blocks as they land (wide chunks: after the intra products)
            if (!wide) {
                for (int j = 0; ok && j < NSUB; ++j) {
                    const int b = c * NSUB + j;
                    if (!swait(&bars[B_VF + b % NKV], (b / NKV) & 1)) { ok = false; break; }
                    scale_v(b, gb);
                }
                if (!ok) break;
            }
            // (2) per sub-block: the wide-chunk query rows, then h
            for (int j = 0; ok && j < NSUB; ++j) {
                const int b = c * NSUB + j;
                if (wide) {
                    if (!swait(&bars[B_SQ], nw & 1)) { ok = false; break; }
                    ++nw;
                    zero_late_rows(b, gb);
                    sync_state();
                    if (leader) mbar_arrive(&bars[B_QZ]);
                }
                if (!out_pass(b, gb)) { ok = false; break; }
            }
            if (!ok) break;
            if (wide) {
                if (!swait(&bars[B_ID], nwc & 1)) { ok = false; break; }
                ++nwc;
                for (int j = 0; j < NSUB; ++j) scale_v(c * NSUB + j, gb);
            }
            // (3) fold the chunk's update into the fp32 state, then the next chunk's parts
            RS_TRACE(leader, c, 8);
            if (!swait(&bars[B_UF], c & 1)) { ok = false; break; }
            RS_TRACE(leader, c, 10);
            tc_fence_after();
#pragma unroll
            for (int pc = 0; pc < KPT / 16; ++pc) {
                uint32_t r[16];
                tmem_ld16(tU + lane_addr + kbase + 16 * pc, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) Cs[16 * pc + e] = fmaf(a, Cs[16 * pc + e], __uint_as_float(r[e]));
            }
            tc_fence_before();
            sync_state();                         // every read of U precedes the parts' writes
            tc_fence_after();
            RS_TRACE(leader, c, 11);
            if (c + 1 < nch) {
                if (!swait(&bars[B_GR + (c + 1) % GB], ((c + 1) / GB) & 1)) { ok = false; break; }
                write_parts<KPT, KC>(Cs, tR + lane_addr, kbase);
                tc_fence_before();
                sync_state();
                if (leader) mbar_arrive(&bars[B_RR]);
                RS_TRACE(leader, c, 12);
            }
            if (leader) mbar_arrive(&bars[B_GE + gb]);
        }
        // final state (last segment only)
        if (ok && g == P - 1 && nch > 0 && !*abort_flag && C_out && has_row) {
            float4 *dst = reinterpret_cast<float4 *>(C_out + ((size_t)bh * D + i0 + i) * D + k0 + kbase);
#pragma unroll
            for (int e = 0; e < KPT / 4; ++e)
                dst[e] = make_float4(Cs[4 * e], Cs[4 * e + 1], Cs[4 * e + 2], Cs[4 * e + 3]);
        }
        tc_fence_before();
    } else {
        if (KC == 256) regs_dec<104>();
        // ------------------------------------------------------------ scores
        const int xt = tid - 384;                    // 0..127
        const bool xleader = xt == 0;
        const int tr = 16 * q4 + (lane & 15);        // score row in the sub-block (M = 64 layout: lanes 0-15)
        const int hh = lane >> 4;                    // column half of this lane
        bool ok = true;
        auto xwait = [&](uint64_t *bar, uint32_t parity) -> bool {
            const bool r = xleader ? rs_wait(bar, parity, abort_flag, status) : true;
            return group_all<2, 128>(r);
        };
        float rowsum = 0.f;
        for (int c = 0; ok && c < nch; ++c) {
            const int gb = c % GB;
            if (!xwait(&bars[B_GR + gb], (c / GB) & 1)) { ok = false; break; }
            const float *gs = gS + gb * 8;
            const bool wide = gs[GS_WIDE] != 0.f;
            const int Lc = (int)gs[GS_LC];
            const float rho = gs[GS_RHO];
            for (int tt = 0; tt < TPC; ++tt) {
                const int gt_ = c * TPC + tt;
                int j, i;
                tile_ji(tt, j, i);
                if (!xwait(&bars[B_SF], gt_ & 1) || (gt_ >= 1 && !xwait(&bars[B_PE], (gt_ - 1) & 1))) { ok = false; break; }
                RS_TRACE(xleader && tt == 0, c, 16);
                tc_fence_after();
                uint32_t sa[32], sb[32], sn[8];
                tmem_ld16(tS + lane_addr + 0, *reinterpret_cast<uint32_t(*)[16]>(&sa[0]));
                tmem_ld16(tS + lane_addr + 16, *reinterpret_cast<uint32_t(*)[16]>(&sa[16]));
                tmem_ld16(tS + lane_addr + 32, *reinterpret_cast<uint32_t(*)[16]>(&sb[0]));
                tmem_ld16(tS + lane_addr + 48, *reinterpret_cast<uint32_t(*)[16]>(&sb[16]));
                tmem_ld8(tS + lane_addr + 64, sn);
                tmem_wait_ld();
                tc_fence_before();
                sync_so();
                if (xleader) mbar_arrive(&bars[B_SE]);           // S may be overwritten by the next tile
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const uint32_t up = __shfl_sync(0xffffffffu, sb[e], lane & 15);
                    sa[e] = hh ? up : sa[e];
                }
                const int t = 64 * j + tr;                   // token of this row within the chunk
                const bool valid = t < Lc;
                const float ref_t = garr(gb, G_REF)[t];
                const bool late = garr(gb, G_LATE)[t] != 0.f;
                // masked, weighted scores as bf16 (the B operand of the intra product) and their row sum
                const float *w = garr(gb, G_W) + 64 * i + 32 * hh;
                const float *us = garr(gb, G_U) + 64 * i + 32 * hh;
                if (i == 0) rowsum = 0.f;
#pragma unroll
                for (int cq = 0; cq < 4; ++cq) {
                    uint32_t p4[4], l4[4];
#pragma unroll
                    for (int p2 = 0; p2 < 4; ++p2) {
                        float pv[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int sl2 = cq * 8 + p2 * 2 + e;
                            const int s = 64 * i + 32 * hh + sl2;     // key token within the chunk
                            const bool keep = valid && s <= t;
                            const float sc = keep ? __uint_as_float(sa[sl2]) : 0.f;
                            if (!wide) {
                                pv[e] = rho * sc;
                                rowsum += w[sl2] * sc;
                            } else {     // exp(u_s - ref_t) <= e^40 only where s <= t
                                pv[e] = keep ? sc * (expf(us[sl2] - ref_t) * inv_sqrt_d) : 0.f;
                                rowsum += pv[e];
                            }
                        }
                        p4[p2] = cvt_bf16x2(pv[0], pv[1]);
                        if (KS > 1) l4[p2] = cvt_bf16x2(pv[0] - bf_lo(p4[p2]), pv[1] - bf_hi(p4[p2]));
                    }
                    *reinterpret_cast<uint4 *>(sP + sw128_offset(tr, 4 * hh + cq)) = make_uint4(p4[0], p4[1], p4[2], p4[3]);
                    if (KS > 1)
                        *reinterpret_cast<uint4 *>(sP + 8192 + sw128_offset(tr, 4 * hh + cq)) =
                            make_uint4(l4[0], l4[1], l4[2], l4[3]);
                }
                if (i == j) {       // the sub-block's last tile: denominators of its rows
                    const float rs = rowsum + __shfl_xor_sync(0xffffffffu, rowsum, 16);
                    if (hh == 0) {
                        // n'.q_t from the normaliser columns (hi + mid + lo parts)
                        const float nq = __uint_as_float(sn[0]) + __uint_as_float(sn[1]) + __uint_as_float(sn[2]);
                        const float gt = garr(gb, G_G)[t];
                        float den;
                        if (!wide) den = gt * (nq + rho * rs);
                        else if (!late) den = gt * (nq + rs);
                        else den = rs;            // the old state's share is below fp32 resolution
                        // 0.5: sigma(o) = (1 + tanh(o / 2)) / 2
                        garr(gb, G_INV)[t] = valid ? 0.5f * garr(gb, G_OF)[t] / fmaxf(fabsf(den), garr(gb, G_FL)[t]) : 0.f;
                        if (KS > 1 && tile == 0 && valid) {   // this CTA's share of the denominator, and the row factors
                            const size_t tk = tok0 + (size_t)tseg + (size_t)c * L + t;
                            dpart[(size_t)kh * gridDim.z * S + tk] = den;
                            if (kh == 0) tokrec[tk] = make_float2(garr(gb, G_OF)[t], garr(gb, G_FL)[t]);
                        }
                    }
                }
                fence_async_smem();
                sync_so();
                if (xleader) {
                    mbar_arrive(&bars[B_PR]);
                    if (i == j) mbar_arrive(&bars[B_INV + ((c * NSUB + j) & 1)]);   // the sub-block's 1 / denominators
                }
                RS_TRACE(xleader && tt == 0, c, 17);
            }
            if (!ok) break;
            sync_so();                                       // G_INV written before the chunk's gates are released
            if (xleader) mbar_arrive(&bars[B_GE + gb]);
        }
        tc_fence_before();
    }
    pdl_launch_dependents();      // the combining kernel may be scheduled; it waits for this one
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

// Split key columns (DH 512, and DH 256 at chunk 256): the two halves'
// numerators and denominators are summed and the output formed,
// h = sigma(o) * f_t (N_0 + N_1) / max(|d_0 + d_1|, e^{-m_t}); f_t is the row
// factor (g_t, or 1 in a wide chunk's rows whose retrieval was dropped).  An
// HBM stream: four value columns of one token per thread.
__global__ void __launch_bounds__(256)
combine_keysplit_kernel(const float *__restrict__ part, const float *__restrict__ dpart,
                        const float2 *__restrict__ tokrec, const float *__restrict__ o_pre,
                        __nv_bfloat16 *__restrict__ h, size_t tokens, int D) {
    pdl_wait();                                    // the output kernel's partial sums
    const size_t n4 = tokens * (size_t)(D / 4);
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += stride) {
        const size_t tk = e / (D / 4);
        const float4 a = reinterpret_cast<const float4 *>(part)[e];
        const float4 b = reinterpret_cast<const float4 *>(part + tokens * D)[e];
        const float4 o = reinterpret_cast<const float4 *>(o_pre)[e];
        const float2 tr = tokrec[tk];
        const float f = tr.x / fmaxf(fabsf(dpart[tk] + dpart[tokens + tk]), tr.y);
        const float x0 = (a.x + b.x) * f, x1 = (a.y + b.y) * f, x2 = (a.z + b.z) * f, x3 = (a.w + b.w) * f;
        uint2 out;
        out.x = cvt_bf16x2(x0 * sigmoid(o.x), x1 * sigmoid(o.y));
        out.y = cvt_bf16x2(x2 * sigmoid(o.z), x3 * sigmoid(o.w));
        reinterpret_cast<uint2 *>(h)[e] = out;
    }
}

template <int D, int NSUB>
cudaError_t launch_rs_t(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    using Cfg = RsCfg<D, NSUB>;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map_bf16(&mq, a.q, p.BH, p.S, D) || !make_map_bf16(&mk, a.k, p.BH, p.S, D) ||
        !make_map_bf16(&mv, a.v, p.BH, p.S, D) || !make_map_f32_rows(&mo, a.o_pre, p.BH, p.S, D, Cfg::RV, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = launch_segment_summaries(a, p, st);
    if (e != cudaSuccess) return e;
    float *ws = (float *)a.workspace;
    // at least 116 KB so that one CTA runs per SM: each allocates all 512 TMEM columns
    const int sm = Cfg::kBytes > 118784 ? Cfg::kBytes : 118784;
    e = cudaFuncSetAttribute(segment_output_rs_kernel<D, NSUB>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    float *part = Cfg::KS > 1 ? ws + p.off_part : nullptr;
    float *dpart = Cfg::KS > 1 ? ws + p.off_dpart : nullptr;
    float2 *tokrec = Cfg::KS > 1 ? (float2 *)(ws + p.off_tok) : nullptr;
    {
        KernelTimer timer("segment_output_rs", st);
        e = launch_chained(segment_output_rs_kernel<D, NSUB>, dim3((D / Cfg::RV) * Cfg::KS, p.P, p.BH),
                           dim3(kRsThreads), sm, st, mq, mk, mv, mo, (__nv_bfloat16 *)a.h, a.i_pre, a.C0, a.n0,
                           a.m0, a.C_out, a.n_out, a.m_out, (const float *)(ws + p.off_bcum),
                           (const float *)(ws + p.off_pmax), (const float2 *)(ws + p.off_cstat),
                           (const float2 *)(ws + p.off_sstat), (const float *)(ws + p.off_summ), part, dpart,
                           tokrec, a.status, p.S, p.nchunks, p.P, p.cps);
        if (e != cudaSuccess) return e;
    }
    if (Cfg::KS > 1) {
        KernelTimer timer("combine_keysplit", st);
        const size_t n4 = (size_t)p.BH * p.S * (D / 4);
        const unsigned blocks = (unsigned)((n4 + 255) / 256 < (size_t)8 * num_sms_current_device()
                                               ? (n4 + 255) / 256 : (size_t)8 * num_sms_current_device());
        e = launch_chained(combine_keysplit_kernel, dim3(blocks), dim3(256), 0, st, (const float *)part,
                           (const float *)dpart, (const float2 *)tokrec, a.o_pre, (__nv_bfloat16 *)a.h,
                           (size_t)p.BH * p.S, D);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int NSUB>
cudaError_t launch_rs_nsub(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    switch (p.DH) {
        case 64: return launch_rs_t<64, NSUB>(a, p, st);
        case 128: return launch_rs_t<128, NSUB>(a, p, st);
        case 256: return launch_rs_t<256, NSUB>(a, p, st);
        case 512: return launch_rs_t<512, NSUB < 4 ? NSUB : 2>(a, p, st);   // DH 512 takes chunks 64 and 128
    }
    return cudaErrorInvalidValue;
}

}  // namespace

#ifdef XLSTM_RS_TRACE
extern "C" int xlstm_debug_set_rs_trace(void *buf) {
    return cudaMemcpyToSymbol(g_rs_trace, &buf, sizeof(buf)) == cudaSuccess ? 0 : 1;
}
#endif

bool rs_path_supports(int DH, int L) {
    if (DH != 64 && DH != 128 && DH != 256 && DH != 512) return false;
    if (L == 64 || L == 128) return true;
    return L == 256 && DH <= 256;
}

int rs_key_splits(int DH, int L) { return DH > 256 || (DH == 256 && L == 256) ? 2 : 1; }

cudaError_t launch_fwd_rs(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    if (!a.bf16 || !rs_path_supports(p.DH, p.L)) return cudaErrorInvalidValue;
    cudaError_t e = launch_gate_prologue(a, p, st);
    if (e != cudaSuccess) return e;
    switch (p.L) {
        case 64: return launch_rs_nsub<1>(a, p, st);
        case 128: return launch_rs_nsub<2>(a, p, st);
        case 256: return launch_rs_nsub<4>(a, p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace xlstm
