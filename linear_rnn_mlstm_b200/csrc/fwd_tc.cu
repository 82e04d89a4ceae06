// Chunkwise mLSTM forward on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// Computes the same chunkwise-parallel form as the fp32 SIMT kernels (see
// fwd_simt.cu for the notation) for bf16 q/k/v, chunk L = 64, DH in {128, 256},
// with value rows tiled by 128 per CTA ("xLSTM: Extended Long Short-Term
// Memory" section 2.3: retrieval by matrix multiplication, covariance update of
// the matrix memory).  Per chunk of a segment, on the tensor cores:
//
//   S    = Q [K ; n'_prev hi ; n'_prev lo]^T           M=64,  N=72, K=DH (bf16)
//   H~^T = Cs Q^T                                      M=128, N=64, K=DH (tf32, Cs in TMEM)
//   H~^T += (w^ V)^T (Shi + Slo)^T  (scores masked s<=t) M=128, N=64, K=64 (bf16)
//   Cs  += (w^ V)^T K                                  M=128, N=DH, K=64 (bf16)
//
// Cs is the CTA's 128 value rows of the state, resident in TMEM in fp32 for the
// whole segment and lazily scaled, C' = Lambda Cs; w^_s = e^{u_s + b_L - m_next}
// / (sqrt(d) Lambda_c) folds the gates, the key scaling and the lazy scale into
// V.  With that choice the decayed intra-chunk weight factorises exactly,
//   e^{b_t - b_s + itilde_s - m_t} / sqrt(d) = F_t w^_s,  F_t = g_t Lambda_prev,
// and F_t is also the retrieval's row scale, so
//   h_t = o_t F_t H~_t / max(|g_t n'_prev.q_t + F_t sum_s w^_s S_ts|, e^{-m_t})
// needs no per-element exponential and the retrieval uses Q as loaded.  The
// normaliser n' rides in two extra key rows of S (hi and lo bf16 parts); the
// masked scores go to the MMA as hi + lo bf16 parts, since the intra term can
// nearly cancel against the normaliser and one bf16 rounding there would be
// amplified in h.
//
// Every wait is bounded (tc_ptx.cuh): on a timeout the kernel raises the device
// status word and unwinds.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "tc_ptx.cuh"

namespace xlstm {

using namespace tc;

namespace {

constexpr int kL = 64;             // tokens per chunk on this path
constexpr int kRows = 128;         // value rows per CTA
constexpr int kKRows = 72;         // key-tile rows: 64 keys, n' hi, n' lo, 6 spare rows
constexpr int kKBlock = kKRows * 128;   // bytes per 64-column block of the key tile
// Key rows 66-71 of the first block only feed score columns 66-71, which nothing
// reads: a chunk's per-token u, b and prefix maxima ride there (3 x 256 bytes).
constexpr int kGateRow = 66;
constexpr int kThreads = 320;       // segment summaries: TMA warp, MMA warp, 8 compute warps
constexpr int kMaxCps = 256;       // chunks per segment the tables hold
constexpr float kLnLambdaFloor = -40.f;  // rescale the TMEM state below this log scale
constexpr float kLnChunkFloor = -60.f;   // smallest decay of the state's scale over one chunk (see below)

__device__ __forceinline__ void named_sync_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

#ifdef XLSTM_TC_TRACE
// Timing trace of the pipeline steps (diagnostic builds only): 32 globaltimer
// stamps per (CTA, chunk).
__device__ unsigned long long *g_tc_trace = nullptr;
#define TC_TRACE(cond, c, slot)                                                                    \
    do {                                                                                           \
        if (g_tc_trace && (cond)) {                                                                \
            const size_t cta_ = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x; \
            g_tc_trace[(cta_ * kMaxCps + (c)) * 32 + (slot)] = clock64();                          \
        }                                                                                          \
    } while (0)
#define TC_TRACE_NS(cond, slot)                                                                    \
    do {                                                                                           \
        if (g_tc_trace && (cond)) {                                                                \
            const size_t cta_ = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x; \
            g_tc_trace[cta_ * kMaxCps * 32 + (slot)] = globaltimer_ns();                           \
        }                                                                                          \
    } while (0)
// the segment-summary kernel's records, after the output kernel's (CTA index + 1024)
#define TC_TRACE_SUM(cond, c, slot)                                                                \
    do {                                                                                           \
        if (g_tc_trace && (cond) && (c) < kMaxCps) {                                               \
            const size_t cta_ = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x + 1024; \
            g_tc_trace[(cta_ * kMaxCps + (c)) * 32 + (slot)] = clock64();                          \
        }                                                                                          \
    } while (0)
#else
#define TC_TRACE(cond, c, slot) do { } while (0)
#define TC_TRACE_NS(cond, slot) do { } while (0)
#define TC_TRACE_SUM(cond, c, slot) do { } while (0)
#endif

// A bounded wait taken by all 128 compute threads, with a group-uniform result.
__device__ __forceinline__ bool compute_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             unsigned int *status) {
    return group_wait<1, 256>(bar, parity, threadIdx.x == 64, abort_flag, status);
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------ segment outputs
template <int D>
struct OutLayout {
    static constexpr int kQ = 0;                          // Q  bf16 K-major: D/64 blocks x 8 KB
    static constexpr int kKslot = (D / 64) * kKBlock;     // one key slot: D/64 blocks x 72 rows
    static constexpr int kK = kQ + D * 128;
    static constexpr int kV = kK + 2 * kKslot;            // V, scaled in place to w^ V: 2 blocks x 8 KB
    static constexpr int kQt = kV + 16384;                // Q as fp32 (tf32 operand), K-major: D/32 blocks x 8 KB
    static constexpr int kP = kQt + D * 256;              // masked scores, high bf16 part, K-major: 64 x 128 B
    static constexpr int kPl = kP + 8192;                 // masked scores, low bf16 part
    static constexpr int kO = kPl + 8192;                 // o-gate tile: 32 tokens x 128 value rows fp32 (TMA)
    static constexpr int kF = kO + 16384;                 // float arrays (see kernel)
    static constexpr int kNF = 16 * 64;
    static constexpr int kTab = kF + kNF * 4;             // per-chunk tables
    static constexpr int kBar = kTab + 5 * kMaxCps * 4;
    static constexpr int kNumBars = 40;
    static constexpr int kMisc = kBar + kNumBars * 8;     // tmem base, abort flag, o-tile counters
    static constexpr int kEnd = kMisc + 32;
    static constexpr int kBytes = kEnd + 1024;            // slack for 1024-byte alignment
};

constexpr int kMaxSmemPerCta = 232448;   // 227 KB of opt-in shared memory per CTA on sm_100
static_assert(OutLayout<256>::kBytes <= kMaxSmemPerCta, "output kernel shared memory");

enum {
    B_FULL_Q = 0, B_Q_FREE, B_FULL_K0, B_FULL_K1, B_K_FREE0, B_K_FREE1, B_FULL_V, B_V_FREE,
    B_VHAT_READY, B_QT_READY, B_QT_FREE, B_S_FULL, B_S_FREE, B_P_READY, B_P_FREE,
    B_H_FULL0, B_H_FULL1, B_H_FREE0, B_H_FREE1, B_NROW_READY0, B_NROW_READY1, B_RESC_DONE, B_DONE,
    B_GATES_READY0, B_GATES_READY1, B_GATES_FREE0, B_GATES_FREE1,
    B_FINV_READY0, B_FINV_READY1, B_FINV_FREE0, B_FINV_FREE1, B_INTRA_DONE, B_STATE_READY,
    B_O_FULL0, B_O_FULL1, B_NUM
};
static_assert(B_NUM <= OutLayout<128>::kNumBars, "barrier slots");
// Every barrier is waited by parity, so no producer may complete a barrier twice
// ahead of a waiter.  Buffers that a producer can refill before the consumer of
// the previous fill has waited are double-buffered with their own barriers
// (key-slot normaliser rows, gate arrays, denominators, H accumulators).

// Per-CTA tables built from the chunk statistics: for each chunk of the
// segment, the stabiliser at its start, the state scale used by its retrieval,
// the rescale factor applied before it (0 = none), ln(1/Lambda) after its
// update, and whether it is a wide chunk.
//
// A chunk is wide when its largest input-gate term outweighs the decayed state
// it starts from by more than e^60 (m_prev - max_s u_s < -60).  The factorised
// intra weights F_t w^_s would then leave the fp32 range, so a wide chunk takes
// exact weights instead: the score group forms e^{u_s + b_t - m_t} S_ts / sqrt(d)
// per element, the retrieval operand is g_t q_t, and V is scaled by w^ only
// after the intra-chunk MMA has read it (MMA order retrieval, intra, update).
struct ChunkTab {
    float *mprev, *lamret, *resc, *lnupd, *wide;
};

// Warp roles: 0 TMA, 1 MMA (and TMEM owner), 2-5 operand group (gates, Q as
// fp32, normaliser chain, w^ V, rescale, final state), 6-9 score group (masked
// scores and the denominators; one warp per TMEM lane quadrant), 10-13 output
// group (h; one warp per quadrant, the chunk's tokens in two passes of 32).
// Each group has its own named barrier and one thread that polls mbarriers for
// it.  14 warps: at most 4 per SM sub-partition, so 128 registers fit.
constexpr int kOutThreads = 448;

__device__ __forceinline__ void sync_ops() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void sync_sco() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void sync_out() { asm volatile("bar.sync 3, 128;" ::: "memory"); }
__device__ __forceinline__ bool wait_ops(uint64_t *bar, uint32_t parity, volatile int *abort_flag, unsigned int *status) {
    return group_wait<1, 128>(bar, parity, threadIdx.x == 64, abort_flag, status);
}
__device__ __forceinline__ bool wait_sco(uint64_t *bar, uint32_t parity, volatile int *abort_flag, unsigned int *status) {
    return group_wait<2, 128>(bar, parity, threadIdx.x == 192, abort_flag, status);
}
__device__ __forceinline__ bool wait_out(uint64_t *bar, uint32_t parity, volatile int *abort_flag, unsigned int *status) {
    return group_wait<3, 128>(bar, parity, threadIdx.x == 320, abort_flag, status);
}

template <int D>
__global__ void __launch_bounds__(kOutThreads, 1)
segment_output_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                         __nv_bfloat16 *__restrict__ h_out,
                         const float *__restrict__ i_pre, const float *__restrict__ o_pre,
                         const float *__restrict__ C0, const float *__restrict__ n0, const float *__restrict__ m0,
                         float *__restrict__ C_out, float *__restrict__ n_out, float *__restrict__ m_out,
                         const float *__restrict__ upad, const float *__restrict__ bpad,
                         const float *__restrict__ xpad, const float2 *__restrict__ cstat,
                         const float2 *__restrict__ sstat, const float *__restrict__ summ,
                         unsigned int *status, int S, int Spad, int nchunks, int P, int cps) {
    using Lay = OutLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sQ = smem + Lay::kQ;
    uint8_t *sK = smem + Lay::kK;
    uint8_t *sV = smem + Lay::kV;
    uint8_t *sQt = smem + Lay::kQt;
    uint8_t *sP = smem + Lay::kP;
    uint8_t *sPl = smem + Lay::kPl;
    const float *sO = reinterpret_cast<const float *>(smem + Lay::kO);
    // per-token arrays, [2][64] by chunk parity, written by the operand group
    float *fm = reinterpret_cast<float *>(smem + Lay::kF);   // m_t
    float *fg = fm + 128;                                    // g_t = e^{b_t + m_prev - m_t}
    float *fF = fg + 128;                                    // F_t = g_t * Lambda_prev (row scale of H)
    float *fw = fF + 128;                                    // w^_s: weight folded into V (per key)
    float *fpw = fw + 128;                                   // [64] normaliser weight (operand group only)
    float *finv = fpw + 64;                                  // [2][64] F_t / denominator (score -> output)
    float *fu = finv + 128;                                  // [2][64] u_s (wide chunks)
    float *frun = fu + 128;                                  // [2][64] m_t - b_t (wide chunks)
    ChunkTab tab;
    tab.mprev = reinterpret_cast<float *>(smem + Lay::kTab);
    tab.lamret = tab.mprev + kMaxCps;
    tab.resc = tab.lamret + kMaxCps;
    tab.lnupd = tab.resc + kMaxCps;
    tab.wide = tab.lnupd + kMaxCps;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kMisc + 4);
    // o-gate tiles issued into / taken from the shared tile, per pass (hq = 0, 1)
    int *o_issued = reinterpret_cast<int *>(smem + Lay::kMisc + 8);
    int *o_taken = reinterpret_cast<int *>(smem + Lay::kMisc + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, g = blockIdx.y, bh = blockIdx.z;
    const int i0 = tile * kRows;
    const int c0 = g * cps;
    const int nch = min(nchunks, c0 + cps) - c0;
    const size_t tok0 = (size_t)bh * S;
    const float inv_sqrt_d = rsqrtf((float)D);
    const int q4 = warp & 3;                                 // TMEM lane quadrant of this warp
    const uint32_t lane_addr = ((uint32_t)(32 * q4)) << 16;
    const bool is_ops = warp >= 2 && warp < 6;
    const bool is_sco = warp >= 6 && warp < 10;
    const bool is_out = warp >= 10;
    const int ct = tid - 64;                                 // operand-group thread 0..127
    const int st_ = tid - 192;                               // score-group thread 0..127
    const int xt = tid - 320;                                // output-group thread 0..127

    // ------------------------------------------------------------ set-up
    TC_TRACE_NS(tid == 0, 30);
    if (tid == 0) {
        for (int i = 0; i < B_NUM; ++i) {
            const bool two = i == B_Q_FREE || i == B_H_FREE0 || i == B_H_FREE1 || i == B_FINV_FREE0 ||
                             i == B_FINV_FREE1;
            mbar_init(&bars[i], two ? 2 : 1);
        }
        *abort_flag = 0;
        o_issued[0] = o_issued[1] = o_taken[0] = o_taken[1] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tc_fence_before();
    }
    float nreg[D / 128];                           // operand group: n' entries j = nj(r)
    // key column of the operand group's r-th normaliser register (adjacent pairs for DH = 256)
    auto nj = [&](int r) { return D == 256 ? 2 * (tid - 64) + r : (tid - 64); };
    __syncthreads();
    tc_fence_after();
    pdl_wait();                                    // the segment scan's states and the gate statistics
    const uint32_t tbase = *tmem_slot;
    const uint32_t t_state = tbase;                // columns [0, D)
    const uint32_t t_S = tbase + 256;              // columns [256, 328)
    const uint32_t t_H0 = tbase + 384;             // columns [384, 448) and [448, 512)

    if (is_ops) {
        // incoming normaliser (the incoming C' goes to TMEM from the output group)
        const float m_init = m0 ? m0[bh] : 0.f;
        const float *nsrc = g == 0 ? (n0 ? n0 + (size_t)bh * D : nullptr)
                                   : summ + ((size_t)bh * (P - 1) + g - 1) * ((size_t)D * D + D) + (size_t)D * D;
#pragma unroll
        for (int r = 0; r < D / 128; ++r) nreg[r] = nsrc ? nsrc[nj(r)] : 0.f;
        // zero the extra key rows 64..71 of both slots, then n'_in (hi, lo) in slot 0
        for (int e = ct; e < 2 * (D / 64) * 8 * 8; e += 128) {      // (slot, block, row, chunk)
            const int ch = e & 7, row = 64 + ((e >> 3) & 7), blk = (e >> 6) % (D / 64), slot = e / (64 * (D / 64));
            *reinterpret_cast<uint4 *>(sK + slot * Lay::kKslot + blk * kKBlock + sw128_offset(row, ch)) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        sync_ops();
#pragma unroll
        for (int r = 0; r < D / 128; ++r) {
            const int j = nj(r);
            const float hi = __bfloat162float(__float2bfloat16_rn(nreg[r]));
            uint8_t *blkp = sK + (j / 64) * kKBlock;
            const int cc = (j % 64) / 8, within = (j % 8) * 2;
            *reinterpret_cast<__nv_bfloat16 *>(blkp + sw128_offset(64, cc) + within) = __float2bfloat16_rn(hi);
            *reinterpret_cast<__nv_bfloat16 *>(blkp + sw128_offset(65, cc) + within) = __float2bfloat16_rn(nreg[r] - hi);
        }
        // per-chunk tables: the chunk statistics are staged in shared memory by all
        // operand-group threads (one load each), then one thread scans them
        for (int c = ct; c < nch; c += 128) {
            const float2 cs = cstat[(size_t)bh * nchunks + c0 + c];
            tab.mprev[c] = cs.x;
            tab.lamret[c] = cs.y;
        }
        for (int gp = ct; gp < g; gp += 128) {
            const float2 st = sstat[(size_t)bh * P + gp];
            tab.resc[gp] = st.x;
            tab.lnupd[gp] = st.y;
        }
        sync_ops();
        if (ct == 0) {
            float mc = m_init;
            for (int gp = 0; gp < g; ++gp) mc = fmaxf(tab.resc[gp] + mc, tab.lnupd[gp]);
            // ln Lambda stays in [-60, 0]: a chunk whose own decay of the stabilised
            // state, m_prev - max_s u_s, is below -60 is taken as -60.  That chunk
            // holds a term e^60 times heavier than the whole earlier state, so the
            // earlier state's share after it is below fp32 resolution either way.
            float lnlam = 0.f;
            for (int c = 0; c < nch; ++c) {
                const float2 cs = make_float2(tab.mprev[c], tab.lamret[c]);
                const float mn = cs.x + fmaxf(mc, cs.y);
                const float lna_true = cs.x + mc - mn;       // <= 0
                const float lna = fmaxf(lna_true, kLnChunkFloor);
                tab.mprev[c] = mc;
                tab.wide[c] = lna_true < kLnChunkFloor ? 1.f : 0.f;
                if (lnlam + lna < kLnLambdaFloor && c > 0) {
                    tab.resc[c] = expf(lnlam);               // Cs <- Lambda Cs before chunk c
                    lnlam = 0.f;
                } else {
                    tab.resc[c] = 0.f;
                }
                tab.lamret[c] = expf(lnlam);
                lnlam += lna;
                tab.lnupd[c] = -lnlam;                       // ln (1 / Lambda) after chunk c
                mc = mn;
            }
        }
        fence_async_smem();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();

    const uint32_t idesc_S = idesc_f32acc(kFmtBF16, kFmtBF16, false, false, 64, kKRows);
    const uint32_t idesc_R = idesc_f32acc(kFmtTF32, kFmtTF32, false, false, 128, 64);
    const uint32_t idesc_I = idesc_f32acc(kFmtBF16, kFmtBF16, true, false, 128, 64);
    const uint32_t idesc_U = idesc_f32acc(kFmtBF16, kFmtBF16, true, true, 128, D);

    // The o gates of one epilogue pass reach shared memory by TMA, one tile of
    // 32 tokens x 128 value rows at a time: the output group takes tokens 0-31 of
    // each chunk (hq = 0), the score group tokens 32-63 (hq = 1).  Whichever group
    // has just read the tile issues the load of the next one, so the epilogue
    // threads never hold a global load across a barrier or an arrival.
    auto issue_o = [&](int c, int hq) {
        uint64_t *bar = &bars[B_O_FULL0 + hq];
        mbar_arrive_expect_tx(bar, 32 * kRows * 4);
        tma_load_3d(const_cast<float *>(sO), &map_o, bar, i0, (c0 + c) * kL + 32 * hq, bh);
        ++o_issued[hq];
    };
    // This thread's 32 gates of the tile in shared memory (thread = value row i;
    // a warp reads 32 consecutive floats per token).
    auto read_gates = [&](float (&og)[32]) {
        const int i = 32 * q4 + lane;
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) og[kk] = sO[kk * kRows + i];
    };
    // One epilogue pass: h for tokens [32 hq, 32 hq + 32) of chunk c, from the H~
    // accumulator (thread = value row i = TMEM lane), the gates `og` of those
    // tokens and the per-token factors F_t / (2 den_t); each h element is stored
    // straight to global memory (a warp writes 64 contiguous bytes per token).
    auto epilogue_pass = [&](int c, int hq, const float (&og)[32]) {
        const int hb = c & 1;
        const int i = 32 * q4 + lane;
        const int tb = (c0 + c) * kL + 32 * hq;
        const int n = min(32, S - tb);
        __nv_bfloat16 *hrow = h_out + (tok0 + tb) * D + i0 + i;
        uint32_t r[32];
        tmem_ld16(t_H0 + 64 * hb + lane_addr + 32 * hq, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
        tmem_ld16(t_H0 + 64 * hb + lane_addr + 32 * hq + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
        tmem_wait_ld();
        const float *inv = finv + 64 * hb + 32 * hq;          // holds F_t / (2 den_t)
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
            // sigma(o) = (1 + tanh(o / 2)) / 2, the 1/2 folded into inv
            const float hv = __uint_as_float(r[kk]) * inv[kk];
            if (kk < n) hrow[(size_t)kk * D] = __float2bfloat16_rn(fmaf(hv, tanh_approx(0.5f * og[kk]), hv));
        }
    };
    // After a pass the group's share of H[hb] and finv[hb] is released.
    auto finish_pass = [&](int c, bool leader) {
        if (leader) {
            mbar_arrive(&bars[B_H_FREE0 + (c & 1)]);
            mbar_arrive(&bars[B_FINV_FREE0 + (c & 1)]);
        }
    };

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&map_q);
            tma_prefetch_desc(&map_k);
            tma_prefetch_desc(&map_v);
            tma_prefetch_desc(&map_o);
            // The operands of the chunk after next go to L2 ahead of their loads; the
            // output gates, which the output group reads with plain loads, likewise.
            auto prefetch = [&](int c) {
                const int t0 = (c0 + c) * kL;
                for (int jb = 0; jb < D / 64; ++jb) {
                    tma_prefetch_l2_3d(&map_q, jb * 64, t0, bh);
                    tma_prefetch_l2_3d(&map_k, jb * 64, t0, bh);
                }
                tma_prefetch_l2_3d(&map_v, i0, t0, bh);
                tma_prefetch_l2_3d(&map_v, i0 + 64, t0, bh);
                tma_prefetch_l2_3d(&map_o, i0, t0, bh);
                tma_prefetch_l2_3d(&map_o, i0, t0 + 32, bh);
            };
            for (int c = 0; c < min(nch, 2); ++c) prefetch(c);
            int issued_q = 0, issued_k[2] = {0, 0}, issued_v = 0;
            for (int c = 0; c < nch; ++c) {
                const int t0 = (c0 + c) * kL;
                if (c + 2 < nch) prefetch(c + 2);
                if (c >= 1 && !mbar_wait(&bars[B_Q_FREE], (c - 1) & 1, abort_flag, status)) break;
                mbar_arrive_expect_tx(&bars[B_FULL_Q], kL * D * 2);
                for (int jb = 0; jb < D / 64; ++jb)
                    tma_load_3d(sQ + jb * 8192, &map_q, &bars[B_FULL_Q], jb * 64, t0, bh);
                ++issued_q;
                TC_TRACE(true, c, 29);
                const int slot = c & 1;
                if (c >= 2 && !mbar_wait(&bars[B_K_FREE0 + slot], ((c >> 1) - 1) & 1, abort_flag, status)) break;
                mbar_arrive_expect_tx(&bars[B_FULL_K0 + slot], kL * D * 2 + 3 * kL * 4);
                for (int jb = 0; jb < D / 64; ++jb)
                    tma_load_3d(sK + slot * Lay::kKslot + jb * kKBlock, &map_k, &bars[B_FULL_K0 + slot],
                                jb * 64, t0, bh);
                {   // the chunk's u, b and prefix maxima, into the slot's spare rows
                    uint8_t *gdst = sK + slot * Lay::kKslot + kGateRow * 128;
                    const size_t gsrc = (size_t)bh * Spad + t0;
                    bulk_load(gdst, upad + gsrc, kL * 4, &bars[B_FULL_K0 + slot]);
                    bulk_load(gdst + 256, bpad + gsrc, kL * 4, &bars[B_FULL_K0 + slot]);
                    bulk_load(gdst + 512, xpad + gsrc, kL * 4, &bars[B_FULL_K0 + slot]);
                }
                ++issued_k[slot];
                if (c >= 1 && !mbar_wait(&bars[B_V_FREE], (c - 1) & 1, abort_flag, status)) break;
                mbar_arrive_expect_tx(&bars[B_FULL_V], kL * kRows * 2);
                for (int b = 0; b < 2; ++b)
                    tma_load_3d(sV + b * 8192, &map_v, &bars[B_FULL_V], i0 + 64 * b, t0, bh);
                ++issued_v;
            }
            // never leave a load in flight into shared memory
            if (issued_q) mbar_wait(&bars[B_FULL_Q], (issued_q - 1) & 1, nullptr, status);
            for (int s = 0; s < 2; ++s)
                if (issued_k[s]) mbar_wait(&bars[B_FULL_K0 + s], (issued_k[s] - 1) & 1, nullptr, status);
            if (issued_v) mbar_wait(&bars[B_FULL_V], (issued_v - 1) & 1, nullptr, status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int nresc = 0;
            bool ok = true;
            auto issue_S = [&](int c) {
                const int slot = c & 1;
                // Descriptors are built once and stepped in place: +32 B (2 units of 16 B)
                // per K step inside a 128-byte row, one block per four steps.  Shared
                // addresses are below 256 KB, so the 14-bit address field cannot carry
                // out.  Four MMAs per loop body keep the issuing thread's code small.
                uint64_t dq = sdesc_sw128(smem_u32(sQ), 16, 1024);
                uint64_t dk = sdesc_sw128(smem_u32(sK + slot * Lay::kKslot), 16, 1024);
#pragma unroll 1
                for (int jb = 0; jb < D / 64; ++jb) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) mma_bf16_ss(t_S, dq + 2 * k4, dk + 2 * k4, idesc_S, (jb | k4) != 0);
                    dq += 8192 >> 4;
                    dk += kKBlock >> 4;
                }
                mma_commit(&bars[B_S_FULL]);
                mma_commit(&bars[B_Q_FREE]);
            };
            ok = mbar_wait(&bars[B_FULL_Q], 0, abort_flag, status) &&
                 mbar_wait(&bars[B_FULL_K0], 0, abort_flag, status);
            if (ok) {
                tc_fence_after();
                issue_S(0);
            }
            for (int c = 0; ok && c < nch; ++c) {
                const int hb = c & 1;
                const uint32_t t_H = t_H0 + 64 * hb;
                if (tab.resc[c] != 0.f) {
                    if (!mbar_wait(&bars[B_RESC_DONE], nresc & 1, abort_flag, status)) { ok = false; break; }
                    ++nresc;
                }
                TC_TRACE(true, c, 25);
                if (!mbar_wait(&bars[B_QT_READY], c & 1, abort_flag, status)) { ok = false; break; }
                TC_TRACE(true, c, 26);
                if (c == 0 && !mbar_wait(&bars[B_STATE_READY], 0, abort_flag, status)) { ok = false; break; }
                if (c >= 2 && !mbar_wait(&bars[B_H_FREE0 + hb], ((c >> 1) - 1) & 1, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                TC_TRACE(true, c, 12);
                {   // retrieval from the state at the chunk start: H^T = Cs Q^T (tf32, Cs in TMEM)
                    uint64_t dqt = sdesc_sw128(smem_u32(sQt), 16, 1024);
                    uint32_t ta = t_state;
#pragma unroll 1
                    for (int blk = 0; blk < D / 32; ++blk) {
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) mma_tf32_ts(t_H, ta + 8 * k4, dqt + 2 * k4, idesc_R, (blk | k4) != 0);
                        dqt += 8192 >> 4;
                        ta += 32;
                    }
                    mma_commit(&bars[B_QT_FREE]);
                }
                TC_TRACE(true, c, 27);
                auto update = [&]() -> bool {   // state update: Cs += (w^ V)^T K
                    if (!mbar_wait(&bars[B_VHAT_READY], c & 1, abort_flag, status)) return false;
                    tc_fence_after();
                    TC_TRACE(true, c, 15);
                    const uint32_t va = smem_u32(sV), ka = smem_u32(sK + (c & 1) * Lay::kKslot);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ss(t_state, sdesc_sw128(va + ks * 2048, 8192, 1024),
                                    sdesc_sw128(ka + ks * 2048, kKBlock, 1024), idesc_U, 1);
                    mma_commit(&bars[B_K_FREE0 + (c & 1)]);
                    return true;
                };
                auto intra = [&]() -> bool {    // H^T += Vs^T (Phi + Plo)^T over the masked scores
                    if (!mbar_wait(&bars[B_P_READY], c & 1, abort_flag, status)) return false;
                    tc_fence_after();
                    TC_TRACE(true, c, 13);
                    const uint32_t va = smem_u32(sV), pa = smem_u32(sP), pla = smem_u32(sPl);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ss(t_H, sdesc_sw128(va + ks * 2048, 8192, 1024),
                                    sdesc_sw128(pa + ks * 32, 16, 1024), idesc_I, 1);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ss(t_H, sdesc_sw128(va + ks * 2048, 8192, 1024),
                                    sdesc_sw128(pla + ks * 32, 16, 1024), idesc_I, 1);
                    mma_commit(&bars[B_H_FULL0 + hb]);
                    mma_commit(&bars[B_P_FREE]);
                    return true;
                };
                if (tab.wide[c] == 0.f) {       // V already holds w^ V
                    if (!update() || !intra()) { ok = false; break; }
                } else {                        // V unscaled for the intra term, then w^ V
                    if (!intra()) { ok = false; break; }
                    mma_commit(&bars[B_INTRA_DONE]);
                    if (!update()) { ok = false; break; }
                }
                mma_commit(&bars[B_V_FREE]);
                if (c + 1 < nch) {   // scores of the next chunk
                    const int slot = (c + 1) & 1;
                    if (!mbar_wait(&bars[B_FULL_Q], (c + 1) & 1, abort_flag, status)) { ok = false; break; }
                    TC_TRACE(true, c + 1, 30);
                    if (!mbar_wait(&bars[B_FULL_K0 + slot], ((c + 1) >> 1) & 1, abort_flag, status)) { ok = false; break; }
                    TC_TRACE(true, c + 1, 31);
                    if (!mbar_wait(&bars[B_NROW_READY0 + slot], (c >> 1) & 1, abort_flag, status) ||
                        !mbar_wait(&bars[B_S_FREE], c & 1, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    TC_TRACE(true, c, 14);
                    issue_S(c + 1);
                    TC_TRACE(true, c, 24);
                }
            }
            mma_commit(&bars[B_DONE]);
            // drain: every MMA issued has completed before TMEM is released
            mbar_wait(&bars[B_DONE], 0, nullptr, status);
        }
    } else if (is_ops) {
        // --------------------------------------------------------- operand group
        bool ok = true;
        int nwide = 0;
        for (int c = 0; ok && c < nch; ++c) {
            const int t0 = (c0 + c) * kL;
            const int Lc = min(kL, S - t0);
            const int pb = c & 1;
            const float mprev = tab.mprev[c];
            const bool wide = tab.wide[c] != 0.f;
            TC_TRACE(ct == 0, c, 0);
            // (1) lazy rescale of the TMEM state before this chunk's retrieval
            if (tab.resc[c] != 0.f) {
                if (!wait_ops(&bars[B_K_FREE0 + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag, status)) { ok = false; break; }
                __syncwarp();
                tc_fence_after();
                const float f = tab.resc[c];
                for (int jb = 0; jb < D; jb += 16) {
                    uint32_t r[16];
                    tmem_ld16(t_state + lane_addr + jb, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
                    tmem_st16(t_state + lane_addr + jb, r);
                }
                tmem_wait_st();
                tc_fence_before();
                sync_ops();
                if (ct == 0) mbar_arrive(&bars[B_RESC_DONE]);
            }
            // (2) per-token gates of this chunk (parity buffer pb):
            //     m_t = b_t + max(m_prev, chunk prefix max of u)
            // u, b and the prefix maximum of u arrived with the chunk's keys, in the
            // key slot's spare rows; the chunk totals are their values at the last token
            if (!wait_ops(&bars[B_FULL_K0 + (c & 1)], (c >> 1) & 1, abort_flag, status) ||
                (c >= 2 && !wait_ops(&bars[B_GATES_FREE0 + pb], ((c >> 1) - 1) & 1, abort_flag, status))) { ok = false; break; }
            const float *g_u = reinterpret_cast<const float *>(sK + (c & 1) * Lay::kKslot + kGateRow * 128);
            const float *g_b = g_u + 64, *g_x = g_u + 128;
            const float2 cs = make_float2(g_b[Lc - 1], g_x[Lc - 1]);   // (sum of log f, max of u) of this chunk
            const float mnext = cs.x + fmaxf(mprev, cs.y);
            if (ct < kL) {
                const int t = ct;
                const bool valid = t < Lc;
                const float b = valid ? g_b[t] : 0.f;
                const float u = valid ? g_u[t] : -INFINITY;
                const float run = fmaxf(mprev, valid ? g_x[t] : mprev);
                const float gt = valid ? expf(mprev - run) : 0.f;     // = e^{b_t + m_prev - m_t}
                const float wn = valid ? expf(u + cs.x - mnext) * inv_sqrt_d : 0.f;
                const float wl = valid ? expf(u + cs.x - mnext + tab.lnupd[c]) * inv_sqrt_d : 0.f;
                fm[64 * pb + t] = b + run;
                fg[64 * pb + t] = gt;
                fF[64 * pb + t] = wide ? 1.f : gt * tab.lamret[c];
                fw[64 * pb + t] = wl;
                fpw[t] = wn;
                fu[64 * pb + t] = u;
                frun[64 * pb + t] = run;
            }
            sync_ops();
            if (ct == 0) mbar_arrive(&bars[B_GATES_READY0 + pb]);
            TC_TRACE(ct == 0, c, 1);
            // (3) Q as fp32 (K-major, tf32 operand of the retrieval); lanes take rows so a
            // warp's 16-byte stores land on distinct bank groups
            if (!wait_ops(&bars[B_FULL_Q], c & 1, abort_flag, status)) { ok = false; break; }
            if (c >= 1 && !wait_ops(&bars[B_QT_FREE], (c - 1) & 1, abort_flag, status)) { ok = false; break; }
            TC_TRACE(ct == 0, c, 2);
            if (!wide) {
#pragma unroll 4
                for (int e = ct; e < kL * (D / 8); e += 128) {
                    const int t = e & 63, ch = e >> 6;
                    const int jb = ch >> 3, cc = ch & 7;
                    const uint4 src = *reinterpret_cast<const uint4 *>(sQ + jb * 8192 + sw128_offset(t, cc));
                    const int blk = 2 * jb + (cc >> 2), cd = (cc & 3) * 2;
                    uint8_t *dst = sQt + blk * 8192;
                    *reinterpret_cast<float4 *>(dst + sw128_offset(t, cd)) =
                        make_float4(bf16_lo(src.x), bf16_hi(src.x), bf16_lo(src.y), bf16_hi(src.y));
                    *reinterpret_cast<float4 *>(dst + sw128_offset(t, cd + 1)) =
                        make_float4(bf16_lo(src.z), bf16_hi(src.z), bf16_lo(src.w), bf16_hi(src.w));
                }
            } else {     // wide chunk: the retrieval operand is g_t q_t
                for (int e = ct; e < kL * (D / 8); e += 128) {
                    const int t = e & 63, ch = e >> 6;
                    const int jb = ch >> 3, cc = ch & 7;
                    const uint4 src = *reinterpret_cast<const uint4 *>(sQ + jb * 8192 + sw128_offset(t, cc));
                    const int blk = 2 * jb + (cc >> 2), cd = (cc & 3) * 2;
                    const float gq = fg[64 * pb + t];
                    uint8_t *dst = sQt + blk * 8192;
                    *reinterpret_cast<float4 *>(dst + sw128_offset(t, cd)) =
                        make_float4(gq * bf16_lo(src.x), gq * bf16_hi(src.x), gq * bf16_lo(src.y), gq * bf16_hi(src.y));
                    *reinterpret_cast<float4 *>(dst + sw128_offset(t, cd + 1)) =
                        make_float4(gq * bf16_lo(src.z), gq * bf16_hi(src.z), gq * bf16_lo(src.w), gq * bf16_hi(src.w));
                }
            }
            fence_async_smem();
            sync_ops();
            if (ct == 0) {
                mbar_arrive(&bars[B_QT_READY]);
                mbar_arrive(&bars[B_Q_FREE]);
            }
            TC_TRACE(ct == 0, c, 3);
            // (4) normaliser chain n'_c = a n'_{c-1} + sum_s w_s k^_s, into the next key slot
            {
                const int slot = c & 1;
                if (!wait_ops(&bars[B_FULL_K0 + slot], (c >> 1) & 1, abort_flag, status)) { ok = false; break; }
                TC_TRACE(ct == 0, c, 4);
                const float a = expf(cs.x + mprev - mnext);
                const uint8_t *kt = sK + slot * Lay::kKslot;
                if (D == 256) {      // this thread's pair of key columns j = 2 ct, 2 ct + 1
                    const int j = 2 * ct;
                    const uint8_t *blkp = kt + (j / 64) * kKBlock;
                    const int cc = (j % 64) / 8, within = (j % 8) * 2;
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
                    for (int s = 0; s < kL; ++s) {
                        const uint32_t kv = *reinterpret_cast<const uint32_t *>(blkp + sw128_offset(s, cc) + within);
                        const float w = fpw[s];
                        a0 += w * bf16_lo(kv);
                        a1 += w * bf16_hi(kv);
                    }
                    nreg[0] = a * nreg[0] + a0;
                    nreg[1] = a * nreg[1] + a1;
                } else {
                    const int j = ct;
                    const uint8_t *blkp = kt + (j / 64) * kKBlock;
                    const int cc = (j % 64) / 8, within = (j % 8) * 2;
                    float acc = 0.f;
#pragma unroll 8
                    for (int s = 0; s < kL; ++s)
                        acc += fpw[s] * __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(
                                            blkp + sw128_offset(s, cc) + within));
                    nreg[0] = a * nreg[0] + acc;
                }
                if (c + 1 < nch) {
                    const int ns = (c + 1) & 1;
                    if (c >= 1 && !wait_ops(&bars[B_K_FREE0 + ns], ((c - 1) >> 1) & 1, abort_flag, status)) { ok = false; break; }
                    uint8_t *nt = sK + ns * Lay::kKslot;
#pragma unroll
                    for (int r = 0; r < D / 128; ++r) {
                        const int j = nj(r);
                        uint8_t *blkp = nt + (j / 64) * kKBlock;
                        const int cc = (j % 64) / 8, within = (j % 8) * 2;
                        const float hi = __bfloat162float(__float2bfloat16_rn(nreg[r]));
                        *reinterpret_cast<__nv_bfloat16 *>(blkp + sw128_offset(64, cc) + within) = __float2bfloat16_rn(hi);
                        *reinterpret_cast<__nv_bfloat16 *>(blkp + sw128_offset(65, cc) + within) =
                            __float2bfloat16_rn(nreg[r] - hi);
                    }
                    fence_async_smem();
                    sync_ops();
                    if (ct == 0) mbar_arrive(&bars[B_NROW_READY0 + ns]);
                }
            }
            TC_TRACE(ct == 0, c, 5);
            // (5) V scaled in place by w^ (the operand of both the update and the intra term)
            if (!wait_ops(&bars[B_FULL_V], c & 1, abort_flag, status)) { ok = false; break; }
            if (wide) {      // the intra-chunk MMA reads V unscaled first
                if (!wait_ops(&bars[B_INTRA_DONE], nwide & 1, abort_flag, status)) { ok = false; break; }
                ++nwide;
            }
            TC_TRACE(ct == 0, c, 6);
            {
                const float *wv = fw + 64 * pb;
#pragma unroll 4
                for (int e = ct; e < 2 * kL * 8; e += 128) {       // (block, row s, chunk)
                    const int blk = e / (kL * 8), s = (e / 8) % kL, cc = e & 7;
                    uint4 *p = reinterpret_cast<uint4 *>(sV + blk * 8192 + sw128_offset(s, cc));
                    const uint4 src = *p;
                    const float w = wv[s];
                    uint4 dst;
                    dst.x = pack_bf16x2(bf16_lo(src.x) * w, bf16_hi(src.x) * w);
                    dst.y = pack_bf16x2(bf16_lo(src.y) * w, bf16_hi(src.y) * w);
                    dst.z = pack_bf16x2(bf16_lo(src.z) * w, bf16_hi(src.z) * w);
                    dst.w = pack_bf16x2(bf16_lo(src.w) * w, bf16_hi(src.w) * w);
                    *p = dst;
                }
            }
            fence_async_smem();
            sync_ops();
            if (ct == 0) mbar_arrive(&bars[B_VHAT_READY]);
            TC_TRACE(ct == 0, c, 7);
        }
        // final state (last segment only): Lambda * Cs, n', m
        if (ok && g == P - 1 && nch > 0) {
            if (wait_ops(&bars[B_DONE], 0, abort_flag, status)) {
                __syncwarp();
                tc_fence_after();
                const int cl = nch - 1;
                const float2 cs = cstat[(size_t)bh * nchunks + c0 + cl];
                const float mn = cs.x + fmaxf(tab.mprev[cl], cs.y);
                const float lam_last = expf(-tab.lnupd[cl]);
                if (C_out) {
                    const int i = 32 * q4 + lane;
                    for (int jb = 0; jb < D; jb += 16) {
                        uint32_t r[16];
                        tmem_ld16(t_state + lane_addr + jb, r);
                        tmem_wait_ld();
                        float4 *dst = reinterpret_cast<float4 *>(C_out + ((size_t)bh * D + i0 + i) * D + jb);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_float4(__uint_as_float(r[4 * e]) * lam_last,
                                                 __uint_as_float(r[4 * e + 1]) * lam_last,
                                                 __uint_as_float(r[4 * e + 2]) * lam_last,
                                                 __uint_as_float(r[4 * e + 3]) * lam_last);
                    }
                }
                if (tile == 0) {
                    if (n_out) {
#pragma unroll
                        for (int r = 0; r < D / 128; ++r) n_out[(size_t)bh * D + nj(r)] = nreg[r];
                    }
                    if (m_out && ct == 0) m_out[bh] = mn;
                }
            }
        }
        tc_fence_before();
    } else if (is_sco) {
        // ---------------------------------------------------------- score group
        // Rows t = 16 q4 + (lane & 15) of S sit in TMEM lanes 0-15 of the warp's
        // quadrant (M = 64 layout); lanes 16-31 take the same rows' upper 32
        // columns via shuffles, so every lane masks 32 scores.
        // After the scores of chunk c it writes h for tokens 32-63 of chunk c - 1.
        bool ok = true;
        const int t = 16 * q4 + (lane & 15);
        const int hh = lane >> 4;                             // column half of this lane
        auto pass1 = [&](int cp) -> bool {                    // epilogue of tokens 32-63 of chunk cp
            if (!wait_sco(&bars[B_H_FULL0 + (cp & 1)], (cp >> 1) & 1, abort_flag, status) ||
                !wait_sco(&bars[B_O_FULL1], cp & 1, abort_flag, status)) return false;
            float og[32];
            read_gates(og);
            sync_sco();                                       // every thread has its gates: the tile is free
            if (st_ == 0) {
                ++o_taken[1];
                if (cp + 1 < nch) issue_o(cp + 1, 0);         // tokens 0-31 of the next chunk
            }
            __syncwarp();
            tc_fence_after();
            TC_TRACE(st_ == 0, cp, 22);
            epilogue_pass(cp, 1, og);
            TC_TRACE(st_ == 0, cp, 23);
            tc_fence_before();
            sync_sco();
            finish_pass(cp, st_ == 0);
            TC_TRACE(st_ == 0, cp, 28);
            return true;
        };
        for (int c = 0; ok && c < nch; ++c) {
            const int t0 = (c0 + c) * kL;
            const int Lc = min(kL, S - t0);
            const int pb = c & 1;
            if (!wait_sco(&bars[B_GATES_READY0 + pb], (c >> 1) & 1, abort_flag, status) ||
                !wait_sco(&bars[B_S_FULL], c & 1, abort_flag, status) ||
                (c >= 1 && !wait_sco(&bars[B_P_FREE], (c - 1) & 1, abort_flag, status)) ||
                (c >= 2 && !wait_sco(&bars[B_FINV_FREE0 + pb], ((c >> 1) - 1) & 1, abort_flag, status))) { ok = false; break; }
            TC_TRACE(st_ == 0, c, 8);
            __syncwarp();
            tc_fence_after();
            uint32_t sa[32], sb[32], sn[8];
            tmem_ld16(t_S + lane_addr + 0, *reinterpret_cast<uint32_t(*)[16]>(&sa[0]));
            tmem_ld16(t_S + lane_addr + 16, *reinterpret_cast<uint32_t(*)[16]>(&sa[16]));
            tmem_ld16(t_S + lane_addr + 32, *reinterpret_cast<uint32_t(*)[16]>(&sb[0]));
            tmem_ld16(t_S + lane_addr + 48, *reinterpret_cast<uint32_t(*)[16]>(&sb[16]));
            tmem_ld8(t_S + lane_addr + 64, sn);
            tmem_wait_ld();
            TC_TRACE(st_ == 0, c, 16);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const uint32_t up = __shfl_sync(0xffffffffu, sb[e], lane & 15);
                sa[e] = hh ? up : sa[e];
            }
            const bool valid = t < Lc;
            float rowsum = 0.f;
            if (tab.wide[c] != 0.f) {
                // exact weights e^{u_s - (m_t - b_t)} / sqrt(d); exponents <= 0 for s <= t
                const float rt = frun[64 * pb + t];
                const float *us = fu + 64 * pb + 32 * hh;
                for (int cq = 0; cq < 4; ++cq) {
                    const int cc = 4 * hh + cq;
                    uint32_t w4[4], l4[4];
#pragma unroll
                    for (int p2 = 0; p2 < 4; ++p2) {
                        float pv[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int sl = cq * 8 + p2 * 2 + e;
                            const int s = 32 * hh + sl;
                            pv[e] = (valid && s <= t) ? expf(us[sl] - rt) * inv_sqrt_d * __uint_as_float(sa[sl]) : 0.f;
                            rowsum += pv[e];
                        }
                        w4[p2] = pack_bf16x2(pv[0], pv[1]);
                        l4[p2] = pack_bf16x2(pv[0] - bf16_lo(w4[p2]), pv[1] - bf16_hi(w4[p2]));
                    }
                    *reinterpret_cast<uint4 *>(sP + sw128_offset(t, cc)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    *reinterpret_cast<uint4 *>(sPl + sw128_offset(t, cc)) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
                }
            } else {
            const float4 *wv4 = reinterpret_cast<const float4 *>(fw + 64 * pb + 32 * hh);
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {
                const int cc = 4 * hh + cq;
                const float4 wa = wv4[2 * cq], wb = wv4[2 * cq + 1];
                const float wk[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                uint32_t w4[4], l4[4];
#pragma unroll
                for (int p2 = 0; p2 < 4; ++p2) {
                    float pv[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int sl = cq * 8 + p2 * 2 + e;
                        const int s = 32 * hh + sl;
                        const float sc = (valid && s <= t) ? __uint_as_float(sa[sl]) : 0.f;
                        pv[e] = sc;
                        rowsum += wk[p2 * 2 + e] * sc;
                    }
                    w4[p2] = pack_bf16x2(pv[0], pv[1]);
                    l4[p2] = pack_bf16x2(pv[0] - bf16_lo(w4[p2]), pv[1] - bf16_hi(w4[p2]));
                }
                *reinterpret_cast<uint4 *>(sP + sw128_offset(t, cc)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                *reinterpret_cast<uint4 *>(sPl + sw128_offset(t, cc)) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
            }
            }
            TC_TRACE(st_ == 0, c, 17);
            rowsum += __shfl_xor_sync(0xffffffffu, rowsum, 16);
            if (hh == 0) {
                // den = g_t (n'_prev . q_t) + F_t sum_s w^_s S_ts;  h_t = o_t F_t H~_t / max(|den|, e^-m_t)
                const float nq = __uint_as_float(sn[0]) + __uint_as_float(sn[1]);
                const float Ft = fF[64 * pb + t];
                const float den = fg[64 * pb + t] * nq + Ft * rowsum;
                finv[64 * pb + t] = valid ? 0.5f * Ft / fmaxf(fabsf(den), expf(-fm[64 * pb + t])) : 0.f;
            }
            TC_TRACE(st_ == 0, c, 18);
            fence_async_smem();
            TC_TRACE(st_ == 0, c, 19);
            tc_fence_before();
            sync_sco();
            if (st_ == 0) {
                mbar_arrive(&bars[B_P_READY]);
                mbar_arrive(&bars[B_S_FREE]);
                mbar_arrive(&bars[B_GATES_FREE0 + pb]);
                mbar_arrive(&bars[B_FINV_READY0 + pb]);
            }
            TC_TRACE(st_ == 0, c, 9);
            if (c >= 1 && !pass1(c - 1)) { ok = false; break; }
        }
        if (ok && nch > 0) ok = pass1(nch - 1);
    } else if (is_out) {
        // --------------------------------------------------------- output group
        // Thread = value row i of H^T (TMEM lane); h for tokens 0-31 of each chunk
        // goes through the shared h tile and leaves by TMA store, so the global
        // writes are whole 128-byte rows.  The gates are loaded a chunk ahead.
        bool ok = true;
        if (xt == 0 && nch > 0) issue_o(0, 0);             // gates of tokens 0-31 of chunk 0
        {   // Incoming state into TMEM, while the other groups start on chunk 0: the
            // initial state for segment 0, else the state at the end of segment g - 1,
            // which segment_scan_kernel left in summary slot g - 1.
            const int i = 32 * q4 + lane;
            const float *src = g == 0 ? (C0 ? C0 + (size_t)bh * D * D : nullptr)
                                      : summ + ((size_t)bh * (P - 1) + g - 1) * ((size_t)D * D + D);
#pragma unroll 4
            for (int jb = 0; jb < D; jb += 16) {
                uint32_t r[16];
                if (src) {
                    const float4 *row = reinterpret_cast<const float4 *>(src + (size_t)(i0 + i) * D + jb);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 x = row[e];
                        r[4 * e] = __float_as_uint(x.x);
                        r[4 * e + 1] = __float_as_uint(x.y);
                        r[4 * e + 2] = __float_as_uint(x.z);
                        r[4 * e + 3] = __float_as_uint(x.w);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) r[e] = 0u;
                }
                tmem_st16(t_state + lane_addr + jb, r);
            }
            tmem_wait_st();
            tc_fence_before();
            sync_out();
            if (xt == 0) mbar_arrive(&bars[B_STATE_READY]);
        }
        for (int c = 0; ok && c < nch; ++c) {
            const int hb = c & 1;
            if (!wait_out(&bars[B_H_FULL0 + hb], (c >> 1) & 1, abort_flag, status) ||
                !wait_out(&bars[B_FINV_READY0 + hb], (c >> 1) & 1, abort_flag, status) ||
                !wait_out(&bars[B_O_FULL0], c & 1, abort_flag, status)) { ok = false; break; }
            TC_TRACE(xt == 0, c, 10);
            float og[32];
            read_gates(og);
            sync_out();                                      // every thread has its gates: the tile is free
            if (xt == 0) {
                ++o_taken[0];
                issue_o(c, 1);                               // tokens 32-63 of this chunk
            }
            __syncwarp();
            tc_fence_after();
            TC_TRACE(xt == 0, c, 20);
            epilogue_pass(c, 0, og);
            TC_TRACE(xt == 0, c, 21);
            tc_fence_before();
            sync_out();
            finish_pass(c, xt == 0);
            TC_TRACE(xt == 0, c, 11);
        }
        tc_fence_before();
    }
    __syncthreads();
    TC_TRACE_NS(tid == 0, 31);
    // never leave an o-gate load in flight into shared memory (a group that gave
    // up a wait may not have taken the last tile issued for it)
    if (tid == 0) {
        for (int hq = 0; hq < 2; ++hq)
            if (o_issued[hq] > o_taken[hq])
                mbar_wait(&bars[B_O_FULL0 + hq], (o_issued[hq] - 1) & 1, nullptr, status, 200000000ull);
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
        tmem_relinquish();
    }
}

// ------------------------------------------------------------ segment scan
// Turns the segment summaries into incoming states, in place: slot g of the
// summary buffer becomes the state (C', n') at the end of segment g, i.e. the
// incoming state of segment g + 1:
//   X_g = e^{F_g + M_{g-1} - M_g} X_{g-1} + e^{mloc_g - M_g} dX_g,
//   M_g = max(F_g + M_{g-1}, mloc_g),  X_{-1} = initial state,  M_{-1} = m_0,
// with (F_g, mloc_g) the segment's total log forget and own stabiliser.  One
// thread per 4 consecutive floats of a head's (C', n'), all segments in order.
__global__ void __launch_bounds__(256)
segment_scan_kernel(const float2 *__restrict__ sstat, float *__restrict__ summ, const float *__restrict__ C0,
                    const float *__restrict__ n0, const float *__restrict__ m0, int D, int P) {
    pdl_wait();
    const int bh = blockIdx.y;
    const size_t per = (size_t)D * D + D;
    const size_t e4 = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (e4 >= per) return;
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const size_t idx = e4 + e;
        x[e] = idx < (size_t)D * D ? (C0 ? C0[(size_t)bh * D * D + idx] : 0.f)
                                   : (n0 ? n0[(size_t)bh * D + idx - (size_t)D * D] : 0.f);
    }
    float mc = m0 ? m0[bh] : 0.f;
    float4 *slot = reinterpret_cast<float4 *>(summ + (size_t)bh * (P - 1) * per + e4);
    const size_t stride4 = per / 4;
#pragma unroll 4
    for (int g = 0; g < P - 1; ++g) {
        const float2 st = sstat[(size_t)bh * P + g];
        const float mn = fmaxf(st.x + mc, st.y);
        const float al = expf(st.x + mc - mn), be = expf(st.y - mn);
        const float4 d = slot[g * stride4];
        x[0] = al * x[0] + be * d.x;
        x[1] = al * x[1] + be * d.y;
        x[2] = al * x[2] + be * d.z;
        x[3] = al * x[3] + be * d.w;
        slot[g * stride4] = make_float4(x[0], x[1], x[2], x[3]);
        mc = mn;
    }
    pdl_launch_dependents();
}

// ------------------------------------------------------------ segment summaries
// Per (value tile, segment g < P-1, head): dC = sum_s w_s v_s k_s^T over the
// segment, w_s = e^{u_s + E_c - mloc} / sqrt(d) (all exponents <= 0), on the
// tensor cores with the accumulator in TMEM; dn = sum_s w_s k_s on the tensor
// cores too, as rows 0 and 1 (w in bf16 high and low parts) of an M=64 product
// with the same K tile.  K and V stream through a 4-stage ring; V is scaled by
// w in place.  The tile's u = log i - b travels with it: a bulk copy puts the
// 64 floats into rows 2-3 of the stage's W tile, rows whose products (rows 2-3
// of the dn accumulator) are never read, so the compute warps hold no global
// load across their barriers.
// DH 512 splits the key columns over two CTAs (KC = 256 each); their summaries
// are independent column blocks of the same dC, so nothing is exchanged.
template <int D>
struct SumLayout {
    static constexpr int KC = D > 256 ? 256 : D;          // key columns per CTA
    static constexpr int KS = D / KC;                     // key splits
    static constexpr int NT = (D + 127) / 128;            // value-row tiles
    static constexpr int kStages = 4;
    static constexpr int kKslot = (KC / 64) * 8192;       // K bf16: KC/64 blocks x 64 rows
    static constexpr int kSlot = kKslot + 16384 + 8192;   // + V (2 blocks x 8 KB) + W (64 x 64 bf16, rows 0-1 used)
    static constexpr int kF = kStages * kSlot;            // w[64]
    static constexpr int kTab = kF + 64 * 4;              // E per chunk
    static constexpr int kBar = kTab + kMaxCps * 4;       // full[4], free[4], ready[4], done
    static constexpr int kMisc = kBar + 16 * 8;
    static constexpr int kBytes = kMisc + 16 + 1024;
};
static_assert(SumLayout<512>::kBytes <= kMaxSmemPerCta, "summary kernel shared memory");

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
segment_summary_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                          const float *__restrict__ upad, const float2 *__restrict__ cstat,
                          float2 *__restrict__ sstat, float *__restrict__ summ,
                          unsigned int *status, int S, int Spad, int nchunks, int P, int cps, int L) {
    using Lay = SumLayout<D>;
    constexpr int NS = Lay::kStages;
    // value rows of this CTA: 128, or all DH when DH < 128 (the MMAs keep M = 128;
    // the second 64-row block of V stays zero, so rows >= DH of dC are zero)
    constexpr int kVBlocks = D < 128 ? 1 : 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    float *fw = reinterpret_cast<float *>(smem + Lay::kF);
    float *tabE = reinterpret_cast<float *>(smem + Lay::kTab);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::kBar);
    uint64_t *b_full = bars, *b_free = bars + NS, *b_ready = bars + 2 * NS, *b_done = bars + 3 * NS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kMisc + 4);
    __shared__ float s_mloc, s_etot;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int KC = Lay::KC, KS = Lay::KS, NT = Lay::NT;
    const int tile = blockIdx.x / KS, kh = blockIdx.x % KS, g = blockIdx.y, bh = blockIdx.z;
    const int i0 = tile * kRows, k0 = kh * KC;
    const int c0 = g * cps;
    const int nch = min(nchunks, c0 + cps) - c0;
    // 64-token tiles of the segment; tile tl lies in chunk tl / nsub (chunks of L tokens)
    const int nsub = L / kL;
    const int tseg = c0 * L;
    const int ntl = (min(S, (c0 + nch) * L) - tseg + kL - 1) / kL;
    const float inv_sqrt_d = rsqrtf((float)D);

    pdl_wait();
    float *tabM = fw;                                  // chunk maxima, staged (fw is free until the loop)
    for (int c = tid; c < nch; c += blockDim.x) {
        const float2 cs = cstat[(size_t)bh * nchunks + c0 + c];
        tabE[c] = cs.x;
        if (c < 64) tabM[c] = cs.y;
    }
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < 3 * NS + 1; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        // segment statistics: E_c = sum_{c' >= c} btot, mloc = max_c (cmax_c + E_c)
        float E = 0.f, mloc = -INFINITY;
        for (int c = nch - 1; c >= 0; --c) {
            const float cy = c < 64 ? tabM[c] : cstat[(size_t)bh * nchunks + c0 + c].y;
            E += tabE[c];
            tabE[c] = E;
            mloc = fmaxf(mloc, cy + E);
        }
        s_mloc = mloc;
        s_etot = E;
        if (blockIdx.x == 0) sstat[(size_t)bh * P + g] = make_float2(E, mloc);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tc_fence_before();
    }
    for (int e = tid; e < NS * 512; e += blockDim.x) {     // the W tiles start all zero
        const int st = e >> 9, off = (e & 511) * 16;
        *reinterpret_cast<uint4 *>(smem + st * Lay::kSlot + Lay::kKslot + 16384 + off) = make_uint4(0u, 0u, 0u, 0u);
        if (kVBlocks == 1)                                  // and so does an unloaded V block
            *reinterpret_cast<uint4 *>(smem + st * Lay::kSlot + Lay::kKslot + 8192 + off) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = *tmem_slot;                  // dC in columns [0, KC), dn rows in [256, 256 + KC)
    const float mloc = s_mloc;
    const uint32_t idesc_U = idesc_f32acc(kFmtBF16, kFmtBF16, true, true, 128, KC);
    const uint32_t idesc_N = idesc_f32acc(kFmtBF16, kFmtBF16, false, true, 64, KC);

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&map_k);
            tma_prefetch_desc(&map_v);
            int issued[NS] = {};
            for (int c = 0; c < ntl; ++c) {
                const int slot = c % NS, t0 = tseg + c * kL;
                if (c >= NS && !mbar_wait(&b_free[slot], ((c / NS) - 1) & 1, abort_flag, status)) break;
                TC_TRACE_SUM(true, c, 0);
                uint8_t *base = smem + slot * Lay::kSlot;
                mbar_arrive_expect_tx(&b_full[slot], kL * KC * 2 + kL * kVBlocks * 64 * 2 + kL * 4);
                for (int jb = 0; jb < KC / 64; ++jb)
                    tma_load_3d(base + jb * 8192, &map_k, &b_full[slot], k0 + jb * 64, t0, bh);
                for (int b = 0; b < kVBlocks; ++b)
                    tma_load_3d(base + Lay::kKslot + b * 8192, &map_v, &b_full[slot], i0 + 64 * b, t0, bh);
                bulk_load(base + Lay::kKslot + 16384 + 256, upad + (size_t)bh * Spad + t0, kL * 4, &b_full[slot]);
                ++issued[slot];
            }
            // never leave a load in flight into shared memory
            for (int st = 0; st < NS; ++st)
                if (issued[st]) mbar_wait(&b_full[st], (issued[st] - 1) & 1, nullptr, status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int c = 0; c < ntl; ++c) {
                const int slot = c % NS;
                if (!mbar_wait(&b_ready[slot], (c / NS) & 1, abort_flag, status)) break;
                TC_TRACE_SUM(true, c, 1);
                tc_fence_after();
                const uint32_t va = smem_u32(smem + slot * Lay::kSlot + Lay::kKslot);
                const uint32_t ka = smem_u32(smem + slot * Lay::kSlot);
                const uint32_t wa = va + 16384;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tacc, sdesc_sw128(va + ks * 2048, 8192, 1024),
                                sdesc_sw128(ka + ks * 2048, 8192, 1024), idesc_U, (c > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tacc + 256, sdesc_sw128(wa + ks * 32, 16, 1024),
                                sdesc_sw128(ka + ks * 2048, 8192, 1024), idesc_N, (c > 0 || ks > 0) ? 1u : 0u);
                mma_commit(&b_free[slot]);
            }
            mma_commit(b_done);
            mbar_wait(b_done, 0, nullptr, status);
        }
    } else {
        // 8 compute warps: w and its bf16 parts (threads 0-63), V scaled in place
        // (all); for the readout, the two warps of each TMEM lane quadrant take
        // one half of the columns each.
        const int ct = tid - 64, q4 = warp & 3;
        bool ok = true;
        for (int c = 0; c < ntl; ++c) {
            const int slot = c % NS, t0 = tseg + c * kL, Lc = min(kL, S - t0);
            if (!compute_wait(&b_full[slot], (c / NS) & 1, abort_flag, status)) { ok = false; break; }
            TC_TRACE_SUM(ct == 0, c, 2);
            uint8_t *base = smem + slot * Lay::kSlot;
            uint8_t *sV = base + Lay::kKslot;
            if (ct < kL) {       // rows 0 and 1 of W: w in bf16 high and low parts
                const float u = reinterpret_cast<const float *>(sV + 16384 + 256)[ct];
                const float wv = ct < Lc ? expf(u + tabE[c / nsub] - mloc) * inv_sqrt_d : 0.f;
                fw[ct] = wv;
                const __nv_bfloat16 whi = __float2bfloat16_rn(wv);
                uint8_t *sW = sV + 16384;
                *reinterpret_cast<__nv_bfloat16 *>(sW + sw128_offset(0, ct >> 3) + (ct & 7) * 2) = whi;
                *reinterpret_cast<__nv_bfloat16 *>(sW + sw128_offset(1, ct >> 3) + (ct & 7) * 2) =
                    __float2bfloat16_rn(wv - __bfloat162float(whi));
            }
            named_sync_compute();
#pragma unroll 4
            for (int e = ct; e < kVBlocks * kL * 8; e += 256) {   // V rows scaled in place by w
                const int blk = e / (kL * 8), s = (e / 8) % kL, cc = e & 7;
                uint4 *pv = reinterpret_cast<uint4 *>(sV + blk * 8192 + sw128_offset(s, cc));
                const uint4 src = *pv;
                const float ws = fw[s];
                uint4 dst;
                dst.x = pack_bf16x2(bf16_lo(src.x) * ws, bf16_hi(src.x) * ws);
                dst.y = pack_bf16x2(bf16_lo(src.y) * ws, bf16_hi(src.y) * ws);
                dst.z = pack_bf16x2(bf16_lo(src.z) * ws, bf16_hi(src.z) * ws);
                dst.w = pack_bf16x2(bf16_lo(src.w) * ws, bf16_hi(src.w) * ws);
                *pv = dst;
            }
            fence_async_smem();
            named_sync_compute();
            if (ct == 0) mbar_arrive(&b_ready[slot]);
            TC_TRACE_SUM(ct == 0, c, 3);
        }
        if (ok && compute_wait(b_done, 0, abort_flag, status)) {
            __syncwarp();
            tc_fence_after();
            float *out = summ + ((size_t)bh * (P - 1) + g) * ((size_t)D * D + D);
            const int i = 32 * q4 + lane;
            const uint32_t lane_addr = ((uint32_t)(32 * q4)) << 16;
            const int jhalf = (ct >> 7) * (KC / 2);
            for (int jb = jhalf; jb < jhalf + KC / 2; jb += 16) {
                uint32_t r[16];
                tmem_ld16(tacc + lane_addr + jb, r);
                tmem_wait_ld();
                if (i0 + i >= D) continue;                  // padding rows (DH < 128)
                float4 *dst = reinterpret_cast<float4 *>(out + (size_t)(i0 + i) * D + k0 + jb);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                         __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
            }
            if (q4 == 0) {      // dn = rows 0 + 1 of the M=64 product (TMEM lanes 0 and 1)
                for (int jb = jhalf; jb < jhalf + KC / 2; jb += 16) {
                    uint32_t r[16];
                    tmem_ld16(tacc + 256 + jb, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float v = __uint_as_float(r[e]) + __shfl_down_sync(0xffffffffu, __uint_as_float(r[e]), 1);
                        if (lane == 0 && (jb + e) / (KC / NT) == tile)   // the value tiles share out the columns
                            out[(size_t)D * D + k0 + jb + e] = v;
                    }
                }
            }
        }
        tc_fence_before();
    }
    pdl_launch_dependents();      // the next kernel may be scheduled; it waits for this one
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tacc, 512);
        tmem_relinquish();
    }
}

// ------------------------------------------------------------------- host
template <int D>
cudaError_t launch_summaries_t(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    if (p.P <= 1) return cudaSuccess;
    CUtensorMap mk, mv;
    if (!make_map_bf16(&mk, a.k, p.BH, p.S, D) || !make_map_bf16(&mv, a.v, p.BH, p.S, D))
        return cudaErrorInvalidValue;
    float *ws = (float *)a.workspace;
    const float2 *cstat = (const float2 *)(ws + p.off_cstat);
    float2 *sstat = (float2 *)(ws + p.off_sstat);
    float *summ = ws + p.off_summ;
    const int sm = SumLayout<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(segment_summary_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    {
        KernelTimer timer("segment_summary_tc", st);
        e = launch_chained(segment_summary_tc_kernel<D>, dim3(SumLayout<D>::NT * SumLayout<D>::KS, p.P - 1, p.BH),
                           dim3(kThreads), sm, st, mk, mv, (const float *)(ws + p.off_upad), cstat, sstat, summ,
                           a.status, p.S, p.Spad, p.nchunks, p.P, p.cps, p.L);
        if (e != cudaSuccess) return e;
    }
    KernelTimer timer("segment_scan", st);
    const size_t per4 = ((size_t)D * D + D) / 4;
    return launch_chained(segment_scan_kernel, dim3((unsigned)((per4 + 255) / 256), p.BH), dim3(256), 0, st,
                          (const float2 *)sstat, summ, a.C0, a.n0, a.m0, D, p.P);
}

template <int D>
cudaError_t launch_tc_t(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map_bf16(&mq, a.q, p.BH, p.S, D) || !make_map_bf16(&mk, a.k, p.BH, p.S, D) ||
        !make_map_bf16(&mv, a.v, p.BH, p.S, D) || !make_map_f32_rows(&mo, a.o_pre, p.BH, p.S, D, kRows, 32))
        return cudaErrorInvalidValue;
    float *ws = (float *)a.workspace;
    const float2 *cstat = (const float2 *)(ws + p.off_cstat);
    float2 *sstat = (float2 *)(ws + p.off_sstat);
    float *summ = ws + p.off_summ;
    cudaError_t e = launch_summaries_t<D>(a, p, st);
    if (e != cudaSuccess) return e;
    const int sm = OutLayout<D>::kBytes;
    e = cudaFuncSetAttribute(segment_output_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    KernelTimer timer("segment_output_tc", st);
    return launch_chained(segment_output_tc_kernel<D>, dim3(D / kRows, p.P, p.BH), dim3(kOutThreads), sm, st,
                          mq, mk, mv, mo, (__nv_bfloat16 *)a.h, a.i_pre, a.o_pre, a.C0, a.n0, a.m0, a.C_out,
                          a.n_out, a.m_out, (const float *)(ws + p.off_upad), (const float *)(ws + p.off_bpad),
                          (const float *)(ws + p.off_xpad), cstat, (const float2 *)sstat, (const float *)summ,
                          a.status, p.S, p.Spad, p.nchunks, p.P, p.cps);
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map_f32_rows(CUtensorMap *m, const void *base, int BH, int S, int D, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)S * D * 4};
    cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_bf16(CUtensorMap *m, const void *base, int BH, int S, int D, bool swizzle, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_segment_summaries(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    switch (p.DH) {
        case 64: return launch_summaries_t<64>(a, p, st);
        case 128: return launch_summaries_t<128>(a, p, st);
        case 256: return launch_summaries_t<256>(a, p, st);
        case 512: return launch_summaries_t<512>(a, p, st);
    }
    return cudaErrorInvalidValue;
}

bool tensor_path_supports(int DH, int L) { return L == kL && (DH == 128 || DH == 256); }

#ifdef XLSTM_TC_TRACE
extern "C" int xlstm_debug_set_trace(void *buf) {
    return cudaMemcpyToSymbol(g_tc_trace, &buf, sizeof(buf)) == cudaSuccess ? 0 : 1;
}
#endif

int tensor_path_max_chunks_per_segment() { return kMaxCps; }

cudaError_t launch_fwd_tensor(const FwdArgs &a, const FwdPlan &p, cudaStream_t st) {
    if (!a.bf16 || !tensor_path_supports(p.DH, p.L) || p.cps > kMaxCps) return cudaErrorInvalidValue;
    cudaError_t e = launch_gate_prologue(a, p, st);
    if (e != cudaSuccess) return e;
    if (p.DH == 128) return launch_tc_t<128>(a, p, st);
    return launch_tc_t<256>(a, p, st);
}

}  // namespace xlstm
