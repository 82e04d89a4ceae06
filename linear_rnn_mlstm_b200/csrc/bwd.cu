// Backward of the mLSTM cell: gradients with respect to q, k, v and the three
// gate pre-activations, fp32 arithmetic on CUDA cores ("xLSTM: Extended Long
// Short-Term Memory" section 2.3; the stabiliser held fixed as section 2.2
// allows).  Six launches, each a thin wrapper around a per-thread body in
// bwd_body.cuh (the algorithm is described there):
//   K1 bwd_gates       one warp per head       log f, chunk-local cumsum, m_t
//   K2 bwd_states      one thread per state row  chunk-start states C'_c, n'_c
//                      (DH a multiple of 32: one CTA per 32 rows, bwd_rows_kernel)
//   K3 bwd_token_fwd   one thread per token    num', nq', den', dotilde, dnum', dnq'
//                      (DH a multiple of 32: one warp per token; bf16 with DH 128 or
//                      256: one CTA per chunk)
//   K4 bwd_reverse     one thread per state row  reverse state at each chunk end
//                      (DH a multiple of 32: one CTA per 32 rows, bwd_rows_kernel)
//   K5 bwd_token_grad  one thread per token    dq, dk, dv, ditilde
//                      (DH a multiple of 32: one warp per token; bf16 with DH 128 or
//                      256: one CTA per chunk)
//   K6 bwd_forget      one warp per head       dftilde (reverse cumulative sum)
// The chunk-start and reverse states are materialised in the workspace
// (2 (NC + 1) DH^2 floats per head); this is the correctness-first form of the
// backward, not a tuned one.
#include <stdint.h>

#include "../../include/xlstm_mlstm.h"
#include "bwd_body.cuh"
#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "bwd_tc.cuh"

namespace xlstm {
namespace {

using bwd::BwdPtrs;

constexpr int kThreads = 128;

__device__ __forceinline__ long long thread_index() {
    return (long long)blockIdx.x * blockDim.x + threadIdx.x;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_states_kernel(BwdPtrs p) {
    const long long i = thread_index();
    const long long rows = (long long)p.DH + 1;
    if (i < (long long)p.BH * rows) bwd::states_row<T>(p, (int)(i / rows), (int)(i % rows));
}

template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_token_fwd_kernel(BwdPtrs p) {
    const long long i = thread_index();
    if (i < (long long)p.BH * p.S) bwd::token_fwd<T>(p, (int)(i / p.S), (int)(i % p.S));
}

template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_reverse_kernel(BwdPtrs p) {
    const long long i = thread_index();
    const long long rows = (long long)p.DH + 1;
    if (i < (long long)p.BH * rows) bwd::reverse_row<T>(p, (int)(i / rows), (int)(i % rows));
}

template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_token_grad_kernel(BwdPtrs p) {
    const long long i = thread_index();
    if (i < (long long)p.BH * p.S) bwd::token_grad<T>(p, (int)(i / p.S), (int)(i % p.S));
}

// K2 and K4 for DH a multiple of 32 (up to 512), one CTA per (32 state rows,
// head) instead of one thread per row: lanes take the key columns (DH / 32
// each), a warp four rows, so the rows stay in registers across chunks; per
// chunk the key tile (K2) or query tile (K4) and the 32 rows' coefficients are
// staged in shared memory once and shared by all 32 rows.  Same arithmetic,
// in the same order per element, as states_row / reverse_row.
constexpr int kRowBlock = 32;
constexpr int kRowThreads = 256;      // 8 warps x 4 rows

template <typename T>
__host__ __device__ size_t rows_stage_bytes(int L, int DH) {     // a multiple of 128 bytes
    return ((size_t)L * DH * sizeof(T) + (size_t)L * kRowBlock * 4 + (size_t)3 * L * 4 + 127) & ~(size_t)127;
}
template <typename T>
size_t rows_smem_bytes(int L, int DH) { return 2 * rows_stage_bytes<T>(L, DH) + (size_t)L * kRowBlock * 4; }

__device__ __forceinline__ uint32_t tc_smem_u32(const void *ptr) {
    return (uint32_t)__cvta_generic_to_shared(ptr);
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc_smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tc_smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Stages (two, by chunk parity) hold a chunk's key (K2) or query (K4) tile, the
// 32 rows' raw coefficients (v or dnum' entries) and the per-token scalars;
// the next chunk's stage is filled by cp.async while this one is used, so the
// walk over chunks waits on no global-memory round trip.
template <typename T, int NCL, bool REVERSE>
__global__ void __launch_bounds__(kRowThreads) bwd_rows_kernel(BwdPtrs p) {
    constexpr int DH = 32 * NCL;
    extern __shared__ __align__(16) uint8_t rows_smem[];
    const int L = p.L, S = p.S, NC = p.NC;
    const size_t stage_bytes = rows_stage_bytes<T>(L, DH);
    float *coef = reinterpret_cast<float *>(rows_smem + 2 * stage_bytes);     // [L][32]
    const int bh = blockIdx.y, r0 = blockIdx.x * kRowBlock;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t DD = (size_t)DH * DH;
    const float inv_sqrt = 1.f / sqrtf((float)DH);
    const T *src = (const T *)(REVERSE ? p.q : p.k);
    const T *v = (const T *)p.v;
    auto stage = [&](int buf, T *&tile, float *&raw, float *&sc) {
        uint8_t *base = rows_smem + buf * stage_bytes;
        tile = reinterpret_cast<T *>(base);
        raw = reinterpret_cast<float *>(base + (size_t)L * DH * sizeof(T));
        sc = raw + (size_t)L * kRowBlock;                                   // [3][L]
    };
    // the copies of chunk c into stage buf
    auto issue = [&](int c, int buf) {
        T *tile; float *raw, *sc;
        stage(buf, tile, raw, sc);
        const int a = c * L, n = bwd::imin(S, a + L) - a;
        const size_t row0 = (size_t)bh * S + a;
        constexpr int EPV = 16 / (int)sizeof(T);                            // elements per 16 bytes
        for (int e = threadIdx.x; e < n * DH / EPV; e += kRowThreads)
            cp_async16(tile + (size_t)e * EPV, src + row0 * DH + (size_t)e * EPV);
        for (int e = threadIdx.x; e < n * kRowBlock; e += kRowThreads) {
            const int s = e / kRowBlock, rr = e % kRowBlock, r = r0 + rr;
            const size_t ts = row0 + s;
            if (r < DH) {
                if (REVERSE) cp_async4(raw + e, p.dnum + ts * DH + r);
                else if (sizeof(T) == 4) cp_async4(raw + e, v + ts * DH + r);
                else    // bf16: the 4-byte word holding element r (picked apart below)
                    cp_async4(raw + e, reinterpret_cast<const uint8_t *>(v) + ((ts * DH + r) & ~(size_t)1) * 2);
            } else {
                if (REVERSE && r == DH) cp_async4(raw + e, p.dnq + ts);
                else raw[e] = r == DH ? 1.f : 0.f;
            }
        }
        for (int s = threadIdx.x; s < n; s += kRowThreads) {
            cp_async4(sc + s, p.b + row0 + s);
            if (REVERSE) cp_async4(sc + L + s, p.mt + row0 + s);
            else cp_async4(sc + L + s, p.ip + row0 + s);
        }
    };
    // this warp's rows r0 + 4 warp + i (row DH is the normaliser; rows past it unused)
    float st[4][NCL];
    auto slot_ptr = [&](int r, int slot) -> float * {
        if (r == DH) return (REVERSE ? p.dnb + (size_t)bh * NC * DH : p.nst + (size_t)bh * (NC + 1) * DH) +
                            (size_t)slot * DH;
        return (REVERSE ? p.dCb + (size_t)bh * NC * DD : p.Cst + (size_t)bh * (NC + 1) * DD) +
               (size_t)slot * DD + (size_t)r * DH;
    };
    // row r's values (lane + 32 j) into `slot`
    auto store_row = [&](int r, int slot, const float (&x)[NCL]) {
        float *dst = slot_ptr(r, slot);
#pragma unroll
        for (int j = 0; j < NCL; ++j) dst[lane + 32 * j] = x[j];
    };
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + 4 * warp + i;
#pragma unroll
        for (int j = 0; j < NCL; ++j) {
            const int col = lane + 32 * j;
            float x = 0.f;
            if (REVERSE && r < DH && p.dC) x = p.dC[(size_t)bh * DD + (size_t)r * DH + col];
            if (REVERSE && r == DH && p.dn) x = p.dn[(size_t)bh * DH + col];
            st[i][j] = x;
        }
        if (r <= DH) store_row(r, REVERSE ? NC - 1 : 0, st[i]);
    }
    // chunks walked: 0 .. NC-1 forward; NC-1 .. 1 in reverse (slot c-1 from chunk c)
    const int nsteps = REVERSE ? NC - 1 : NC;
    auto chunk_of = [&](int k) { return REVERSE ? NC - 1 - k : k; };
    if (nsteps > 0) issue(chunk_of(0), 0);
    cp_async_commit();
    // the chunk scalars are loaded one chunk ahead too (a barrier would wait for them)
    float nBs = 0.f, nmprev = 0.f, nmend = 0.f;
    if (nsteps > 0) {
        const size_t h0 = (size_t)bh * NC + chunk_of(0);
        nBs = p.Bsum[h0]; nmprev = p.mprev[h0]; nmend = p.mend[h0];
    }
    for (int k = 0; k < nsteps; ++k) {
        const int c = chunk_of(k), buf = k & 1;
        const float Bs = nBs, mprev = nmprev, mend = nmend;
        __syncthreads();                       // everyone is done with stage buf ^ 1 and the coefficients
        if (k + 1 < nsteps) issue(chunk_of(k + 1), buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();                    // this chunk's copies (the newest group may still fly)
        __syncthreads();
        T *tile; float *raw, *sc;
        stage(buf, tile, raw, sc);
        const int a = c * L, n = bwd::imin(S, a + L) - a;
        for (int e = threadIdx.x; e < n * kRowBlock; e += kRowThreads) {
            const int s = e / kRowBlock, r = r0 + e % kRowBlock;
            const float w = REVERSE ? expf(sc[s] + mprev - sc[L + s])
                                    : expf(Bs - sc[s] + sc[L + s] - mend) * inv_sqrt;
            float x = raw[e];
            if (!REVERSE && sizeof(T) == 2 && r < DH) {
                const uint32_t word = __float_as_uint(x);
                x = __uint_as_float((r & 1) ? (word & 0xffff0000u) : (word << 16));
            }
            coef[e] = w * x;
        }
        __syncthreads();
        if (k + 1 < nsteps) {                  // in flight during this chunk's products
            const size_t hn = (size_t)bh * NC + chunk_of(k + 1);
            nBs = p.Bsum[hn]; nmprev = p.mprev[hn]; nmend = p.mend[hn];
        }
        const float decay = expf(Bs + mprev - mend);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < NCL; ++j) st[i][j] *= decay;
        for (int s = 0; s < n; ++s) {
            float kv[NCL];
#pragma unroll
            for (int j = 0; j < NCL; ++j) kv[j] = bwd::ld(tile, (size_t)s * DH + lane + 32 * j);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float cf = coef[s * kRowBlock + 4 * warp + i];
#pragma unroll
                for (int j = 0; j < NCL; ++j) st[i][j] += cf * kv[j];
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = r0 + 4 * warp + i;
            if (r > DH) continue;
            store_row(r, REVERSE ? c - 1 : c + 1, st[i]);
        }
    }
    cp_async_wait<0>();
}

template <typename T, bool REVERSE>
bool launch_rows(const BwdPtrs &p, cudaStream_t st) {
    const int ncl = p.DH / 32;
    if (p.DH % 32 != 0 || (ncl != 1 && ncl != 2 && ncl != 4 && ncl != 8 && ncl != 16)) return false;
    const size_t sm = rows_smem_bytes<T>(p.L, p.DH);
    if (sm > 232448) return false;        // two stages do not fit (fp32 at DH 512): per-thread kernel
    const dim3 grid((unsigned)((p.DH + 1 + kRowBlock - 1) / kRowBlock), (unsigned)p.BH);
#define XLSTM_BWD_ROWS(N)                                                                         \
    if (ncl == N) {                                                                                \
        cudaFuncSetAttribute(bwd_rows_kernel<T, N, REVERSE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm); \
        bwd_rows_kernel<T, N, REVERSE><<<grid, kRowThreads, sm, st>>>(p);                          \
        return true;                                                                               \
    }
    XLSTM_BWD_ROWS(1)
    XLSTM_BWD_ROWS(2)
    XLSTM_BWD_ROWS(4)
    XLSTM_BWD_ROWS(8)
    XLSTM_BWD_ROWS(16)
#undef XLSTM_BWD_ROWS
    return false;
}

// K3 and K5 for DH a multiple of 32 (up to 512), one warp per token instead of
// one thread: each lane takes the columns lane + 32 i, the dot products over
// DH are warp sums, and the products with the chunk's DH x DH states are read
// row by row in coalesced 128-byte pieces (row-indexed vectors come in as
// uniform loads).  The same quantities as token_fwd / token_grad; only the
// summation order inside each dot product differs.
constexpr int kTokWarps = 8;

__device__ __forceinline__ float wsum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename T, int NCL>
__global__ void __launch_bounds__(32 * kTokWarps) bwd_token_fwd_warp_kernel(BwdPtrs p) {
    constexpr int DH = 32 * NCL;
    __shared__ float s_ws[kTokWarps][bwd::kMaxChunk];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gt = (long long)blockIdx.x * kTokWarps + warp;
    if (gt >= (long long)p.BH * p.S) return;
    const int bh = (int)(gt / p.S), t = (int)(gt % p.S);
    const int S = p.S, L = p.L, NC = p.NC;
    const size_t DD = (size_t)DH * DH;
    const float inv_sqrt = 1.f / sqrtf((float)DH);
    const T *q = (const T *)p.q, *k = (const T *)p.k, *v = (const T *)p.v, *dh = (const T *)p.dh;
    const size_t ts = (size_t)bh * S + t;
    const int c = t / L, a = c * L;
    const size_t hc = (size_t)bh * NC + c;
    const float m_t = p.mt[ts], b_t = p.b[ts];
    const float g = expf(b_t + p.mprev[hc] - m_t);
    const float *Cc = p.Cst + ((size_t)bh * (NC + 1) + c) * DD;
    const float *nc = p.nst + ((size_t)bh * (NC + 1) + c) * DH;
    float qv[NCL];
#pragma unroll
    for (int i = 0; i < NCL; ++i) qv[i] = bwd::ld(q, ts * DH + lane + 32 * i);
    float *ws = s_ws[warp];
    float nq = 0.f;
    for (int s = a; s <= t; ++s) {
        const size_t ss = (size_t)bh * S + s;
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < NCL; ++i) dot += qv[i] * bwd::ld(k, ss * DH + lane + 32 * i);
        dot = wsum(dot);
        const float w = expf(b_t - p.b[ss] + p.ip[ss] - m_t) * dot * inv_sqrt;
        if (lane == 0) ws[s - a] = w;
        nq += w;
    }
    __syncwarp();
    float ni = 0.f;
#pragma unroll
    for (int i = 0; i < NCL; ++i) ni += nc[lane + 32 * i] * qv[i];
    nq += g * wsum(ni);
    // num'[r]: lane r % 32 keeps row r = lane + 32 i
    float num[NCL];
#pragma unroll
    for (int i = 0; i < NCL; ++i) num[i] = 0.f;
#pragma unroll
    for (int rb = 0; rb < NCL; ++rb) {
        for (int rl = 0; rl < 32; ++rl) {
            const int r = 32 * rb + rl;
            float part = 0.f;
#pragma unroll
            for (int i = 0; i < NCL; ++i) part += Cc[(size_t)r * DH + lane + 32 * i] * qv[i];
            part = wsum(part);
            if (rl == lane) num[rb] = part;
        }
    }
#pragma unroll
    for (int i = 0; i < NCL; ++i) {
        const int r = lane + 32 * i;
        float acc = num[i] * g;
        for (int s = a; s <= t; ++s) acc += ws[s - a] * bwd::ld(v, ((size_t)bh * S + s) * DH + r);
        num[i] = acc;
        p.num[ts * DH + r] = acc;
    }
    const float floor_ = expf(-m_t);
    const float den = fmaxf(fabsf(nq), floor_);
    float sdot = 0.f, A = 0.f;
#pragma unroll
    for (int i = 0; i < NCL; ++i) {
        const int r = lane + 32 * i;
        const float o = bwd::sigmoid_hd(p.op[ts * DH + r]);
        const float hv = num[i] / den;
        const float dhr = bwd::ld(dh, ts * DH + r);
        const float dht = dhr * o;
        p.dO[ts * DH + r] = dhr * hv * o * (1.f - o);
        const float dn_r = dht / den;
        p.dnum[ts * DH + r] = dn_r;
        sdot += dht * hv;
        A += dn_r * num[i];
    }
    sdot = wsum(sdot);
    A = wsum(A);
    if (lane == 0) {
        const float dnq = fabsf(nq) > floor_ ? -sdot / den * (nq > 0.f ? 1.f : -1.f) : 0.f;
        p.dnq[ts] = dnq;
        p.nq[ts] = nq;
        p.den[ts] = den;
        p.A[ts] = A + dnq * nq;
    }
}

template <typename T, int NCL>
__global__ void __launch_bounds__(32 * kTokWarps) bwd_token_grad_warp_kernel(BwdPtrs p) {
    constexpr int DH = 32 * NCL;
    __shared__ float s_w[kTokWarps][3][bwd::kMaxChunk];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gs = (long long)blockIdx.x * kTokWarps + warp;
    if (gs >= (long long)p.BH * p.S) return;
    const int bh = (int)(gs / p.S), s = (int)(gs % p.S);
    const int S = p.S, L = p.L, NC = p.NC;
    const size_t DD = (size_t)DH * DH;
    const float inv_sqrt = 1.f / sqrtf((float)DH);
    const T *q = (const T *)p.q, *k = (const T *)p.k, *v = (const T *)p.v;
    T *dq = (T *)p.dq, *dk = (T *)p.dk, *dv = (T *)p.dv;
    const size_t ss = (size_t)bh * S + s;
    const int c = s / L, a = c * L, e = bwd::imin(S, a + L);
    const size_t hc = (size_t)bh * NC + c;
    const float m_s = p.mt[ss], b_s = p.b[ss], i_s = p.ip[ss];
    const float *dnum_s = p.dnum + ss * DH;
    float *wdp_a = s_w[warp][0], *wdp_b = s_w[warp][1], *wsc_b = s_w[warp][2];
    float dns[NCL], vs[NCL], ks[NCL];
#pragma unroll
    for (int i = 0; i < NCL; ++i) {
        const int j = lane + 32 * i;
        dns[i] = dnum_s[j];
        vs[i] = bwd::ld(v, ss * DH + j);
        ks[i] = bwd::ld(k, ss * DH + j);
    }
    const float dnq_s = p.dnq[ss];
    for (int u = a; u <= s; ++u) {
        const size_t us = (size_t)bh * S + u;
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < NCL; ++i) dot += dns[i] * bwd::ld(v, us * DH + lane + 32 * i);
        dot = wsum(dot);
        if (lane == 0) wdp_a[u - a] = expf(b_s - p.b[us] + p.ip[us] - m_s) * (dot + dnq_s);
    }
    for (int t = s; t < e; ++t) {
        const size_t tt = (size_t)bh * S + t;
        float dot = 0.f, sc = 0.f;
#pragma unroll
        for (int i = 0; i < NCL; ++i) {
            const int j = lane + 32 * i;
            dot += p.dnum[tt * DH + j] * vs[i];
            sc += bwd::ld(q, tt * DH + j) * ks[i];
        }
        dot = wsum(dot);
        sc = wsum(sc);
        if (lane == 0) {
            const float w = expf(p.b[tt] - b_s + i_s - p.mt[tt]);
            wdp_b[t - s] = w * (dot + p.dnq[tt]);
            wsc_b[t - s] = w * sc * inv_sqrt;
        }
    }
    __syncwarp();
    const float g = expf(b_s + p.mprev[hc] - m_s);
    const float wk = expf(p.Bsum[hc] - b_s + i_s - p.mend[hc]);
    const float *Cc = p.Cst + ((size_t)bh * (NC + 1) + c) * DD;
    const float *ncs = p.nst + ((size_t)bh * (NC + 1) + c) * DH;
    const float *dCc = p.dCb + ((size_t)bh * NC + c) * DD;
    const float *dnc = p.dnb + ((size_t)bh * NC + c) * DH;
    // dq and dk: lanes own the key columns j; the states are read row by row
    float aq[NCL], ak[NCL], inter[NCL], rv[NCL];
#pragma unroll
    for (int i = 0; i < NCL; ++i) aq[i] = ak[i] = inter[i] = rv[i] = 0.f;
    for (int u = a; u <= s; ++u) {
        const float w = wdp_a[u - a];
#pragma unroll
        for (int i = 0; i < NCL; ++i) aq[i] += w * bwd::ld(k, ((size_t)bh * S + u) * DH + lane + 32 * i);
    }
    for (int t = s; t < e; ++t) {
        const float w = wdp_b[t - s];
#pragma unroll
        for (int i = 0; i < NCL; ++i) ak[i] += w * bwd::ld(q, ((size_t)bh * S + t) * DH + lane + 32 * i);
    }
    for (int r = 0; r < DH; ++r) {
        const float dr = dnum_s[r], vr = bwd::ld(v, ss * DH + r);
#pragma unroll
        for (int i = 0; i < NCL; ++i) {
            inter[i] += Cc[(size_t)r * DH + lane + 32 * i] * dr;
            rv[i] += dCc[(size_t)r * DH + lane + 32 * i] * vr;
        }
    }
    float di = 0.f;
#pragma unroll
    for (int i = 0; i < NCL; ++i) {
        const int j = lane + 32 * i;
        const float dqj = aq[i] * inv_sqrt + g * (inter[i] + dnq_s * ncs[j]);
        bwd::st(dq, ss * DH + j, dqj);
        const float dkh = ak[i] + wk * (rv[i] + dnc[j]);
        di += dkh * ks[i] * inv_sqrt;
        bwd::st(dk, ss * DH + j, dkh * inv_sqrt);
    }
    di = wsum(di);
    // dv: lanes own the value rows r = lane + 32 i; dC k_s by one warp sum per row
    float av[NCL];
#pragma unroll
    for (int i = 0; i < NCL; ++i) av[i] = 0.f;
    for (int t = s; t < e; ++t) {
        const float w = wsc_b[t - s];
#pragma unroll
        for (int i = 0; i < NCL; ++i) av[i] += w * p.dnum[((size_t)bh * S + t) * DH + lane + 32 * i];
    }
#pragma unroll
    for (int rb = 0; rb < NCL; ++rb) {
        for (int rl = 0; rl < 32; ++rl) {
            const int r = 32 * rb + rl;
            float part = 0.f;
#pragma unroll
            for (int i = 0; i < NCL; ++i) part += dCc[(size_t)r * DH + lane + 32 * i] * ks[i];
            part = wsum(part);
            if (rl == lane) av[rb] += wk * part * inv_sqrt;
        }
    }
#pragma unroll
    for (int i = 0; i < NCL; ++i) bwd::st(dv, ss * DH + lane + 32 * i, av[i]);
    if (lane == 0) {
        p.di[ss] = di;
        p.dF[ss] = p.A[ss] - di;
    }
}

template <typename T, bool GRAD>
bool launch_token_warp(const BwdPtrs &p, cudaStream_t st) {
    const int ncl = p.DH / 32;
    if (p.DH % 32 != 0 || (ncl != 1 && ncl != 2 && ncl != 4 && ncl != 8 && ncl != 16)) return false;
    const long long tokens = (long long)p.BH * p.S;
    const unsigned blocks = (unsigned)((tokens + kTokWarps - 1) / kTokWarps);
#define XLSTM_BWD_TOK(N)                                                                          \
    if (ncl == N) {                                                                                \
        if (GRAD) bwd_token_grad_warp_kernel<T, N><<<blocks, 32 * kTokWarps, 0, st>>>(p);          \
        else bwd_token_fwd_warp_kernel<T, N><<<blocks, 32 * kTokWarps, 0, st>>>(p);                \
        return true;                                                                               \
    }
    XLSTM_BWD_TOK(1)
    XLSTM_BWD_TOK(2)
    XLSTM_BWD_TOK(4)
    XLSTM_BWD_TOK(8)
    XLSTM_BWD_TOK(16)
#undef XLSTM_BWD_TOK
    return false;
}

// K1 and K6 with one warp per head instead of one thread: 32 tokens at a time
// with warp scans.  K1's stabiliser uses the unrolled form of the recurrence,
// m_t = b_t + max(m_prev, max_{s <= t in the chunk} (itilde_s - b_s)) with b
// chunk-local (equal to the sequential max-plus recurrence up to rounding; the
// backward only needs one consistent m with all exponents <= 0).
// K1 and K6 with one CTA per head: the per-chunk work (scans over a chunk's
// tokens, one warp per chunk) runs in parallel, and only the short chain over
// chunks (the stabiliser carried from chunk to chunk; the suffix sums of the
// chunks' d log f totals) is walked by one thread, from shared memory.
constexpr int kSeqThreads = 1024;
constexpr int kSeqTile = 2048;                 // chunks per pass through shared memory

// K1: (a) per chunk, log f, the chunk-local cumulative log forget b and the
// chunk-local prefix maximum of itilde - b (held in mt for now), the chunk's
// total (Bsum) and maximum; (b) the chunk-to-chunk stabiliser
// m_end = Bsum + max(m_prev, chunk maximum), m_0 = 0; (c) per token
// m_t = b_t + max(m_prev, prefix maximum).  Same operations per value as the
// token-by-token unrolled form b_t + max(m_prev, max_{s<=t}(itilde_s - b_s)).
__global__ void __launch_bounds__(kSeqThreads) bwd_gates_seq_kernel(BwdPtrs p) {
    __shared__ float s_u[kSeqTile], s_B[kSeqTile], s_m[kSeqTile];
    __shared__ float s_carry;
    const int bh = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.S, L = p.L, NC = p.NC;
    const size_t base = (size_t)bh * S, cbase = (size_t)bh * NC;
    for (int c0 = 0; c0 < NC; c0 += kSeqTile) {
        const int nt = bwd::imin(kSeqTile, NC - c0);
        for (int cc = warp; cc < nt; cc += kSeqThreads / 32) {
            const int a = (c0 + cc) * L, e = bwd::imin(S, a + L);
            float carry = 0.f, umax = -INFINITY;
            for (int t0 = a; t0 < e; t0 += 32) {
                const int t = t0 + lane;
                const bool ok = t < e;
                const float fpre = ok ? p.fp[base + t] : 0.f;
                const float lf = ok ? (p.fgate_exp ? fpre : bwd::log_sigmoid_hd(fpre)) : 0.f;
                float b = lf;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, b, o);
                    if (lane >= o) b += y;
                }
                b += carry;
                float u = ok ? p.ip[base + t] - b : -INFINITY;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, u, o);
                    if (lane >= o) u = fmaxf(u, y);
                }
                u = fmaxf(u, umax);
                if (ok) {
                    p.logf[base + t] = lf;
                    p.b[base + t] = b;
                    p.mt[base + t] = u;
                }
                const int last = bwd::imin(31, e - 1 - t0);
                carry = __shfl_sync(0xffffffffu, b, last);
                umax = __shfl_sync(0xffffffffu, u, last);
            }
            if (lane == 0) {
                s_B[cc] = carry;
                s_u[cc] = umax;
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float m = c0 == 0 ? 0.f : s_carry;
            for (int cc = 0; cc < nt; ++cc) {
                s_m[cc] = m;
                p.mprev[cbase + c0 + cc] = m;
                p.Bsum[cbase + c0 + cc] = s_B[cc];
                m = s_B[cc] + fmaxf(m, s_u[cc]);
                p.mend[cbase + c0 + cc] = m;
            }
            s_carry = m;
        }
        __syncthreads();
        for (int cc = warp; cc < nt; cc += kSeqThreads / 32) {
            const int a = (c0 + cc) * L, e = bwd::imin(S, a + L);
            const float m = s_m[cc];
            for (int t = a + lane; t < e; t += 32) p.mt[base + t] = p.b[base + t] + fmaxf(m, p.mt[base + t]);
        }
        __syncthreads();
    }
}

// K6, first part (only with final-state cotangents), one warp per head: the
// returned state's stabiliser m_T = F_T + max(0, max_s(itilde_s - F_s)); its
// explicit dependence moves A_final = sum dC' o C'_T + sum dn' o n'_T from
// itilde to F at the maximising key s*.
__global__ void __launch_bounds__(128) bwd_final_state_kernel(BwdPtrs p) {
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= p.BH) return;
    const int bh = (int)w, S = p.S, DH = p.DH, NC = p.NC;
    const size_t base = (size_t)bh * S, DD = (size_t)DH * DH;
    float a_final = 0.f;
    const float *CT = p.Cst + ((size_t)bh * (NC + 1) + NC) * DD;
    const float *nT = p.nst + ((size_t)bh * (NC + 1) + NC) * DH;
    if (p.dC && p.tc) {                    // C'_T as bf16 high + low planes
        const uint8_t *pl = reinterpret_cast<const uint8_t *>(CT);
        for (size_t i = lane; i < DD; i += 32) {
            const uint32_t off = bwdtc::plane_offset((int)(i / DH), (int)(i % DH), DH);
            const float x = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(pl + off)) +
                            __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(pl + DD * 2 + off));
            a_final += p.dC[(size_t)bh * DD + i] * x;
        }
    } else if (p.dC) {
        for (size_t i = lane; i < DD; i += 32) a_final += p.dC[(size_t)bh * DD + i] * CT[i];
    }
    if (p.dn)
        for (int j = lane; j < DH; j += 32) a_final += p.dn[(size_t)bh * DH + j] * nT[j];
    a_final = wsum(a_final);
    // the first t with the largest itilde_t - F_t, if that is > 0 (m_T's maximising key)
    float F0 = 0.f, best = 0.f;
    int sstar = -1;
    for (int t0 = 0; t0 < S; t0 += 32) {
        const int t = t0 + lane;
        float F = t < S ? p.logf[base + t] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, F, o);
            if (lane >= o) F += y;
        }
        F += F0;
        float cand = t < S ? p.ip[base + t] - F : -INFINITY;
        int ct = t;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {             // max, earliest token on ties
            const float oc = __shfl_xor_sync(0xffffffffu, cand, o);
            const int ot = __shfl_xor_sync(0xffffffffu, ct, o);
            if (oc > cand || (oc == cand && ot < ct)) { cand = oc; ct = ot; }
        }
        if (cand > best) { best = cand; sstar = ct; }
        F0 = __shfl_sync(0xffffffffu, F, 31);
    }
    if (lane == 0 && sstar >= 0) {
        p.di[base + sstar] -= a_final;
        p.dF[base + sstar] += a_final;
    }
}

// K6, second part: d log f_j = sum_{t >= j} dF_t.  (a) each chunk's total,
// (b) the suffix sums of the totals (one thread, last chunk first), (c) each
// chunk's own reverse cumulative sum started from its suffix; then the forget
// activation's derivative.
__global__ void __launch_bounds__(kSeqThreads) bwd_forget_seq_kernel(BwdPtrs p) {
    __shared__ float s_sum[kSeqTile];
    __shared__ float s_carry;
    const int bh = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.S, L = p.L, NC = p.NC;
    const size_t base = (size_t)bh * S;
    for (int c1 = NC; c1 > 0; c1 -= kSeqTile) {
        const int c0 = c1 > kSeqTile ? c1 - kSeqTile : 0, nt = c1 - c0;
        for (int cc = warp; cc < nt; cc += kSeqThreads / 32) {
            const int a = (c0 + cc) * L, e = bwd::imin(S, a + L);
            float x = 0.f;
            for (int t = a + lane; t < e; t += 32) x += p.dF[base + t];
            x = wsum(x);
            if (lane == 0) s_sum[cc] = x;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float acc = c1 == NC ? 0.f : s_carry;
            for (int cc = nt - 1; cc >= 0; --cc) {
                const float x = s_sum[cc];
                s_sum[cc] = acc;                 // total of the chunks after cc
                acc += x;
            }
            s_carry = acc;
        }
        __syncthreads();
        for (int cc = warp; cc < nt; cc += kSeqThreads / 32) {
            const int a = (c0 + cc) * L, e = bwd::imin(S, a + L);
            float acc = s_sum[cc];
            for (int g0 = a + ((e - a - 1) / 32) * 32; g0 >= a; g0 -= 32) {
                const int t = g0 + lane;
                float x = t < e ? p.dF[base + t] : 0.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_down_sync(0xffffffffu, x, o);
                    if (lane + o < 32) x += y;
                }
                x += acc;
                if (t < e) p.df[base + t] = p.fgate_exp ? x : x * bwd::sigmoid_hd(-p.fp[base + t]);
                acc = __shfl_sync(0xffffffffu, x, 0);
            }
        }
        __syncthreads();
    }
}

size_t align64(size_t x) { return (x + 63) & ~size_t(63); }

// Workspace layout in floats, each array 256-byte aligned; when `p` is given
// its workspace pointers are set from `base`.  Returns the number of floats.
size_t bwd_layout(long long BH, long long S, long long DH, long long NC, bool tc, float *base,
                  BwdPtrs *p) {
    const size_t ng = (size_t)(BH * S), nc = (size_t)(BH * NC), DD = (size_t)(DH * DH);
    const size_t xt = tc ? ng * DH : 0;
    const size_t sizes[] = {ng, ng, ng, ng, ng, ng, ng, ng,                 // per token
                            nc, nc, nc,                                     // per chunk
                            (size_t)BH * (NC + 1) * DD, (size_t)BH * (NC + 1) * DH,
                            ng * DH, tc ? 0 : ng * DH,                      // num', dnum' (fp32 kernels)
                            (size_t)BH * NC * DD, (size_t)BH * NC * DH,
                            xt, xt, xt,                                     // dnum' planes, dk / dv products
                            tc ? nc * 128 : 0, tc ? nc : 0};                // walk records, decays
    BwdPtrs unused;
    BwdPtrs *t = p ? p : &unused;
    float *dnhl = nullptr;
    float **dst[] = {&t->logf, &t->b, &t->mt, &t->den, &t->nq, &t->A, &t->dF, &t->dnq,
                     &t->mprev, &t->mend, &t->Bsum, &t->Cst, &t->nst, &t->num, &t->dnum,
                     &t->dCb, &t->dnb, &dnhl, &t->dki, &t->dvi, &t->wrec, &t->decay};
    static_assert(sizeof(sizes) / sizeof(sizes[0]) == sizeof(dst) / sizeof(dst[0]),
                  "one size per workspace array");
    size_t off = 0;
    for (size_t i = 0; i < sizeof(sizes) / sizeof(sizes[0]); ++i) {
        *dst[i] = base && sizes[i] ? base + off : nullptr;
        off = align64(off + sizes[i]);
    }
    t->dnhl = dnhl;
    t->tc = tc ? 1 : 0;
    return off;
}

// The backward runs on the tensor cores for bf16 inputs with DH 64, 128 or
// 256 (DH 64: one 128-row tile whose upper half is padding).
bool bwd_uses_tc(xlstm_dtype dt, int DH) { return dt == XLSTM_BF16 && (DH == 64 || DH == 128 || DH == 256); }

bool misaligned16(const void *p) { return ((uintptr_t)p & 15u) != 0; }

xlstm_status check_bwd_shape(int B, int NH, int S, int DH, int chunk, xlstm_dtype dt) {
    if (dt != XLSTM_F32 && dt != XLSTM_BF16) return XLSTM_ERR_DTYPE;
    if (B < 0 || NH < 0 || S < 0) return XLSTM_ERR_SHAPE;
    if (DH < 16 || DH > 512 || DH % 16 != 0) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH * S * DH > (1LL << 40)) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH > 0x7fffffffLL) return XLSTM_ERR_SHAPE;     // heads index an int
    if (chunk < 1 || chunk > bwd::kMaxChunk) return XLSTM_ERR_CHUNK;
    return XLSTM_OK;
}

unsigned blocks_for(long long n) { return (unsigned)((n + kThreads - 1) / kThreads); }

// One of the four state products (bwd_tc.cuh) for every chunk: `states` holds
// the planes of C' (NC + 1 slots per head) or dC~ (NC slots), `b` (and `b2`,
// the low plane, when B_SPLIT) the token rows, `out` [BH, S, D] fp32.
template <int D, bool A_T, bool B_SPLIT>
cudaError_t launch_state_mma_t(const BwdPtrs &p, const float *states, int slots_per_head, const void *b,
                               const void *b2, float *out, cudaStream_t st) {
    CUtensorMap m1, m2;
    if (!make_map_bf16(&m1, b, p.BH, p.S, D, true, 64)) return cudaErrorInvalidValue;
    if (!make_map_bf16(&m2, B_SPLIT ? b2 : b, p.BH, p.S, D, true, 64)) return cudaErrorInvalidValue;
    const size_t slot_bytes = (size_t)D * D * sizeof(float);
    const int sm = bwdtc::MmaLay<D, B_SPLIT>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(bwdtc::state_mma_kernel<D, A_T, B_SPLIT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    bwdtc::state_mma_kernel<D, A_T, B_SPLIT><<<dim3((unsigned)((long long)p.NC * p.BH), bwdtc::kTiles<D>),
                                               bwdtc::kMmaThreads, sm, st>>>(
        m1, m2, reinterpret_cast<const uint8_t *>(states), (size_t)slots_per_head * slot_bytes, slot_bytes, out,
        p.S, p.L, p.NC, device_status_ptr());
    return cudaGetLastError();
}

// which: 0 C' q (-> num), 1 C'^T dnum' (-> num), 2 dC~^T v (-> dki), 3 dC~ k (-> dvi)
template <int D>
cudaError_t launch_state_mma(const BwdPtrs &p, int which, cudaStream_t st) {
    const __nv_bfloat16 *dn_hi = reinterpret_cast<const __nv_bfloat16 *>(p.dnhl);
    switch (which) {
        case 0: return launch_state_mma_t<D, false, false>(p, p.Cst, p.NC + 1, p.q, nullptr, p.num, st);
        case 1: return launch_state_mma_t<D, true, true>(p, p.Cst, p.NC + 1, dn_hi,
                                                         dn_hi + (size_t)p.BH * p.S * D, p.num, st);
        case 2: return launch_state_mma_t<D, true, false>(p, p.dCb, p.NC, p.v, nullptr, p.dki, st);
        default: return launch_state_mma_t<D, false, false>(p, p.dCb, p.NC, p.k, nullptr, p.dvi, st);
    }
}

// The state recurrences on the tensor cores (bwd_tc.cuh): one walk over the
// chunks per (head, 128-row tile, 64-column block), writing every slot once.
template <int D, bool REVERSE>
cudaError_t launch_state_recurrence_t(const BwdPtrs &p, cudaStream_t st) {
    CUtensorMap ma, ma2, mb;
    const __nv_bfloat16 *dn_hi = reinterpret_cast<const __nv_bfloat16 *>(p.dnhl);
    const void *a1 = REVERSE ? (const void *)dn_hi : p.v;
    const void *a2 = REVERSE ? (const void *)(dn_hi + (size_t)p.BH * p.S * D) : p.v;
    if (!make_map_bf16(&ma, a1, p.BH, p.S, D, true, 64) || !make_map_bf16(&ma2, a2, p.BH, p.S, D, true, 64) ||
        !make_map_bf16(&mb, REVERSE ? p.q : p.k, p.BH, p.S, D, true, 64))
        return cudaErrorInvalidValue;
    const int sm = bwdtc::WalkLay<D, REVERSE>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(bwdtc::state_walk_kernel<D, REVERSE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    KernelTimer timer(REVERSE ? "bwd_reverse_walk" : "bwd_states_walk", st);
    const long long slots = (long long)p.BH * p.NC * 64;
    bwdtc::walk_weights_kernel<REVERSE><<<(unsigned)((slots + 255) / 256), 256, 0, st>>>(p);
    bwdtc::state_walk_kernel<D, REVERSE><<<dim3((unsigned)p.BH, bwdtc::kTiles<D>, D / 64), bwdtc::kWalkThreads, sm,
                                           st>>>(ma, ma2, mb, p, device_status_ptr());
    return cudaGetLastError();
}

cudaError_t launch_state_recurrence(const BwdPtrs &p, bool reverse, cudaStream_t st) {
    if (p.DH == 64)
        return reverse ? launch_state_recurrence_t<64, true>(p, st) : launch_state_recurrence_t<64, false>(p, st);
    if (p.DH == 128)
        return reverse ? launch_state_recurrence_t<128, true>(p, st) : launch_state_recurrence_t<128, false>(p, st);
    return reverse ? launch_state_recurrence_t<256, true>(p, st) : launch_state_recurrence_t<256, false>(p, st);
}

template <int D>
cudaError_t launch_token_fwd_tc_t(const BwdPtrs &p, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!make_map_bf16(&mq, p.q, p.BH, p.S, D, true, 64) || !make_map_bf16(&mk, p.k, p.BH, p.S, D, true, 64) ||
        !make_map_bf16(&mv, p.v, p.BH, p.S, D, true, 64))
        return cudaErrorInvalidValue;
    const int sm = bwdtc::TokLay<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(bwdtc::token_fwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    bwdtc::token_fwd_tc_kernel<D><<<(unsigned)((long long)p.NC * p.BH), bwdtc::kTokThreads, sm, st>>>(
        mq, mk, mv, p, device_status_ptr());
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_token_grad_tc_t(const BwdPtrs &p, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mdh, mdl;
    const __nv_bfloat16 *dn_hi = reinterpret_cast<const __nv_bfloat16 *>(p.dnhl);
    if (!make_map_bf16(&mq, p.q, p.BH, p.S, D, true, 64) || !make_map_bf16(&mk, p.k, p.BH, p.S, D, true, 64) ||
        !make_map_bf16(&mv, p.v, p.BH, p.S, D, true, 64) || !make_map_bf16(&mdh, dn_hi, p.BH, p.S, D, true, 64) ||
        !make_map_bf16(&mdl, dn_hi + (size_t)p.BH * p.S * D, p.BH, p.S, D, true, 64))
        return cudaErrorInvalidValue;
    const int sm = bwdtc::GradLay<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(bwdtc::token_grad_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    const long long items = (long long)p.NC * p.BH, sms = num_sms_current_device();
    bwdtc::token_grad_tc_kernel<D><<<(unsigned)(items < sms ? items : sms), bwdtc::kTokThreads, sm, st>>>(
        mq, mk, mv, mdh, mdl, p, device_status_ptr());
    return cudaGetLastError();
}

cudaError_t launch_state_products(const BwdPtrs &p, int which, cudaStream_t st) {
    KernelTimer timer("bwd_state_mma", st);
    return p.DH == 64    ? launch_state_mma<64>(p, which, st)
           : p.DH == 128 ? launch_state_mma<128>(p, which, st)
                         : launch_state_mma<256>(p, which, st);
}

template <typename T>
cudaError_t launch_bwd(const BwdPtrs &p, cudaStream_t st) {
    const long long heads = p.BH, rows = (long long)p.BH * (p.DH + 1),
                    tokens = (long long)p.BH * p.S;
    {
        KernelTimer timer("bwd_gates", st);
        bwd_gates_seq_kernel<<<(unsigned)heads, kSeqThreads, 0, st>>>(p);
    }
    cudaError_t e;
    if (p.tc) {
        if ((e = launch_state_recurrence(p, false, st)) != cudaSuccess) return e;
        if ((e = launch_state_products(p, 0, st)) != cudaSuccess) return e;
    } else {
        KernelTimer timer("bwd_states", st);
        if (!launch_rows<T, false>(p, st)) bwd_states_kernel<T><<<blocks_for(rows), kThreads, 0, st>>>(p);
    }
    if (p.tc) {
        KernelTimer timer("bwd_token_fwd_tc", st);
        e = p.DH == 64    ? launch_token_fwd_tc_t<64>(p, st)
            : p.DH == 128 ? launch_token_fwd_tc_t<128>(p, st)
                          : launch_token_fwd_tc_t<256>(p, st);
        if (e != cudaSuccess) return e;
    } else {
        KernelTimer timer("bwd_token_fwd", st);
        if (!launch_token_warp<T, false>(p, st))
            bwd_token_fwd_kernel<T><<<blocks_for(tokens), kThreads, 0, st>>>(p);
    }
    if (p.tc) {
        if ((e = launch_state_recurrence(p, true, st)) != cudaSuccess) return e;
        for (int which = 1; which <= 3; ++which)
            if ((e = launch_state_products(p, which, st)) != cudaSuccess) return e;
    } else {
        KernelTimer timer("bwd_reverse", st);
        if (!launch_rows<T, true>(p, st)) bwd_reverse_kernel<T><<<blocks_for(rows), kThreads, 0, st>>>(p);
    }
    if (p.tc) {
        KernelTimer timer("bwd_token_grad_tc", st);
        e = p.DH == 64    ? launch_token_grad_tc_t<64>(p, st)
            : p.DH == 128 ? launch_token_grad_tc_t<128>(p, st)
                          : launch_token_grad_tc_t<256>(p, st);
        if (e != cudaSuccess) return e;
    } else {
        KernelTimer timer("bwd_token_grad", st);
        if (!launch_token_warp<T, true>(p, st))
            bwd_token_grad_kernel<T><<<blocks_for(tokens), kThreads, 0, st>>>(p);
    }
    {
        KernelTimer timer("bwd_forget", st);
        if (p.dC || p.dn) bwd_final_state_kernel<<<(unsigned)((heads * 32 + 127) / 128), 128, 0, st>>>(p);
        bwd_forget_seq_kernel<<<(unsigned)heads, kSeqThreads, 0, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace
}  // namespace xlstm

using namespace xlstm;

extern "C" xlstm_status xlstm_mlstm_bwd_workspace_size(int B, int NH, int S, int DH, int chunk,
                                                       xlstm_dtype dt, size_t *bytes) {
    if (!bytes) return XLSTM_ERR_NULL;
    const xlstm_status st = check_bwd_shape(B, NH, S, DH, chunk, dt);
    if (st != XLSTM_OK) return st;
    const long long BH = (long long)B * NH;
    if (BH == 0 || S == 0) {
        *bytes = 0;
        return XLSTM_OK;
    }
    const long long NC = (S + chunk - 1) / chunk;
    *bytes = bwd_layout(BH, S, DH, NC, bwd_uses_tc(dt, DH), nullptr, nullptr) * sizeof(float);
    return XLSTM_OK;
}

extern "C" xlstm_status xlstm_mlstm_bwd(const void *q, const void *k, const void *v,
                                        const float *i_pre, const float *f_pre,
                                        const float *o_pre, const void *dh, const float *dC,
                                        const float *dn, void *dq, void *dk, void *dv,
                                        float *di, float *df, float *d_o, int B, int NH, int S,
                                        int DH, int chunk, xlstm_dtype dt, xlstm_fgate fg,
                                        void *workspace, size_t workspace_bytes,
                                        void *cuda_stream) {
    CallRange range("xlstm_mlstm_bwd");
    xlstm_status st = check_bwd_shape(B, NH, S, DH, chunk, dt);
    if (st != XLSTM_OK) return st;
    if (fg != XLSTM_FGATE_SIGMOID && fg != XLSTM_FGATE_EXP) return XLSTM_ERR_DTYPE;
    const long long BH = (long long)B * NH;
    if (BH == 0 || S == 0) return XLSTM_OK;
    const void *inputs[] = {q, k, v, i_pre, f_pre, o_pre, dh};
    const void *outputs[] = {dq, dk, dv, di, df, d_o};
    for (const void *p : inputs)
        if (!p) return XLSTM_ERR_NULL;
    for (const void *p : outputs)
        if (!p) return XLSTM_ERR_NULL;
    const void *all[] = {q, k, v, i_pre, f_pre, o_pre, dh, dC, dn, dq, dk, dv, di, df, d_o,
                         workspace};
    for (const void *p : all)
        if (misaligned16(p)) return XLSTM_ERR_ALIGN;
    for (const void *o : outputs) {
        for (const void *i : inputs)
            if (o == i) return XLSTM_ERR_UNSUPPORTED;
        if (o == (const void *)dC || o == (const void *)dn || o == workspace)
            return XLSTM_ERR_UNSUPPORTED;
    }
    for (int a = 0; a < 6; ++a)
        for (int b = a + 1; b < 6; ++b)
            if (outputs[a] == outputs[b]) return XLSTM_ERR_UNSUPPORTED;
    const long long NC = (S + chunk - 1) / chunk;
    const bool tc = bwd_uses_tc(dt, DH);
    const size_t need = bwd_layout(BH, S, DH, NC, tc, nullptr, nullptr) * sizeof(float);
    if (!workspace || workspace_bytes < need) return XLSTM_ERR_WORKSPACE;

    bwd::BwdPtrs p;
    p.q = q; p.k = k; p.v = v;
    p.ip = i_pre; p.fp = f_pre; p.op = o_pre; p.dh = dh;
    p.dC = dC; p.dn = dn;
    p.dq = dq; p.dk = dk; p.dv = dv; p.di = di; p.df = df; p.dO = d_o;
    bwd_layout(BH, S, DH, NC, tc, (float *)workspace, &p);
    p.BH = (int)BH; p.S = S; p.DH = DH; p.L = chunk; p.NC = (int)NC;
    p.fgate_exp = fg == XLSTM_FGATE_EXP;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    const cudaError_t e = dt == XLSTM_BF16 ? launch_bwd<__nv_bfloat16>(p, stream)
                                           : launch_bwd<float>(p, stream);
    return e == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}
