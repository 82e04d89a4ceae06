// Backward of the mLSTM cell: gradients with respect to q, k, v and the three
// gate pre-activations, fp32 arithmetic on CUDA cores ("xLSTM: Extended Long
// Short-Term Memory" section 2.3; the stabiliser held fixed as section 2.2
// allows).  Six launches, each a thin wrapper around a per-thread body in
// bwd_body.cuh (the algorithm is described there):
//   K1 bwd_gates       one thread per head     log f, chunk-local cumsum, m_t
//   K2 bwd_states      one thread per state row  chunk-start states C'_c, n'_c
//                      (DH a multiple of 32: one CTA per 32 rows, bwd_rows_kernel)
//   K3 bwd_token_fwd   one thread per token    num', nq', den', dotilde, dnum', dnq'
//   K4 bwd_reverse     one thread per state row  reverse state at each chunk end
//                      (DH a multiple of 32: one CTA per 32 rows, bwd_rows_kernel)
//   K5 bwd_token_grad  one thread per token    dq, dk, dv, ditilde
//   K6 bwd_forget      one thread per head     dftilde (reverse cumulative sum)
// The chunk-start and reverse states are materialised in the workspace
// (2 (NC + 1) DH^2 floats per head); this is the correctness-first form of the
// backward, not a tuned one.
#include <stdint.h>

#include "../../include/xlstm_mlstm.h"
#include "bwd_body.cuh"
#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace xlstm {
namespace {

using bwd::BwdPtrs;

constexpr int kThreads = 128;

__device__ __forceinline__ long long thread_index() {
    return (long long)blockIdx.x * blockDim.x + threadIdx.x;
}

__global__ void __launch_bounds__(kThreads) bwd_gates_kernel(BwdPtrs p) {
    const long long i = thread_index();
    if (i < p.BH) bwd::gates_head(p, (int)i);
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
size_t rows_smem_bytes(int L, int DH) { return (size_t)L * DH * sizeof(T) + (size_t)L * (kRowBlock + 1) * 4; }

template <typename T, int NCL, bool REVERSE>
__global__ void __launch_bounds__(kRowThreads) bwd_rows_kernel(BwdPtrs p) {
    constexpr int DH = 32 * NCL;
    extern __shared__ __align__(16) uint8_t rows_smem[];
    const int L = p.L, S = p.S, NC = p.NC;
    T *tile = reinterpret_cast<T *>(rows_smem);                           // [L][DH]
    float *coef = reinterpret_cast<float *>(rows_smem + (size_t)L * DH * sizeof(T));   // [L][32]
    float *wt = coef + (size_t)L * kRowBlock;                             // [L] per-token weight
    const int bh = blockIdx.y, r0 = blockIdx.x * kRowBlock;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t DD = (size_t)DH * DH;
    const float inv_sqrt = 1.f / sqrtf((float)DH);
    const T *src = (const T *)(REVERSE ? p.q : p.k);
    const T *v = (const T *)p.v;
    // this warp's rows r0 + 4 warp + i (row DH is the normaliser; rows past it unused)
    float st[4][NCL];
    auto slot_ptr = [&](int r, int slot) -> float * {
        if (r == DH) return (REVERSE ? p.dnb + (size_t)bh * NC * DH : p.nst + (size_t)bh * (NC + 1) * DH) +
                            (size_t)slot * DH;
        return (REVERSE ? p.dCb + (size_t)bh * NC * DD : p.Cst + (size_t)bh * (NC + 1) * DD) +
               (size_t)slot * DD + (size_t)r * DH;
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
            if (r <= DH) slot_ptr(r, REVERSE ? NC - 1 : 0)[col] = x;
        }
    }
    const int c_first = REVERSE ? NC - 1 : 0, c_end = REVERSE ? 0 : NC, dir = REVERSE ? -1 : 1;
    for (int c = c_first; c != c_end; c += dir) {
        const size_t hc = (size_t)bh * NC + c;
        const int a = c * L, n = bwd::imin(S, a + L) - a;
        __syncthreads();                       // the previous chunk's tile and coefficients are read
        for (int e = threadIdx.x; e < n * DH / 8; e += kRowThreads) {
            const int s = e / (DH / 8), part = e % (DH / 8);
            const size_t g = ((size_t)bh * S + a + s) * DH + part * 8;
            if (sizeof(T) == 2) {
                reinterpret_cast<uint4 *>(tile)[(size_t)s * DH / 8 + part] = *reinterpret_cast<const uint4 *>(src + g);
            } else {
                reinterpret_cast<uint4 *>(tile)[(size_t)s * DH / 4 + 2 * part] = *reinterpret_cast<const uint4 *>(src + g);
                reinterpret_cast<uint4 *>(tile)[(size_t)s * DH / 4 + 2 * part + 1] =
                    *reinterpret_cast<const uint4 *>(src + g + 4);
            }
        }
        const float mend = p.mend[hc], mprev = p.mprev[hc];
        for (int s = threadIdx.x; s < n; s += kRowThreads) {
            const size_t ts = (size_t)bh * S + a + s;
            wt[s] = REVERSE ? expf(p.b[ts] + mprev - p.mt[ts]) : expf(p.Bsum[hc] - p.b[ts] + p.ip[ts] - mend) * inv_sqrt;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < n * kRowBlock; e += kRowThreads) {
            const int s = e / kRowBlock, rr = e % kRowBlock, r = r0 + rr;
            const size_t ts = (size_t)bh * S + a + s;
            float x = 0.f;
            if (r < DH) x = REVERSE ? p.dnum[ts * DH + r] : bwd::ld(v, ts * DH + r);
            else if (r == DH) x = REVERSE ? p.dnq[ts] : 1.f;
            coef[s * kRowBlock + rr] = wt[s] * x;
        }
        __syncthreads();
        const float decay = expf(p.Bsum[hc] + mprev - mend);
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
            float *dst = slot_ptr(r, REVERSE ? c - 1 : c + 1);
#pragma unroll
            for (int j = 0; j < NCL; ++j) dst[lane + 32 * j] = st[i][j];
        }
    }
}

template <typename T, bool REVERSE>
bool launch_rows(const BwdPtrs &p, cudaStream_t st) {
    const int ncl = p.DH / 32;
    if (p.DH % 32 != 0 || (ncl != 1 && ncl != 2 && ncl != 4 && ncl != 8 && ncl != 16)) return false;
    const size_t sm = rows_smem_bytes<T>(p.L, p.DH);
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

__global__ void __launch_bounds__(kThreads) bwd_forget_kernel(BwdPtrs p) {
    const long long i = thread_index();
    if (i < p.BH) bwd::forget_head(p, (int)i);
}

size_t align64(size_t x) { return (x + 63) & ~size_t(63); }

// Workspace layout in floats, each array 256-byte aligned; when `p` is given
// its workspace pointers are set from `base`.  Returns the number of floats.
size_t bwd_layout(long long BH, long long S, long long DH, long long NC, float *base,
                  BwdPtrs *p) {
    const size_t ng = (size_t)(BH * S), nc = (size_t)(BH * NC), DD = (size_t)(DH * DH);
    const size_t sizes[] = {ng, ng, ng, ng, ng, ng, ng, ng,                 // per token
                            nc, nc, nc,                                     // per chunk
                            (size_t)BH * (NC + 1) * DD, (size_t)BH * (NC + 1) * DH,
                            ng * DH, ng * DH,                               // num', dnum'
                            (size_t)BH * NC * DD, (size_t)BH * NC * DH};
    BwdPtrs unused;
    BwdPtrs *t = p ? p : &unused;
    float **dst[] = {&t->logf, &t->b, &t->mt, &t->den, &t->nq, &t->A, &t->dF, &t->dnq,
                     &t->mprev, &t->mend, &t->Bsum, &t->Cst, &t->nst, &t->num, &t->dnum,
                     &t->dCb, &t->dnb};
    static_assert(sizeof(sizes) / sizeof(sizes[0]) == sizeof(dst) / sizeof(dst[0]),
                  "one size per workspace array");
    size_t off = 0;
    for (size_t i = 0; i < sizeof(sizes) / sizeof(sizes[0]); ++i) {
        *dst[i] = base ? base + off : nullptr;
        off = align64(off + sizes[i]);
    }
    return off;
}

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

template <typename T>
cudaError_t launch_bwd(const BwdPtrs &p, cudaStream_t st) {
    const long long heads = p.BH, rows = (long long)p.BH * (p.DH + 1),
                    tokens = (long long)p.BH * p.S;
    {
        KernelTimer timer("bwd_gates", st);
        bwd_gates_kernel<<<blocks_for(heads), kThreads, 0, st>>>(p);
    }
    {
        KernelTimer timer("bwd_states", st);
        if (!launch_rows<T, false>(p, st)) bwd_states_kernel<T><<<blocks_for(rows), kThreads, 0, st>>>(p);
    }
    {
        KernelTimer timer("bwd_token_fwd", st);
        bwd_token_fwd_kernel<T><<<blocks_for(tokens), kThreads, 0, st>>>(p);
    }
    {
        KernelTimer timer("bwd_reverse", st);
        if (!launch_rows<T, true>(p, st)) bwd_reverse_kernel<T><<<blocks_for(rows), kThreads, 0, st>>>(p);
    }
    {
        KernelTimer timer("bwd_token_grad", st);
        bwd_token_grad_kernel<T><<<blocks_for(tokens), kThreads, 0, st>>>(p);
    }
    {
        KernelTimer timer("bwd_forget", st);
        bwd_forget_kernel<<<blocks_for(heads), kThreads, 0, st>>>(p);
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
    *bytes = bwd_layout(BH, S, DH, NC, nullptr, nullptr) * sizeof(float);
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
    const size_t need = bwd_layout(BH, S, DH, NC, nullptr, nullptr) * sizeof(float);
    if (!workspace || workspace_bytes < need) return XLSTM_ERR_WORKSPACE;

    bwd::BwdPtrs p;
    p.q = q; p.k = k; p.v = v;
    p.ip = i_pre; p.fp = f_pre; p.op = o_pre; p.dh = dh;
    p.dC = dC; p.dn = dn;
    p.dq = dq; p.dk = dk; p.dv = dv; p.di = di; p.df = df; p.dO = d_o;
    bwd_layout(BH, S, DH, NC, (float *)workspace, &p);
    p.BH = (int)BH; p.S = S; p.DH = DH; p.L = chunk; p.NC = (int)NC;
    p.fgate_exp = fg == XLSTM_FGATE_EXP;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    const cudaError_t e = dt == XLSTM_BF16 ? launch_bwd<__nv_bfloat16>(p, stream)
                                           : launch_bwd<float>(p, stream);
    return e == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}
