// C ABI of the mLSTM library: argument validation, launch planning, dispatch.
// The operation and every argument are documented in include/xlstm_mlstm.h.
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "profile.h"

namespace xlstm {

__device__ unsigned int g_device_status = 0;

// Address of the device status word on the current device (nullptr on failure).
unsigned int *device_status_ptr() {
    unsigned int *p = nullptr;
    return cudaGetSymbolAddress((void **)&p, g_device_status) == cudaSuccess ? p : nullptr;
}

constexpr int kMaxHeads = 65535;           // B * NH rides in a grid dimension

// SM count of the current device, which the forward's segment plan fills one
// wave of.  Without a usable device (a host-only process asking for a
// workspace size) the plan is made for a full B200 (148 SMs).
int num_sms_current_device() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();   // a failed query must not leak into a later launch check
        return 148;
    }
    return n;
}

static size_t align64(size_t x) { return (x + 63) & ~size_t(63); }

bool make_fwd_plan(int B, int NH, int S, int DH, int L, int path, int forced_segments,
                   int num_sms, FwdPlan *p) {
    memset(p, 0, sizeof(*p));
    p->B = B; p->NH = NH; p->S = S; p->DH = DH; p->L = L;
    p->BH = B * NH;
    p->path = path;
    p->nchunks = S > 0 ? (S + L - 1) / L : 0;
    p->Spad = (S + 63) / 64 * 64;
    const bool tensor = path == XLSTM_PATH_TENSOR || path == XLSTM_PATH_TENSOR_TMEM || path == XLSTM_PATH_TENSOR_RS;
    if (tensor) {
        p->rows = DH < 128 ? DH : 128;
    } else {
        p->rows = DH < 32 ? DH : 32;
    }
    p->ntiles = (DH + p->rows - 1) / p->rows;
    if (p->nchunks == 0 || p->BH == 0) {
        p->P = 0; p->cps = 0;
        p->total_floats = 0;
        return true;
    }
    int P;
    // DH 512 on the tensor path splits each value tile's keys over two CTAs
    const int ksplit = tensor ? rs_key_splits(DH, L) : 1;
    const long per_set = (long)p->BH * p->ntiles * ksplit;
    if (forced_segments > 0) {
        P = forced_segments;
    } else if (tensor) {
        // one CTA per SM (shared memory and TMEM are sized for that): fill one wave
        P = (int)(num_sms / per_set);
    } else {
        const long target = 2L * num_sms;
        P = (int)((target + per_set - 1) / per_set);
    }
    if (P < 1) P = 1;
    if (tensor) {
        // the per-CTA chunk tables hold a bounded number of chunks
        const int cap = tensor_path_max_chunks_per_segment();
        const int need = (p->nchunks + cap - 1) / cap;
        if (P < need) P = need;
    }
    if (P > p->nchunks) P = p->nchunks;
    if (P > kMaxHeads) P = kMaxHeads;
    p->cps = (p->nchunks + P - 1) / P;
    p->P = (p->nchunks + p->cps - 1) / p->cps;
    layout_fwd_workspace(p);
    return true;
}

void layout_fwd_workspace(FwdPlan *p) {
    const int S = p->S, DH = p->DH;
    const bool tensor = p->path == XLSTM_PATH_TENSOR || p->path == XLSTM_PATH_TENSOR_TMEM ||
                        p->path == XLSTM_PATH_TENSOR_RS;
    const int ksplit = tensor ? rs_key_splits(DH, p->L) : 1;
    size_t off = 0;
    p->off_bcum = off;  off = align64(off + (size_t)p->BH * S);
    p->off_pmax = off;  off = align64(off + (size_t)p->BH * S);
    p->off_upad = off;  off = align64(off + (size_t)p->BH * p->Spad);
    p->off_bpad = off;  off = align64(off + (size_t)p->BH * p->Spad);
    p->off_xpad = off;  off = align64(off + (size_t)p->BH * p->Spad);
    p->off_cstat = off; off = align64(off + (size_t)p->BH * p->nchunks * 2);
    p->off_sstat = off; off = align64(off + (size_t)p->BH * p->P * 2);
    p->off_summ = off;  off = align64(off + (size_t)p->BH * (p->P - 1) * ((size_t)DH * DH + DH));
    if (ksplit > 1) {
        p->off_part = off;  off = align64(off + 2 * (size_t)p->BH * S * DH);
        p->off_dpart = off; off = align64(off + 2 * (size_t)p->BH * S);
        p->off_tok = off;   off = align64(off + 2 * (size_t)p->BH * S);
    }
    p->total_floats = off;
}

// Copies (or zero-fills) the initial state into the final-state outputs: the
// S == 0 forward.
__global__ void state_passthrough_kernel(const float *C0, const float *n0, const float *m0,
                                         float *C_out, float *n_out, float *m_out, int BH, int DH) {
    const size_t nC = (size_t)BH * DH * DH, nn = (size_t)BH * DH;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nC; i += stride) {
        if (C_out) C_out[i] = C0 ? C0[i] : 0.f;
        if (i < nn && n_out) n_out[i] = n0 ? n0[i] : 0.f;
        if (i < (size_t)BH && m_out) m_out[i] = m0 ? m0[i] : 0.f;
    }
}

cudaError_t launch_state_passthrough(const FwdArgs &a, int BH, int DH, cudaStream_t st) {
    if (!a.C_out && !a.n_out && !a.m_out) return cudaSuccess;
    KernelTimer timer("state_passthrough", st);
    state_passthrough_kernel<<<4 * num_sms_current_device(), 256, 0, st>>>(a.C0, a.n0, a.m0, a.C_out, a.n_out,
                                                          a.m_out, BH, DH);
    return cudaGetLastError();
}

}  // namespace xlstm

using namespace xlstm;

static bool misaligned(const void *p) { return ((uintptr_t)p & 15u) != 0; }

static xlstm_status check_fwd_shape(int B, int NH, int S, int DH, int chunk, xlstm_dtype dt) {
    if (dt != XLSTM_F32 && dt != XLSTM_BF16) return XLSTM_ERR_DTYPE;
    if (B < 0 || NH < 0 || S < 0) return XLSTM_ERR_SHAPE;
    if (DH < 16 || DH > 512 || DH % 16 != 0) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH > kMaxHeads) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH * S * DH > (1LL << 40)) return XLSTM_ERR_SHAPE;
    if (dt == XLSTM_BF16) {
        if (chunk != 64 && chunk != 128 && chunk != 256) return XLSTM_ERR_CHUNK;
    } else {
        if (chunk < 1 || chunk > 1024) return XLSTM_ERR_CHUNK;
    }
    return XLSTM_OK;
}

static bool any_tensor_path(int DH, int chunk) {
    return rs_path_supports(DH, chunk) || tensor_path_supports(DH, chunk);
}

static int resolve_path(xlstm_dtype dt, int DH, int chunk, const xlstm_fwd_options *opts,
                        xlstm_status *st) {
    *st = XLSTM_OK;
    const int want = opts ? opts->path : XLSTM_PATH_AUTO;
    if (want == XLSTM_PATH_SIMT) return XLSTM_PATH_SIMT;
    if (want == XLSTM_PATH_TENSOR || want == XLSTM_PATH_TENSOR_TMEM || want == XLSTM_PATH_TENSOR_RS) {
        const bool ok = dt == XLSTM_BF16 && (want == XLSTM_PATH_TENSOR      ? any_tensor_path(DH, chunk)
                                             : want == XLSTM_PATH_TENSOR_RS ? rs_path_supports(DH, chunk)
                                                                            : tensor_path_supports(DH, chunk));
        if (!ok) {
            *st = XLSTM_ERR_UNSUPPORTED;
            return 0;
        }
        return want;
    }
    if (want != XLSTM_PATH_AUTO) {
        *st = XLSTM_ERR_UNSUPPORTED;
        return 0;
    }
    if (dt == XLSTM_BF16 && any_tensor_path(DH, chunk)) return XLSTM_PATH_TENSOR;
    return XLSTM_PATH_SIMT;
}

extern "C" {

int xlstm_abi_version(void) { return XLSTM_ABI_VERSION; }

const char *xlstm_status_string(xlstm_status s) {
    switch (s) {
        case XLSTM_OK: return "ok";
        case XLSTM_ERR_NULL: return "a required pointer is NULL";
        case XLSTM_ERR_SHAPE: return "unsupported or inconsistent shape";
        case XLSTM_ERR_DTYPE: return "unsupported dtype or gate kind";
        case XLSTM_ERR_CHUNK: return "unsupported chunk size for this dtype";
        case XLSTM_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case XLSTM_ERR_CUDA: return "CUDA runtime or launch error";
        case XLSTM_ERR_TIMEOUT: return "a bounded device-side wait ran out";
        case XLSTM_ERR_WORKSPACE: return "workspace missing or too small";
        case XLSTM_ERR_UNSUPPORTED: return "unsupported option combination";
    }
    return "unknown status";
}

xlstm_status xlstm_mlstm_fwd_workspace_size_ex(int B, int NH, int S, int DH, int chunk,
                                               xlstm_dtype dt, const xlstm_fwd_options *opts,
                                               size_t *bytes) {
    if (!bytes) return XLSTM_ERR_NULL;
    xlstm_status st = check_fwd_shape(B, NH, S, DH, chunk, dt);
    if (st != XLSTM_OK) return st;
    const int path = resolve_path(dt, DH, chunk, opts, &st);
    if (st != XLSTM_OK) return st;
    FwdPlan p;
    if (!make_fwd_plan(B, NH, S, DH, chunk, path, opts ? opts->segments : 0, num_sms_current_device(), &p))
        return XLSTM_ERR_SHAPE;
    *bytes = p.bytes();
    return XLSTM_OK;
}

xlstm_status xlstm_mlstm_fwd_path(int DH, int chunk, xlstm_dtype dt, const xlstm_fwd_options *opts,
                                  int *path) {
    if (!path) return XLSTM_ERR_NULL;
    xlstm_status st = check_fwd_shape(1, 1, 1, DH, chunk, dt);
    if (st != XLSTM_OK) return st;
    if (opts && opts->segments < 0) return XLSTM_ERR_UNSUPPORTED;
    const int p = resolve_path(dt, DH, chunk, opts, &st);
    if (st != XLSTM_OK) return st;
    *path = p;
    return XLSTM_OK;
}

xlstm_status xlstm_mlstm_fwd_workspace_size(int B, int NH, int S, int DH, int chunk,
                                            xlstm_dtype dt, size_t *bytes) {
    return xlstm_mlstm_fwd_workspace_size_ex(B, NH, S, DH, chunk, dt, nullptr, bytes);
}

xlstm_status xlstm_mlstm_fwd_ex(const void *q, const void *k, const void *v,
                                const float *i_pre, const float *f_pre, const float *o_pre,
                                void *h, const float *C0, const float *n0, const float *m0,
                                float *C_out, float *n_out, float *m_out,
                                int B, int NH, int S, int DH, int chunk,
                                xlstm_dtype dt, xlstm_fgate fg,
                                void *workspace, size_t workspace_bytes,
                                const xlstm_fwd_options *opts, void *cuda_stream) {
    CallRange range("xlstm_mlstm_fwd");
    xlstm_status st = check_fwd_shape(B, NH, S, DH, chunk, dt);
    if (st != XLSTM_OK) return st;
    if (fg != XLSTM_FGATE_SIGMOID && fg != XLSTM_FGATE_EXP) return XLSTM_ERR_DTYPE;
    if (opts && opts->segments < 0) return XLSTM_ERR_UNSUPPORTED;
    const int path = resolve_path(dt, DH, chunk, opts, &st);
    if (st != XLSTM_OK) return st;
    if ((long long)B * NH == 0) return XLSTM_OK;
    if (S > 0 && (!q || !k || !v || !i_pre || !f_pre || !o_pre || !h)) return XLSTM_ERR_NULL;
    const void *ptrs[] = {q, k, v, i_pre, f_pre, o_pre, h, C0, n0, m0, C_out, n_out, m_out, workspace};
    for (const void *p : ptrs)
        if (misaligned(p)) return XLSTM_ERR_ALIGN;

    if ((C_out && C_out == C0) || (n_out && n_out == n0) || (m_out && m_out == m0))
        return XLSTM_ERR_UNSUPPORTED;
    FwdPlan plan;
    if (!make_fwd_plan(B, NH, S, DH, chunk, path, opts ? opts->segments : 0, num_sms_current_device(), &plan))
        return XLSTM_ERR_SHAPE;
    if (plan.bytes() > 0 && (!workspace || workspace_bytes < plan.bytes())) return XLSTM_ERR_WORKSPACE;

    FwdArgs a;
    a.q = q; a.k = k; a.v = v; a.i_pre = i_pre; a.f_pre = f_pre; a.o_pre = o_pre; a.h = h;
    a.C0 = C0; a.n0 = n0; a.m0 = m0; a.C_out = C_out; a.n_out = n_out; a.m_out = m_out;
    a.workspace = workspace;
    a.status = nullptr;
    if (cudaGetSymbolAddress((void **)&a.status, g_device_status) != cudaSuccess) return XLSTM_ERR_CUDA;
    a.bf16 = dt == XLSTM_BF16;
    a.fgate_exp = fg == XLSTM_FGATE_EXP;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    cudaError_t e;
    if (S == 0) {
        e = launch_state_passthrough(a, plan.BH, DH, stream);
    } else if (path == XLSTM_PATH_TENSOR_RS ||
               (path == XLSTM_PATH_TENSOR && !tensor_path_supports(DH, chunk))) {
        // the register-state kernels: where the tensor-memory-state kernel does not
        // apply (DH 64), or when asked for
        e = launch_fwd_rs(a, plan, stream);
    } else if (path == XLSTM_PATH_TENSOR || path == XLSTM_PATH_TENSOR_TMEM) {
        // measured faster at DH 128 / 256 with chunk 64 (the long workload)
        e = launch_fwd_tensor(a, plan, stream);
    } else {
        e = launch_fwd_simt(a, plan, stream);
    }
    return e == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

xlstm_status xlstm_mlstm_fwd(const void *q, const void *k, const void *v,
                             const float *i_pre, const float *f_pre, const float *o_pre,
                             void *h, const float *C0, const float *n0, const float *m0,
                             float *C_out, float *n_out, float *m_out,
                             int B, int NH, int S, int DH, int chunk,
                             xlstm_dtype dt, xlstm_fgate fg,
                             void *workspace, size_t workspace_bytes, void *cuda_stream) {
    return xlstm_mlstm_fwd_ex(q, k, v, i_pre, f_pre, o_pre, h, C0, n0, m0, C_out, n_out, m_out,
                              B, NH, S, DH, chunk, dt, fg, workspace, workspace_bytes, nullptr,
                              cuda_stream);
}

// ---------------------------------------------------------- sequence parallelism
static size_t seg_state_floats(long long BH, int DH) {
    const size_t n = (size_t)BH * ((size_t)DH * DH + DH + 2);
    return (n + 3) & ~size_t(3);
}

static xlstm_status check_state_shape(int B, int NH, int DH) {
    if (B < 0 || NH < 0) return XLSTM_ERR_SHAPE;
    if (DH < 16 || DH > 512 || DH % 16 != 0) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH > kMaxHeads) return XLSTM_ERR_SHAPE;
    return XLSTM_OK;
}

// The segment-state pass reuses the forward's segmentation and summary kernels
// with every segment summarised (the forward leaves the last one to its output
// kernel), then folds the summaries; a BH-float buffer after the forward's
// layout holds the fold's starting stabiliser for the in-place scan.
static xlstm_status make_seg_state_plan(int B, int NH, int S, int DH, int chunk, xlstm_dtype dt,
                                        FwdPlan *p, size_t *off_mstart, size_t *total_floats) {
    xlstm_status st;
    const int path = resolve_path(dt, DH, chunk, nullptr, &st);
    if (st != XLSTM_OK) return st;
    if (!make_fwd_plan(B, NH, S, DH, chunk, path, 0, num_sms_current_device(), p)) return XLSTM_ERR_SHAPE;
    if (p->P == 0) {
        *off_mstart = 0;
        *total_floats = 0;
        return XLSTM_OK;
    }
    p->P += 1;
    layout_fwd_workspace(p);
    *off_mstart = p->total_floats;
    *total_floats = align64(p->total_floats + (size_t)p->BH);
    return XLSTM_OK;
}

xlstm_status xlstm_mlstm_seg_state_floats(int B, int NH, int DH, size_t *floats) {
    if (!floats) return XLSTM_ERR_NULL;
    xlstm_status st = check_state_shape(B, NH, DH);
    if (st != XLSTM_OK) return st;
    *floats = seg_state_floats((long long)B * NH, DH);
    return XLSTM_OK;
}

xlstm_status xlstm_mlstm_seg_state_workspace_size(int B, int NH, int S, int DH, int chunk,
                                                  xlstm_dtype dt, size_t *bytes) {
    if (!bytes) return XLSTM_ERR_NULL;
    xlstm_status st = check_fwd_shape(B, NH, S, DH, chunk, dt);
    if (st != XLSTM_OK) return st;
    FwdPlan p;
    size_t off_m, total;
    st = make_seg_state_plan(B, NH, S, DH, chunk, dt, &p, &off_m, &total);
    if (st != XLSTM_OK) return st;
    *bytes = total * sizeof(float);
    return XLSTM_OK;
}

xlstm_status xlstm_mlstm_seg_state(const void *k, const void *v, const float *i_pre, const float *f_pre,
                                   float *packed, int B, int NH, int S, int DH, int chunk,
                                   xlstm_dtype dt, xlstm_fgate fg, void *workspace,
                                   size_t workspace_bytes, void *cuda_stream) {
    CallRange range("xlstm_mlstm_seg_state");
    xlstm_status st = check_fwd_shape(B, NH, S, DH, chunk, dt);
    if (st != XLSTM_OK) return st;
    if (fg != XLSTM_FGATE_SIGMOID && fg != XLSTM_FGATE_EXP) return XLSTM_ERR_DTYPE;
    const int BH = B * NH;
    if (BH == 0) return XLSTM_OK;
    if (!packed) return XLSTM_ERR_NULL;
    if (S > 0 && (!k || !v || !i_pre || !f_pre)) return XLSTM_ERR_NULL;
    const void *ptrs[] = {k, v, i_pre, f_pre, packed, workspace};
    for (const void *p : ptrs)
        if (misaligned(p)) return XLSTM_ERR_ALIGN;
    FwdPlan plan;
    size_t off_m, total;
    st = make_seg_state_plan(B, NH, S, DH, chunk, dt, &plan, &off_m, &total);
    if (st != XLSTM_OK) return st;
    if (total > 0 && (!workspace || workspace_bytes < total * sizeof(float))) return XLSTM_ERR_WORKSPACE;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    float *Cp = packed, *np = packed + (size_t)BH * DH * DH, *mp = np + (size_t)BH * DH, *Fp = mp + BH;
    FoldSource src = {};
    if (S == 0) {
        // an empty run: zero state, stabiliser -inf, no forgetting
        return launch_state_fold(src, 0, 0, nullptr, nullptr, nullptr, 1, Cp, np, mp, Fp, BH, DH, stream) ==
                       cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
    }
    FwdArgs a = {};
    a.k = k; a.v = v; a.i_pre = i_pre; a.f_pre = f_pre;
    a.workspace = workspace;
    if (cudaGetSymbolAddress((void **)&a.status, g_device_status) != cudaSuccess) return XLSTM_ERR_CUDA;
    a.bf16 = dt == XLSTM_BF16;
    a.fgate_exp = fg == XLSTM_FGATE_EXP;
    float *ws = (float *)workspace;
    const bool tensor = plan.path != XLSTM_PATH_SIMT;
    cudaError_t e = cudaSuccess;
    if (tensor && plan.Spad > S) {
        // the tensor-core summaries fetch 64-token tiles of log i - b; past the
        // end of the run every byte 0xFE (-1.7e38) makes the token's weight 0
        e = cudaMemset2DAsync(ws + plan.off_upad + S, (size_t)plan.Spad * sizeof(float), 0xFE,
                              (size_t)(plan.Spad - S) * sizeof(float), BH, stream);
        if (e != cudaSuccess) return XLSTM_ERR_CUDA;
    }
    if ((e = launch_gate_prologue(a, plan, stream)) != cudaSuccess) return XLSTM_ERR_CUDA;
    if (tensor) {
        // summaries + the in-place segment scan, started from stabiliser -1.7e38
        // (bytes 0xFE): the same fold as from -inf for any finite statistics
        float *mstart = ws + off_m;
        if (cudaMemsetAsync(mstart, 0xFE, (size_t)BH * sizeof(float), stream) != cudaSuccess)
            return XLSTM_ERR_CUDA;
        a.m0 = mstart;
        e = launch_segment_summaries(a, plan, stream);
    } else {
        e = launch_segment_summaries_simt(a, plan, stream);
    }
    if (e != cudaSuccess) return XLSTM_ERR_CUDA;
    const size_t per = (size_t)DH * DH + DH;
    float *summ = ws + plan.off_summ;
    const float *sst = ws + plan.off_sstat;
    src.C = summ;
    src.n = summ + (size_t)DH * DH;
    src.F = sst;
    src.m = sst + 1;
    src.cg = src.ng = per;
    src.cbh = src.nbh = (size_t)(plan.P - 1) * per;
    src.sg = 2;
    src.sbh = 2 * (size_t)plan.P;
    e = launch_state_fold(src, plan.P - 1, tensor ? 1 : 0, nullptr, nullptr, nullptr, 1, Cp, np, mp, Fp, BH, DH,
                          stream);
    return e == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

xlstm_status xlstm_mlstm_state_combine(const float *parts, int count, const float *C0, const float *n0,
                                       const float *m0, float *C_out, float *n_out, float *m_out,
                                       int B, int NH, int DH, void *cuda_stream) {
    CallRange range("xlstm_mlstm_state_combine");
    xlstm_status st = check_state_shape(B, NH, DH);
    if (st != XLSTM_OK) return st;
    if (count < 0) return XLSTM_ERR_SHAPE;
    const int BH = B * NH;
    if (BH == 0) return XLSTM_OK;
    if (!C_out || !n_out || !m_out || (count > 0 && !parts)) return XLSTM_ERR_NULL;
    const void *ptrs[] = {parts, C0, n0, m0, C_out, n_out, m_out};
    for (const void *p : ptrs)
        if (misaligned(p)) return XLSTM_ERR_ALIGN;
    if ((C0 && C_out == C0) || (n0 && n_out == n0) || (m0 && m_out == m0)) return XLSTM_ERR_UNSUPPORTED;
    const size_t packed = seg_state_floats(BH, DH);
    FoldSource src = {};
    src.C = parts;
    src.n = parts ? parts + (size_t)BH * DH * DH : nullptr;
    src.m = parts ? src.n + (size_t)BH * DH : nullptr;
    src.F = parts ? src.m + BH : nullptr;
    src.cg = src.ng = src.sg = packed;
    src.cbh = (size_t)DH * DH;
    src.nbh = DH;
    src.sbh = 1;
    return launch_state_fold(src, count, 0, C0, n0, m0, 0, C_out, n_out, m_out, nullptr, BH, DH,
                             (cudaStream_t)cuda_stream) == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

xlstm_status xlstm_mlstm_step(const void *q, const void *k, const void *v,
                              const float *i_pre, const float *f_pre, const float *o_pre,
                              void *h, float *C, float *n, float *m,
                              int B, int NH, int DH, xlstm_dtype dt, xlstm_fgate fg,
                              void *cuda_stream) {
    CallRange range("xlstm_mlstm_step");
    if (dt != XLSTM_F32 && dt != XLSTM_BF16) return XLSTM_ERR_DTYPE;
    if (fg != XLSTM_FGATE_SIGMOID && fg != XLSTM_FGATE_EXP) return XLSTM_ERR_DTYPE;
    if (B < 0 || NH < 0 || DH < 16 || DH > 512 || DH % 16 != 0) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH > kMaxHeads) return XLSTM_ERR_SHAPE;
    if ((long long)B * NH == 0) return XLSTM_OK;
    if (!q || !k || !v || !i_pre || !f_pre || !o_pre || !h || !C || !n || !m) return XLSTM_ERR_NULL;
    const void *ptrs[] = {q, k, v, i_pre, f_pre, o_pre, h, C, n, m};
    for (const void *p : ptrs)
        if (misaligned(p)) return XLSTM_ERR_ALIGN;
    StepArgs a;
    a.q = q; a.k = k; a.v = v; a.i_pre = i_pre; a.f_pre = f_pre; a.o_pre = o_pre; a.h = h;
    a.C = C; a.n = n; a.m = m;
    a.BH = B * NH; a.DH = DH;
    a.bf16 = dt == XLSTM_BF16;
    a.fgate_exp = fg == XLSTM_FGATE_EXP;
    a.status = nullptr;
    if (cudaGetSymbolAddress((void **)&a.status, g_device_status) != cudaSuccess) return XLSTM_ERR_CUDA;
    return launch_step(a, (cudaStream_t)cuda_stream) == cudaSuccess ? XLSTM_OK : XLSTM_ERR_CUDA;
}

xlstm_status xlstm_device_status(void *cuda_stream) {
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return XLSTM_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_device_status, sizeof(word)) != cudaSuccess) return XLSTM_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess)
        return XLSTM_ERR_CUDA;
    return word ? XLSTM_ERR_TIMEOUT : XLSTM_OK;
}

}  // extern "C"
