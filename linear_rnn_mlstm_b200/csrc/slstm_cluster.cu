// sLSTM forward on a cluster of CTAs per (batch, head), for DH 64, 128, 256 or 512
// ("xLSTM: Extended Long Short-Term Memory" section 2.2: scalar memory cells
// with exponential gating and memory mixing through recurrent connections
// within a head; the per-unit step is the one written out in slstm_body.cuh).
//
// The recurrence is sequential in t and each step needs the four DH x DH
// recurrent blocks of the head against h_{t-1}.  Here those blocks stay in
// registers for the whole sequence: the head's DH units are split over
// DH / 32 CTAs of one cluster, 32 units per CTA, four units per warp; a warp
// holds the 16 rows (4 units x 4 gates) of its units, each lane the columns
// lane + 32 k (128 floats per lane at DH 256).  Per step a warp forms 16
// partial dot products per lane, sums them across the warp with a halving
// butterfly (16 shuffles leave each lane pair with one row's total), gathers a
// unit's four gates into one lane, updates (c, n, m) there, and writes h_t[j]
// into every CTA's copy of h by distributed shared memory; one cluster barrier
// per step orders those writes before the next step reads them.  The gate
// pre-activations of 16 steps at a time reach shared memory by TMA (one
// 32-unit x 16-step box per gate) through a 4-stage ring.
#include <cuda.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "slstm_body.cuh"
#include "tc_ptx.cuh"

namespace xlstm {
namespace {

constexpr int kClThreads = 256;      // 8 warps x 4 units
constexpr int kClSteps = 16;         // steps per input stage
constexpr int kClStages = 4;

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Store to the same shared-memory variable in CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster(float *local, uint32_t rank, float v) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(tc::smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

// Columns per lane held in registers; at DH 512 (a 16-CTA cluster) the other
// eight per lane live in shared memory (128 KB per CTA), laid out so that a
// lane reads only its own words: [warp][row][column - 8][lane].
template <int DH> struct ClSplit {
    static constexpr int NC = DH / 32;                  // columns per lane
    static constexpr int NREG = NC < 8 ? NC : 8;
    static constexpr int NSM = NC - NREG;
    static constexpr size_t kSmem = (size_t)(kClThreads / 32) * 16 * NSM * 32 * 4;
};

template <int DH>
__global__ void __launch_bounds__(kClThreads, 1)
slstm_cluster_kernel(const __grid_constant__ CUtensorMap map_z, const __grid_constant__ CUtensorMap map_i,
                     const __grid_constant__ CUtensorMap map_f, const __grid_constant__ CUtensorMap map_o,
                     const __grid_constant__ CUtensorMap map_h, slstm::SlstmPtrs p, unsigned int *status) {
    constexpr int CS = DH / 32;                  // CTAs per cluster
    constexpr int NC = DH / 32;                  // columns per lane
    constexpr int NREG = ClSplit<DH>::NREG, NSM = ClSplit<DH>::NSM;
    extern __shared__ __align__(16) float rsm[];   // [8 warps][16 rows][NSM][32 lanes]
    __shared__ __align__(128) float pre[kClStages][4][kClSteps][32];   // gate pre-activations
    __shared__ __align__(16) float hbuf[2][DH];                       // h_{t-1} / h_t of the whole head
    // this CTA's h of a 16-step block, sent out by one TMA store per block (a
    // per-step global store would sit inside every step's release)
    __shared__ __align__(128) float hst[2][kClSteps][32];
    __shared__ __align__(8) uint64_t full[kClStages];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int bh = blockIdx.x / CS, head = bh % p.NH;
    const int S = p.S;
    const int ul = 4 * warp + (lane >> 3);       // this lane's unit within the CTA (lanes 8u..8u+7)
    const int j = (int)rank * 32 + ul;           // ... within the head
    const bool unit_lane = (lane & 7) == 0;
    const int nblk = (S + kClSteps - 1) / kClSteps;

    // the warp's 16 rows (row r = 4 u + g: unit 4 warp + u, gate g in z, i, f, o)
    float Rr[16][NREG];
    float *Rs = rsm + (size_t)warp * 16 * NSM * 32;
    {
        const size_t DD = (size_t)DH * DH;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int jr = (int)rank * 32 + 4 * warp + (r >> 2);
            const float *row = p.R + ((size_t)head * 4 + (r & 3)) * DD + (size_t)jr * DH;
#pragma unroll
            for (int k = 0; k < NREG; ++k) Rr[r][k] = __ldg(row + lane + 32 * k);
#pragma unroll
            for (int k = 0; k < NSM; ++k) Rs[(r * NSM + k) * 32 + lane] = __ldg(row + lane + 32 * (NREG + k));
        }
    }
    float c = 0.f, n = 0.f, m = 0.f;
    if (unit_lane) {
        const size_t s0 = (size_t)bh * DH + j;
        c = p.c0 ? p.c0[s0] : 0.f;
        n = p.n0 ? p.n0[s0] : 0.f;
        m = p.m0 ? p.m0[s0] : 0.f;
    }
    for (int e = threadIdx.x; e < DH; e += kClThreads) hbuf[0][e] = p.h0 ? p.h0[(size_t)bh * DH + e] : 0.f;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kClStages; ++s) tc::mbar_init(&full[s], 1);
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    auto load_block = [&](int blk) {             // thread 0: steps [16 blk, 16 blk + 16) of the 4 gates
        const int s = blk % kClStages;
        tc::mbar_arrive_expect_tx(&full[s], 4 * kClSteps * 32 * 4);
        tc::tma_load_3d(&pre[s][0][0][0], &map_z, &full[s], (int)rank * 32, blk * kClSteps, bh);
        tc::tma_load_3d(&pre[s][1][0][0], &map_i, &full[s], (int)rank * 32, blk * kClSteps, bh);
        tc::tma_load_3d(&pre[s][2][0][0], &map_f, &full[s], (int)rank * 32, blk * kClSteps, bh);
        tc::tma_load_3d(&pre[s][3][0][0], &map_o, &full[s], (int)rank * 32, blk * kClSteps, bh);
    };
    int issued = 0;
    if (threadIdx.x == 0) {
        for (; issued < min(nblk, kClStages - 1); ++issued) load_block(issued);
    }
    cluster_sync_all();                          // every CTA's h copy initialised before any remote write

    bool ok = true;
    for (int t = 0; t < S; ++t) {
        const int blk = t / kClSteps, tin = t % kClSteps, s = blk % kClStages;
        if (tin == 0) {
            // the stage refilled here held block blk - 1, which every thread
            // finished before the cluster barrier that ended step t - 1
            if (threadIdx.x == 0 && issued < nblk && issued == blk + kClStages - 1) load_block(issued++);
            if (blk >= 2) {                      // block blk - 2's h store has read hst[blk & 1]
                if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                __syncthreads();
            }
            bool got = true;
            if (lane == 0) got = tc::mbar_wait(&full[s], (blk / kClStages) & 1, &abort_flag, status);
            got = __shfl_sync(0xffffffffu, got, 0);
            if (!__all_sync(0xffffffffu, got)) ok = false;
        }
        // a warp that gave up still takes every barrier below, so the cluster
        // never waits on it; its results are discarded with the status latched
        const float *hp = hbuf[t & 1];
        float hc[NC];
#pragma unroll
        for (int k = 0; k < NC; ++k) hc[k] = hp[lane + 32 * k];
        float v[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float a = 0.f;
#pragma unroll
            for (int k = 0; k < NREG; ++k) a = fmaf(Rr[r][k], hc[k], a);
#pragma unroll
            for (int k = 0; k < NSM; ++k) a = fmaf(Rs[(r * NSM + k) * 32 + lane], hc[NREG + k], a);
            v[r] = a;
        }
        // halving butterfly: after it lanes 2r and 2r + 1 hold row r's total
#pragma unroll
        for (int w = 16, half = 8; w >= 2; w >>= 1, half >>= 1) {
            const bool upper = (lane & w) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = upper ? v[i] : v[i + half];
                const float keep = upper ? v[i + half] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
            }
        }
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
        // gates of unit u sit in lanes 8u (z), 8u + 2 (i), 8u + 4 (f), 8u + 6 (o)
        const int base = lane & ~7;
        const float ri = __shfl_sync(0xffffffffu, v[0], base + 2);
        const float rf = __shfl_sync(0xffffffffu, v[0], base + 4);
        const float ro = __shfl_sync(0xffffffffu, v[0], base + 6);
        if (unit_lane) {
            const float zt = pre[s][0][tin][ul] + v[0];
            const float it = pre[s][1][tin][ul] + ri;
            const float ft = pre[s][2][tin][ul] + rf;
            const float ot = pre[s][3][tin][ul] + ro;
            const float zz = tanhf(zt);
            const float log_f = p.fgate_exp ? ft : slstm::log_sigmoid_hd(ft);
            const float o = slstm::sigmoid_hd(ot);
            const float m_new = fmaxf(log_f + m, it);
            const float fg = expf(log_f + m - m_new);
            const float ig = expf(it - m_new);
            m = m_new;
            c = fg * c + ig * zz;
            n = fg * n + ig;
            const float h = o * c / n;
            hst[blk & 1][tin][ul] = h;
            float *dst = &hbuf[(t + 1) & 1][j];
#pragma unroll
            for (int r2 = 0; r2 < CS; ++r2) st_cluster(dst, (uint32_t)r2, h);
        }
        if (tin == kClSteps - 1 || t == S - 1) tc::fence_async_smem();   // hst visible to the TMA store
        cluster_sync_all();                      // h_t complete in every CTA
        if (threadIdx.x == 0 && (tin == kClSteps - 1 || t == S - 1)) {
            tc::tma_store_3d(&map_h, &hst[blk & 1][0][0], (int)rank * 32, blk * kClSteps, bh);
            tc::bulk_commit();
        }
    }
    if (!ok && lane == 0 && warp == 0) atomicOr(status, kStatusTimeout);
    if (unit_lane) {
        const size_t s0 = (size_t)bh * DH + j;
        if (p.c_out) p.c_out[s0] = c;
        if (p.n_out) p.n_out[s0] = n;
        if (p.m_out) p.m_out[s0] = m;
        if (p.h_out) p.h_out[s0] = hbuf[S & 1][j];
    }
    if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // h written
    if (threadIdx.x == 0) {                      // never leave a load in flight into shared memory
        for (int b = max(0, issued - kClStages); b < issued; ++b)
            tc::mbar_wait(&full[b % kClStages], (b / kClStages) & 1, nullptr, status, 200000000ull);
    }
    cluster_sync_all();                          // no CTA leaves while a peer may still read its memory
}

template <int DH>
cudaError_t launch_cluster_t(const slstm::SlstmPtrs &p, cudaStream_t st) {
    CUtensorMap mz, mi, mf, mo;
    const unsigned long long dims[3] = {(unsigned long long)DH, (unsigned long long)p.S, (unsigned long long)p.BH};
    const unsigned long long strides[2] = {(unsigned long long)DH * 4, (unsigned long long)p.S * DH * 4};
    const unsigned box[3] = {32u, (unsigned)kClSteps, 1u};
    CUtensorMap mh;
    if (p.S > 0 && (!make_tensor_map_3d(&mh, p.h, 4, dims, strides, box) ||
                    !make_tensor_map_3d(&mz, p.zx, 4, dims, strides, box) ||
                    !make_tensor_map_3d(&mi, p.ix, 4, dims, strides, box) ||
                    !make_tensor_map_3d(&mf, p.fx, 4, dims, strides, box) ||
                    !make_tensor_map_3d(&mo, p.ox, 4, dims, strides, box)))
        return cudaErrorInvalidValue;
    const int sm = (int)ClSplit<DH>::kSmem;
    cudaError_t e;
    if (sm > 0 && (e = cudaFuncSetAttribute(slstm_cluster_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            sm)) != cudaSuccess)
        return e;
    if (DH / 32 > 8 && (e = cudaFuncSetAttribute(slstm_cluster_kernel<DH>,
                                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.BH * (DH / 32));
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = (size_t)sm;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = DH / 32;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, slstm_cluster_kernel<DH>, mz, mi, mf, mo, mh, p, device_status_ptr());
}

}  // namespace

// DH 512 needs a 16-CTA cluster (beyond the portable 8): taken only where the
// device can place one with this kernel's resources.
bool slstm_cluster_supports(int DH) {
    if (DH == 64 || DH == 128 || DH == 256) return true;
    if (DH != 512) return false;
    static int ok = -1;
    if (ok < 0) {
        int n = 0;
        const int sm = (int)ClSplit<512>::kSmem;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16);
        cfg.blockDim = dim3(kClThreads);
        cfg.dynamicSmemBytes = (size_t)sm;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        ok = cudaFuncSetAttribute(slstm_cluster_kernel<512>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) ==
                     cudaSuccess &&
                 cudaFuncSetAttribute(slstm_cluster_kernel<512>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                     cudaSuccess &&
                 cudaOccupancyMaxActiveClusters(&n, slstm_cluster_kernel<512>, &cfg) == cudaSuccess && n >= 1
             ? 1 : 0;
        cudaGetLastError();   // a refused query must not leak into a later launch check
    }
    return ok == 1;
}

cudaError_t launch_slstm_cluster(const slstm::SlstmPtrs &p, cudaStream_t st) {
    switch (p.DH) {
        case 64: return launch_cluster_t<64>(p, st);
        case 128: return launch_cluster_t<128>(p, st);
        case 256: return launch_cluster_t<256>(p, st);
        case 512: return launch_cluster_t<512>(p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace xlstm
