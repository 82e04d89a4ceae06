// Tensor-map (TMA descriptor) construction for the kernels that move 2- and
// 3-dimensional boxes without swizzling.  The driver's encoder is reached
// through the runtime's entry-point query, so the library links no driver
// library directly.
#include <mutex>

#include "kernels.h"

namespace xlstm {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
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

}  // namespace

bool make_tensor_map_3d(CUtensorMap *m, const void *base, int elem_bytes, const unsigned long long dims[3],
                        const unsigned long long strides_bytes[2], const unsigned box[3]) {
    EncodeTiledFn fn = encoder();
    if (!fn || (elem_bytes != 2 && elem_bytes != 4)) return false;
    cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    cuuint64_t s[2] = {strides_bytes[0], strides_bytes[1]};
    cuuint32_t b[3] = {box[0], box[1], box[2]};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
              const_cast<void *>(base), d, s, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace xlstm
