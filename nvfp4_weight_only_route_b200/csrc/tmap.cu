// tmap.cu -- tensor-map (TMA descriptor) encoding shared by the expert kernels.
#include "internal.h"

namespace tfmoe {
namespace {

// cuTensorMapEncodeTiled, looked up through the runtime so the library does not
// link the driver library directly (it loads on machines without a GPU driver).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

}  // namespace

CUresult encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType type, void *base, uint64_t dim0,
                              uint64_t dim1, uint64_t row_stride_bytes, uint32_t box0, uint32_t box1,
                              CUtensorMapSwizzle swizzle)
{
    EncodeTiledFn encode = encode_tiled_fn();
    if (!encode) return CUDA_ERROR_NOT_FOUND;
    const cuuint64_t gdim[2] = {(cuuint64_t)dim0, (cuuint64_t)dim1};
    const cuuint64_t gstride[1] = {(cuuint64_t)row_stride_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)box0, (cuuint32_t)box1};
    const cuuint32_t estride[2] = {1, 1};
    return encode(map, type, 2, base, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace tfmoe
