// Host side of the TMA helpers: the tensor-map encoder is taken from the driver
// through the runtime's entry-point query, so the library links no driver stub.
#include <cudaTypedefs.h>

#include "tma.cuh"

namespace gdn {
namespace tma {

static PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

cudaError_t map2d(CUtensorMap *m, CUtensorMapDataType dtype, const void *base, uint64_t cols, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle)
{
    auto fn = encoder();
    if (!fn || !base || cols == 0 || rows == 0) return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t map_heads(CUtensorMap *m, CUtensorMapDataType dtype, const void *base, uint64_t dim, uint64_t heads,
                      uint64_t rows, uint32_t box_rows)
{
    auto fn = encoder();
    if (!fn || !base || dim == 0 || heads == 0 || rows == 0) return cudaErrorInvalidValue;
    const cuuint64_t dims[3] = {dim, heads, rows};
    const cuuint64_t strides[2] = {dim * 2, heads * dim * 2};  // bytes; 16-bit elements
    const cuuint32_t box[3] = {64, 1, box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, dtype, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace tma
}  // namespace gdn
