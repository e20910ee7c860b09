// q4_tma.cu -- host side of the TMA kernels: tensor-map encoding through the
// driver entry point obtained from the CUDA runtime (no libcuda link needed).
#include <mutex>

#include "q4_sm100.cuh"

namespace q4 {
namespace {

EncodeTiledFn g_encode = nullptr;
std::once_flag g_once;

void resolve() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}

}  // namespace

cudaError_t encode_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                                 int elem_bytes, uint64_t rows, uint64_t cols, uint64_t row_bytes,
                                 uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swizzle) {
    std::call_once(g_once, resolve);
    if (!g_encode) return cudaErrorNotSupported;
    (void)elem_bytes;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace q4
