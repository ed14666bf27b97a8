// tensor_map.cu — 2-D TMA tensor maps over row-major [rows, 128] byte
// matrices with the 128-byte swizzle (key caches, indexer queries).
//
// The encode function is the driver's, resolved at run time through the
// runtime's entry-point query, so the library does not link libcuda.
#include <cuda.h>

#include "internal.h"

namespace lsa {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D uint8 tensor map over [rows, 128] with a box of [box_rows, 128] and the
// 128-byte swizzle; rows past the end read as zero.
bool make_map_impl(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)128, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)128};
    const cuuint32_t box[2] = {(cuuint32_t)128, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tensor_maps_available() { return encode_fn() != nullptr; }

bool tensor_map_rows128(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    return make_map_impl(m, base, rows, box_rows);
}

}  // namespace lsa
