// Host side of the TMA path: tensor-map encoding through the runtime's driver entry point.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_common.cuh"

namespace mla {

bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, int rank,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            encode = (PFN_cuTensorMapEncodeTiled_v12000)p;
    });
    if (!encode || rank < 1 || rank > 5) return false;
    if (swizzle_bytes != 128 && swizzle_bytes != 64 && swizzle_bytes != 0) return false;
    if (swizzle_bytes && box[0] * (uint32_t)elem_bytes > (uint32_t)swizzle_bytes) return false;
    if ((box[0] * (uint32_t)elem_bytes) % 16 != 0) return false;   // the inner box extent
    if (((uintptr_t)base & 15) != 0) return false;
    for (int i = 0; i + 1 < rank; ++i)
        if (strides_bytes[i] % 16 != 0) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank) s[i] = strides_bytes[i];
    }
    const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                        : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r = encode(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), d, s, b, e,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
    return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rank, dims, strides_bytes, box, swizzle_bytes);
}

}  // namespace mla
