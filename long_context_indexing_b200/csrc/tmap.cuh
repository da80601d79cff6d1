// tmap.cuh -- host-side encoding of TMA tensor maps (cuTensorMapEncodeTiled,
// reached through the runtime's driver entry point so that the library does
// not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace lsa {

typedef CUresult (*TmapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The encoder, or nullptr when the driver does not provide it.
inline TmapEncodeFn tmap_encode_fn()
{
    static const TmapEncodeFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return (TmapEncodeFn)p;
        return (TmapEncodeFn) nullptr;
    }();
    return fn;
}

// A [rows][64] bf16 array read in boxes of box_rows rows, 128-byte swizzle
// (the tensor-core operand layout of the scoring kernels).  False when the
// encoder is missing or refuses the map.
inline bool tmap_rows64_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows)
{
    TmapEncodeFn enc = tmap_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {64, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {64 * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lsa
