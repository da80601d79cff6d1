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

}  // namespace lsa
