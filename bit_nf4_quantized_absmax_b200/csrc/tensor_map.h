// Host access to the driver's tiled tensor-map encoder (cuTensorMapEncodeTiled),
// resolved once through the runtime's driver entry point.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace qlora {

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline PFN_encodeTiled get_encoder() {
  static PFN_encodeTiled fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_encodeTiled>(nullptr);
    return reinterpret_cast<PFN_encodeTiled>(p);
  }();
  return fn;
}

}  // namespace qlora
