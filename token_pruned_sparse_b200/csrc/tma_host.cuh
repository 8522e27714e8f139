// Host side of TMA: the driver's tensor-map encoder, reached at run time
// through the runtime's driver entry-point query (the library links the
// static CUDA runtime only, never libcuda directly).
#pragma once

#include <cuda.h>   // CUtensorMap and the encoder's argument types

#include <mutex>

#include "tps_internal.cuh"

namespace tps {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled, looked up once per process. On failure returns
// TPS_ERR_CUDA with a message naming `who`.
inline int tensor_map_encoder(EncodeTiledFn* fn, const char* who) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && f)
      cached = reinterpret_cast<EncodeTiledFn>(f);
  });
  *fn = cached;
  if (!cached) return fail(TPS_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", who);
  return TPS_OK;
}

}  // namespace tps
