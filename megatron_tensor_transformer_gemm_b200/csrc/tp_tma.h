// Host-side access to cuTensorMapEncodeTiled without linking libcuda: the
// driver entry point is fetched once through the runtime.
#pragma once

#include <cuda.h>

#include "tp_internal.h"

namespace tpi {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

tp_status tma_encoder(EncodeTiledFn* out);

// bf16 tensor map with 128-byte swizzle and zero fill out of bounds.
// dims[0] is the contiguous extent; strides are bytes of dims 1..rank-1.
tp_status encode_bf16(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims,
                      const cuuint64_t* strides, const cuuint32_t* box, const char* what);

}  // namespace tpi
