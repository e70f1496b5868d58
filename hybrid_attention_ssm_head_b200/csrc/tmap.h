// Host-side construction of TMA tensor maps (cuTensorMapEncodeTiled reached
// through the runtime's driver entry point, so the library does not link libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hymba {

// 128-byte swizzled tiled map of a row-major tensor with up to 3 dims.
// dims[0] is the contiguous dimension (elements); strides_bytes[i] is the byte
// stride of dims[i+1].  box[i] elements per copy.  Out-of-range elements read 0.
bool make_tmap(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int rank,
               const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box);

}  // namespace hymba
