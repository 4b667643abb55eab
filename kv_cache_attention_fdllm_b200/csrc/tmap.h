// Host-side creation of TMA tensor maps (cuTensorMapEncodeTiled, fetched from
// the driver at run time so that the library does not link against libcuda).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace fdllm {

// Encodes a tiled bf16 tensor map.  dims[0] is the contiguous dimension;
// strides_bytes[i] is the byte stride of dims[i + 1].  Returns false on error.
bool encode_bf16_map(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box,
                     CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promo);

}  // namespace fdllm
