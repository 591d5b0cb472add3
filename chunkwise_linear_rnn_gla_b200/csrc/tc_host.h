// Host-side helper: TMA tensor-map encoding through the driver entry point
// (fetched once with cudaGetDriverEntryPoint, so the library needs no link
// against libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace gla {
namespace tc {

// Encode a tiled tensor map. dims/box are innermost-first; strides_bytes has
// rank-1 entries (strides of dims 1..rank-1). Returns false on failure.
bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, uint32_t rank, const void* base, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle);

// Number of SMs of the current device (148 if the query fails).
int sm_count();

}  // namespace tc
}  // namespace gla
