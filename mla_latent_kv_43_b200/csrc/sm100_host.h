// Host helpers of the tensor-core path: TMA descriptor encoding and device facts.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {
namespace sm100 {

// Encode a bf16 tiled tensor map.  dims/box are innermost first; strides are
// the byte strides of dims 1..rank-1.  Out-of-bounds elements read as zero.
// Returns false when the driver rejects the description.
bool make_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle);

// Streaming multiprocessors of the current device (148 on B200 when unknown).
int sm_count();

}  // namespace sm100
}  // namespace mla
