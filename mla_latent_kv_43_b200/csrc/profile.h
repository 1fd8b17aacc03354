// Optional per-kernel CUDA-event timing (mla_profile_enable / mla_profile_read).
#pragma once
#include <cuda_runtime.h>

namespace mla {
// Record the "before" event of a kernel named `name` on `stream` (no-op when
// profiling is off).  Pair every call with prof_end on the same stream.
void prof_begin(cudaStream_t stream, const char* name);
void prof_end(cudaStream_t stream);
}  // namespace mla
