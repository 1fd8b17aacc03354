// Self-test of the failure path: every kernel of the library waits through the
// same bounded mbarrier wait (sm100_ptx.cuh, mbar_wait), which gives up after a
// time limit, records MLA_ERR_TIMEOUT and lets the kernel leave normally (no
// trap, no fault).  This entry point runs that wait on a barrier nothing ever
// arrives on, with a caller-chosen limit, so a test can check the status and
// that the context is still usable afterwards.
#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0, nullptr, limit_ns)) set_status(status, MLA_ERR_TIMEOUT);
}

}  // namespace
}  // namespace mla

extern "C" MLA_API int mla_selftest_wait_timeout(int32_t* status, int64_t limit_ns, void* stream) {
    if (!status || limit_ns <= 0 || limit_ns > 10000000000LL) return MLA_ERR_ARG;
    mla::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status, (uint64_t)limit_ns);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
