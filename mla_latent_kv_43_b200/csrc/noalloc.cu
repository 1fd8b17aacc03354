// mla_decode_noalloc: the decode step for callers that cannot allocate device
// memory themselves (see include/mla.h).  The scratch lives in one static
// device array; each device that loads this library holds it until the
// process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "mla.h"

namespace {

constexpr size_t kScratchBytes = MLA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device.  In host code the
// array's name only stands for the symbol; the address must come from the
// runtime, once per device, with that device current.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MLA_OK;
}

}  // namespace

extern "C" int mla_decode_noalloc(const mla_dims* dims, int32_t batch, int32_t n_q, const void* q_nope,
                                  const void* q_rope, const void* W_uk, const void* W_uv, const void* cache,
                                  int64_t capacity, const int32_t* seq_lens, int64_t max_len, void* out,
                                  int32_t splits, int32_t* status, void* stream) {
    // The layout call checks dims and sizes exactly as mla_decode does.
    mla_ws_layout L;
    int rc = mla_decode_workspace_layout(dims, batch, n_q, max_len, splits, &L);
    if (rc == MLA_OK && (batch == 0 || n_q == 0)) {
        // the empty problem: mla_decode's own answer, without touching the device
        return mla_decode(dims, batch, n_q, q_nope, q_rope, W_uk, W_uv, cache, capacity, seq_lens, max_len, out,
                          nullptr, 0, splits, status, stream);
    }
    if (rc == MLA_OK && L.total > kScratchBytes) rc = MLA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (rc == MLA_OK && scratch_address(&scratch) != MLA_OK) rc = MLA_ERR_CUDA;
    if (rc != MLA_OK) {
        mla::clear_last_launch_count();     // nothing was enqueued by this call
        return rc;
    }
    // Every region of the workspace is written before it is read within one
    // call, so nothing left by an earlier call needs clearing.
    return mla_decode(dims, batch, n_q, q_nope, q_rope, W_uk, W_uv, cache, capacity, seq_lens, max_len, out, scratch,
                      kScratchBytes, splits, status, stream);
}
