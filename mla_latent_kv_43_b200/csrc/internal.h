// Internal interface between the C ABI (mla_api.cu) and the kernel files.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mla.h"

namespace mla {

struct DecodeCall {
    mla_dims d;
    int batch, n_q;
    const void *q_nope, *q_rope, *W_uk, *W_uv, *cache;
    int64_t capacity;
    const int32_t* seq_lens;
    int64_t max_len;
    void* out;
    char* ws;
    mla_ws_layout L;
    int32_t* status;
    cudaStream_t stream;
    // sparse decode (mla_decode_sparse): selected slots, counts, row length
    const int32_t* sel = nullptr;
    const int32_t* n_sel = nullptr;
    int max_sel = 0;
};

struct AppendCall {
    mla_dims d;
    int batch, n_new, hidden;
    const void *x, *W_dkv;
    const float* rms_gamma;   // [d_c] or nullptr
    const int32_t* positions;
    void* cache;
    int64_t capacity;
    int32_t* status;
    cudaStream_t stream;
};

// Dense tensor-core decode: the CTA-pair attention kernel (heads split across
// the pair, cta_group::2 MMAs; true) or the latent-split kernel (false).
constexpr bool kDecodePairKernel = false;

// True when the tensor-core path serves these dims: bf16 with the
// DeepSeek-V3 head geometry (128 heads, latent 512, rope 64, nope 128, value 128).
bool sm100_decode_supported(const mla_dims& d);
bool sm100_append_supported(const mla_dims& d, int hidden);

// Workspace layouts (offsets 256-byte aligned).
void generic_layout(const mla_dims& d, int batch, int n_q, int64_t max_len, int splits,
                    mla_ws_layout* L);
void sm100_layout(const mla_dims& d, int batch, int n_q, int64_t max_len, int splits,
                  mla_ws_layout* L);

// Each returns MLA_OK or MLA_ERR_CUDA and adds the kernels it enqueued to *launches.
int generic_decode(const DecodeCall& c, int* launches);
int sm100_decode(const DecodeCall& c, int* launches);
int generic_append(const AppendCall& c, int* launches);
int sm100_append(const AppendCall& c, int* launches);
int rope_rows(const mla_dims& d, int64_t n_rows, void* x, int64_t row_stride,
              const int32_t* positions, cudaStream_t stream);
// The output projection y = x W (x [M][K], W [K][n_out]): tcgen05 (bf16) and CUDA-core versions.
namespace sm100 {
int gemm_xw_launch(const void* x, const void* W, int M, int K, int n_out, __nv_bfloat16* y, int32_t* status,
                   cudaStream_t stream, const char* name, int* launches);

// Prefill: the materialised form (per-head keys and values, then causal attention).
struct PrefillCall {
    mla_dims d;
    int batch, n_q;
    const void *q_nope, *q_rope, *W_uk, *W_uv, *cache;
    int64_t capacity;
    const int32_t* seq_lens;
    int64_t max_len;
    void* out;
    char* ws;
    int32_t* status;
    cudaStream_t stream;
};
struct PrefillLayout {
    int64_t q_rot, kn, v, total;   // byte offsets (256-aligned) and the total
};
void prefill_layout(const mla_dims& d, int batch, int n_q, int64_t max_len, PrefillLayout* L);
int prefill_launch(const PrefillCall& c, int* launches);
}
int generic_gemm_xw(mla_dtype dtype, const void* x, const void* W, int M, int K, int n_out, void* y,
                    cudaStream_t stream, int* launches);
// RMSNorm of the latent of every appended row (after either append kernel).
int rms_norm_rows(const AppendCall& c, int* launches);

// Sets the count mla_last_launch_count reports to 0 (for an entry point that
// returns before enqueuing anything).
void clear_last_launch_count();

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// RoPE pair frequencies theta_i = base^(-2i/d_rope), i < d_rope / 2, as
// fractions of a turn in 64-bit fixed point: turn[i] = round(theta_i / (2 pi) * 2^64),
// computed in long double (rope_pair_turn in common.cuh uses them).
void rope_turn_table(float base, int d_rope, uint64_t* turn);

}  // namespace mla
