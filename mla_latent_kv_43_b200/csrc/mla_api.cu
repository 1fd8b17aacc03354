// C ABI of libmla: argument validation, workspace planning and dispatch.
// Every check here runs on the host before anything is enqueued.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "mla.h"

namespace {

thread_local int32_t g_last_launches = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_dims(const mla_dims* d) {
    if (!d) return MLA_ERR_ARG;
    if (d->heads <= 0 || d->d_c <= 0 || d->d_rope <= 0 || d->qk_nope <= 0 || d->v_dim <= 0)
        return MLA_ERR_ARG;
    if ((d->d_rope & 1) || (d->d_c & 1)) return MLA_ERR_ARG;
    if (d->dtype != MLA_BF16 && d->dtype != MLA_FP32) return MLA_ERR_ARG;
    if (!(d->softmax_scale > 0.f) || !isfinite(d->softmax_scale)) return MLA_ERR_ARG;
    if (!(d->rope_base > 1.f) || !isfinite(d->rope_base)) return MLA_ERR_ARG;
    return MLA_OK;
}

bool use_sm100_decode(const mla_dims& d) { return mla::sm100_decode_supported(d); }

int layout_for(const mla_dims* dims, int32_t batch, int32_t n_q, int64_t max_len, int32_t splits,
               mla_ws_layout* L) {
    int rc = validate_dims(dims);
    if (rc) return rc;
    if (batch < 0 || n_q < 0 || splits < 0 || max_len < 0) return MLA_ERR_ARG;
    if (batch > 0 && n_q > 0 && max_len < n_q) return MLA_ERR_ARG;
    if (use_sm100_decode(*dims))
        mla::sm100_layout(*dims, batch, n_q, max_len, splits, L);
    else
        mla::generic_layout(*dims, batch, n_q, max_len, splits, L);
    return MLA_OK;
}

}  // namespace

namespace mla {

void clear_last_launch_count() { g_last_launches = 0; }

void rope_turn_table(float base, int d_rope, uint64_t* turn) {
    const long double two_pi = 6.283185307179586476925286766559005768L;
    for (int i = 0; i < d_rope / 2; ++i) {
        const long double theta = powl((long double)base, -2.0L * i / d_rope);
        turn[i] = (uint64_t)llroundl(theta / two_pi * 18446744073709551616.0L);   // 2^64
    }
}

}  // namespace mla

extern "C" {

size_t mla_decode_workspace_bytes(const mla_dims* dims, int32_t batch, int32_t n_q, int64_t max_len,
                                  int32_t splits) {
    mla_ws_layout L;
    if (layout_for(dims, batch, n_q, max_len, splits, &L)) return 0;
    return L.total;
}

int mla_decode_workspace_layout(const mla_dims* dims, int32_t batch, int32_t n_q, int64_t max_len,
                                int32_t splits, mla_ws_layout* layout) {
    if (!layout) return MLA_ERR_ARG;
    return layout_for(dims, batch, n_q, max_len, splits, layout);
}

int mla_rope(const mla_dims* dims, int64_t n_rows, void* x, int64_t row_stride,
             const int32_t* positions, void* stream) {
    int rc = validate_dims(dims);
    if (rc) return rc;
    if (n_rows < 0 || row_stride < dims->d_rope) return MLA_ERR_ARG;
    if (n_rows == 0) return MLA_OK;
    if (!x || !positions) return MLA_ERR_ARG;
    return mla::rope_rows(*dims, n_rows, x, row_stride, positions, (cudaStream_t)stream);
}

int mla_append(const mla_dims* dims, int32_t batch, int32_t n_new, int32_t hidden, const void* x,
               const void* W_dkv, const float* rms_gamma, const int32_t* positions, void* cache,
               int64_t capacity, int32_t* status, void* stream) {
    g_last_launches = 0;
    int rc = validate_dims(dims);
    if (rc) return rc;
    if (batch < 0 || n_new < 0 || hidden <= 0 || capacity <= 0) return MLA_ERR_ARG;
    if (batch == 0 || n_new == 0) return MLA_OK;
    if (!x || !W_dkv || !positions || !cache || !status) return MLA_ERR_ARG;
    mla::AppendCall c{*dims, batch, n_new, hidden, x, W_dkv, rms_gamma, positions, cache, capacity, status,
                      (cudaStream_t)stream};
    int launches = 0;
    if (mla::sm100_append_supported(*dims, hidden)) {
        if (!aligned16(x) || !aligned16(W_dkv) || !aligned16(cache)) return MLA_ERR_ALIGN;
        rc = mla::sm100_append(c, &launches);
    } else {
        rc = mla::generic_append(c, &launches);
    }
    if (rc == MLA_OK && rms_gamma) rc = mla::rms_norm_rows(c, &launches);
    g_last_launches = launches;
    return rc;
}

int mla_decode(const mla_dims* dims, int32_t batch, int32_t n_q, const void* q_nope,
               const void* q_rope, const void* W_uk, const void* W_uv, const void* cache,
               int64_t capacity, const int32_t* seq_lens, int64_t max_len, void* out,
               void* workspace, size_t workspace_bytes, int32_t splits, int32_t* status,
               void* stream) {
    g_last_launches = 0;
    int rc = validate_dims(dims);
    if (rc) return rc;
    if (batch < 0 || n_q < 0 || splits < 0 || capacity <= 0) return MLA_ERR_ARG;
    if (batch == 0 || n_q == 0) return MLA_OK;
    if (max_len < n_q || max_len > capacity) return MLA_ERR_ARG;
    if (!q_nope || !q_rope || !W_uk || !W_uv || !cache || !seq_lens || !out || !workspace || !status)
        return MLA_ERR_ARG;
    mla_ws_layout L;
    if ((rc = layout_for(dims, batch, n_q, max_len, splits, &L))) return rc;
    if (workspace_bytes < L.total) return MLA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLA_ERR_ALIGN;
    const bool tc = use_sm100_decode(*dims);
    if (tc && (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_uk) || !aligned16(W_uv) ||
               !aligned16(cache) || !aligned16(out)))
        return MLA_ERR_ALIGN;
    mla::DecodeCall c{*dims, batch, n_q, q_nope, q_rope, W_uk, W_uv, cache, capacity, seq_lens,
                      max_len, out, static_cast<char*>(workspace), L, status, (cudaStream_t)stream};
    int launches = 0;
    rc = tc ? mla::sm100_decode(c, &launches) : mla::generic_decode(c, &launches);
    g_last_launches = launches;
    return rc;
}

int mla_decode_sparse(const mla_dims* dims, int32_t batch, int32_t n_q, const void* q_nope,
                      const void* q_rope, const void* W_uk, const void* W_uv, const void* cache,
                      int64_t capacity, const int32_t* seq_lens, int64_t max_len, const int32_t* sel,
                      const int32_t* n_sel, int32_t max_sel, void* out, void* workspace,
                      size_t workspace_bytes, int32_t splits, int32_t* status, void* stream) {
    g_last_launches = 0;
    int rc = validate_dims(dims);
    if (rc) return rc;
    if (batch < 0 || n_q < 0 || splits < 0 || capacity <= 0) return MLA_ERR_ARG;
    if (batch == 0 || n_q == 0) return MLA_OK;
    if (max_len < n_q || max_len > capacity || max_sel < 1 || max_sel > max_len) return MLA_ERR_ARG;
    if (!q_nope || !q_rope || !W_uk || !W_uv || !cache || !seq_lens || !sel || !n_sel || !out || !workspace ||
        !status)
        return MLA_ERR_ARG;
    if (!use_sm100_decode(*dims)) return MLA_ERR_UNSUPPORTED;
    if ((int64_t)batch * capacity >= ((int64_t)1 << 31)) return MLA_ERR_UNSUPPORTED;
    mla_ws_layout L;
    if ((rc = layout_for(dims, batch, n_q, max_sel, splits, &L))) return rc;
    if (workspace_bytes < L.total) return MLA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLA_ERR_ALIGN;
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_uk) || !aligned16(W_uv) || !aligned16(cache) ||
        !aligned16(out))
        return MLA_ERR_ALIGN;
    mla::DecodeCall c{*dims, batch, n_q, q_nope, q_rope, W_uk, W_uv, cache, capacity, seq_lens,
                      max_len, out, static_cast<char*>(workspace), L, status, (cudaStream_t)stream};
    c.sel = sel;
    c.n_sel = n_sel;
    c.max_sel = max_sel;
    int launches = 0;
    rc = mla::sm100_decode(c, &launches);
    g_last_launches = launches;
    return rc;
}

static bool prefill_dims_ok(const mla_dims* d) {
    return d->dtype == MLA_BF16 && d->d_c == 512 && d->d_rope == 64 && d->qk_nope == 128 && d->v_dim == 128;
}

size_t mla_prefill_workspace_bytes(const mla_dims* dims, int32_t batch, int32_t n_q, int64_t max_len) {
    if (validate_dims(dims) || batch < 0 || n_q < 0 || max_len < 0) return 0;
    mla::sm100::PrefillLayout L;
    mla::sm100::prefill_layout(*dims, batch, n_q, max_len, &L);
    return (size_t)L.total;
}

int mla_prefill(const mla_dims* dims, int32_t batch, int32_t n_q, const void* q_nope, const void* q_rope,
                const void* W_uk, const void* W_uv, const void* cache, int64_t capacity, const int32_t* seq_lens,
                int64_t max_len, void* out, void* workspace, size_t workspace_bytes, int32_t* status,
                void* stream) {
    g_last_launches = 0;
    int rc = validate_dims(dims);
    if (rc) return rc;
    if (batch < 0 || n_q < 0 || capacity <= 0) return MLA_ERR_ARG;
    if (batch == 0 || n_q == 0) return MLA_OK;
    if (max_len < n_q || max_len > capacity) return MLA_ERR_ARG;
    if (!q_nope || !q_rope || !W_uk || !W_uv || !cache || !seq_lens || !out || !workspace || !status)
        return MLA_ERR_ARG;
    if (!prefill_dims_ok(dims)) return MLA_ERR_UNSUPPORTED;
    const int64_t lim = (int64_t)1 << 31;
    if ((int64_t)batch * n_q >= lim || (int64_t)dims->heads * batch * max_len >= lim ||
        (int64_t)batch * capacity >= lim)
        return MLA_ERR_UNSUPPORTED;
    if (workspace_bytes < mla_prefill_workspace_bytes(dims, batch, n_q, max_len)) return MLA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLA_ERR_ALIGN;
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_uk) || !aligned16(W_uv) || !aligned16(cache) ||
        !aligned16(out))
        return MLA_ERR_ALIGN;
    mla::sm100::PrefillCall c{*dims, batch, n_q, q_nope, q_rope, W_uk, W_uv, cache, capacity, seq_lens,
                              max_len, out, static_cast<char*>(workspace), status, (cudaStream_t)stream};
    int launches = 0;
    rc = mla::sm100::prefill_launch(c, &launches);
    g_last_launches = launches;
    return rc;
}

int mla_output_projection(const mla_dims* dims, int32_t tokens, int32_t hidden, const void* out, const void* W_O,
                          void* y, int32_t* status, void* stream) {
    g_last_launches = 0;
    int rc = validate_dims(dims);
    if (rc) return rc;
    if (tokens < 0 || hidden <= 0) return MLA_ERR_ARG;
    if (tokens == 0) return MLA_OK;
    if (!out || !W_O || !y || !status) return MLA_ERR_ARG;
    const int K = dims->heads * dims->v_dim;
    int launches = 0;
    if (dims->dtype == MLA_BF16 && hidden % 8 == 0 && K % 8 == 0) {
        if (!aligned16(out) || !aligned16(W_O) || !aligned16(y)) return MLA_ERR_ALIGN;
        rc = mla::sm100::gemm_xw_launch(out, W_O, tokens, K, hidden, (__nv_bfloat16*)y, status, (cudaStream_t)stream,
                                        "sm100_oproj", &launches);
    } else {
        rc = mla::generic_gemm_xw((mla_dtype)dims->dtype, out, W_O, tokens, K, hidden, y, (cudaStream_t)stream, &launches);
    }
    g_last_launches = launches;
    return rc;
}

int mla_get_status(int32_t* status, void* stream, int32_t* host_status) {
    if (!status || !host_status) return MLA_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(host_status, status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MLA_ERR_CUDA;
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_OK;
}

const char* mla_status_string(int code) {
    switch (code) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_ARG: return "MLA_ERR_ARG";
        case MLA_ERR_ALIGN: return "MLA_ERR_ALIGN";
        case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
        case MLA_ERR_LEN: return "MLA_ERR_LEN";
        case MLA_ERR_POS: return "MLA_ERR_POS";
        case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
        case MLA_ERR_INDEX: return "MLA_ERR_INDEX";
        default: return "MLA_ERR_UNKNOWN";
    }
}

int32_t mla_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
