/*
 * mla.h -- C ABI of libmla.so: Multi-head Latent Attention against the
 * compressed latent cache -- absorbed decode (dense and over a top-k
 * selection), cache append, output projection, and prefill in the
 * materialised factorisation.
 *
 * Multi-head Latent Attention caches, per token and layer, one 576-wide entry:
 * a 512-wide latent c_KV followed by a 64-wide rope key that is already
 * rotated at the token's position ("Understanding MLA (Multi-head Latent
 * Attention)", section 5 "What gets cached").  Decode scores every head's
 * query directly against that cache after moving the key up-projection onto
 * the query side (same page, section 4), and applies the value up-projection
 * to the softmax-weighted latent (aicassindra "Multi-head latent attention",
 * "End-to-end flow").
 *
 * Conventions for every entry point:
 *  - Pointers marked (device) are CUDA device pointers; nothing is copied to
 *    or from the host except where stated.  The caller allocates every buffer
 *    (inputs, outputs, workspace, the 4-byte status word); the library
 *    allocates no memory and keeps no pointer after the call returns.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *    stream.  All work is enqueued on it and the call returns without waiting.
 *  - Tensors are dense, row-major, in the element type `dims->dtype`
 *    (MLA_BF16: bfloat16, MLA_FP32: float) unless stated otherwise.
 *  - Return value: MLA_OK, or an error code for problems found on the host
 *    before anything is enqueued (nothing runs in that case).  Problems only
 *    the device can see (a bad length or position) are recorded in the status
 *    word with an atomic "first error wins" update and never trap; read and
 *    clear it with mla_get_status.
 *  - Empty work (batch == 0, n_q == 0, n_new == 0, n_rows == 0) returns MLA_OK
 *    and enqueues nothing.
 */
#ifndef MLA_H
#define MLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum mla_dtype { MLA_BF16 = 0, MLA_FP32 = 1 };

enum mla_status {
    MLA_OK = 0,
    MLA_ERR_ARG = 1,          /* null pointer, non-positive or odd size, bad dtype */
    MLA_ERR_ALIGN = 2,        /* a pointer the kernels load with TMA is not 16-byte aligned */
    MLA_ERR_WORKSPACE = 3,    /* workspace_bytes below the call's size (mla_*_workspace_bytes) */
    MLA_ERR_UNSUPPORTED = 4,  /* a valid request the library does not implement */
    MLA_ERR_CUDA = 5,         /* a CUDA launch or API call failed */
    MLA_ERR_LEN = 6,          /* device: len_b < n_q, len_b > capacity or len_b > max_len */
    MLA_ERR_POS = 7,          /* device: an append position outside [0, capacity) */
    MLA_ERR_TIMEOUT = 8,      /* device: a bounded wait inside a kernel expired */
    MLA_ERR_INDEX = 9         /* device: a selected cache slot outside the query's visible keys */
};

/* Model geometry.  The per-head query/key width is qk_nope + d_rope and the
 * value width is v_dim ("Understanding MLA", Phase C step C1 and Phase D
 * step D1).  softmax_scale is normally 1/sqrt(qk_nope + d_rope) (Phase D,
 * step D2); rope_base is the RoPE base (10000). */
typedef struct {
    int32_t heads;
    int32_t d_c;       /* latent width (512 for DeepSeek-V3) */
    int32_t d_rope;    /* rope key width (64), even */
    int32_t qk_nope;   /* content part of the query/key (128) */
    int32_t v_dim;     /* value width per head (128) */
    int32_t dtype;     /* enum mla_dtype */
    float softmax_scale;
    float rope_base;
} mla_dims;

/* Workspace regions of one mla_decode call (byte offsets from the workspace
 * base; a size of 0 means the region is not used).  Exposed so tests can
 * inspect the intermediate results of a call. */
typedef struct {
    size_t total;          /* bytes the call needs */
    size_t q_lat;          /* absorbed queries [B][n_q][H][d_c + d_rope], compute dtype */
    size_t q_lat_bytes;
    size_t o_lat;          /* latent outputs [B][n_q][H][d_c], compute dtype: combined on the
                              generic path; on the tensor-core path only for query tokens whose
                              key tiles one work item covered (a token cut across items keeps its
                              pieces in part_o / part_lse, merged after the up-projection) */
    size_t o_lat_bytes;
    size_t part_o;         /* split-KV partial latent outputs, each normalised by its own sum:
                              compute dtype on the tensor-core path, float otherwise.  On the
                              tensor-core path head-major and blocked by 64 latent columns:
                              element (piece slot s, head h, column c) at
                              ((h * d_c / 64 + c / 64) * 2 splits + s) * 64 + c % 64 */
    size_t part_o_bytes;
    size_t part_lse;       /* split-KV partial log-sum-exp values, float (tensor-core path: base 2,
                              [H][2 splits][2 latent halves], the halves normalised separately) */
    size_t part_lse_bytes;
    size_t sched;          /* device-built work schedule (tensor-core path, int32: the key-tile
                              prefix of the query tokens [B n_q + 1], each item's first token
                              [splits], each piece slot's query token [2 splits], -1 if unused) */
    size_t sched_bytes;
    int32_t compute_dtype; /* enum mla_dtype of q_lat, o_lat (and part_o on the tensor-core path) */
    int32_t splits;        /* key splits per query (generic path) or work items (tensor-core path) */
} mla_ws_layout;

/* Workspace needed by mla_decode for these sizes (0 on invalid arguments).
 * max_len is a host-known upper bound on every len_b; splits as in
 * mla_decode (0 = automatic). */
MLA_API size_t mla_decode_workspace_bytes(const mla_dims* dims, int32_t batch, int32_t n_q,
                                  int64_t max_len, int32_t splits);

/* Same sizes as mla_decode_workspace_bytes, with the region offsets.
 * Returns MLA_OK or MLA_ERR_ARG. */
MLA_API int mla_decode_workspace_layout(const mla_dims* dims, int32_t batch, int32_t n_q,
                                int64_t max_len, int32_t splits, mla_ws_layout* layout);

/* In-place RoPE on strided rows ("Understanding MLA", Phase B step B2 and
 * Phase C step C2): every interleaved pair (x[2i], x[2i+1]) of row r is
 * rotated by the angle positions[r] * rope_base^(-2i/d_rope).
 *   x          (device) first element of row 0; row r starts at x + r*row_stride
 *              elements; d_rope elements per row are rotated.
 *   row_stride elements between rows (>= d_rope).
 *   positions  (device) int32[n_rows], each >= 0.
 * Used to build a cache's rope keys from raw values (as the append step would
 * have stored them); the decode and append kernels apply the same rotation
 * internally. */
MLA_API int mla_rope(const mla_dims* dims, int64_t n_rows, void* x, int64_t row_stride,
             const int32_t* positions, void* stream);

/* Append n_new tokens to each of `batch` sequences (aicassindra "Multi-head
 * latent attention", "End-to-end flow"; "Understanding MLA", Phase A step A1):
 * y = x W_dkv (float accumulation), latent = y[0:d_c], rope key =
 * RoPE(y[d_c:d_c+d_rope], position), and cache[b][pos][:] = latent || rope key,
 * rounded once to dims->dtype.
 *   x          (device) [batch*n_new][hidden]; token i of sequence b is row b*n_new+i.
 *   W_dkv      (device) [hidden][d_c + d_rope].
 *   rms_gamma  (device) float[d_c] or NULL.  Non-NULL: the latent alone is
 *              RMS-normalised before it is stored, latent = gamma * y[0:d_c] /
 *              sqrt(mean(y[0:d_c]^2) + 1e-6) ("Understanding MLA", Phase A step
 *              A2; the pages give no epsilon, 1e-6 is the usual choice); the rope
 *              key is not normalised.  On the bf16 path y[0:d_c] is rounded to
 *              bf16 once before the normalisation and once after it.
 *   positions  (device) int32[batch*n_new]: slot of each new token, distinct
 *              within a sequence.  A position outside [0, capacity) sets
 *              MLA_ERR_POS and that row is not written.
 *   cache      (device) [batch][capacity][d_c + d_rope]; only the addressed slots
 *              are written, every other byte is left untouched.
 *   status     (device) int32 status word. */
MLA_API int mla_append(const mla_dims* dims, int32_t batch, int32_t n_new, int32_t hidden,
               const void* x, const void* W_dkv, const float* rms_gamma,
               const int32_t* positions, void* cache, int64_t capacity,
               int32_t* status, void* stream);

/* Absorbed MLA decode for n_q query tokens per sequence.
 * For sequence b holding len_b cached tokens (its queries' own entries
 * included), query j sits at position p = len_b - n_q + j and attends keys
 * 0..p.  Per head h:
 *   q_lat  = [ W_uk[h] q_nope  ||  RoPE(q_rope, p) ]            (width d_c + d_rope)
 *   s_n    = softmax_scale * < q_lat , cache[b][n][:] >,  n <= p
 *   o_lat  = sum_n softmax(s)_n * cache[b][n][0:d_c]
 *   out    = o_lat W_uv[h]
 * which equals softmax(Q K^T / sqrt(qk_nope + d_rope)) V with K = [c W_uk[h] ||
 * rope key] and V = c W_uv[h] ("Understanding MLA", sections 3-4; "Multi-Head
 * Latent Attention", section 2 "Computational complexity").
 *   q_nope    (device) [batch][n_q][heads][qk_nope]
 *   q_rope    (device) [batch][n_q][heads][d_rope], not yet rotated
 *   W_uk      (device) [heads][d_c][qk_nope]   (K^(h) = c W_uk[h])
 *   W_uv      (device) [heads][d_c][v_dim]     (V^(h) = c W_uv[h])
 *   cache     (device) [batch][capacity][d_c + d_rope], rope keys already rotated
 *   seq_lens  (device) int32[batch]; a length < n_q, > capacity or > max_len sets
 *             MLA_ERR_LEN in the status word and that sequence's outputs are zero.
 *   max_len   host-known bound on every len_b (n_q <= max_len <= capacity).
 *   out       (device) [batch][n_q][heads][v_dim]
 *   workspace (device) >= mla_decode_workspace_bytes(...) bytes, 256-byte aligned.
 *   splits    0 = automatic; k > 0 asks for k key splits per query.
 *   status    (device) int32 status word. */
MLA_API int mla_decode(const mla_dims* dims, int32_t batch, int32_t n_q,
               const void* q_nope, const void* q_rope, const void* W_uk, const void* W_uv,
               const void* cache, int64_t capacity, const int32_t* seq_lens, int64_t max_len,
               void* out, void* workspace, size_t workspace_bytes, int32_t splits,
               int32_t* status, void* stream);

/* Absorbed MLA decode over a selected subset of each query's cached keys
 * ("Multi-Head Latent Attention", section 4: a selector picks a top-k subset of
 * the cached latents for every query -- k = 2048 in DeepSeek-V3.2 -- and MLA
 * runs unchanged on that subset; the selector itself is not part of this
 * library).  Arguments as mla_decode, plus
 *   sel      (device) int32[batch][n_q][max_sel]: the cache slots query (b, j)
 *            attends, distinct, each in [0, p] for the query's position p;
 *            entries past n_sel are ignored.  Their order does not matter.
 *   n_sel    (device) int32[batch][n_q]: how many leading entries of sel are
 *            used, 1 <= n_sel <= min(max_sel, p + 1); any other count sets
 *            MLA_ERR_LEN and that query's outputs are zero.
 *   max_sel  (host) row length of sel, 1 <= max_sel <= max_len.
 * A slot outside [0, p] sets MLA_ERR_INDEX and the call's outputs are then
 * unspecified (finite).  Implemented on the tensor-core path (bf16 with the
 * DeepSeek-V3 head geometry); other dims return MLA_ERR_UNSUPPORTED.  The
 * workspace is mla_decode_workspace_bytes(dims, batch, n_q, max_sel, splits)
 * bytes; batch * capacity must fit in 31 bits. */
MLA_API int mla_decode_sparse(const mla_dims* dims, int32_t batch, int32_t n_q,
               const void* q_nope, const void* q_rope, const void* W_uk, const void* W_uv,
               const void* cache, int64_t capacity, const int32_t* seq_lens, int64_t max_len,
               const int32_t* sel, const int32_t* n_sel, int32_t max_sel,
               void* out, void* workspace, size_t workspace_bytes, int32_t splits,
               int32_t* status, void* stream);

/* The output projection ("Understanding MLA", Phase D step D2): the per-head
 * outputs of a decode step, concatenated head after head, projected to the
 * hidden width: y[t] = [out[t][0] || out[t][1] || ... || out[t][H-1]] W_O.
 *   tokens  number of query tokens (batch * n_q of the decode).
 *   hidden  output width; a multiple of 8 for the tensor-core path.
 *   out     (device) [tokens][heads][v_dim] (mla_decode's output), dims->dtype.
 *   W_O     (device) [heads * v_dim][hidden], dims->dtype.
 *   y       (device) [tokens][hidden], dims->dtype; float accumulation, one rounding.
 *   status  (device) int32 status word.
 * bf16 runs a tcgen05 GEMM with K split over a cluster of 2, 4 or 8 CTAs (the
 * widest split whose grid runs in one wave); fp32 (or a width that is not a
 * multiple of 8) runs on CUDA cores.
 * Errors: MLA_ERR_ARG (tokens < 0, hidden <= 0, a null pointer when tokens > 0),
 * MLA_ERR_ALIGN (a bf16 tensor-core operand not 16-byte aligned),
 * MLA_ERR_UNSUPPORTED (more than 65535 * 256 tokens on the tensor-core path);
 * tokens == 0 returns MLA_OK and touches nothing. */
MLA_API int mla_output_projection(const mla_dims* dims, int32_t tokens, int32_t hidden, const void* out,
               const void* W_O, void* y, int32_t* status, void* stream);

/* Prefill: the same attention as mla_decode (same inputs, same outputs, the
 * queries' own entries already in the cache) evaluated in the materialised
 * factorisation, for many query tokens per sequence: each cached latent of the
 * first max_len rows of a sequence is expanded once into per-head keys c W_uk[h]
 * and values c W_uv[h], then ordinary causal attention runs per head over the
 * 192-wide key [c W_uk[h] || k_rope] and the 128-wide value ("Understanding MLA",
 * sections "Reference code vs serving engines" and 6; "Multi-Head Latent
 * Attention", section 3).  The materialised rows live in the workspace.
 * Arguments as for mla_decode (without splits); workspace >=
 * mla_prefill_workspace_bytes(dims, batch, n_q, max_len), 256-byte aligned.
 * bf16 with d_c 512, d_rope 64, qk_nope 128, v_dim 128 and any head count;
 * other dims return MLA_ERR_UNSUPPORTED, as do sizes whose batch * n_q,
 * heads * batch * max_len or batch * capacity reach 2^31.  Host errors as for
 * mla_decode (MLA_ERR_ARG, MLA_ERR_WORKSPACE, MLA_ERR_ALIGN for q_nope, q_rope,
 * W_uk, W_uv, cache or out not 16-byte aligned).  A sequence with a bad length
 * sets MLA_ERR_LEN and gets zero outputs. */
MLA_API size_t mla_prefill_workspace_bytes(const mla_dims* dims, int32_t batch, int32_t n_q, int64_t max_len);
MLA_API int mla_prefill(const mla_dims* dims, int32_t batch, int32_t n_q, const void* q_nope, const void* q_rope,
                        const void* W_uk, const void* W_uv, const void* cache, int64_t capacity,
                        const int32_t* seq_lens, int64_t max_len, void* out, void* workspace,
                        size_t workspace_bytes, int32_t* status, void* stream);

/* Failure-path self-test.  Every kernel of the library waits on its
 * barriers through one bounded wait that gives up after a time limit,
 * records MLA_ERR_TIMEOUT in the status word and lets the kernel leave
 * normally (no trap, no fault).  This call runs that wait in one CTA on a
 * barrier that nothing ever arrives on, with the limit limit_ns (0 < limit_ns
 * <= 10 s): afterwards the status word holds MLA_ERR_TIMEOUT and the context
 * remains usable.  It has no counterpart on the pages; it exists for tests.
 *   status  (device) int32 status word. */
MLA_API int mla_selftest_wait_timeout(int32_t* status, int64_t limit_ns, void* stream);

/* Size of the fixed scratch area behind mla_decode_noalloc. */
#define MLA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* mla_decode without a caller-provided workspace, for callers that cannot
 * allocate device memory: code that runs where cudaMalloc is not allowed or
 * must not block (inside an allocator-free serving loop, a plugin that may
 * only use memory its host framework hands it, a real-time thread that cannot
 * risk the device-wide synchronisation an allocation may cause).  It has no
 * counterpart on the pages; it is a packaging variant of mla_decode.
 *
 * Arguments and results are those of mla_decode minus workspace and
 * workspace_bytes.  The workspace is a fixed MLA_NOALLOC_SCRATCH_BYTES static
 * device array inside the library: every GPU that loads the library holds it
 * until the process exits, and the call allocates nothing.  A request whose
 * workspace (mla_decode_workspace_bytes with the same sizes and splits) would
 * exceed it returns MLA_ERR_WORKSPACE; pass a small `splits` (for example 4)
 * to fit larger batches, since split-KV partial results dominate the size.
 * The first call on each device looks up the array's device address (with
 * that device current).  With CUDA's lazy module loading that lookup is also
 * what loads the library's device code on that device and reserves the
 * array, and it may synchronise the device: make the first call during
 * set-up, before any stream capture.  The address is cached per device for
 * the life of the process; it is no longer valid after the device is reset
 * (cudaDeviceReset), so do not call this entry point again after a reset.
 * Argument checks and their order are mla_decode's (an empty problem returns
 * MLA_OK without touching the device); a call that returns an error
 * enqueued nothing and mla_last_launch_count then reports 0.
 * All calls share the one array and it keeps the last call's contents (no
 * region needs clearing: each is written before it is read), so calls whose
 * execution overlaps on the GPU -- on different streams, or from different
 * host threads -- race with each other; serialise them. */
MLA_API int mla_decode_noalloc(const mla_dims* dims, int32_t batch, int32_t n_q,
                               const void* q_nope, const void* q_rope, const void* W_uk,
                               const void* W_uv, const void* cache, int64_t capacity,
                               const int32_t* seq_lens, int64_t max_len, void* out,
                               int32_t splits, int32_t* status, void* stream);

/* Waits for `stream`, copies the status word to *host_status and resets it to
 * MLA_OK.  Returns MLA_OK or MLA_ERR_CUDA. */
MLA_API int mla_get_status(int32_t* status, void* stream, int32_t* host_status);

/* Name of a status code ("MLA_OK", "MLA_ERR_LEN", ...). */
MLA_API const char* mla_status_string(int code);

/* Number of CUDA kernels the most recent mla_decode / mla_append call on this
 * host thread enqueued (for launch accounting). */
MLA_API int32_t mla_last_launch_count(void);

/* Per-kernel timing on the launching stream.  mla_profile_enable(1) makes
 * every later call record a CUDA event before and after each kernel it
 * enqueues (events are created on first use and destroyed by
 * mla_profile_enable(0); no device memory is involved).  mla_profile_read
 * waits for the recorded events and returns, per kernel name, the launch
 * count and the summed milliseconds since the previous read:
 *   names      host buffer receiving NUL-separated kernel names
 *   counts     host int32[max_kernels]; total_ms host float[max_kernels]
 * Returns the number of kernel names written (>= 0), or -MLA_ERR_CUDA /
 * -MLA_ERR_ARG. */
MLA_API int mla_profile_enable(int on);
MLA_API int mla_profile_read(char* names, size_t names_len, int32_t* counts, float* total_ms,
                             int32_t max_kernels);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H */
