// CUDA-core (FFMA) kernels of the decode step for any head geometry.
//
// These serve the fp32 dtype, where the bf16 tensor-core path cannot meet an
// fp32 accuracy bar, and bf16 problems whose geometry is not the DeepSeek-V3
// one.  All arithmetic is float with float accumulation.  The step follows
// the absorbed form ("Understanding MLA (Multi-head Latent Attention)",
// section 4: W_K moves to the query side; aicassindra "Multi-head latent
// attention", "End-to-end flow": score against the cached latents, weight
// them, up-project with W_UV):
//   absorb   q_lat = [W_uk[h] q_nope || RoPE(q_rope, p)]
//   attend   per key split: online softmax over scale * <q_lat, cache row>,
//            latent output and log-sum-exp of the split
//   combine  merge the splits by their log-sum-exp
//   upproj   out = o_lat W_uv[h]
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "profile.h"

namespace mla {
namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 32;  // keys scored per step of the attend loop

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
absorb_kernel(mla_dims d, int n_q, const T* __restrict__ q_nope, const T* __restrict__ q_rope,
              const T* __restrict__ W_uk, const int32_t* __restrict__ seq_lens, int64_t capacity,
              int64_t max_len, float* __restrict__ q_lat, int32_t* status) {
    extern __shared__ float smem[];
    const int bj = blockIdx.x, h = blockIdx.y;
    const int b = bj / n_q, j = bj % n_q;
    const int D = d.d_c + d.d_rope;
    float* row = q_lat + ((int64_t)bj * d.heads + h) * D;
    const int64_t len = seq_lens[b];
    if (!len_ok(len, n_q, capacity, max_len)) {
        if (threadIdx.x == 0 && h == 0 && j == 0) set_status(status, MLA_ERR_LEN);
        for (int i = threadIdx.x; i < D; i += blockDim.x) row[i] = 0.f;
        return;
    }
    const int64_t p = query_pos(len, n_q, j);
    const T* qn = q_nope + ((int64_t)bj * d.heads + h) * d.qk_nope;
    for (int k = threadIdx.x; k < d.qk_nope; k += blockDim.x) smem[k] = to_f32(qn[k]);
    __syncthreads();
    const T* W = W_uk + (int64_t)h * d.d_c * d.qk_nope;
    for (int i = threadIdx.x; i < d.d_c; i += blockDim.x) {
        float acc = 0.f;
        for (int k = 0; k < d.qk_nope; ++k) acc = fmaf(to_f32(W[(int64_t)i * d.qk_nope + k]), smem[k], acc);
        row[i] = acc;
    }
    const T* qr = q_rope + ((int64_t)bj * d.heads + h) * d.d_rope;
    for (int r = threadIdx.x; r < d.d_rope / 2; r += blockDim.x) {
        float y0, y1;
        rope_pair(to_f32(qr[2 * r]), to_f32(qr[2 * r + 1]), p, r, d.d_rope, d.rope_base, &y0, &y1);
        row[d.d_c + 2 * r] = y0;
        row[d.d_c + 2 * r + 1] = y1;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
attend_kernel(mla_dims d, int n_q, int splits, const float* __restrict__ q_lat,
              const T* __restrict__ cache, int64_t capacity, const int32_t* __restrict__ seq_lens,
              int64_t max_len, float* __restrict__ part_o, float* __restrict__ part_lse) {
    extern __shared__ float smem[];
    const int D = d.d_c + d.d_rope;
    float* q = smem;                 // [D]
    float* o = q + D;                // [d_c]
    float* sc = o + d.d_c;           // [kChunk] scores, then weights
    const int idx = blockIdx.x, s = blockIdx.y;
    const int bj = idx / d.heads, h = idx % d.heads;
    const int b = bj / n_q, j = bj % n_q;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    float* po = part_o + (((int64_t)bj * splits + s) * d.heads + h) * d.d_c;
    float* pl = part_lse + ((int64_t)bj * splits + s) * d.heads + h;
    const int64_t len = seq_lens[b];
    int64_t kb = 0, ke = 0;
    if (len_ok(len, n_q, capacity, max_len)) {
        const int64_t chunk = (max_len + splits - 1) / splits;
        kb = (int64_t)s * chunk;
        ke = min(kb + chunk, query_pos(len, n_q, j) + 1);
    }
    if (ke <= kb) {  // nothing visible in this split (or an invalid length)
        for (int i = threadIdx.x; i < d.d_c; i += blockDim.x) po[i] = 0.f;
        if (threadIdx.x == 0) *pl = -INFINITY;
        return;
    }
    const float* qsrc = q_lat + ((int64_t)bj * d.heads + h) * D;
    for (int i = threadIdx.x; i < D; i += blockDim.x) q[i] = qsrc[i];
    for (int i = threadIdx.x; i < d.d_c; i += blockDim.x) o[i] = 0.f;
    __syncthreads();
    const T* base = cache + (int64_t)b * capacity * D;
    float m = -INFINITY, l = 0.f;
    for (int64_t n0 = kb; n0 < ke; n0 += kChunk) {
        for (int kk = warp; kk < kChunk; kk += nwarps) {
            const int64_t n = n0 + kk;
            float acc = 0.f;
            if (n < ke) {
                const T* r = base + n * D;
                for (int i = lane; i < D; i += 32) acc = fmaf(q[i], to_f32(r[i]), acc);
            }
            acc = warp_sum(acc);
            if (lane == 0) sc[kk] = (n < ke) ? acc * d.softmax_scale : -INFINITY;
        }
        __syncthreads();
        float cmax = -INFINITY;
        for (int kk = 0; kk < kChunk; ++kk) cmax = fmaxf(cmax, sc[kk]);
        const float m_new = fmaxf(m, cmax);
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
        __syncthreads();  // every thread has read the raw scores
        if (threadIdx.x < kChunk) {
            const int64_t n = n0 + threadIdx.x;
            sc[threadIdx.x] = (n < ke) ? expf(sc[threadIdx.x] - m_new) : 0.f;
        }
        __syncthreads();
        float psum = 0.f;
        for (int kk = 0; kk < kChunk; ++kk) psum += sc[kk];
        const int kmax = (int)min((int64_t)kChunk, ke - n0);
        for (int i = threadIdx.x; i < d.d_c; i += blockDim.x) {
            float acc = o[i] * alpha;
            for (int kk = 0; kk < kmax; ++kk) acc = fmaf(sc[kk], to_f32(base[(n0 + kk) * D + i]), acc);
            o[i] = acc;
        }
        l = l * alpha + psum;
        m = m_new;
        __syncthreads();
    }
    const float inv = 1.f / l;
    for (int i = threadIdx.x; i < d.d_c; i += blockDim.x) po[i] = o[i] * inv;
    if (threadIdx.x == 0) *pl = m + logf(l);
}

__global__ void __launch_bounds__(kThreads)
combine_kernel(mla_dims d, int splits, const float* __restrict__ part_o,
               const float* __restrict__ part_lse, float* __restrict__ o_lat) {
    const int bj = blockIdx.x, h = blockIdx.y;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, part_lse[((int64_t)bj * splits + s) * d.heads + h]);
    float* dst = o_lat + ((int64_t)bj * d.heads + h) * d.d_c;
    if (M == -INFINITY) {  // invalid sequence: zero output
        for (int i = threadIdx.x; i < d.d_c; i += blockDim.x) dst[i] = 0.f;
        return;
    }
    float wsum = 0.f;
    for (int s = 0; s < splits; ++s) wsum += expf(part_lse[((int64_t)bj * splits + s) * d.heads + h] - M);
    const float inv = 1.f / wsum;
    for (int i = threadIdx.x; i < d.d_c; i += blockDim.x) {
        float acc = 0.f;
        for (int s = 0; s < splits; ++s) {
            const float w = expf(part_lse[((int64_t)bj * splits + s) * d.heads + h] - M);
            if (w != 0.f) acc = fmaf(w, part_o[(((int64_t)bj * splits + s) * d.heads + h) * d.d_c + i], acc);
        }
        dst[i] = acc * inv;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
upproj_kernel(mla_dims d, const float* __restrict__ o_lat, const T* __restrict__ W_uv,
              T* __restrict__ out) {
    extern __shared__ float smem[];
    const int bj = blockIdx.x, h = blockIdx.y;
    const float* src = o_lat + ((int64_t)bj * d.heads + h) * d.d_c;
    for (int i = threadIdx.x; i < d.d_c; i += blockDim.x) smem[i] = src[i];
    __syncthreads();
    const T* W = W_uv + (int64_t)h * d.d_c * d.v_dim;
    T* dst = out + ((int64_t)bj * d.heads + h) * d.v_dim;
    for (int v = threadIdx.x; v < d.v_dim; v += blockDim.x) {
        float acc = 0.f;
        for (int i = 0; i < d.d_c; ++i) acc = fmaf(smem[i], to_f32(W[(int64_t)i * d.v_dim + v]), acc);
        dst[v] = from_f32<T>(acc);
    }
}

template <typename T>
__global__ void rope_kernel(int64_t n_rows, int d_rope, float base, T* x, int64_t row_stride,
                            const int32_t* __restrict__ positions) {
    const int half = d_rope / 2;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n_rows * half) return;
    const int64_t r = t / half;
    const int i = (int)(t % half);
    T* p = x + r * row_stride + 2 * i;
    float y0, y1;
    rope_pair(to_f32(p[0]), to_f32(p[1]), positions[r], i, d_rope, base, &y0, &y1);
    p[0] = from_f32<T>(y0);
    p[1] = from_f32<T>(y1);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
append_kernel(mla_dims d, int n_new, int hidden, const T* __restrict__ x,
              const T* __restrict__ W_dkv, const int32_t* __restrict__ positions, T* cache,
              int64_t capacity, int32_t* status) {
    extern __shared__ float xs[];
    const int m = blockIdx.x;
    const int D = d.d_c + d.d_rope;
    const int64_t pos = positions[m];
    if (pos < 0 || pos >= capacity) {
        if (threadIdx.x == 0 && blockIdx.y == 0) set_status(status, MLA_ERR_POS);
        return;
    }
    for (int k = threadIdx.x; k < hidden; k += blockDim.x) xs[k] = to_f32(x[(int64_t)m * hidden + k]);
    __syncthreads();
    const int n = 2 * (blockIdx.y * blockDim.x + threadIdx.x);
    if (n >= D) return;
    float a0 = 0.f, a1 = 0.f;
    for (int k = 0; k < hidden; ++k) {
        a0 = fmaf(xs[k], to_f32(W_dkv[(int64_t)k * D + n]), a0);
        a1 = fmaf(xs[k], to_f32(W_dkv[(int64_t)k * D + n + 1]), a1);
    }
    if (n >= d.d_c) {  // rope key: rotate the pair at the token's position
        float y0, y1;
        rope_pair(a0, a1, pos, (n - d.d_c) / 2, d.d_rope, d.rope_base, &y0, &y1);
        a0 = y0;
        a1 = y1;
    }
    const int b = m / n_new;
    T* dst = cache + ((int64_t)b * capacity + pos) * D + n;
    dst[0] = from_f32<T>(a0);
    dst[1] = from_f32<T>(a1);
}

int check(int* launches) {
    if (launches) ++*launches;
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

template <typename T>
int decode_t(const DecodeCall& c, int* launches) {
    const mla_dims& d = c.d;
    const int D = d.d_c + d.d_rope, S = c.L.splits, BJ = c.batch * c.n_q;
    float* q_lat = reinterpret_cast<float*>(c.ws + c.L.q_lat);
    float* o_lat = reinterpret_cast<float*>(c.ws + c.L.o_lat);
    float* part_o = reinterpret_cast<float*>(c.ws + c.L.part_o);
    float* part_lse = reinterpret_cast<float*>(c.ws + c.L.part_lse);
    int rc;
    prof_begin(c.stream, "generic_absorb");
    absorb_kernel<T><<<dim3(BJ, d.heads), kThreads, d.qk_nope * sizeof(float), c.stream>>>(
        d, c.n_q, (const T*)c.q_nope, (const T*)c.q_rope, (const T*)c.W_uk, c.seq_lens, c.capacity,
        c.max_len, q_lat, c.status);
    prof_end(c.stream);
    if ((rc = check(launches))) return rc;
    const size_t att_smem = (size_t)(D + d.d_c + kChunk) * sizeof(float);
    prof_begin(c.stream, "generic_attend");
    attend_kernel<T><<<dim3(BJ * d.heads, S), kThreads, att_smem, c.stream>>>(
        d, c.n_q, S, q_lat, (const T*)c.cache, c.capacity, c.seq_lens, c.max_len, part_o, part_lse);
    prof_end(c.stream);
    if ((rc = check(launches))) return rc;
    prof_begin(c.stream, "generic_combine");
    combine_kernel<<<dim3(BJ, d.heads), kThreads, 0, c.stream>>>(d, S, part_o, part_lse, o_lat);
    prof_end(c.stream);
    if ((rc = check(launches))) return rc;
    prof_begin(c.stream, "generic_upproj");
    upproj_kernel<T><<<dim3(BJ, d.heads), kThreads, d.d_c * sizeof(float), c.stream>>>(
        d, o_lat, (const T*)c.W_uv, (T*)c.out);
    prof_end(c.stream);
    return check(launches);
}

template <typename T>
int append_t(const AppendCall& c, int* launches) {
    const int D = c.d.d_c + c.d.d_rope;
    const int M = c.batch * c.n_new;
    const dim3 grid(M, (D / 2 + kThreads - 1) / kThreads);
    const size_t smem = (size_t)c.hidden * sizeof(float);
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(append_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return MLA_ERR_CUDA;
    }
    prof_begin(c.stream, "generic_append");
    append_kernel<T><<<grid, kThreads, smem, c.stream>>>(c.d, c.n_new, c.hidden, (const T*)c.x,
                                                       (const T*)c.W_dkv, c.positions, (T*)c.cache,
                                                       c.capacity, c.status);
    prof_end(c.stream);
    return check(launches);
}

}  // namespace

void generic_layout(const mla_dims& d, int batch, int n_q, int64_t max_len, int splits,
                    mla_ws_layout* L) {
    const int64_t BJ = (int64_t)batch * n_q;
    const int D = d.d_c + d.d_rope;
    int S = splits;
    if (S <= 0) S = (int)std::min<int64_t>(64, std::max<int64_t>(1, (max_len + 511) / 512));
    *L = mla_ws_layout{};
    size_t off = 0;
    auto take = [&](size_t bytes, size_t* o, size_t* sz) {
        *o = off;
        *sz = bytes;
        off = align_up(off + bytes, 256);
    };
    take(BJ * d.heads * D * sizeof(float), &L->q_lat, &L->q_lat_bytes);
    take(BJ * d.heads * d.d_c * sizeof(float), &L->o_lat, &L->o_lat_bytes);
    take(BJ * S * d.heads * d.d_c * sizeof(float), &L->part_o, &L->part_o_bytes);
    take(BJ * S * d.heads * sizeof(float), &L->part_lse, &L->part_lse_bytes);
    L->total = off;
    L->compute_dtype = MLA_FP32;
    L->splits = S;
}

int generic_decode(const DecodeCall& c, int* launches) {
    return c.d.dtype == MLA_FP32 ? decode_t<float>(c, launches) : decode_t<__nv_bfloat16>(c, launches);
}

int generic_append(const AppendCall& c, int* launches) {
    return c.d.dtype == MLA_FP32 ? append_t<float>(c, launches) : append_t<__nv_bfloat16>(c, launches);
}

namespace {

// RMSNorm of the latent of each appended row, in place ("Understanding MLA",
// Phase A step A2): row[0:d_c] = gamma * row / sqrt(mean(row^2) + 1e-6), the
// rope columns untouched.  One block per new token; rows whose position is
// outside the cache were not written (the append kernel set MLA_ERR_POS).
template <typename T>
__global__ void rms_rows_kernel(int d_c, int D, int n_new, const int32_t* __restrict__ positions,
                                const float* __restrict__ gamma, T* cache, int64_t capacity) {
    __shared__ float part[32];
    const int m = blockIdx.x;
    const int64_t pos = positions[m];
    if (pos < 0 || pos >= capacity) return;
    T* row = cache + ((int64_t)(m / n_new) * capacity + pos) * D;
    float ss = 0.f;
    for (int i = threadIdx.x; i < d_c; i += blockDim.x) {
        const float v = to_f32(row[i]);
        ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.f;
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) part[0] = v;
    }
    __syncthreads();
    const float inv = 1.f / sqrtf(part[0] / (float)d_c + 1e-6f);
    for (int i = threadIdx.x; i < d_c; i += blockDim.x) row[i] = from_f32<T>(gamma[i] * to_f32(row[i]) * inv);
}

}  // namespace

namespace {

// y[t][n] = sum_k x[t][k] W[k][n]: one thread per output element, float
// accumulation (the CUDA-core output projection).
template <typename T>
__global__ void gemm_xw_kernel(const T* __restrict__ x, const T* __restrict__ W, int M, int K, int n_out,
                               T* __restrict__ y) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= n_out) return;
    for (int t = blockIdx.y; t < M; t += gridDim.y) {
        float acc = 0.f;
        for (int k = 0; k < K; ++k)
            acc = fmaf(to_f32(x[(int64_t)t * K + k]), to_f32(W[(int64_t)k * n_out + n]), acc);
        y[(int64_t)t * n_out + n] = from_f32<T>(acc);
    }
}

}  // namespace

int generic_gemm_xw(mla_dtype dtype, const void* x, const void* W, int M, int K, int n_out, void* y,
                    cudaStream_t stream, int* launches) {
    const dim3 grid((n_out + 127) / 128, M < 65535 ? M : 65535);
    prof_begin(stream, "generic_oproj");
    if (dtype == MLA_FP32)
        gemm_xw_kernel<float><<<grid, 128, 0, stream>>>((const float*)x, (const float*)W, M, K, n_out, (float*)y);
    else
        gemm_xw_kernel<__nv_bfloat16><<<grid, 128, 0, stream>>>((const __nv_bfloat16*)x, (const __nv_bfloat16*)W, M,
                                                                K, n_out, (__nv_bfloat16*)y);
    prof_end(stream);
    if (launches) ++*launches;
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int rms_norm_rows(const AppendCall& c, int* launches) {
    const int M = c.batch * c.n_new, D = c.d.d_c + c.d.d_rope;
    if (M == 0) return MLA_OK;
    prof_begin(c.stream, "rms_norm_rows");
    if (c.d.dtype == MLA_FP32)
        rms_rows_kernel<float><<<M, 128, 0, c.stream>>>(c.d.d_c, D, c.n_new, c.positions, c.rms_gamma,
                                                        (float*)c.cache, c.capacity);
    else
        rms_rows_kernel<__nv_bfloat16><<<M, 128, 0, c.stream>>>(c.d.d_c, D, c.n_new, c.positions, c.rms_gamma,
                                                                (__nv_bfloat16*)c.cache, c.capacity);
    prof_end(c.stream);
    if (launches) ++*launches;
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int rope_rows(const mla_dims& d, int64_t n_rows, void* x, int64_t row_stride,
              const int32_t* positions, cudaStream_t stream) {
    const int64_t total = n_rows * (d.d_rope / 2);
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    if (d.dtype == MLA_FP32)
        rope_kernel<float><<<(unsigned)blocks, threads, 0, stream>>>(n_rows, d.d_rope, d.rope_base,
                                                                   (float*)x, row_stride, positions);
    else
        rope_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, stream>>>(
            n_rows, d.d_rope, d.rope_base, (__nv_bfloat16*)x, row_stride, positions);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
