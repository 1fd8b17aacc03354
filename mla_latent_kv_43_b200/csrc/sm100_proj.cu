// Per-head projections of the decode step on tcgen05 tensor cores.
//
// absorb  ("Understanding MLA (Multi-head Latent Attention)", section 4:
//          the key up-projection is moved to the query side)
//     q_lat[n][h][i] = sum_k W_uk[h][i][k] q_nope[n][h][k]          i < 512
//     q_lat[n][h][512 + r] = RoPE(q_rope[n][h], p_n)[r]              (Phase C, step C2)
//   plus the key-tile plan of the attention kernel (tiles per query token).
// upproj  (aicassindra "Multi-head latent attention", "End-to-end flow": the
//          value up-projection applied to the weighted latent)
//     out[n][h][v] = sum_i W_uv[h][i][v] o_lat[n][h][i]
//
// Both are batched over heads: one CTA computes a 128 x N tile D = A_h B_h^T
// with M = 128 weight rows, N = query tokens, K = 128 (absorb) or 512
// (upproj).  The weight tile is the A operand (K-major W_uk rows; MN-major
// W_uv columns), the activations the K-major B operand, staged by TMA with
// 128-byte swizzle, accumulated in TMEM, written back as bf16.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "profile.h"
#include "sm100_host.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {
namespace {

constexpr int kThreads = 128;
constexpr int kStages = 4;
constexpr int kStageBytes = 32768;   // A k-block (16 KB) + B k-block (<= 16 KB)
constexpr int kKeysPerTile = 64;

struct ProjArgs {
    int BJ, H, n_q, n_tile;
    // absorb
    const __nv_bfloat16* q_rope;
    const int32_t* seq_lens;
    int64_t capacity, max_len;
    float rope_base;
    __nv_bfloat16* q_lat;
    int32_t* cum;            // [BJ + 1] key tiles prefix of each query token
    // upproj
    __nv_bfloat16* out;
    int32_t* status;
};

template <int MODE>  // 0: absorb, 1: upproj
struct ProjShape {
    static constexpr int kBlocks = MODE == 0 ? 2 : 8;   // K / 64
};

__device__ void plan_tiles(const ProjArgs& a, int tid) {
    // Tiles of 64 keys each query token attends; 0 for an invalid length.
    __shared__ int32_t part[kThreads + 1];
    const int per = (a.BJ + kThreads - 1) / kThreads;
    const int lo = min(a.BJ, tid * per), hi = min(a.BJ, lo + per);
    int32_t sum = 0;
    bool bad = false;
    for (int bj = lo; bj < hi; ++bj) {
        const int b = bj / a.n_q, j = bj % a.n_q;
        const int64_t len = a.seq_lens[b];
        if (len_ok(len, a.n_q, a.capacity, a.max_len))
            sum += (int32_t)((query_pos(len, a.n_q, j) + kKeysPerTile) / kKeysPerTile);
        else
            bad = true;
    }
    if (bad) set_status(a.status, MLA_ERR_LEN);
    part[tid + 1] = sum;
    if (tid == 0) part[0] = 0;
    __syncthreads();
    if (tid == 0)
        for (int i = 1; i <= kThreads; ++i) part[i] += part[i - 1];
    __syncthreads();
    int32_t run = part[tid];
    if (tid == 0) a.cum[0] = 0;
    for (int bj = lo; bj < hi; ++bj) {
        const int b = bj / a.n_q, j = bj % a.n_q;
        const int64_t len = a.seq_lens[b];
        if (len_ok(len, a.n_q, a.capacity, a.max_len))
            run += (int32_t)((query_pos(len, a.n_q, j) + kKeysPerTile) / kKeysPerTile);
        a.cum[bj + 1] = run;
    }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
proj_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB, ProjArgs a) {
    constexpr int KB = ProjShape<MODE>::kBlocks;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kStages], empty[kStages], done;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int h = blockIdx.x, mt = blockIdx.y, nt = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = a.n_tile;
    const uint32_t ncols = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t a_bytes = 16384, b_bytes = (uint32_t)N * 128;

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch(&mapA);
            tma_prefetch(&mapB);
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % kStages;
                if (kb >= kStages && !mbar_wait(&empty[s], ((kb / kStages) - 1) & 1, &abort_flag)) {
                    abort_flag = 1;
                    break;
                }
                uint8_t* sa = smem + s * kStageBytes;
                uint8_t* sb = sa + 16384;
                mbar_expect_tx(&full[s], a_bytes + b_bytes);
                if (MODE == 0) {
                    tma_load_2d(sa, &mapA, &full[s], kb * 64, h * 512 + mt * 128);
                } else {
                    tma_load_2d(sa, &mapA, &full[s], 0, h * 512 + kb * 64);
                    tma_load_2d(sa + 8192, &mapA, &full[s], 64, h * 512 + kb * 64);
                }
                tma_load_3d(sb, &mapB, &full[s], kb * 64, h, nt * N);
            }
        }
    } else if (warp == 1) {
        if (elect_one()) {
            const uint32_t idesc = idesc_bf16(128, N, MODE == 1, false);
            bool ok = true;
            for (int kb = 0; kb < KB && ok; ++kb) {
                const int s = kb % kStages;
                if (!mbar_wait(&full[s], (kb / kStages) & 1, &abort_flag)) {
                    abort_flag = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * kStageBytes), sb = sa + 16384;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = MODE == 0 ? sdesc(sa + ks * 32, 16, 1024, kSwizzle128)
                                                  : sdesc(sa + ks * 2048, 8192, 1024, kSwizzle128);
                    const uint64_t bd = sdesc(sb + ks * 32, 16, 1024, kSwizzle128);
                    mma_ss(tmem, ad, bd, idesc, (kb | ks) ? 1u : 0u);
                }
                mma_commit(&empty[s]);
            }
            mma_commit(&done);
        }
    }
    __syncwarp();

    // absorb extras while the MMAs run: query RoPE and the key-tile plan
    if (MODE == 0) {
        if (mt == 0) {
            for (int t = threadIdx.x; t < N * 32; t += kThreads) {
                const int n = nt * N + t / 32, r = t % 32;
                if (n >= a.BJ) continue;
                const int b = n / a.n_q, j = n % a.n_q;
                const int64_t p = query_pos(a.seq_lens[b], a.n_q, j);
                const __nv_bfloat16* qr = a.q_rope + ((int64_t)n * a.H + h) * 64;
                float y0, y1;
                rope_pair(__bfloat162float(qr[2 * r]), __bfloat162float(qr[2 * r + 1]), p, r, 64, a.rope_base, &y0,
                          &y1);
                __nv_bfloat16* dst = a.q_lat + ((int64_t)n * a.H + h) * 576 + 512 + 2 * r;
                dst[0] = __float2bfloat16_rn(y0);
                dst[1] = __float2bfloat16_rn(y1);
            }
        }
        if (h == 0 && mt == 0 && nt == 0) plan_tiles(a, threadIdx.x);
    }

    // epilogue: TMEM row (32*warp + lane) -> bf16 outputs
    const bool ok = mbar_wait(&done, 0, &abort_flag);
    tc_fence_after();
    if (!ok) {
        if (threadIdx.x == 0) set_status(a.status, MLA_ERR_TIMEOUT);
    } else {
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < N; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int n = nt * N + c0 + c;
                if (c0 + c >= N || n >= a.BJ) continue;
                const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r[c]));
                if (MODE == 0)
                    a.q_lat[((int64_t)n * a.H + h) * 576 + mt * 128 + m] = v;
                else
                    a.out[((int64_t)n * a.H + h) * 128 + m] = v;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, ncols);
}

int round_n(int bj) {
    int n = bj < 128 ? bj : 128;
    n = (n + 15) / 16 * 16;
    return n < 16 ? 16 : n;
}

template <int MODE>
int launch(const CUtensorMap& A, const CUtensorMap& B, const ProjArgs& a, dim3 grid, cudaStream_t st,
           const char* name, int* launches) {
    const size_t smem = kStages * kStageBytes + 1024;
    if (cudaFuncSetAttribute(proj_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return MLA_ERR_CUDA;
    prof_begin(st, name);
    proj_kernel<MODE><<<grid, kThreads, smem, st>>>(A, B, a);
    prof_end(st);
    if (launches) ++*launches;
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

// absorb + q-RoPE + plan.  q_nope [BJ][H][128], W_uk [H][512][128], q_rope [BJ][H][64]
int launch_absorb(const DecodeCall& c, __nv_bfloat16* q_lat, int32_t* cum, int* launches) {
    const int BJ = c.batch * c.n_q, H = c.d.heads, N = round_n(BJ);
    CUtensorMap A, B;
    {
        const uint64_t dims[2] = {128, (uint64_t)H * 512}, str[1] = {128 * 2};
        const uint32_t box[2] = {64, 128};
        if (!make_map(&A, c.W_uk, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        const uint64_t dims[3] = {128, (uint64_t)H, (uint64_t)BJ}, str[2] = {128 * 2, (uint64_t)H * 128 * 2};
        const uint32_t box[3] = {64, 1, (uint32_t)N};
        if (!make_map(&B, c.q_nope, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    ProjArgs a{};
    a.BJ = BJ;
    a.H = H;
    a.n_q = c.n_q;
    a.n_tile = N;
    a.q_rope = (const __nv_bfloat16*)c.q_rope;
    a.seq_lens = c.seq_lens;
    a.capacity = c.capacity;
    a.max_len = c.max_len;
    a.rope_base = c.d.rope_base;
    a.q_lat = q_lat;
    a.cum = cum;
    a.status = c.status;
    const dim3 grid(H, 4, (BJ + N - 1) / N);
    return launch<0>(A, B, a, grid, c.stream, "sm100_absorb", launches);
}

// up-projection.  o_lat [BJ][H][512] bf16, W_uv [H][512][128], out [BJ][H][128]
int launch_upproj(const DecodeCall& c, const __nv_bfloat16* o_lat, int* launches) {
    const int BJ = c.batch * c.n_q, H = c.d.heads, N = round_n(BJ);
    CUtensorMap A, B;
    {
        const uint64_t dims[2] = {128, (uint64_t)H * 512}, str[1] = {128 * 2};
        const uint32_t box[2] = {64, 64};
        if (!make_map(&A, c.W_uv, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        const uint64_t dims[3] = {512, (uint64_t)H, (uint64_t)BJ}, str[2] = {512 * 2, (uint64_t)H * 512 * 2};
        const uint32_t box[3] = {64, 1, (uint32_t)N};
        if (!make_map(&B, o_lat, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    ProjArgs a{};
    a.BJ = BJ;
    a.H = H;
    a.n_q = c.n_q;
    a.n_tile = N;
    a.out = (__nv_bfloat16*)c.out;
    a.status = c.status;
    const dim3 grid(H, 1, (BJ + N - 1) / N);
    return launch<1>(A, B, a, grid, c.stream, "sm100_upproj", launches);
}

}  // namespace sm100
}  // namespace mla
