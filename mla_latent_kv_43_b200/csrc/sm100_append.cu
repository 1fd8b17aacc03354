// Cache append (and the output projection's plain product) on tcgen05 tensor cores.
//
// For the new tokens m (x [M][hidden], M = batch * n_new) at their slots
// pos_m ("Understanding MLA (Multi-head Latent Attention)", Phase A step A1
// and Phase B step B2; aicassindra "Multi-head latent attention", the append
// step of "End-to-end flow"):
//     y[m][n] = sum_k x[m][k] W_dkv[k][n]                       n < 576
//     cache[b][pos_m][n] = y[m][n]                              n < 512 (latent)
//     cache[b][pos_m][512 + 2i .. +1] = RoPE(y[m][512 + 2i .. +1], pos_m)
//
// Work split.  The transposed product D = W_dkv^T x^T puts 128 output features
// on the M dimension (5 feature tiles; the last one holds the 64 rope
// features, the rest of its box is zero fill) and the tokens on N; W_dkv is
// read as an MN-major A operand straight from its [hidden][576] layout.  K =
// hidden is split across a cluster of 8 CTAs, so 40 SMs stream the 8.3 MB of
// weights.  Each CTA leaves its fp32 partial in shared memory; after a cluster
// barrier CTA r sums feature rows [16r, 16r + 16) of the tile over the eight
// partials through distributed shared memory, rotates the rope pairs and
// stores bf16 cache entries.
//
// The output projection ("Understanding MLA", Phase D step D2: the heads'
// outputs flattened and projected to the hidden width) is the same product
// y = x W with x = the decode output [tokens][heads * v_dim] and W = W_O
// [heads * v_dim][hidden]; the same kernel stores y rows instead of cache
// entries.
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
constexpr int kSplitMax = 8;             // CTAs per cluster splitting K (the append's split)
constexpr int kStages = 4;
constexpr int kBoxA = 8192;              // 64 k rows x 64 features x 2 B
constexpr int kMaxN = 256;               // tokens per launch tile
constexpr int kFeatures = 576;

struct AppendArgs {
    int M, n_new, kblocks, N;            // tokens, tokens per sequence, k blocks of 64, token tile
    int n_out;                           // output width: 576 for the append, the hidden width for W_O
    __nv_bfloat16* y;                    // plain product [M][n_out] (the output projection)
    const int32_t* positions;
    __nv_bfloat16* cache;
    int64_t capacity;
    uint64_t rope_turn[32];              // pair frequencies, fractions of a turn (rope_turn_table)
    int32_t* status;
};

__host__ __device__ constexpr uint32_t tmem_cols_for(int n) {
    return n <= 32 ? 32u : (n <= 64 ? 64u : (n <= 128 ? 128u : 256u));
}

// kAppend: rotate the rope features and store cache entries at the tokens'
// slots; otherwise store the plain product y = x W (the output projection).
// kSplit CTAs of a cluster share one 128-feature tile, each over 1/kSplit of K.
template <bool kAppend, int kSplit>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(kThreads, 1)
append_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapX, AppendArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kStages], empty[kStages], done;
    __shared__ uint32_t tmem_base;
    __shared__ int flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x / kSplit, nt = blockIdx.y;
    const uint32_t rank = cluster_rank();
    const int N = a.N;
    const int stage_bytes = 2 * kBoxA + N * 128;
    const int kb0 = (int)((int64_t)rank * a.kblocks / kSplit), kb1 = (int)((int64_t)(rank + 1) * a.kblocks / kSplit);
    const int nk = kb1 - kb0;
    const uint32_t ncols = tmem_cols_for(N);
    // fp32 partial [128 rows][N], row stride N * 4 + 16 bytes; aliases the stages once the MMAs are done
    const int row_bytes = N * 4 + 16;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done, 1);
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
    grid_dep_wait();         // no-op under a plain launch

    if (warp == 0) {
        if (elect_one()) {
            for (int i = 0; i < nk; ++i) {
                const int s = i % kStages, kb = kb0 + i;
                if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, nullptr)) break;
                uint8_t* st = smem + s * stage_bytes;
                mbar_expect_tx(&full[s], stage_bytes);
                tma_load_2d(st, &mapW, &full[s], 128 * mt, kb * 64);
                tma_load_2d(st + kBoxA, &mapW, &full[s], 128 * mt + 64, kb * 64);
                tma_load_2d(st + 2 * kBoxA, &mapX, &full[s], kb * 64, nt * N);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // whole warp, one elected lane issues
        const uint32_t idesc = idesc_bf16(128, N, true, false);
        const uint64_t da = sdesc(smem_u32(smem), kBoxA, 1024, kSwizzle128);
        const uint64_t db = sdesc(smem_u32(smem) + 2 * kBoxA, 16, 1024, kSwizzle128);
        for (int i = 0; i < nk; ++i) {
            const int s = i % kStages;
            int ready = 0;
            if (lane == 0) ready = mbar_wait(&full[s], (i / kStages) & 1, nullptr) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ready, 0)) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ss_w(tmem, sdesc_add(da, s * stage_bytes + ks * 2048), sdesc_add(db, s * stage_bytes + ks * 32),
                         idesc, (i | ks) ? 1u : 0u);
            mma_commit_w(&empty[s]);
        }
        mma_commit_w(&done);
    }
    __syncwarp();
    grid_dep_trigger();

    // every MMA of this CTA done: TMEM row t (feature 128 mt + t) -> smem partial row t
    if (threadIdx.x == 0) {
        flag = mbar_wait(&done, 0, nullptr) ? 1 : 0;
        if (!flag) set_status(a.status, MLA_ERR_TIMEOUT);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t part = smem_u32(smem);
    const int t = threadIdx.x;
    for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t r[16];
        if (nk > 0 && flag) {
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(part + t * row_bytes + (c0 + 4 * j) * 4),
                         "r"(r[4 * j]), "r"(r[4 * j + 1]), "r"(r[4 * j + 2]), "r"(r[4 * j + 3])
                         : "memory");
    }
    tc_fence_before();
    cluster_sync();          // every partial of the cluster is in place

    // CTA `rank` finishes feature rows [R rank, R rank + R) of the tile, R = 128 /
    // kSplit: thread (pair p, token group g) sums rows 2p, 2p + 1 for tokens
    // 4g .. 4g + 3 (+ multiples of 4 * kGroups).
    constexpr int kRows = 128 / kSplit, kGroups = kThreads / (kRows / 2);
    static_assert(kRows % 2 == 0 && kThreads % (kRows / 2) == 0, "feature rows per CTA");
    const int p = t / kGroups, g = t % kGroups;
    const int row = kRows * (int)rank + 2 * p;
    const int n = 128 * mt + row;
    uint32_t peer_part[kSplit];
#pragma unroll
    for (int c = 0; c < kSplit; ++c) peer_part[c] = map_peer(part, (uint32_t)c);
    for (int m4 = 4 * g; m4 < N; m4 += 4 * kGroups) {
        float v0[4] = {0.f, 0.f, 0.f, 0.f}, v1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < kSplit; ++c) {
            float4 u0, u1;
            asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(u0.x), "=f"(u0.y), "=f"(u0.z), "=f"(u0.w)
                         : "r"(peer_part[c] + row * row_bytes + m4 * 4));
            asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(u1.x), "=f"(u1.y), "=f"(u1.z), "=f"(u1.w)
                         : "r"(peer_part[c] + (row + 1) * row_bytes + m4 * 4));
            v0[0] += u0.x; v0[1] += u0.y; v0[2] += u0.z; v0[3] += u0.w;
            v1[0] += u1.x; v1[1] += u1.y; v1[2] += u1.z; v1[3] += u1.w;
        }
        if (n >= a.n_out) continue;                    // zero fill past the last feature
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = nt * N + m4 + i;
            if (m >= a.M) break;
            if constexpr (!kAppend) {
                *reinterpret_cast<uint32_t*>(a.y + (int64_t)m * a.n_out + n) = pack_bf16(v0[i], v1[i]);
                continue;
            }
            const int64_t pos = a.positions[m];
            if (pos < 0 || pos >= a.capacity) {
                set_status(a.status, MLA_ERR_POS);
                continue;
            }
            float y0 = v0[i], y1 = v1[i];
            if (n >= 512) rope_pair_turn_bf16(v0[i], v1[i], pos, a.rope_turn[(n - 512) >> 1], &y0, &y1);
            const int b = m / a.n_new;
            *reinterpret_cast<uint32_t*>(a.cache + ((int64_t)b * a.capacity + pos) * kFeatures + n) = pack_bf16(y0, y1);
        }
    }
    cluster_sync();          // no CTA frees its smem while a peer may still read it
    if (warp == 1) tmem_dealloc(tmem, ncols);
}

}  // namespace

int append_launch(const AppendCall& c, int* launches) {
    const int M = c.batch * c.n_new;
    int N = (M + 15) / 16 * 16;
    if (N > kMaxN) N = kMaxN;
    CUtensorMap mw, mx;
    {
        const uint64_t dims[2] = {(uint64_t)kFeatures, (uint64_t)c.hidden}, str[1] = {kFeatures * 2};
        const uint32_t box[2] = {64, 64};
        if (!make_map(&mw, c.W_dkv, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        const uint64_t dims[2] = {(uint64_t)c.hidden, (uint64_t)M}, str[1] = {(uint64_t)c.hidden * 2};
        const uint32_t box[2] = {64, (uint32_t)N};
        if (!make_map(&mx, c.x, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    AppendArgs a{};
    a.M = M;
    a.n_out = kFeatures;
    a.n_new = c.n_new;
    a.kblocks = (c.hidden + 63) / 64;
    a.N = N;
    a.positions = c.positions;
    a.cache = (__nv_bfloat16*)c.cache;
    a.capacity = c.capacity;
    rope_turn_table(c.d.rope_base, 64, a.rope_turn);
    a.status = c.status;
    const int stage_bytes = 2 * kBoxA + N * 128;
    const int part_bytes = 128 * (N * 4 + 16);
    const size_t smem = (size_t)(kStages * stage_bytes > part_bytes ? kStages * stage_bytes : part_bytes) + 1024;
    if (cudaFuncSetAttribute(append_kernel<true, kSplitMax>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    const dim3 grid((kFeatures + 127) / 128 * kSplitMax, (M + N - 1) / N);
    prof_begin(c.stream, "sm100_append");
    const cudaError_t e =
        launch_plain(append_kernel<true, kSplitMax>, grid, dim3(kThreads), smem, c.stream, mw, mx, a);
    prof_end(c.stream);
    if (launches) ++*launches;
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

// y [M][n_out] = x [M][K] W [K][n_out], bf16 in and out, fp32 accumulation:
// the same split-K cluster kernel without the cache epilogue.
int gemm_xw_launch(const void* x, const void* W, int M, int K, int n_out, __nv_bfloat16* y, int32_t* status,
                   cudaStream_t stream, const char* name, int* launches) {
    int N = (M + 15) / 16 * 16;
    if (N > kMaxN) N = kMaxN;
    if ((M + N - 1) / N > 65535) return MLA_ERR_UNSUPPORTED;    // token tiles on grid.y
    CUtensorMap mw, mx;
    {
        const uint64_t dims[2] = {(uint64_t)n_out, (uint64_t)K}, str[1] = {(uint64_t)n_out * 2};
        const uint32_t box[2] = {64, 64};
        if (!make_map(&mw, W, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M}, str[1] = {(uint64_t)K * 2};
        const uint32_t box[2] = {64, (uint32_t)N};
        if (!make_map(&mx, x, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    AppendArgs a{};
    a.M = M;
    a.n_out = n_out;
    a.y = y;
    a.n_new = 1;
    a.kblocks = (K + 63) / 64;
    a.N = N;
    a.status = status;
    const int stage_bytes = 2 * kBoxA + N * 128;
    const int part_bytes = 128 * (N * 4 + 16);
    const size_t smem = (size_t)(kStages * stage_bytes > part_bytes ? kStages * stage_bytes : part_bytes) + 1024;
    // the widest split whose grid still runs in one wave (two CTAs per SM when
    // their shared memory fits: a 448-CTA grid at 7168 columns took 1.5 waves)
    const int tiles = (n_out + 127) / 128 * ((M + N - 1) / N);
    const int per_sm = smem <= 112 * 1024 ? 2 : 1;
    int split = kSplitMax;
    while (split > 2 && tiles * split > per_sm * sm_count()) split /= 2;
    auto kern = split == 8 ? append_kernel<false, 8> : split == 4 ? append_kernel<false, 4> : append_kernel<false, 2>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    const dim3 grid((n_out + 127) / 128 * split, (M + N - 1) / N);
    prof_begin(stream, name);
    const cudaError_t e = launch_plain(kern, grid, dim3(kThreads), smem, stream, mw, mx, a);
    prof_end(stream);
    if (launches) ++*launches;
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100

bool sm100_append_supported(const mla_dims& d, int hidden) {
    return d.dtype == MLA_BF16 && d.d_c == 512 && d.d_rope == 64 && hidden % 8 == 0;
}

int sm100_append(const AppendCall& c, int* launches) { return sm100::append_launch(c, launches); }

}  // namespace mla
