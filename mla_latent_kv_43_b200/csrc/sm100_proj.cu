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
constexpr int kKeysPerTile = 64;

struct ProjArgs {
    int BJ, H, n_q, n_tile;
    // absorb
    const __nv_bfloat16* q_rope;
    const int32_t* seq_lens;
    int64_t capacity, max_len;
    uint64_t rope_turn[32];  // pair frequencies, fractions of a turn (rope_turn_table)
    __nv_bfloat16* q_lat;
    int32_t* cum;            // [BJ + 1] key tiles prefix of each query token
    int32_t* first_bj;       // [pairs] first query token of each attention cluster's tile range
    int pairs;
    const int32_t* n_sel;    // sparse decode: selected keys per query token (nullptr: dense)
    int max_sel;
    // upproj
    __nv_bfloat16* out;
    int32_t* status;
};

// Key tiles query token bj attends: its visible keys 0..p, or its selected
// keys in the sparse decode; 0 (and *bad) when its length or count is invalid.
__device__ __forceinline__ int32_t tiles_of(const ProjArgs& a, int bj, bool* bad) {
    const int b = bj / a.n_q, j = bj % a.n_q;
    const int64_t len = a.seq_lens[b];
    if (!len_ok(len, a.n_q, a.capacity, a.max_len)) {
        *bad = true;
        return 0;
    }
    const int64_t p = query_pos(len, a.n_q, j);
    if (a.n_sel) {
        const int32_t n = a.n_sel[bj];
        if (n < 1 || n > a.max_sel || (int64_t)n > p + 1) {
            *bad = true;
            return 0;
        }
        return (n + kKeysPerTile - 1) / kKeysPerTile;
    }
    return (int32_t)((p + kKeysPerTile) / kKeysPerTile);
}

__device__ void plan_tiles(const ProjArgs& a, int tid) {
    // Tiles of 64 keys each query token attends; 0 for an invalid length.
    __shared__ int32_t part[kThreads / 32];
    const int per = (a.BJ + kThreads - 1) / kThreads;
    const int lo = min(a.BJ, tid * per), hi = min(a.BJ, lo + per);
    int32_t sum = 0;
    bool bad = false;
    for (int bj = lo; bj < hi; ++bj) sum += tiles_of(a, bj, &bad);
    if (bad) set_status(a.status, MLA_ERR_LEN);
    // exclusive prefix of the per-thread sums: shuffle scan in each warp, then
    // the four warp totals
    const int lane = tid & 31, warp = tid >> 5;
    int32_t incl = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
    }
    if (lane == 31) part[warp] = incl;
    __syncthreads();
    int32_t run = incl - sum;
    for (int w = 0; w < warp; ++w) run += part[w];
    if (tid == 0) a.cum[0] = 0;
    const int32_t run_lo = run;                 // cum[lo]
    bool ignored = false;
    for (int bj = lo; bj < hi; ++bj) {
        run += tiles_of(a, bj, &ignored);
        a.cum[bj + 1] = run;
    }
    // First query token of every cluster's tile range [p T / pairs, (p + 1) T / pairs):
    // the first bj with cum[bj + 1] > floor(p T / pairs).  The thread whose prefix
    // range [cum[lo], cum[hi]) holds that start answers from its own values: those
    // are the clusters p with ceil(cum[lo] pairs / T) <= p < ceil(cum[hi] pairs / T).
    int32_t T = 0;
    for (int w = 0; w < kThreads / 32; ++w) T += part[w];
    if (T == 0) {
        for (int p = tid; p < a.pairs; p += kThreads) a.first_bj[p] = a.BJ;
        return;
    }
    const int p0 = (int)(((int64_t)run_lo * a.pairs + T - 1) / T);
    const int p1 = min(a.pairs, (int)(((int64_t)run * a.pairs + T - 1) / T));
    for (int p = p0; p < p1; ++p) {
        const int s0 = (int)(((uint32_t)p * (uint32_t)T) / (uint32_t)a.pairs);
        int32_t c = run_lo;
        for (int bj = lo; bj < hi; ++bj) {
            c += tiles_of(a, bj, &ignored);
            if (c > s0) {
                a.first_bj[p] = bj;
                break;
            }
        }
    }
}

__host__ __device__ constexpr uint32_t tmem_cols_for(int n) {
    return n <= 32 ? 32u : (n <= 64 ? 64u : (n <= 128 ? 128u : (n <= 256 ? 256u : 512u)));
}

// Thread 0 waits for `bar` (bounded); the block learns the outcome through
// smem after a __syncthreads, so no warp diverges on a timeout.
__device__ bool block_wait(uint64_t* bar, int* flag, int32_t* status) {
    if (threadIdx.x == 0) {
        *flag = mbar_wait(bar, 0, nullptr) ? 1 : 0;
        if (!*flag) set_status(status, MLA_ERR_TIMEOUT);
    }
    __syncthreads();
    return *flag != 0;
}

// One CTA per (head h, row tile mt of W_uk[h], token tile): the 128 latent
// rows [128 mt, 128 mt + 128) against the tile's tokens, M = 128, N = tokens,
// K = 128 (2 boxes of 64).  Four CTAs of 48 KB fit on an SM, so one CTA's
// loads overlap another's MMAs and epilogue.  This is the first kernel of a
// decode call and is launched without programmatic dependence: its TMA loads
// read the caller's inputs.
__global__ void __launch_bounds__(kThreads, 4)
absorb_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB, ProjArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full, done;
    __shared__ uint32_t tmem_base;
    __shared__ int flag;
    const int h = blockIdx.x, mt = blockIdx.y, nt = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = a.n_tile;
    const uint32_t ncols = tmem_cols_for(N);
    uint8_t* sA = smem;                    // [kb] 16 KB boxes: 128 rows x 64 k
    uint8_t* sB = smem + 2 * 16384;        // [kb] N x 128 B

    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
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

    if (warp == 0 && elect_one()) {
        mbar_expect_tx(&full, 2 * 16384 + 2 * N * 128);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_2d(sA + kb * 16384, &mapA, &full, kb * 64, h * 512 + mt * 128);
            tma_load_3d(sB + kb * N * 128, &mapB, &full, kb * 64, h, nt * N);
        }
    } else if (warp == 1) {
        // whole warp, one elected lane issues (warp-uniform descriptors)
        int ready = 0;
        if (lane == 0) ready = mbar_wait(&full, 0, nullptr) ? 1 : 0;
        if (__shfl_sync(0xffffffffu, ready, 0)) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, N, false, false);
            const uint64_t da = sdesc(smem_u32(sA), 16, 1024, kSwizzle128);
            const uint64_t db = sdesc(smem_u32(sB), 16, 1024, kSwizzle128);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss_w(tmem, sdesc_add(da, kb * 16384 + ks * 32), sdesc_add(db, kb * N * 128 + ks * 32), idesc,
                             (kb | ks) ? 1u : 0u);
        }
        mma_commit_w(&done);
    }
    __syncwarp();
    grid_dep_trigger();

    // query RoPE (CTAs of row tile 0; one thread per token row, N <= kThreads)
    // and the key-tile plan while the MMAs run
    const int n_row = nt * N + threadIdx.x;
    if (mt == 0 && threadIdx.x < N && n_row < a.BJ) {
        const int b = n_row / a.n_q, j = n_row % a.n_q;
        const int64_t p = query_pos(a.seq_lens[b], a.n_q, j);
        const uint4* src = reinterpret_cast<const uint4*>(a.q_rope + ((int64_t)n_row * a.H + h) * 64);
        uint4* dst = reinterpret_cast<uint4*>(a.q_lat + ((int64_t)n_row * a.H + h) * 576 + 512);
        uint4 rot[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) rot[c] = src[c];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t w[4] = {rot[c].x, rot[c].y, rot[c].z, rot[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
                float y0, y1;
                rope_pair_turn(x.x, x.y, p, a.rope_turn[4 * c + i], &y0, &y1);
                w[i] = pack_bf16(y0, y1);
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    if (h == 0 && mt == 0 && nt == 0) plan_tiles(a, threadIdx.x);

    if (block_wait(&done, &flag, a.status)) {
        // TMEM row m holds q_lat[n][h][128 mt + m] for the N tokens; stage as
        // [n][128] bf16 in smem (the operand area is free now), then write each
        // token's 256-byte segment with 16-byte stores.
        tc_fence_after();
        __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem);
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < N; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) stage[(c0 + c) * 128 + m] = __float2bfloat16_rn(__uint_as_float(r[c]));
        }
        __syncthreads();
        const int nvalid = min(N, a.BJ - nt * N);
        for (int i = threadIdx.x; i < nvalid * 16; i += kThreads) {
            const int n = i >> 4, c = i & 15;
            reinterpret_cast<uint4*>(a.q_lat + ((int64_t)(nt * N + n) * a.H + h) * 576 + 128 * mt)[c] =
                reinterpret_cast<const uint4*>(stage + n * 128)[c];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, ncols);
}

// One CTA per (head, token tile of <= 64): out[n][h][v] = sum_i W_uv[h][i][v] o_lat[n][h][i].
// A = W_uv[h] read MN-major (v contiguous), 8 k-blocks of 64 rows, all in flight.
__global__ void __launch_bounds__(kThreads, 1)
upproj_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB, ProjArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[8], done;
    __shared__ uint32_t tmem_base;
    __shared__ int flag;
    const int h = blockIdx.x, nt = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = a.n_tile;
    const uint32_t ncols = tmem_cols_for(N);
    const int stage = 16384 + N * 128;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(&full[i], 1);
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

    if (warp == 0 && elect_one()) {
        // W_uv is an input: fetch it before waiting for the previous kernel
        for (int kb = 0; kb < 8; ++kb) {
            uint8_t* st = smem + kb * stage;
            mbar_expect_tx(&full[kb], 16384 + N * 128);
            tma_load_2d(st, &mapA, &full[kb], 0, h * 512 + kb * 64);
            tma_load_2d(st + 8192, &mapA, &full[kb], 64, h * 512 + kb * 64);
        }
        grid_dep_wait();         // o_lat comes from the previous kernels
        for (int kb = 0; kb < 8; ++kb)
            tma_load_3d(smem + kb * stage + 16384, &mapB, &full[kb], kb * 64, h, nt * N);
    } else if (warp == 1) {
        // whole warp, one elected lane issues (warp-uniform descriptors)
        const uint32_t idesc = idesc_bf16(128, N, true, false);
        const uint64_t da = sdesc(smem_u32(smem), 8192, 1024, kSwizzle128);
        const uint64_t db = sdesc(smem_u32(smem) + 16384, 16, 1024, kSwizzle128);
        for (int kb = 0; kb < 8; ++kb) {
            int ready = 0;
            if (lane == 0) ready = mbar_wait(&full[kb], 0, nullptr) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ready, 0)) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ss_w(tmem, sdesc_add(da, kb * stage + ks * 2048), sdesc_add(db, kb * stage + ks * 32), idesc,
                         (kb | ks) ? 1u : 0u);
        }
        mma_commit_w(&done);
    }
    __syncwarp();
    grid_dep_wait();
    grid_dep_trigger();

    if (block_wait(&done, &flag, a.status)) {
        // stage out[n][h][0:128] as [n][128] bf16 in smem, then 16-byte stores
        tc_fence_after();
        __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem);
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < N; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) stage[(c0 + c) * 128 + m] = __float2bfloat16_rn(__uint_as_float(r[c]));
        }
        __syncthreads();
        const int nvalid = min(N, a.BJ - nt * N);
        for (int i = threadIdx.x; i < nvalid * 16; i += kThreads) {
            const int n = i >> 4, c = i & 15;
            reinterpret_cast<uint4*>(a.out + ((int64_t)(nt * N + n) * a.H + h) * 128)[c] =
                reinterpret_cast<const uint4*>(stage + n * 128)[c];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, ncols);
}

int round_n(int bj, int cap) {
    int n = bj < cap ? bj : cap;
    n = (n + 15) / 16 * 16;
    return n < 16 ? 16 : n;
}

template <typename K>
int launch(K kernel, const CUtensorMap& A, const CUtensorMap& B, const ProjArgs& a, dim3 grid, size_t smem,
           cudaStream_t st, const char* name, int* launches, bool pdl = true) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    prof_begin(st, name);
    const cudaError_t e = pdl ? launch_pdl(kernel, grid, dim3(kThreads), smem, st, A, B, a)
                              : launch_plain(kernel, grid, dim3(kThreads), smem, st, A, B, a);
    prof_end(st);
    if (launches) ++*launches;
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

// absorb + q-RoPE + plan.  q_nope [BJ][H][128], W_uk [H][512][128], q_rope [BJ][H][64]
int launch_absorb(const DecodeCall& c, __nv_bfloat16* q_lat, int32_t* cum, int32_t* first_bj, int pairs,
                  int* launches) {
    // (sparse decode: c.n_sel / c.max_sel give the tile counts)
    const int BJ = c.batch * c.n_q, H = c.d.heads, N = round_n(BJ, 128);
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
    rope_turn_table(c.d.rope_base, 64, a.rope_turn);
    a.q_lat = q_lat;
    a.cum = cum;
    a.first_bj = first_bj;
    a.pairs = pairs;
    a.n_sel = c.n_sel;
    a.max_sel = c.max_sel;
    a.status = c.status;
    const dim3 grid(H, 4, (BJ + N - 1) / N);
    return launch(absorb_kernel, A, B, a, grid, 2 * 16384 + 2 * N * 128 + 1024, c.stream, "sm100_absorb", launches,
                  false);
}

// up-projection.  o_lat [BJ][H][512] bf16, W_uv [H][512][128], out [BJ][H][128]
int launch_upproj(const DecodeCall& c, const __nv_bfloat16* o_lat, int* launches) {
    const int BJ = c.batch * c.n_q, H = c.d.heads, N = round_n(BJ, 64);
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
    return launch(upproj_kernel, A, B, a, grid, 8 * (16384 + N * 128) + 1024, c.stream, "sm100_upproj", launches);
}

}  // namespace sm100
}  // namespace mla
