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
//   with the split-KV log-sum-exp merge of the tokens whose key tiles were
//   cut across attention clusters applied after the projection (it is linear).
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

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

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
    int32_t* slot_owner;     // [2 pairs] query token of each split-KV piece slot (-1: unused)
    int32_t* cut;            // [pairs + 1] first key tile of each attention cluster
    int pairs;
    const int32_t* n_sel;    // sparse decode: selected keys per query token (nullptr: dense)
    int max_sel;
    int tile_keys;           // keys per attention tile (64)
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
        return (n + a.tile_keys - 1) / a.tile_keys;
    }
    return (int32_t)((p + a.tile_keys) / a.tile_keys);
}

// Cluster ranges, given the key-tile prefix cum of the query tokens.  Cluster
// p covers tiles [cut[p], cut[p + 1]).  The cuts share out a cost that charges
// every query token kItemTiles tiles on top of its own (loading its query
// slice and its epilogue cost about that much time per item), so a cluster
// that gets more items gets fewer tiles; a cut that falls in a token's fixed
// share lands on the token's first tile.  Then each cluster's first token and
// the query token each split-KV piece slot holds: slot 2p the piece in
// cluster p of a token begun in an earlier cluster, slot 2p + 1 the piece of
// a token begun in p that goes on past it (-1: no such piece).
constexpr int kItemTiles = 4;
constexpr int kMaxClusters = 256;
__device__ void plan_clusters(const ProjArgs& a, const int32_t* cum, int tid) {
    __shared__ int32_t s_cut[kMaxClusters + 1];
    const int32_t T = cum[a.BJ];
    const int64_t C = (int64_t)T + (int64_t)kItemTiles * a.BJ;
    for (int p = tid; p <= a.pairs; p += kThreads) {
        int32_t t = T;
        if (p < a.pairs) {
            const int64_t x = (int64_t)p * C / a.pairs;
            int lo = 0, hi = a.BJ;                     // largest bj with cum[bj] + K bj <= x
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if ((int64_t)cum[mid] + (int64_t)kItemTiles * mid <= x) lo = mid; else hi = mid - 1;
            }
            if (lo < a.BJ) {
                const int64_t o = x - ((int64_t)cum[lo] + (int64_t)kItemTiles * lo) - kItemTiles;
                const int64_t len = cum[lo + 1] - cum[lo];
                t = cum[lo] + (int32_t)(o < 0 ? 0 : (o > len ? len : o));
            }
        }
        s_cut[p] = t;
        a.cut[p] = t;
    }
    __syncthreads();
    // the token holding tile t: the first bj with cum[bj + 1] > t
    auto holder = [&](int32_t t) {
        int l = 0, r = a.BJ - 1;
        while (l < r) {
            const int mid = (l + r) >> 1;
            if (cum[mid + 1] > t) r = mid; else l = mid + 1;
        }
        return l;
    };
    for (int p = tid; p < a.pairs; p += kThreads) {
        const int32_t s0 = s_cut[p], s1 = s_cut[p + 1];
        a.first_bj[p] = s0 < T ? holder(s0) : a.BJ;
        int even = -1, odd = -1;
        if (s1 > s0) {
            const int bf = holder(s0);
            if (cum[bf] < s0) even = bf;
            const int bl = holder(s1 - 1);
            if (cum[bl] >= s0 && cum[bl + 1] > s1) odd = bl;
        }
        a.slot_owner[2 * p] = even;
        a.slot_owner[2 * p + 1] = odd;
    }
}

// Key-tile plan, for any number of query tokens: per-thread token ranges and
// global loads throughout (used when the tokens do not fit the staged plan).
__device__ void plan_tiles_long(const ProjArgs& a, int tid) {

    // Tiles of tile_keys keys each query token attends; 0 for an invalid length.
    __shared__ int32_t part_l[kThreads / 32];
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
    if (lane == 31) part_l[warp] = incl;
    __syncthreads();
    int32_t run = incl - sum;
    for (int w = 0; w < warp; ++w) run += part_l[w];
    if (tid == 0) a.cum[0] = 0;
    bool ignored = false;
    for (int bj = lo; bj < hi; ++bj) {
        run += tiles_of(a, bj, &ignored);
        a.cum[bj + 1] = run;
    }
    __syncthreads();         // every cum entry of the block is written (and visible to it)
    plan_clusters(a, a.cum, tid);
}

constexpr int kPlanTokens = 512;           // tokens the staged plan holds in shared memory (2 KB: the absorb CTAs stay four per SM)

// The key-tile plan of the attention kernel: cum[bj + 1] = key tiles of query
// tokens 0..bj, and the first token of every cluster's tile range.  Each
// token's length is loaded once (all loads of a thread issued together), the
// prefix and the cluster starts are then computed from shared memory.
__device__ void plan_tiles(const ProjArgs& a, int tid) {
    if (a.BJ > kPlanTokens) {
        plan_tiles_long(a, tid);
        return;
    }
    __shared__ int32_t part[kThreads / 32];
    __shared__ int32_t s_cum[kPlanTokens + 1];
    constexpr int kPer = kPlanTokens / kThreads;
    const int per = (a.BJ + kThreads - 1) / kThreads;
    const int lo = min(a.BJ, tid * per), hi = min(a.BJ, lo + per);
    int32_t t[kPer];
    int32_t sum = 0;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        t[i] = lo + i < hi ? tiles_of(a, lo + i, &bad) : 0;
        sum += t[i];
    }
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
    if (tid == 0) {
        a.cum[0] = 0;
        s_cum[0] = 0;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        run += t[i];
        if (lo + i < hi) {
            a.cum[lo + i + 1] = run;
            s_cum[lo + i + 1] = run;
        }
    }
    __syncthreads();
    plan_clusters(a, s_cum, tid);
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
// decode call.  It is launched with programmatic dependence so that its
// prologue (barriers, TMEM) overlaps the tail of whatever kernel precedes it
// in the stream; every read of the caller's inputs comes after
// griddepcontrol.wait, which waits for that kernel to complete (a preceding
// copy or a kernel that never triggers simply serialises as usual).
__global__ void __launch_bounds__(kThreads, 4)
absorb_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB, ProjArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full, done;
    __shared__ uint32_t tmem_base;
    __shared__ int flag;
    const int h = blockIdx.x, mt = blockIdx.y, nt = blockIdx.z;
    if (h == a.H) {
        // the extra column of the grid: one CTA builds the attention kernel's
        // key-tile plan, off the critical path of the projection CTAs
        if (mt == 0 && nt == 0) {
            grid_dep_wait();
            plan_tiles(a, threadIdx.x);
        }
        return;
    }
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
    grid_dep_wait();         // every read of the caller's inputs comes after this

    if (warp == 0 && elect_one()) {
        // both 64-column k groups of the weight rows and of the tokens, one copy each
        mbar_expect_tx(&full, 2 * 16384 + 2 * N * 128);
        tma_load_3d(sA, &mapA, &full, 0, h * 512 + mt * 128, 0);
        tma_load_4d(sB, &mapB, &full, 0, nt * N, 0, h);
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

    // query RoPE while the MMAs run (CTAs of row tile 0; one thread per token
    // row, N <= kThreads)
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
                rope_pair_turn_bf16(x.x, x.y, p, a.rope_turn[4 * c + i], &y0, &y1);
                w[i] = pack_bf16(y0, y1);
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }

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

struct UpArgs {
    const int32_t* cum;          // [BJ + 1] key-tile prefix of the query tokens
    const int32_t* slot_owner;   // [2 pairs] query token of each piece slot (-1: unused)
    const int32_t* cut;          // [pairs + 1] first key tile of each attention cluster
    int BJ, H, pairs, n_tok;     // n_tok: tokens per CTA (64)
    int n_cols;                  // MMA N: n_tok + 2 pairs, rounded up to 16 (<= 256)
    const float* part_lse;       // [H][2 pairs][2 latent halves], log2 domain
    __nv_bfloat16* out;          // [BJ][H][128]
    int32_t* status;
};

constexpr int kUpThreads = 256;
constexpr int kUpStages = 3;

// One CTA per (head h, tile of 64 query tokens):
//     out[n][h][v] = sum_i W_uv[h][i][v] o[n][h][i]
// where o is the token's weighted latent row: o_lat as written by the
// attention kernel for a token finished inside one cluster, and for a token
// cut across clusters the log-sum-exp merge of its pieces' normalised
// partial rows part_o[slot][h] with weights 2^(lse_piece - lse) (per latent
// half: the two halves of a piece were normalised by the two CTAs of its
// cluster).  The merge is moved past the projection, which is linear: the
// B operand holds the tile's o_lat rows and every piece row of head h as
// they are (two tensor copies per 64-column k-block, no arithmetic), the
// tensor cores project all of them, D0 over latent columns [0, 256) and D1
// over [256, 512), and the epilogue combines the 128-wide projected rows of a
// cut token's pieces with their weights.
//
// A = W_uv[h] read MN-major (v contiguous): four 32 KB copies of 128 latent
// rows, fetched before waiting for the attention kernel (an input).  B: a
// ring of kUpStages k-blocks of n_cols rows x 128 bytes (128-byte swizzle).
// Warp 0 loads, warp 1 issues the MMAs; meanwhile warps 2-7 find each
// token's pieces and weights.  TMEM: D0 at column 0, D1 at column 256.
__global__ void __launch_bounds__(kUpThreads, 1)
upproj_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapO,
              const __grid_constant__ CUtensorMap mapP, UpArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t fullA[4], fullB[kUpStages], emptyB[kUpStages], done;
    __shared__ uint32_t tmem_base;
    __shared__ int flag;
    // per piece slot s (column n_tok + s of D): the tile-local token it belongs
    // to (-1: none in this tile) and its weights for the two latent halves
    __shared__ int slot_tok[256];
    __shared__ float slot_lse[2][256], slot_w[2][256];
    // per token of the tile: 0 invalid length (zeros), 1 finished in one
    // cluster, 2 cut (merge its pieces)
    __shared__ int tok_mode[64], tok_s0[64], tok_s1[64];
    __shared__ int32_t s_cut[257];
    const int h = blockIdx.x, n0 = blockIdx.z * a.n_tok;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = a.n_cols, S = 2 * a.pairs;
    constexpr int kWBlock = 32768;
    const int kBStage = N * 128;
    uint8_t* sB = smem + 4 * kWBlock;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&fullA[i], 1);
        for (int i = 0; i < kUpStages; ++i) {
            mbar_init(&fullB[i], 1);
            mbar_init(&emptyB[i], 1);
        }
        mbar_init(&done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    if (warp == 0 && elect_one()) {
        // W_uv[h]: one copy per 128 latent rows (both 64-column groups of v)
        for (int j = 0; j < 4; ++j) {
            mbar_expect_tx(&fullA[j], kWBlock);
            tma_load_3d(smem + j * kWBlock, &mapA, &fullA[j], 0, h * 512 + j * 128, 0);
        }
    }
    __syncwarp();
    grid_dep_wait();         // the attention kernel's latents and pieces
    grid_dep_trigger();

    if (warp == 0) {
        if (elect_one()) {
            // k-block kb: the tile's 64 o_lat rows, then all 2 pairs piece rows
            // (rows past the tokens or the slots read as zeros)
            for (int kb = 0; kb < 8; ++kb) {
                const int st = kb % kUpStages;
                if (kb >= kUpStages && !mbar_wait(&emptyB[st], ((kb / kUpStages) - 1) & 1, nullptr)) {
                    set_status(a.status, MLA_ERR_TIMEOUT);
                    break;
                }
                uint8_t* dst = sB + st * kBStage;
                mbar_expect_tx(&fullB[st], (a.n_tok + S) * 128);
                tma_load_4d(dst, &mapO, &fullB[st], 0, n0, kb, h);
                tma_load_4d(dst + a.n_tok * 128, &mapP, &fullB[st], 0, 0, kb, h);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // whole warp, one elected lane issues (warp-uniform descriptors)
        const uint32_t idesc = idesc_bf16(128, N, true, false);
        const uint64_t da = sdesc(smem_u32(smem), kWBlock / 2, 1024, kSwizzle128);   // v groups 16 KB apart
        const uint64_t db = sdesc(smem_u32(sB), 16, 1024, kSwizzle128);
        bool ok = true;
        for (int kb = 0; kb < 8 && ok; ++kb) {
            const int st = kb % kUpStages;
            int ready = 0;
            if (lane == 0)
                ready = ((kb & 1) || mbar_wait(&fullA[kb >> 1], 0, nullptr)) &&
                        mbar_wait(&fullB[st], (kb / kUpStages) & 1, nullptr);
            ok = __shfl_sync(0xffffffffu, ready, 0) != 0;
            if (!ok) {
                if (lane == 0) set_status(a.status, MLA_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ss_w(tmem + (kb < 4 ? 0u : 256u), sdesc_add(da, (kb >> 1) * kWBlock + (kb & 1) * 8192 + ks * 2048),
                         sdesc_add(db, st * kBStage + ks * 32), idesc, ((kb & 3) | ks) ? 1u : 0u);
            mma_commit_w(&emptyB[st]);
        }
        mma_commit_w(&done);
    } else {
        // ---- piece tables (192 threads): each slot's tile-local token (from the
        // plan), each token's mode and slot range, and each slot's weights for
        // the two latent halves, w = 2^(lse - M) / sum over the token's pieces of
        // 2^(lse' - M) with M their maximum
        const int t = threadIdx.x - 64;
        int c0 = 0, c1 = 0;
        if (t < a.n_tok && n0 + t < a.BJ) {
            c0 = a.cum[n0 + t];
            c1 = a.cum[n0 + t + 1];
        }
        for (int p = t; p <= a.pairs; p += 192) s_cut[p] = a.cut[p];
        named_barrier(1, 192);
        if (t < a.n_tok) {
            // the token's pieces lie in slots [2 pf + 1, 2 pl] (pf, pl: the clusters
            // holding its first and last key tile)
            auto pair_of = [&](int32_t tile) {           // largest p with cut[p] <= tile
                int lo = 0, hi = a.pairs - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (s_cut[mid] <= tile) lo = mid; else hi = mid - 1;
                }
                return lo;
            };
            const int pf = pair_of(c0), pl = pair_of(c1 - 1);
            const bool cut = c1 > c0 && pf != pl;
            tok_s0[t] = cut ? 2 * pf + 1 : 256;
            tok_s1[t] = cut ? 2 * pl : -1;
        }
        for (int s = t; s < 256; s += 192) {
            const int owner = s < S ? a.slot_owner[s] - n0 : -1;
            const int tok = owner >= 0 && owner < a.n_tok ? owner : -1;
            slot_tok[s] = tok;
            if (tok >= 0) {
                slot_lse[0][s] = __ldcg(a.part_lse + (h * S + s) * 2);
                slot_lse[1][s] = __ldcg(a.part_lse + (h * S + s) * 2 + 1);
            }
        }
        named_barrier(1, 192);
        if (t < a.n_tok) tok_mode[t] = c1 == c0 ? 0 : (tok_s1[t] >= 0 ? 2 : 1);
        // A token cut into many pieces: one warp, lanes over its slots and
        // shuffle reductions.  Few pieces (the usual case): one thread per token.
        const int gw = warp - 2;
        for (int tt = gw; tt < a.n_tok; tt += 6) {
            const int s0 = tok_s0[tt], s1 = tok_s1[tt];
            if (s1 - s0 < 8) continue;
            float M0 = -INFINITY, M1 = -INFINITY;
            for (int s = s0 + lane; s <= s1; s += 32)
                if (slot_tok[s] == tt) {
                    M0 = fmaxf(M0, slot_lse[0][s]);
                    M1 = fmaxf(M1, slot_lse[1][s]);
                }
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) {
                M0 = fmaxf(M0, __shfl_xor_sync(0xffffffffu, M0, d));
                M1 = fmaxf(M1, __shfl_xor_sync(0xffffffffu, M1, d));
            }
            float S0 = 0.f, S1 = 0.f;
            for (int s = s0 + lane; s <= s1; s += 32)
                if (slot_tok[s] == tt) {
                    S0 += ex2_approx(slot_lse[0][s] - M0);
                    S1 += ex2_approx(slot_lse[1][s] - M1);
                }
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) {
                S0 += __shfl_xor_sync(0xffffffffu, S0, d);
                S1 += __shfl_xor_sync(0xffffffffu, S1, d);
            }
            const float i0 = 1.f / S0, i1 = 1.f / S1;
            for (int s = s0 + lane; s <= s1; s += 32)
                if (slot_tok[s] == tt) {
                    slot_w[0][s] = ex2_approx(slot_lse[0][s] - M0) * i0;
                    slot_w[1][s] = ex2_approx(slot_lse[1][s] - M1) * i1;
                }
        }
        if (t < a.n_tok && tok_s1[t] - tok_s0[t] < 8) {
            const int s0 = tok_s0[t], s1 = tok_s1[t];
            float M0 = -INFINITY, M1 = -INFINITY;
            for (int s = s0; s <= s1; ++s)
                if (slot_tok[s] == t) {
                    M0 = fmaxf(M0, slot_lse[0][s]);
                    M1 = fmaxf(M1, slot_lse[1][s]);
                }
            float S0 = 0.f, S1 = 0.f;
            for (int s = s0; s <= s1; ++s)
                if (slot_tok[s] == t) {
                    S0 += ex2_approx(slot_lse[0][s] - M0);
                    S1 += ex2_approx(slot_lse[1][s] - M1);
                }
            const float i0 = 1.f / S0, i1 = 1.f / S1;
            for (int s = s0; s <= s1; ++s)
                if (slot_tok[s] == t) {
                    slot_w[0][s] = ex2_approx(slot_lse[0][s] - M0) * i0;
                    slot_w[1][s] = ex2_approx(slot_lse[1][s] - M1) * i1;
                }
        }
    }
    __syncthreads();         // piece tables complete

    if (block_wait(&done, &flag, a.status)) {
        // Projected rows straight to out[n][h][0:128] (lane v of a warp writes
        // element v: each store covers 64 contiguous bytes).  Warps w and w + 4
        // share TMEM lane quarter w & 3 (v = 32 (w & 3) + lane): warps 0-3 take
        // the tokens finished in one cluster (D0 + D1 of their own column), warps
        // 4-7 the cut tokens (their pieces' columns, weighted).  Each lane holds
        // one column's token data and the loops take it by shuffle.
        tc_fence_after();
        const int q = warp & 3, v = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const int nvalid = min(a.n_tok, a.BJ - n0);
        __nv_bfloat16* out_hv = a.out + ((int64_t)n0 * a.H + h) * 128 + v;   // token n at + n H 128
        if (warp < 4) {
            for (int c0 = 0; c0 < nvalid; c0 += 32) {
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_off + c0, r0);
                tmem_ld32(tmem + lane_off + 256 + c0, r1);
                const int my_mode = tok_mode[c0 + lane];
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int mode = __shfl_sync(0xffffffffu, my_mode, i);
                    const float val = mode == 1 ? __uint_as_float(r0[i]) + __uint_as_float(r1[i]) : 0.f;
                    if (mode != 2 && c0 + i < nvalid) out_hv[(int64_t)(c0 + i) * a.H * 128] = __float2bfloat16_rn(val);
                }
            }
        } else {
            // slot columns in order; a cut token's pieces are consecutive slots
            // (unused slots between them hold anything and are skipped)
            int prev = -1;
            float acc = 0.f;
            for (int c0 = 0; c0 < S; c0 += 32) {
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_off + a.n_tok + c0, r0);
                tmem_ld32(tmem + lane_off + 256 + a.n_tok + c0, r1);
                const int my_tok = c0 + lane < S ? slot_tok[c0 + lane] : -1;
                const float my_w0 = my_tok >= 0 ? slot_w[0][c0 + lane] : 0.f;
                const float my_w1 = my_tok >= 0 ? slot_w[1][c0 + lane] : 0.f;
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int tok = __shfl_sync(0xffffffffu, my_tok, i);
                    const float w0 = __shfl_sync(0xffffffffu, my_w0, i);
                    const float w1 = __shfl_sync(0xffffffffu, my_w1, i);
                    const float pv = fmaf(w0, __uint_as_float(r0[i]), w1 * __uint_as_float(r1[i]));
                    const float val = tok >= 0 ? pv : 0.f;
                    const bool starts = tok >= 0 && tok != prev;    // a new token's first piece
                    if (starts && prev >= 0) out_hv[(int64_t)prev * a.H * 128] = __float2bfloat16_rn(acc);
                    acc = starts ? val : acc + val;
                    prev = tok >= 0 ? tok : prev;
                }
            }
            if (prev >= 0) out_hv[(int64_t)prev * a.H * 128] = __float2bfloat16_rn(acc);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
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
int launch_absorb(const DecodeCall& c, __nv_bfloat16* q_lat, int32_t* cum, int32_t* first_bj,
                  int pairs, int* launches) {
    // (sparse decode: c.n_sel / c.max_sel give the tile counts)
    const int BJ = c.batch * c.n_q, H = c.d.heads, N = round_n(BJ, 128);
    // The 128-wide rows are viewed as 2 groups of 64 columns (group stride 128
    // bytes, placed after the row dimension) so one box holds both groups
    // group-major -- the layout of two 64-column boxes side by side.
    CUtensorMap A, B;
    {
        const uint64_t dims[3] = {64, (uint64_t)H * 512, 2}, str[2] = {128 * 2, 64 * 2};
        const uint32_t box[3] = {64, 128, 2};
        if (!make_map(&A, c.W_uk, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        // q_nope [BJ][H][128] as (column in group, token, group, head)
        const uint64_t dims[4] = {64, (uint64_t)BJ, 2, (uint64_t)H};
        const uint64_t str[3] = {(uint64_t)H * 128 * 2, 64 * 2, 128 * 2};
        const uint32_t box[4] = {64, (uint32_t)N, 2, 1};
        if (!make_map(&B, c.q_nope, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
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
    a.slot_owner = first_bj + pairs;
    a.cut = first_bj + 3 * pairs;
    a.pairs = pairs;
    a.n_sel = c.n_sel;
    a.max_sel = c.max_sel;
    a.tile_keys = 64;                     // both attention kernels take 64-key tiles
    a.status = c.status;
    const dim3 grid(H + 1, 4, (BJ + N - 1) / N);      // column H: the plan CTA
    return launch(absorb_kernel, A, B, a, grid, 2 * 16384 + 2 * N * 128 + 1024, c.stream, "sm100_absorb", launches);
}

// up-projection with the split-KV merge applied to the projected piece rows.
// o_lat [BJ][H][512] bf16, part_o [H][8][2P][64] bf16, part_lse [H][2P][2],
// W_uv [H][512][128], out [BJ][H][128]
int launch_upproj(const DecodeCall& c, __nv_bfloat16* o_lat, const __nv_bfloat16* part_o, const float* part_lse,
                  const int32_t* cum, int pairs, int* launches) {
    const int BJ = c.batch * c.n_q, H = c.d.heads;
    constexpr int kTok = 64;
    const int n_cols = (kTok + 2 * pairs + 15) / 16 * 16;
    if (n_cols > 256) return MLA_ERR_UNSUPPORTED;
    CUtensorMap A, O, P;
    {
        // W_uv rows [H * 512][128] viewed as (column in group, row, group of 64 columns):
        // one box = 128 rows x both groups, landing group-major
        const uint64_t dims[3] = {64, (uint64_t)H * 512, 2}, str[2] = {128 * 2, 64 * 2};
        const uint32_t box[3] = {64, 128, 2};
        if (!make_map(&A, c.W_uv, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        // o_lat [BJ][H][512] as (column in group, token, group of 64 columns, head):
        // one box = 64 tokens of one group and head
        const uint64_t dims[4] = {64, (uint64_t)BJ, 8, (uint64_t)H};
        const uint64_t str[3] = {(uint64_t)H * 512 * 2, 64 * 2, 512 * 2};
        const uint32_t box[4] = {64, (uint32_t)kTok, 1, 1};
        if (!make_map(&O, o_lat, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        // part_o, head-major and blocked by 64 latent columns ([H][8][2 pairs][64]):
        // one box = every piece slot of one block and head, contiguous
        const uint64_t dims[4] = {64, (uint64_t)(2 * pairs), 8, (uint64_t)H};
        const uint64_t str[3] = {128, (uint64_t)(2 * pairs) * 128, (uint64_t)(2 * pairs) * 8 * 128};
        const uint32_t box[4] = {64, (uint32_t)(2 * pairs), 1, 1};
        if (!make_map(&P, part_o, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    UpArgs a{};
    a.cum = cum;
    a.slot_owner = cum + BJ + 1 + pairs;
    a.cut = cum + BJ + 1 + 3 * pairs;
    a.BJ = BJ;
    a.H = H;
    a.pairs = pairs;
    a.n_tok = kTok;
    a.n_cols = n_cols;
    a.part_lse = part_lse;
    a.out = (__nv_bfloat16*)c.out;
    a.status = c.status;
    const dim3 grid(H, 1, (BJ + kTok - 1) / kTok);
    const size_t smem = 4 * 32768 + (size_t)kUpStages * n_cols * 128 + 1024;
    if (cudaFuncSetAttribute(upproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    prof_begin(c.stream, "sm100_upproj");
    const cudaError_t e = launch_pdl(upproj_kernel, grid, dim3(kUpThreads), smem, c.stream, A, O, P, a);
    prof_end(c.stream);
    if (launches) ++*launches;
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla
