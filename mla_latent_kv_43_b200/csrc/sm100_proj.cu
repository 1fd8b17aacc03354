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
//   with the split-KV log-sum-exp merge of o_lat folded into its operand
//   assembly (tokens whose key tiles were cut across attention clusters).
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
    int tile_keys;           // keys per attention tile: 128 (dense, CTA-pair kernel) or 64 (sparse)
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

__device__ void plan_tiles(const ProjArgs& a, int tid) {
    // Tiles of tile_keys keys each query token attends; 0 for an invalid length.
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

// Split-KV merge of the query tokens' latent rows for head h (log-sum-exp
// over the pieces): the pieces' normalised partial rows weighted by
// 2^(lse_piece - lse), lse = log2 sum_piece 2^lse_piece.  A token finished
// inside one cluster is read from o_lat as it is; a token with an invalid
// length gives zeros.  Merged rows are also written back to o_lat (the
// workspace's weighted latents).
struct MergeArgs {
    const int32_t* cum;
    int BJ, pairs;
    const __nv_bfloat16* part_o;
    const float* part_lse;
    __nv_bfloat16* o_lat;
};

// Pieces of token bj: the clusters pf..pl whose key-tile ranges it spans
// (clusters with an empty range in between hold nothing).  Cluster p covers
// tiles [start(p), start(p + 1)), start(p) = p T / pairs; T * pairs fits 32 bits.
struct PieceRange {
    int T, pairs;
    __device__ int start(int p) const { return (int)(((uint32_t)p * (uint32_t)T) / (uint32_t)pairs); }
    __device__ int pair_of(int t) const {      // largest p with start(p) <= t
        int lo = 0, hi = pairs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (start(mid) <= t) lo = mid; else hi = mid - 1;
        }
        return lo;
    }
    __device__ bool empty(int p) const { return start(p) == (p + 1 < pairs ? start(p + 1) : T); }
    // slot of the piece in cluster p of a token whose first piece is in cluster pf
    __device__ static int slot(int p, int pf) { return p == pf ? 2 * p + 1 : 2 * p; }
};

constexpr int kUpThreads = 256;

// One CTA per (head, token tile of <= 64): out[n][h][v] = sum_i W_uv[h][i][v] o_lat[n][h][i].
// A = W_uv[h] read MN-major (v contiguous), 8 k-blocks of 64 rows, all in flight
// (an input: fetched before waiting for the attention kernel).  The B operand,
// the tokens' weighted latents, is assembled by the whole CTA in shared memory
// (128-byte swizzle, the layout a TMA box would give): each warp merges the
// split-KV pieces of one token row at a time.
__global__ void __launch_bounds__(kUpThreads, 1)
upproj_kernel(const __grid_constant__ CUtensorMap mapA, ProjArgs a, MergeArgs mg) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[4], done;
    __shared__ uint32_t tmem_base;
    __shared__ int flag;
    const int h = blockIdx.x, nt = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = a.n_tile;
    const uint32_t ncols = tmem_cols_for(N);
    // W_uv[h]: four 32 KB blocks of 128 latent rows, each [2 value-column groups][128 rows][64];
    // then the token operand: [8 k-blocks of 64 latent columns][N rows][64]
    constexpr int kWBlock = 32768;
    uint8_t* sB = smem + 4 * kWBlock;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&full[i], 1);
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
        // one copy per 128 latent rows (both 64-column groups of v): a single
        // thread issues about one tensor copy per 0.3 us, so few large ones
        for (int j = 0; j < 4; ++j) {
            mbar_expect_tx(&full[j], kWBlock);
            tma_load_3d(smem + j * kWBlock, &mapA, &full[j], 0, h * 512 + j * 128, 0);
        }
    }
    __syncwarp();
    grid_dep_wait();         // the attention kernel's latents and pieces
    grid_dep_trigger();

    // B operand: row n (token nt * N + n), 64-column block kb at sB + kb * N * 128,
    // 16-byte chunk c of the 128-byte row at ((c ^ (n & 7)) << 4).
    // Phase 1: one thread per token finds its pieces and their log-sum-exp.
    const int nvalid = min(N, a.BJ - nt * N);
    __shared__ int m_pf[64], m_pl[64], m_mode[64];      // mode 0: zeros, 1: o_lat as is, 2: merge
    __shared__ float m_M[64], m_inv[64];
    const PieceRange pr{mg.cum[mg.BJ], mg.pairs};
    if (threadIdx.x < N) {
        const int n = threadIdx.x;
        int mode = 0, pf = 0, pl = -1;
        float M = -INFINITY, S = 0.f;
        if (n < nvalid) {
            const int bj = nt * N + n;
            const int c0 = mg.cum[bj], c1 = mg.cum[bj + 1];
            if (c1 > c0) {
                pf = pr.pair_of(c0);
                pl = pr.pair_of(c1 - 1);
                mode = pf == pl ? 1 : 2;
                if (mode == 2) {
                    for (int p = pf; p <= pl; ++p)
                        if (p == pf || !pr.empty(p)) M = fmaxf(M, mg.part_lse[PieceRange::slot(p, pf) * 128 + h]);
                    for (int p = pf; p <= pl; ++p)
                        if (p == pf || !pr.empty(p)) S += exp2f(mg.part_lse[PieceRange::slot(p, pf) * 128 + h] - M);
                }
            }
        }
        m_pf[n] = pf;
        m_pl[n] = pl;
        m_mode[n] = mode;
        m_M[n] = M;
        m_inv[n] = mode == 2 ? 1.f / S : 0.f;
    }
    __syncthreads();
    // Phase 2: one (token, 64-column block) per thread and pass; a piece's eight
    // 16-byte loads are issued together, two pieces at a time.
    for (int item = threadIdx.x; item < N * 8; item += kUpThreads) {
        const int n = item >> 3, kb = item & 7;
        const int mode = m_mode[n];
        uint32_t w[32];
        const int bj = nt * N + n;
        uint4* orow = reinterpret_cast<uint4*>(mg.o_lat + ((int64_t)bj * 128 + h) * 512 + 64 * kb);
        if (mode == 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = 0u;
            if (n < nvalid) {
#pragma unroll
                for (int c = 0; c < 8; ++c) orow[c] = make_uint4(0u, 0u, 0u, 0u);
            }
        } else if (mode == 1) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = orow[c];
                w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
            }
        } else {
            const int pf = m_pf[n], pl = m_pl[n];
            const float M = m_M[n];
            float acc[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = 0.f;
            int p = pf;
            while (p <= pl) {
                int sl[2] = {-1, -1};
                for (int k = 0; k < 2 && p <= pl; ++p) {
                    if (p == pf || !pr.empty(p)) {
                        if (k == 0) sl[0] = PieceRange::slot(p, pf); else sl[1] = PieceRange::slot(p, pf);
                        ++k;
                    }
                }
                uint4 v[2][8];
                float wt[2] = {0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (sl[i] >= 0) {
                        const uint4* src = reinterpret_cast<const uint4*>(mg.part_o + ((int64_t)sl[i] * 128 + h) * 512 + 64 * kb);
#pragma unroll
                        for (int c = 0; c < 8; ++c) v[i][c] = src[c];
                        wt[i] = exp2f(mg.part_lse[sl[i] * 128 + h] - M);
                    }
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (sl[i] >= 0) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint32_t pw[4] = {v[i][c].x, v[i][c].y, v[i][c].z, v[i][c].w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[j]));
                                acc[8 * c + 2 * j] = fmaf(wt[i], f.x, acc[8 * c + 2 * j]);
                                acc[8 * c + 2 * j + 1] = fmaf(wt[i], f.y, acc[8 * c + 2 * j + 1]);
                            }
                        }
                    }
                }
            }
            const float inv = m_inv[n];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
#pragma unroll
            for (int c = 0; c < 8; ++c) orow[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
        const uint32_t row = smem_u32(sB + (kb * N + n) * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((c ^ (n & 7)) << 4)), "r"(w[4 * c]),
                         "r"(w[4 * c + 1]), "r"(w[4 * c + 2]), "r"(w[4 * c + 3]) : "memory");
    }
    fence_async_smem();      // generic-proxy writes, read by the tensor core
    __syncthreads();

    if (warp == 1) {
        // whole warp, one elected lane issues (warp-uniform descriptors)
        const uint32_t idesc = idesc_bf16(128, N, true, false);
        const uint64_t da = sdesc(smem_u32(smem), kWBlock / 2, 1024, kSwizzle128);   // v groups 16 KB apart
        const uint64_t db = sdesc(smem_u32(sB), 16, 1024, kSwizzle128);
        for (int kb = 0; kb < 8; ++kb) {
            if ((kb & 1) == 0) {
                int ready = 0;
                if (lane == 0) ready = mbar_wait(&full[kb >> 1], 0, nullptr) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, ready, 0)) break;
                tc_fence_after();
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ss_w(tmem, sdesc_add(da, (kb >> 1) * kWBlock + (kb & 1) * 8192 + ks * 2048),
                         sdesc_add(db, kb * N * 128 + ks * 32), idesc, (kb | ks) ? 1u : 0u);
        }
        mma_commit_w(&done);
    }
    __syncwarp();

    if (block_wait(&done, &flag, a.status)) {
        // stage out[n][h][0:128] as [n][128] bf16 in smem, then 16-byte stores;
        // warps w and w + 4 share lane quarter w & 3 and split the token columns
        tc_fence_after();
        __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(smem);
        const int q = warp & 3, m = q * 32 + lane;
        for (int c0 = (warp >> 2) * 16; c0 < N; c0 += 32) {
            uint32_t r[16];
            tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) stg[(c0 + c) * 128 + m] = __float2bfloat16_rn(__uint_as_float(r[c]));
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nvalid * 16; i += kUpThreads) {
            const int n = i >> 4, c = i & 15;
            reinterpret_cast<uint4*>(a.out + ((int64_t)(nt * N + n) * a.H + h) * 128)[c] =
                reinterpret_cast<const uint4*>(stg + n * 128)[c];
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
    a.pairs = pairs;
    a.n_sel = c.n_sel;
    a.max_sel = c.max_sel;
    a.tile_keys = (c.n_sel || !kDecodePairKernel) ? 64 : 128;
    a.status = c.status;
    const dim3 grid(H, 4, (BJ + N - 1) / N);
    return launch(absorb_kernel, A, B, a, grid, 2 * 16384 + 2 * N * 128 + 1024, c.stream, "sm100_absorb", launches);
}

// up-projection with the split-KV merge folded into its operand assembly.
// o_lat [BJ][H][512] bf16, part_o [2P][H][512] bf16, part_lse [2P][H],
// W_uv [H][512][128], out [BJ][H][128]
int launch_upproj(const DecodeCall& c, __nv_bfloat16* o_lat, const __nv_bfloat16* part_o, const float* part_lse,
                  const int32_t* cum, int pairs, int* launches) {
    const int BJ = c.batch * c.n_q, H = c.d.heads, N = round_n(BJ, 64);
    CUtensorMap A;
    {
        // W_uv rows [H * 512][128] viewed as (column in group, row, group of 64 columns):
        // one box = 128 rows x both groups, landing group-major
        const uint64_t dims[3] = {64, (uint64_t)H * 512, 2}, str[2] = {128 * 2, 64 * 2};
        const uint32_t box[3] = {64, 128, 2};
        if (!make_map(&A, c.W_uv, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    ProjArgs a{};
    a.BJ = BJ;
    a.H = H;
    a.n_q = c.n_q;
    a.n_tile = N;
    a.out = (__nv_bfloat16*)c.out;
    a.status = c.status;
    MergeArgs mg{cum, BJ, pairs, part_o, part_lse, o_lat};
    const dim3 grid(H, 1, (BJ + N - 1) / N);
    const size_t smem = 4 * 32768 + 8 * N * 128 + 1024;
    if (cudaFuncSetAttribute(upproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    prof_begin(c.stream, "sm100_upproj");
    const cudaError_t e = launch_pdl(upproj_kernel, grid, dim3(kUpThreads), smem, c.stream, A, a, mg);
    prof_end(c.stream);
    if (launches) ++*launches;
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla
