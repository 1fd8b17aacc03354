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
    for (int w = 0; w < kThreads / 32; ++w) T += part_l[w];
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
    // First query token of every cluster's tile range [p T / pairs, (p + 1) T / pairs):
    // the first bj with cum[bj + 1] > floor(p T / pairs) (BJ when there is none).
    const int32_t T = s_cum[a.BJ];
    for (int p = tid; p < a.pairs; p += kThreads) {
        const int32_t s0 = (int32_t)(((uint32_t)p * (uint32_t)T) / (uint32_t)a.pairs);
        int l = 0, r = a.BJ;
        while (l < r) {
            const int mid = (l + r) >> 1;
            if (s_cum[mid + 1] > s0) r = mid; else l = mid + 1;
        }
        a.first_bj[p] = T == 0 ? a.BJ : l;
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

    const int nvalid = min(N, a.BJ - nt * N);
    {
        // B operand: row n (token nt * N + n), 64-column block kb at sB + kb * N * 128,
        // 16-byte chunk c of the 128-byte row at ((c ^ (n & 7)) << 4).
        // Phase 1: the pieces (slots) of each token and their log-sum-exp.  Many
        // tokens (the usual case: one or two pieces each): one thread per token, up
        // to kFast pieces' log-sum-exps loaded together.  Few tokens (typically
        // cut into many pieces): one warp per token, lanes over pieces.
        // Phase 2 (see below) then assembles the merged rows.
        constexpr int kFast = 4;
        const bool few = nvalid <= 8;
        __shared__ int m_mode[64], m_np[64], m_pf[64], m_pl[64], m_slot[64][kFast];   // mode 0: zeros, 1: o_lat as is, 2: merge
        __shared__ float m_w[64][kFast], m_M[64], m_inv[64];
        const PieceRange pr{mg.cum[mg.BJ], mg.pairs};
        auto token_range = [&](int n, int& mode, int& pf, int& pl) {
            mode = 0;
            pf = 0;
            pl = -1;
            if (n >= nvalid) return;
            const int bj = nt * N + n;
            const int c0 = mg.cum[bj], c1 = mg.cum[bj + 1];
            if (c1 == c0) return;
            pf = pr.pair_of(c0);
            pl = pr.pair_of(c1 - 1);
            mode = pf == pl ? 1 : 2;
        };
        if (few) {
            if (warp < nvalid) {
                const int n = warp;
                int mode, pf, pl;
                token_range(n, mode, pf, pl);
                float M = -INFINITY, S = 0.f;
                if (mode == 2) {
                    for (int p0 = pf; p0 <= pl; p0 += 32) {
                        const int p = p0 + lane;
                        if (p <= pl && (p == pf || !pr.empty(p))) M = fmaxf(M, mg.part_lse[PieceRange::slot(p, pf) * 256 + h]);
                    }
    #pragma unroll
                    for (int d = 16; d > 0; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
                    for (int p0 = pf; p0 <= pl; p0 += 32) {
                        const int p = p0 + lane;
                        if (p <= pl && (p == pf || !pr.empty(p))) S += exp2f(mg.part_lse[PieceRange::slot(p, pf) * 256 + h] - M);
                    }
    #pragma unroll
                    for (int d = 16; d > 0; d >>= 1) S += __shfl_xor_sync(0xffffffffu, S, d);
                }
                if (lane == 0) {
                    m_mode[n] = mode;
                    m_pf[n] = pf;
                    m_pl[n] = pl;
                    m_M[n] = M;
                    m_inv[n] = mode == 2 ? 1.f / S : 0.f;
                }
            }
        } else if (threadIdx.x < N) {
            const int n = threadIdx.x;
            int mode, np = 0, pf, pl;
            token_range(n, mode, pf, pl);
            float M = -INFINITY, S = 0.f;
            if (mode == 2) {
                int sl[kFast];
                for (int p = pf; p <= pl; ++p) {
                    if (p != pf && pr.empty(p)) continue;
                    if (np < kFast) sl[np] = PieceRange::slot(p, pf);
                    ++np;
                }
                float lse[kFast];
    #pragma unroll
                for (int i = 0; i < kFast; ++i) lse[i] = i < np ? mg.part_lse[sl[i] * 256 + h] : -INFINITY;
    #pragma unroll
                for (int i = 0; i < kFast; ++i) M = fmaxf(M, lse[i]);
                if (np > kFast) {            // more pieces: the rest one by one
                    int k = 0;
                    for (int p = pf; p <= pl; ++p) {
                        if (p != pf && pr.empty(p)) continue;
                        if (k++ >= kFast) M = fmaxf(M, mg.part_lse[PieceRange::slot(p, pf) * 256 + h]);
                    }
                }
    #pragma unroll
                for (int i = 0; i < kFast; ++i) {
                    const float w = i < np ? exp2f(lse[i] - M) : 0.f;
                    S += w;
                    m_w[n][i] = w;
                    m_slot[n][i] = i < np ? sl[i] : 0;
                }
                if (np > kFast) {
                    int k = 0;
                    for (int p = pf; p <= pl; ++p) {
                        if (p != pf && pr.empty(p)) continue;
                        if (k++ >= kFast) S += exp2f(mg.part_lse[PieceRange::slot(p, pf) * 256 + h] - M);
                    }
                }
            }
            m_mode[n] = mode;
            m_np[n] = np;
            m_pf[n] = pf;
            m_pl[n] = pl;
            m_M[n] = M;
            m_inv[n] = mode == 2 ? 1.f / S : 0.f;
        }
        __syncthreads();
        // row n of the B operand: 64-column block kb at sB + (kb * N + n) * 128, 16-byte chunk c at ((c ^ (n & 7)) << 4);
        // lane l holds columns [16 l, 16 l + 16): block l / 4, chunks 2 (l % 4) and 2 (l % 4) + 1
        auto put_row = [&](int n, const uint32_t (&w)[8]) {
            const int kb = lane >> 2, c = (lane & 3) * 2;
            const uint32_t row = smem_u32(sB + (kb * N + n) * 128);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((c ^ (n & 7)) << 4)), "r"(w[0]), "r"(w[1]),
                         "r"(w[2]), "r"(w[3]) : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + (((c + 1) ^ (n & 7)) << 4)), "r"(w[4]),
                         "r"(w[5]), "r"(w[6]), "r"(w[7]) : "memory");
        };
        auto accumulate = [&](float (&acc)[16], float wt, const uint4& v0, const uint4& v1) {
            const uint32_t pw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    #pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[j]));
                acc[2 * j] = fmaf(wt, f.x, acc[2 * j]);
                acc[2 * j + 1] = fmaf(wt, f.y, acc[2 * j + 1]);
            }
        };
        if (few) {
            // Few tokens: warp w assembles 64-column block w of every token row, lanes
            // over pieces (each lane one piece's 128-byte segment, weighted), then a
            // butterfly sum across the lanes; rows of tokens past nvalid stay zero.
            const int kb = warp;
            for (int n = 0; n < N; ++n) {
                const int mode = n < nvalid ? m_mode[n] : 0;
                const int bj = nt * N + n;
                float acc[64];
    #pragma unroll
                for (int i = 0; i < 64; ++i) acc[i] = 0.f;
                if (mode == 1 && lane == 0) {
                    const uint4* src = reinterpret_cast<const uint4*>(mg.o_lat + ((int64_t)bj * 128 + h) * 512 + 64 * kb);
    #pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v = src[c];
                        const uint32_t pw[4] = {v.x, v.y, v.z, v.w};
    #pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[j]));
                            acc[8 * c + 2 * j] = f.x;
                            acc[8 * c + 2 * j + 1] = f.y;
                        }
                    }
                } else if (mode == 2) {
                    const int pf = m_pf[n], pl = m_pl[n];
                    const float M = m_M[n], inv = m_inv[n];
                    for (int p0 = pf; p0 <= pl; p0 += 32) {
                        const int p = p0 + lane;
                        if (p <= pl && (p == pf || !pr.empty(p))) {
                            const int sl = PieceRange::slot(p, pf);
                            const uint4* src = reinterpret_cast<const uint4*>(mg.part_o + ((int64_t)sl * 128 + h) * 512 + 64 * kb);
                            uint4 v[8];
    #pragma unroll
                            for (int c = 0; c < 8; ++c) v[c] = src[c];
                            const float wt = exp2f(mg.part_lse[sl * 256 + h] - M) * inv;
    #pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                const uint32_t pw[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
    #pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[j]));
                                    acc[8 * c + 2 * j] = fmaf(wt, f.x, acc[8 * c + 2 * j]);
                                    acc[8 * c + 2 * j + 1] = fmaf(wt, f.y, acc[8 * c + 2 * j + 1]);
                                }
                            }
                        }
                    }
                }
                if (mode == 2) {
    #pragma unroll
                    for (int d = 16; d > 0; d >>= 1)
    #pragma unroll
                        for (int i = 0; i < 64; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], d);
                }
                // lane c (< 8) writes 16-byte chunk c of the 128-byte block: every lane holds
                // the full sums after the butterfly (mode 1: lane 0 only, broadcast below)
                if (mode == 1) {
    #pragma unroll
                    for (int i = 0; i < 64; ++i) acc[i] = __shfl_sync(0xffffffffu, acc[i], 0);
                }
                if (lane < 8) {
                    uint32_t w[4];
    #pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float lo = 0.f, hi = 0.f;
    #pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (c == lane) { lo = acc[8 * c + 2 * j]; hi = acc[8 * c + 2 * j + 1]; }
                        w[j] = pack_bf16(lo, hi);
                    }
                    const uint32_t row = smem_u32(sB + (kb * N + n) * 128);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((lane ^ (n & 7)) << 4)), "r"(w[0]),
                                 "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
                    if (n < nvalid && mode != 1)
                        reinterpret_cast<uint4*>(mg.o_lat + ((int64_t)bj * 128 + h) * 512 + 64 * kb)[lane] =
                            make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        } else {
        // four tokens per warp and round, the first two pieces of each loaded
        // together (most tokens have one or two); further pieces follow one by one
        constexpr int kTok = 4;
        for (int n0 = kTok * warp; n0 < N; n0 += kTok * (kUpThreads / 32)) {
            uint4 v[kTok][2][2];
            int mode[kTok];
    #pragma unroll
            for (int u = 0; u < kTok; ++u) {
                const int n = n0 + u;
                mode[u] = n < N ? m_mode[n] : 0;
                const int bj = nt * N + n;
                if (mode[u] == 1) {
                    const uint4* src = reinterpret_cast<const uint4*>(mg.o_lat + ((int64_t)bj * 128 + h) * 512) + 2 * lane;
                    v[u][0][0] = src[0];
                    v[u][0][1] = src[1];
                } else if (mode[u] == 2) {
    #pragma unroll
                    for (int i = 0; i < 2; ++i) {            // a merged token has at least two pieces
                        const uint4* src = reinterpret_cast<const uint4*>(mg.part_o + ((int64_t)m_slot[n][i] * 128 + h) * 512) + 2 * lane;
                        v[u][i][0] = src[0];
                        v[u][i][1] = src[1];
                    }
                }
            }
    #pragma unroll
            for (int u = 0; u < kTok; ++u) {
                const int n = n0 + u;
                if (n >= N) continue;
                const int bj = nt * N + n;
                uint4* orow = reinterpret_cast<uint4*>(mg.o_lat + ((int64_t)bj * 128 + h) * 512) + 2 * lane;
                uint32_t w[8];
                if (mode[u] == 0) {
    #pragma unroll
                    for (int i = 0; i < 8; ++i) w[i] = 0u;
                    if (n < nvalid) {
                        orow[0] = make_uint4(0u, 0u, 0u, 0u);
                        orow[1] = make_uint4(0u, 0u, 0u, 0u);
                    }
                } else if (mode[u] == 1) {
                    w[0] = v[u][0][0].x; w[1] = v[u][0][0].y; w[2] = v[u][0][0].z; w[3] = v[u][0][0].w;
                    w[4] = v[u][0][1].x; w[5] = v[u][0][1].y; w[6] = v[u][0][1].z; w[7] = v[u][0][1].w;
                } else {
                    float acc[16];
    #pragma unroll
                    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
                    accumulate(acc, m_w[n][0], v[u][0][0], v[u][0][1]);
                    accumulate(acc, m_w[n][1], v[u][1][0], v[u][1][1]);
                    const int np = m_np[n];
                    for (int i = 2; i < min(np, kFast); ++i) {
                        const uint4* src = reinterpret_cast<const uint4*>(mg.part_o + ((int64_t)m_slot[n][i] * 128 + h) * 512) + 2 * lane;
                        accumulate(acc, m_w[n][i], src[0], src[1]);
                    }
                    if (np > kFast) {              // the rest one by one
                        const int pf = m_pf[n];
                        const float M = m_M[n];
                        int k = 0;
                        for (int p = pf; ; ++p) {
                            if (p != pf && pr.empty(p)) continue;
                            if (k++ < kFast) continue;
                            const int sl = PieceRange::slot(p, pf);
                            const uint4* src = reinterpret_cast<const uint4*>(mg.part_o + ((int64_t)sl * 128 + h) * 512) + 2 * lane;
                            accumulate(acc, exp2f(mg.part_lse[sl * 256 + h] - M), src[0], src[1]);
                            if (k == np) break;
                        }
                    }
                    const float inv = m_inv[n];
    #pragma unroll
                    for (int i = 0; i < 8; ++i) w[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
                    orow[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    orow[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
                put_row(n, w);
            }
        }
        }
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
    a.pairs = pairs;
    a.n_sel = c.n_sel;
    a.max_sel = c.max_sel;
    a.tile_keys = 64;                     // both attention kernels take 64-key tiles
    a.status = c.status;
    const dim3 grid(H + 1, 4, (BJ + N - 1) / N);      // column H: the plan CTA
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
