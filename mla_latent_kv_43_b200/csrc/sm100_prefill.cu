// Prefill (materialised) MLA attention on tcgen05 tensor cores.
//
// With many query tokens per sequence the absorbed form stops paying: its
// score and weighted sum run over the 576-wide latent for every (query, key)
// pair, 2 H (576 + 512) flops, while expanding each cached latent once into
// the per-head keys and values costs 2 * 512 * 256 H flops per key and the
// attention itself then runs in the 192/128-wide head space, 2 H (192 + 128)
// flops per pair.  This is the training / reference factorisation of
// "Understanding MLA (Multi-head Latent Attention)" (sections "Reference code
// vs serving engines" and 6, "Training vs decode"), written out in
// "Multi-Head Latent Attention", section 3 (reference implementation):
// k_content = c W_UK, v = c W_UV, the shared rotated rope key broadcast to
// every head, ordinary scaled dot-product attention over the concatenated
// 192 dims, scale 1/sqrt(192).
//
// Steps of one call (same inputs and outputs as the absorbed decode):
//   1. q_rot[t][h] = RoPE(q_rope[t][h], p(t))                       (CUDA cores)
//   2. Kn = c W_uk, V = c W_uv for rows t < max_len of each sequence,
//      rows at or past the sequence's length zeroed, stored head-major
//      [H][B][max_len][128] so that a head's key tile is one contiguous
//      16 KB block                                                    (expand_kernel)
//   3. causal flash attention per (256-query tile, head, sequence)   (this file)
//
// Attention kernel.  One CTA: 256 queries of one head in two groups of 128
// (each group's rows are the TMEM lanes / M of its GEMMs); the two groups
// share every key and value tile.  Per 64-key tile and group:
// S = [q_nope || q_rot] [Kn || k_rope]^T (M 128, N 64, K 192) into one of the
// group's two TMEM score buffers; the softmax warps (one thread per query
// row, the row read from TMEM once and the buffer released at once) mask keys
// past the row's position (only in warps whose rows reach the diagonal; the
// others take a select-free path with paired FMAs), keep a base-2 running maximum that
// moves only when it grows by more than 2^8 (O and the row sum are rescaled
// then) and write P as bf16 over the first 32 columns of the very score
// buffer they read; O += P V (M 128, N 128, K 64) takes P from TMEM (A
// operand) and V MN-major from shared memory, and its completion frees the
// score buffer.  P is thus double-buffered with the scores: a group's softmax
// of tile i waits for the value GEMM of tile i - 1 only when O must be
// rescaled.  Keys and values have rings of their own (three tiles each): a key
// tile is released when its last score GEMM completes, a value tile when its
// last value GEMM does.  The grid runs head
// by head (the query tiles of one head, longest first, then the next head),
// so the CTAs in flight share a few heads' keys and values in L2.  The MMA
// warp issues both groups' score GEMMs of tile i, then their value GEMMs of
// tile i - 1, so one group's softmax runs while the tensor core works for the
// other.
// Roles (384 threads): warp 0 TMA for the queries and keys, warp 10 TMA for
// the values (so a key load never waits behind a value buffer's release),
// warp 1 issues the score GEMMs, warp 11 the value GEMMs, warps 2-5 softmax
// of group 0, warps 6-9 of group 1.  With one issuer, the value GEMM of a
// tile whose P was ready waited about a microsecond behind the issue of the
// next score GEMMs (an issuing thread stalls while the tensor pipe is full),
// and the score GEMM two tiles later waits for that value GEMM; two issuers
// keep that chain short.  The tensor pipe runs both warps' GEMMs in arrival
// order, and each warp's commits track its own GEMMs.
// Each key or value tile arrives in one tensor copy (both 64-column halves
// of its 128-wide rows, viewed as two groups of stride 128 bytes), the rope
// key in a second one.
// TMEM: O of group g at [128 g, 128 g + 128), S double buffers at
// [256 + 128 g, 256 + 128 g + 128) (P over the first half of each).
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "profile.h"
#include "sm100_host.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

namespace {

constexpr int kQ = 128;                            // queries per group
constexpr int kGroups = 2;                         // query groups per CTA
constexpr int kKeys = 64;                          // keys per tile
constexpr int kKStages = 3, kVStages = 3;
constexpr int kBox = 8192;                         // 64 rows x 128 B
constexpr int kQBox = 16384;                       // 128 rows x 128 B
constexpr int kOffK = kGroups * 3 * kQBox;         // Q per group: q_nope[0:64], q_nope[64:128], q_rot
constexpr int kKBytes = 3 * kBox;                  // key tile: Kn[0:64], Kn[64:128], k_rope
constexpr int kVBytes = 2 * kBox;                  // value tile: V[0:64], V[64:128]
constexpr int kOffV = kOffK + kKStages * kKBytes;
constexpr int kSmemBytes = kOffV + kVStages * kVBytes;
constexpr int kThreads = 384;
constexpr uint32_t kColO = 0, kColS = 256, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;          // log2 units

struct PrefillArgs {
    const int32_t* seq_lens;
    int B, n_q, H, q_tiles;
    int64_t capacity, max_len;
    float scale_log2;                              // softmax scale * log2(e)
    __nv_bfloat16* out;                            // [B][n_q][H][128]
    int32_t* status;
};

struct RopeTurns {
    uint64_t turn[32];
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


// a * b + c on two fp32 lanes at once (one paired FMA), denormals flushed
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.ftz.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// q_rot[t][h][0:64] = RoPE(q_rope[t][h], p(t)): one CTA per query token.  The
// rotation of pair i depends only on the token's position, so the token's 32
// (cos, sin) pairs are computed once (the same fixed-point angle reduction as
// the decode path's, so the results are identical) and every head reuses
// them; the token's H x 64 values then stream through in 16-byte chunks that
// consecutive threads take in order (coalesced loads and stores).
__global__ void __launch_bounds__(128) prefill_qrope_kernel(const __nv_bfloat16* __restrict__ q_rope,
                                                            const int32_t* __restrict__ seq_lens, int BJ, int n_q,
                                                            int H, RopeTurns rt, __nv_bfloat16* __restrict__ q_rot) {
    __shared__ float2 cs[32];
    const int t = blockIdx.x;
    if (t >= BJ) return;
    const int b = t / n_q, j = t % n_q;
    const int64_t p = query_pos(seq_lens[b], n_q, j);
    if (threadIdx.x < 32) {
        float c, s;
        rope_cos_sin_turn(p, rt.turn[threadIdx.x], &c, &s);
        cs[threadIdx.x] = make_float2(c, s);
    }
    __syncthreads();
    const uint4* src = reinterpret_cast<const uint4*>(q_rope + (int64_t)t * H * 64);
    uint4* dst = reinterpret_cast<uint4*>(q_rot + (int64_t)t * H * 64);
    for (int i = threadIdx.x; i < H * 8; i += blockDim.x) {
        const uint4 v = src[i];
        const int pair0 = 4 * (i & 7);               // chunk i % 8 of a head row: pairs 4 (i % 8) ..
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
            const float2 r = cs[pair0 + k];
            w[k] = pack_bf16(x.x * r.x - x.y * r.y, x.x * r.y + x.y * r.x);
        }
        dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Expansion of the cached latents into per-head keys and values: one CTA per
// (128 cache rows of a sequence, head h) computes [Kn | V][t][h] = c[t]
// [W_uk[h] | W_uv[h]] as one GEMM with M = 128 rows, N = 256 (the head's
// 128 key and 128 value columns), K = 512 in eight 64-wide blocks through a
// two-stage ring.  Two CTAs share an SM (96 KB each, 256 TMEM columns each),
// so one's epilogue overlaps the other's MMAs.
constexpr int kExThreads = 128;
constexpr int kExStages = 2;
constexpr int kExStageBytes = kQBox + 4 * kBox;    // c rows [128][64], W_uk[h] 64 x 128, W_uv[h] 64 x 128
constexpr int kExSmem = kExStages * kExStageBytes;

struct ExpandArgs {
    const int32_t* seq_lens;
    int B, max_len, row_tiles;                     // row tiles of 128 per sequence
    __nv_bfloat16 *kn, *v;                         // [H][B][max_len][128]
    int32_t* status;
};

__global__ void __launch_bounds__(kExThreads, 2)
expand_kernel(const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_wk,
              const __grid_constant__ CUtensorMap map_wv, ExpandArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kExStages], empty[kExStages], done;
    __shared__ uint32_t tmem_base;
    __shared__ int flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int b = blockIdx.x / a.row_tiles, t0 = (blockIdx.x % a.row_tiles) * 128;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kExStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(&done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    constexpr int kBlocks = 8;                     // K = 512
    if (warp == 0) {
        if (elect_one()) {
            for (int kb = 0; kb < kBlocks; ++kb) {
                const int s = kb % kExStages;
                if (kb >= kExStages && !mbar_wait(&empty[s], ((kb / kExStages) - 1) & 1, nullptr)) break;
                uint8_t* st = smem + s * kExStageBytes;
                mbar_expect_tx(&full[s], kExStageBytes);
                tma_load_3d(st, &map_c, &full[s], kb * 64, t0, b);
                tma_load_3d(st + kQBox, &map_wk, &full[s], 0, kb * 64, h);
                tma_load_3d(st + kQBox + kBox, &map_wk, &full[s], 64, kb * 64, h);
                tma_load_3d(st + kQBox + 2 * kBox, &map_wv, &full[s], 0, kb * 64, h);
                tma_load_3d(st + kQBox + 3 * kBox, &map_wv, &full[s], 64, kb * 64, h);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        constexpr uint32_t idesc = idesc_bf16(128, 256, false, true);
        const uint32_t sb0 = smem_u32(smem);
        const uint64_t da = sdesc(sb0, 16, 1024, kSwizzle128);                 // c rows, K-major
        const uint64_t db = sdesc(sb0 + kQBox, kBox, 1024, kSwizzle128);       // weights, MN-major
        bool ok = true;
        for (int kb = 0; kb < kBlocks && ok; ++kb) {
            const int s = kb % kExStages;
            int r = 0;
            if (lane == 0) r = mbar_wait(&full[s], (kb / kExStages) & 1, nullptr) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, r, 0) != 0;
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ss_w(tmem, sdesc_add(da, s * kExStageBytes + ks * 32),
                         sdesc_add(db, s * kExStageBytes + ks * 2048), idesc, (kb | ks) ? 1u : 0u);
            mma_commit_w(&empty[s]);
        }
        mma_commit_w(&done);
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        flag = mbar_wait(&done, 0, nullptr) ? 1 : 0;
        if (!flag) set_status(a.status, MLA_ERR_TIMEOUT);
    }
    __syncthreads();
    tc_fence_after();
    // row t0 + r of sequence b: 256 columns leave TMEM in eight 32-column chunks
    const int r = warp * 32 + lane, t = t0 + r;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const bool row_ok = t < a.max_len;
    const bool zero = !flag || t >= a.seq_lens[b];
    const int64_t orow = ((int64_t)h * a.B + b) * a.max_len + t;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_off + 32 * c, rr);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
            w[k] = zero ? 0u : pack_bf16(__uint_as_float(rr[2 * k]), __uint_as_float(rr[2 * k + 1]));
        if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>((c < 4 ? a.kn : a.v) + orow * 128 + 32 * (c & 3));
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 256);
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_attend_kernel(const __grid_constant__ CUtensorMap map_qn, const __grid_constant__ CUtensorMap map_qr,
                      const __grid_constant__ CUtensorMap map_kn, const __grid_constant__ CUtensorMap map_kr,
                      const __grid_constant__ CUtensorMap map_v, PrefillArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // Per group g and buffer b: s_full[g][b] the score GEMM into buffer b is
    // done, p_full[g][b] its P is written over it, s_free[g][b] the value GEMM
    // that read that P is done (the buffer may take the next score GEMM);
    // o_done[g][t & 1] completes when O GEMM t of the group is done.  A tile's
    // barrier of buffer b is two completions after the previous one of the same
    // buffer and cannot run ahead of it, so a parity names exactly one completion.
    __shared__ uint64_t q_full, k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
    __shared__ uint64_t s_full[kGroups][2], s_free[kGroups][2], p_full[kGroups][2], o_done[kGroups][2], drain,
        drain_o;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // head by head, then sequence, then query tile (longest first)
    const int per_head = a.q_tiles * a.B;
    const int h = (int)(blockIdx.x / per_head);
    const int rem = (int)(blockIdx.x % per_head);
    const int b = rem / a.q_tiles, qt = a.q_tiles - 1 - rem % a.q_tiles;
    const int q0 = qt * kGroups * kQ;
    const int64_t len = a.seq_lens[b];
    const bool seq_ok = len_ok(len, a.n_q, a.capacity, a.max_len);
    // key tiles of group g: keys 0 .. p of its last query (none for a group past n_q)
    auto tiles_of = [&](int g) -> int {
        const int first = q0 + g * kQ, last = min(first + kQ, a.n_q) - 1;
        return (seq_ok && first < a.n_q) ? (int)((len - a.n_q + last) / kKeys) + 1 : 0;
    };
    const int n_g0 = tiles_of(0), n_g1 = tiles_of(1);
    const int n_all = max(n_g0, n_g1);

    if (threadIdx.x == 0) {
        mbar_init(&q_full, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int g = 0; g < kGroups; ++g) {
            for (int i = 0; i < 2; ++i) {
                mbar_init(&s_full[g][i], 1);
                mbar_init(&s_free[g][i], 1);   // committed after the value GEMM that read buffer i
                mbar_init(&o_done[g][i], 1);
                mbar_init(&p_full[g][i], 4);   // the group's four softmax warps have written P
            }
        }
        mbar_init(&drain, 1);
        mbar_init(&drain_o, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t sbase = smem_u32(smem);
    volatile int* abort = &abort_flag;
    auto fail = [&]() {
        *abort = 1;
        set_status(a.status, MLA_ERR_TIMEOUT);
    };
    // lane 0 waits (bounded), the warp follows its outcome
    auto wait_w = [&](uint64_t* bar, uint32_t parity) -> bool {
        int ok = 1;
        if (lane == 0) ok = mbar_wait(bar, parity, abort) ? 1 : 0;
        return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (n_all > 0 && elect_one()) {
            tma_prefetch(&map_kn);
            tma_prefetch(&map_qn);
            const int qrow = b * a.n_q + q0;
            // both query tiles (rows past n_q belong to the next sequence or are zero filled)
            mbar_expect_tx(&q_full, kGroups * 3 * kQBox);
#pragma unroll
            for (int g = 0; g < kGroups; ++g) {
                uint8_t* qs = smem + g * 3 * kQBox;
                tma_load_4d(qs, &map_qn, &q_full, 0, h, qrow + g * kQ, 0);
                tma_load_3d(qs + 2 * kQBox, &map_qr, &q_full, 0, h, qrow + g * kQ);
            }
            const int krow = (h * a.B + b) * (int)a.max_len, crow = b * (int)a.capacity;
            // rows past the sequence are zero (Kn) or masked (k_rope); past the
            // tensor they are zero filled
            int nk = 0;
            bool ok = true;
            for (int i = 0; ok && i < n_all; ++i) {
                const int sk = i % kKStages;
                if (i >= kKStages && !mbar_wait(&k_empty[sk], ((i / kKStages) - 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                uint8_t* kt = smem + kOffK + sk * kKBytes;
                mbar_expect_tx(&k_full[sk], kKBytes);
                tma_load_3d(kt, &map_kn, &k_full[sk], 0, krow + i * kKeys, 0);
                tma_load_2d(kt + 2 * kBox, &map_kr, &k_full[sk], 512, crow + i * kKeys);
                ++nk;
            }
            if (!ok) fail();
            // no copy of this CTA may still be in flight when it exits
            mbar_wait(&q_full, 0, nullptr);
            for (int k = nk > kKStages ? nk - kKStages : 0; k < nk; ++k)
                mbar_wait(&k_full[k % kKStages], (k / kKStages) & 1, nullptr);
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ TMA producer, values
        if (n_all > 0 && elect_one()) {
            tma_prefetch(&map_v);
            const int krow = (h * a.B + b) * (int)a.max_len;
            int nv = 0;
            bool ok = true;
            for (int i = 0; ok && i < n_all; ++i) {
                const int sv = i % kVStages;
                if (i >= kVStages && !mbar_wait(&v_empty[sv], ((i / kVStages) - 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                uint8_t* vt = smem + kOffV + sv * kVBytes;
                mbar_expect_tx(&v_full[sv], kVBytes);
                tma_load_3d(vt, &map_v, &v_full[sv], 0, krow + i * kKeys, 0);
                ++nv;
            }
            if (!ok) fail();
            for (int k = nv > kVStages ? nv - kVStages : 0; k < nv; ++k)
                mbar_wait(&v_full[k % kVStages], (k / kVStages) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ score GEMM issuer
        // Per key tile i: the score GEMMs of both groups, each into its buffer
        // i & 1 once the value GEMM that read that buffer (tile i - 2) is done.
        if (n_all > 0) {
            constexpr uint32_t idS = idesc_bf16(128, 64, false, false);
            const uint64_t dQ = sdesc(sbase, 16, 1024, kSwizzle128);                   // K-major
            const uint64_t dK = sdesc(sbase + kOffK, 16, 1024, kSwizzle128);           // K-major
            bool ok = wait_w(&q_full, 0);
            for (int i = 0; ok && i < n_all; ++i) {
                const int sk = i % kKStages, sb = i & 1;
                if (!(ok = wait_w(&k_full[sk], (i / kKStages) & 1))) break;
#pragma unroll
                for (int g = 0; g < kGroups; ++g) {
                    if (!ok || i >= (g == 0 ? n_g0 : n_g1)) continue;
                    if (i >= 2 && !(ok = wait_w(&s_free[g][sb], ((i >> 1) - 1) & 1))) break;
                    tc_fence_after();
                    const uint32_t dS = tmem + kColS + 128 * g + 64 * sb;
#pragma unroll
                    for (int kb = 0; kb < 3; ++kb)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_ss_w(dS, sdesc_add(dQ, g * 3 * kQBox + kb * kQBox + ks * 32),
                                     sdesc_add(dK, sk * kKBytes + kb * kBox + ks * 32), idS, (kb | ks) ? 1u : 0u);
                    mma_commit_w(&s_full[g][sb]);
                }
                if (!ok) break;
                mma_commit_w(&k_empty[sk]);
            }
            if (!ok && lane == 0) fail();
            mma_commit_w(&drain);
            if (lane == 0) mbar_wait(&drain, 0, nullptr);
            __syncwarp();
        }
    } else if (warp == 11) {
        // ------------------------------------------------------------ value GEMM issuer
        // Per key tile t and group: O += P V as soon as the group's P and the
        // value tile are in; the commit frees the score buffer that held P.
        if (n_all > 0) {
            constexpr uint32_t idO = idesc_bf16(128, 128, false, true);
            const uint64_t dV = sdesc(sbase + kOffV, kBox, 1024, kSwizzle128);         // MN-major
            bool ok = true;
            for (int t = 0; ok && t < n_all; ++t) {
                const int sv = t % kVStages;
                if (!(ok = wait_w(&v_full[sv], (t / kVStages) & 1))) break;
#pragma unroll
                for (int g = 0; g < kGroups; ++g) {
                    if (!ok || t >= (g == 0 ? n_g0 : n_g1)) continue;
                    if (!(ok = wait_w(&p_full[g][t & 1], (t >> 1) & 1))) break;
                    tc_fence_after();
                    // A = P in TMEM (bf16 pairs, 8 columns per 16 keys)
                    const uint32_t aP = tmem + kColS + 128 * g + 64 * (t & 1);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_ts_w(tmem + kColO + 128 * g, aP + 8 * ks, sdesc_add(dV, sv * kVBytes + ks * 2048), idO,
                                 (t | ks) ? 1u : 0u);
                    mma_commit_w(&o_done[g][t & 1]);
                    mma_commit_w(&s_free[g][t & 1]);
                }
                if (!ok) break;
                mma_commit_w(&v_empty[sv]);
            }
            if (!ok && lane == 0) fail();
            mma_commit_w(&drain_o);
            if (lane == 0) mbar_wait(&drain_o, 0, nullptr);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ softmax groups
        const int g = (warp - 2) >> 2;               // query group: rows q0 + 128 g ..
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int r = q * 32 + lane;                 // query row within the group
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t colO = kColO + 128 * g, colS = kColS + 128 * g;
        const int n_tiles = g == 0 ? n_g0 : n_g1;
        const int j = q0 + g * kQ + r;
        const bool row_ok = j < a.n_q;
        const int64_t p = (seq_ok && row_ok) ? query_pos(len, a.n_q, j) : -1;
        uint4* orow = reinterpret_cast<uint4*>(a.out + (((int64_t)b * a.n_q + j) * a.H + h) * 128);
        if (!seq_ok) {
            if (row_ok)
#pragma unroll
                for (int c = 0; c < 16; ++c) orow[c] = make_uint4(0u, 0u, 0u, 0u);
            if (r == 0 && g == 0) set_status(a.status, MLA_ERR_LEN);
        } else if (n_tiles > 0) {
            float m_used = -INFINITY, l = 0.f;
            bool ok = true;
            for (int i = 0; i < n_tiles; ++i) {
                const int sb = i & 1;
                if (!(ok = wait_w(&s_full[g][sb], (i >> 1) & 1))) break;
                tc_fence_after();
                // The score row is read once; the score buffer is free for the GEMM two
                // tiles later as soon as it is in registers.
                float x[kKeys];
                {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tmem + lane_off + colS + 64 * sb, r0);
                    tmem_ld32(tmem + lane_off + colS + 64 * sb + 32, r1);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        x[k] = __uint_as_float(r0[k]);
                        x[32 + k] = __uint_as_float(r1[k]);
                    }
                }
                // Causal mask: keys past the row's position become -inf (a select, so
                // whatever lies past the sequence never leaks in).  Warp-uniform: a warp
                // takes the masked path if any of its rows needs it.
                const int64_t key0 = (int64_t)i * kKeys;
                const bool masked = __any_sync(0xffffffffu, key0 + kKeys - 1 > p);
                if (masked) {
                    const int lim = (int)max((int64_t)-1, min((int64_t)kKeys, p - key0));   // last visible column
#pragma unroll
                    for (int n = 0; n < kKeys; ++n) x[n] = n > lim ? -INFINITY : x[n];
                }
                float m8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    m8[k] = fmaxf(fmaxf(fmaxf(x[k], x[k + 8]), fmaxf(x[k + 16], x[k + 24])),
                                  fmaxf(fmaxf(x[k + 32], x[k + 40]), fmaxf(x[k + 48], x[k + 56])));
                const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) *
                                 a.scale_log2;
                // the maximum moves only when it grew by more than 2^8 (-inf + 8 is -inf)
                const float m = mx > m_used + kRescaleThreshold ? mx : m_used;
                // O holds tiles 0 .. i - 1 relative to m_used: rescale it when m moved,
                // once the group's O GEMM i - 1 is done.  TMEM accesses are
                // warp-collective, so lanes that need none multiply by 1.
                const bool need = m_used != -INFINITY && m > m_used;
                if (__any_sync(0xffffffffu, need)) {
                    if (i >= 1 && !(ok = wait_w(&o_done[g][(i - 1) & 1], ((i - 1) >> 1) & 1))) break;
                    tc_fence_after();
                    const float alpha = need ? ex2(m_used - m) : 1.f;
#pragma unroll 1
                    for (int c = 0; c < 8; ++c) {
                        uint32_t rr[16];
                        const uint32_t ta = tmem + lane_off + colO + 16 * c;
                        tmem_ld16(ta, rr);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 16; ++k) rr[k] = __float_as_uint(__uint_as_float(rr[k]) * alpha);
                        tmem_st16(ta, rr);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                }
                if (need) l *= ex2(m_used - m);
                m_used = m;
                // P (bf16 pairs of consecutive keys) for the first 32 columns of the buffer
                uint32_t pa[16], pb[16];
                float ps4[4] = {0.f, 0.f, 0.f, 0.f};
                if (!masked) {
                    // every key of the tile is visible to every row of this warp (so the
                    // maximum is finite): p = 2^(s * scale - m), two at a time
                    const float2 sc = make_float2(a.scale_log2, a.scale_log2), nm = make_float2(-m_used, -m_used);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 y = ffma2(make_float2(x[8 * c + 2 * k], x[8 * c + 2 * k + 1]), sc, nm);
                            const float p0 = ex2(y.x), p1 = ex2(y.y);
                            ps4[k] += p0 + p1;
                            (c < 4 ? pa : pb)[4 * (c & 3) + k] = pack_bf16(p0, p1);
                        }
                    }
                } else {
                    // masked keys are -inf (p = 0); a row with no visible key yet keeps P = 0
                    const bool live = m_used != -INFINITY;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int n = 8 * c + 2 * k;
                            const float p0 = live ? ex2(fmaf(x[n], a.scale_log2, -m_used)) : 0.f;
                            const float p1 = live ? ex2(fmaf(x[n + 1], a.scale_log2, -m_used)) : 0.f;
                            ps4[k] += p0 + p1;
                            (c < 4 ? pa : pb)[4 * (c & 3) + k] = pack_bf16(p0, p1);
                        }
                    }
                }
                l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
                // the whole score row is in registers, so P may overwrite it
                tmem_st16(tmem + lane_off + colS + 64 * sb, pa);
                tmem_st16(tmem + lane_off + colS + 64 * sb + 16, pb);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[g][sb]);
            }
            // every O GEMM of the group is done once its last one is
            if (ok) ok = wait_w(&o_done[g][(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1);
            if (!ok) {
                if (lane == 0) fail();
            } else {
                tc_fence_after();
                const float inv = (row_ok && l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(tmem + lane_off + colO + 32 * c, rr);
                    tmem_wait_ld();
                    uint32_t w[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        w[k] = pack_bf16(__uint_as_float(rr[2 * k]) * inv, __uint_as_float(rr[2 * k + 1]) * inv);
                    if (row_ok)
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            orow[4 * c + k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

void prefill_layout(const mla_dims& d, int batch, int n_q, int64_t max_len, PrefillLayout* L) {
    auto up = [](int64_t v) { return (v + 255) / 256 * 256; };
    L->q_rot = 0;
    L->kn = up((int64_t)batch * n_q * d.heads * 64 * 2);
    L->v = L->kn + up((int64_t)batch * max_len * d.heads * 128 * 2);
    L->total = L->v + up((int64_t)batch * max_len * d.heads * 128 * 2);
}

int prefill_launch(const PrefillCall& c, int* launches) {
    const int B = c.batch, H = c.d.heads, n_q = c.n_q;
    const int BJ = B * n_q;
    PrefillLayout L;
    prefill_layout(c.d, B, n_q, c.max_len, &L);
    __nv_bfloat16* q_rot = reinterpret_cast<__nv_bfloat16*>(c.ws + L.q_rot);
    __nv_bfloat16* kn = reinterpret_cast<__nv_bfloat16*>(c.ws + L.kn);
    __nv_bfloat16* v = reinterpret_cast<__nv_bfloat16*>(c.ws + L.v);

    // 1. query rope
    RopeTurns rt;
    rope_turn_table(c.d.rope_base, 64, rt.turn);
    {
        prof_begin(c.stream, "sm100_prefill_qrope");
        prefill_qrope_kernel<<<(unsigned)BJ, 128, 0, c.stream>>>((const __nv_bfloat16*)c.q_rope, c.seq_lens, BJ, n_q,
                                                                 H, rt, q_rot);
        prof_end(c.stream);
        ++*launches;
        if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
    // 2. per-head keys and values from the latent rows
    {
        CUtensorMap mc, mwk, mwv;
        {
            const uint64_t dims[3] = {512, (uint64_t)c.max_len, (uint64_t)B},
                           str[2] = {576 * 2, (uint64_t)c.capacity * 576 * 2};
            const uint32_t box[3] = {64, 128, 1};
            if (!make_map(&mc, c.cache, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
        }
        {
            const uint64_t dims[3] = {128, 512, (uint64_t)H}, str[2] = {256, 512 * 256};
            const uint32_t box[3] = {64, 64, 1};
            if (!make_map(&mwk, c.W_uk, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
            if (!make_map(&mwv, c.W_uv, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
        }
        ExpandArgs e{};
        e.seq_lens = c.seq_lens;
        e.B = B;
        e.max_len = (int)c.max_len;
        e.row_tiles = (int)((c.max_len + 127) / 128);
        e.kn = kn;
        e.v = v;
        e.status = c.status;
        const size_t smem = kExSmem + 1024;
        if (cudaFuncSetAttribute(expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return MLA_ERR_CUDA;
        const int64_t gx = (int64_t)B * e.row_tiles;
        if (gx >= ((int64_t)1 << 31) || H > 65535) return MLA_ERR_UNSUPPORTED;
        prof_begin(c.stream, "sm100_prefill_expand");
        const cudaError_t err =
            launch_plain(expand_kernel, dim3((unsigned)gx, (unsigned)H), dim3(kExThreads), smem, c.stream, mc, mwk,
                         mwv, e);
        prof_end(c.stream);
        ++*launches;
        if (err != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
    // 3. causal attention
    CUtensorMap mqn, mqr, mkn, mkr, mv;
    {
        // q_nope [BJ][H][128] as (column in half, head, token, half): one box = 128
        // tokens of one head, both 64-column halves, landing half-major
        const uint64_t dims[4] = {64, (uint64_t)H, (uint64_t)BJ, 2}, str[3] = {256, (uint64_t)H * 256, 128};
        const uint32_t box[4] = {64, 1, (uint32_t)kQ, 2};
        if (!make_map(&mqn, c.q_nope, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        const uint64_t dims[3] = {64, (uint64_t)H, (uint64_t)BJ}, str[2] = {128, (uint64_t)H * 128};
        const uint32_t box[3] = {64, 1, (uint32_t)kQ};
        if (!make_map(&mqr, q_rot, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        // head-major rows (h * B + b) * max_len + t, as (column in half, row, half):
        // one box = 64 rows, both halves, landing half-major
        const uint64_t dims[3] = {64, (uint64_t)H * B * c.max_len, 2}, str[2] = {256, 128};
        const uint32_t box[3] = {64, (uint32_t)kKeys, 2};
        if (!make_map(&mkn, kn, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
        if (!make_map(&mv, v, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        const uint64_t dims[2] = {576, (uint64_t)B * c.capacity}, str[1] = {576 * 2};
        const uint32_t box[2] = {64, (uint32_t)kKeys};
        if (!make_map(&mkr, c.cache, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    PrefillArgs a{};
    a.seq_lens = c.seq_lens;
    a.B = B;
    a.n_q = n_q;
    a.H = H;
    a.q_tiles = (n_q + kGroups * kQ - 1) / (kGroups * kQ);
    a.capacity = c.capacity;
    a.max_len = c.max_len;
    a.scale_log2 = c.d.softmax_scale * 1.4426950408889634f;
    a.out = (__nv_bfloat16*)c.out;
    a.status = c.status;
    const size_t smem = kSmemBytes + 1024;
    if (cudaFuncSetAttribute(prefill_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return MLA_ERR_CUDA;
    const int64_t blocks = (int64_t)a.q_tiles * H * B;
    prof_begin(c.stream, "sm100_prefill_attend");
    const cudaError_t e = launch_plain(prefill_attend_kernel, dim3((unsigned)blocks), dim3(kThreads), smem, c.stream,
                                       mqn, mqr, mkn, mkr, mv, a);
    prof_end(c.stream);
    ++*launches;
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla
