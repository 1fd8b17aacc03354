// Absorbed MLA attention against the latent cache on tcgen05 tensor cores.
//
// For one query token (b, j) and a range of 64-key tiles of its sequence,
// with q_lat = [W_uk q_nope || RoPE(q_rope)] (576 wide, all 128 heads):
//     S[h][n] = <q_lat[h], cache[b][n][0:576]>                    (score)
//     online softmax over n (base 2, scale folded in), fp32
//     O[h][0:512] += P[h][n] cache[b][n][0:512]                    (weighted latent)
// i.e. the score of "Understanding MLA (Multi-head Latent Attention)",
// section 4 (content part through the absorbed query, position part through
// the shared rope key), weighted over the cached latents as on aicassindra
// "Multi-head latent attention", "End-to-end flow".
//
// Work split.  All heads of a token share each cache row, so the 128 heads
// are the M dimension of both contractions.  The fp32 accumulator of
// 128 heads x 512 latent columns would fill all 512 TMEM columns, so a
// cluster of two CTAs splits the latent: CTA r owns latent columns
// [256r, 256r+256) and rope columns [512+32r, 512+32r+32).  Each CTA loads
// only its 288 columns of every tile (each cache byte crosses HBM once, no
// multicast), computes a partial score over its 288 columns with Q resident
// in TMEM, and the two partials are exchanged through distributed shared
// memory and added in the same order on both CTAs, so both run the identical
// softmax.  Each CTA then accumulates its half of O from the same smem tile
// read as an MN-major operand.
//
// Roles (192 threads): warp 0 issues TMA, warp 1 issues MMAs, warps 2-5 run
// the softmax (thread <-> head <-> TMEM lane) and the epilogues.
//
// Work items.  The key tiles of all query tokens are concatenated and cut
// into one contiguous range per cluster.  A token whose tiles all fall in one
// cluster's range is finished there (normalised latent output, bf16); a token
// cut across clusters leaves fp32 partial outputs plus log2-sum-exp per piece
// for the combine kernel.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "profile.h"
#include "sm100_host.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kAttnKeys = 64;

namespace {

constexpr int kStages = 3;
constexpr int kLatBox = 8192;                      // 64 keys x 64 columns x 2 B
constexpr int kRopeBox = 4096;                     // 64 keys x 32 columns x 2 B
constexpr int kStageBytes = 4 * kLatBox + kRopeBox;
constexpr int kPBytes = 128 * 128;                 // 128 heads x 64 keys bf16
constexpr int kXRow = 272;                         // 64 floats + 16 B pad (bank-conflict free)
constexpr int kXBytes = 128 * kXRow;
constexpr int kOffP = kStages * kStageBytes;
constexpr int kOffX = kOffP + 2 * kPBytes;
constexpr int kSmemBytes = kOffX + 2 * kXBytes;
constexpr int kThreads = 192;
constexpr uint32_t kColO = 0, kColS = 256, kColQ = 320, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;          // log2 units: rescale O only when the max grows by > 2^8

struct AttnArgs {
    const __nv_bfloat16* q_lat;   // [BJ][128][576]
    const int32_t* cum;           // [BJ + 1] tile prefix
    const int32_t* seq_lens;
    int BJ, n_q, pairs;
    float scale_log2;             // softmax_scale * log2(e)
    __nv_bfloat16* o_lat;         // [BJ][128][512]
    float* part_o;                // [2 * pairs][128][512]
    float* part_lse;              // [2 * pairs][128], log2 domain
    int32_t* status;
};

struct Item {
    int bj, t0, t1, n_vis, slot;  // slot < 0: finished here
};

// Iterates the pieces of the concatenated tile range [s0, s1) of one cluster.
struct ItemIter {
    const int32_t* cum;
    int BJ, n_q, bj, s0, s1, pair;
    const int32_t* lens;
    __device__ void init(const AttnArgs& a, int p) {
        cum = a.cum;
        BJ = a.BJ;
        n_q = a.n_q;
        lens = a.seq_lens;
        pair = p;
        const int T = cum[BJ];
        s0 = (int)((int64_t)p * T / a.pairs);
        s1 = (int)((int64_t)(p + 1) * T / a.pairs);
        int lo = 0, hi = BJ;          // first bj with cum[bj + 1] > s0
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (cum[mid + 1] > s0) hi = mid; else lo = mid + 1;
        }
        bj = lo;
    }
    __device__ bool next(Item& it) {
        while (bj < BJ) {
            const int c0 = cum[bj], c1 = cum[bj + 1];
            if (c0 >= s1) return false;
            const int cur = bj++;
            if (c1 == c0) continue;
            const int lo = max(c0, s0), hi = min(c1, s1);
            if (hi <= lo) continue;
            it.bj = cur;
            it.t0 = lo - c0;
            it.t1 = hi - c0;
            const int b = cur / n_q, j = cur % n_q;
            it.n_vis = (int)(query_pos(lens[b], n_q, j) + 1);
            it.slot = (c0 >= s0 && c1 <= s1) ? -1 : (c0 < s0 ? 2 * pair : 2 * pair + 1);
            return true;
        }
        return false;
    }
};

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ float4 ld_shared_v4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attend_kernel(const __grid_constant__ CUtensorMap map_lat, const __grid_constant__ CUtensorMap map_rope,
              AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kStages], empty[kStages];
    __shared__ uint64_t s_full, s_free, q_ready, drain;
    __shared__ uint64_t p_ready[2], p_free[2], x_full[2];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t peer = rank ^ 1u;
    const int pair = blockIdx.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&s_full, 1);
        mbar_init(&s_free, 128);
        mbar_init(&q_ready, 128);
        mbar_init(&drain, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&p_ready[i], 128);
            mbar_init(&p_free[i], 1);
            mbar_init(&x_full[i], 128);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();          // the peer's barriers are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    volatile int* abort = &abort_flag;
    auto fail = [&]() {
        *abort = 1;
        set_status(a.status, MLA_ERR_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch(&map_lat);
            tma_prefetch(&map_rope);
            ItemIter iter;
            iter.init(a, pair);
            Item item;
            uint32_t it = 0;
            bool ok = true;
            while (ok && iter.next(item)) {
                const int b = item.bj / a.n_q;
                for (int t = item.t0; t < item.t1; ++t, ++it) {
                    const int s = it % kStages;
                    if (it >= kStages && !mbar_wait(&empty[s], ((it / kStages) - 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * kStageBytes;
                    mbar_expect_tx(&full[s], kStageBytes);
                    const int key0 = t * kAttnKeys;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        tma_load_3d(st + i * kLatBox, &map_lat, &full[s], 256 * rank + 64 * i, key0, b);
                    tma_load_3d(st + 4 * kLatBox, &map_rope, &full[s], 512 + 32 * rank, key0, b);
                }
            }
            if (!ok) fail();
            // let every issued load land before the CTA can exit
            const uint32_t first = it > kStages ? it - kStages : 0;
            for (uint32_t i = first; i < it; ++i) mbar_wait(&full[i % kStages], (i / kStages) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (elect_one()) {
            constexpr uint32_t idS = idesc_bf16(128, 64, false, false);
            constexpr uint32_t idO = idesc_bf16(128, 256, false, true);
            const uint32_t sbase = smem_u32(smem);
            const uint32_t pbase = sbase + kOffP;
            ItemIter iter;
            iter.init(a, pair);
            Item item;
            uint32_t it = 0, n_items = 0;
            bool ok = true;
            auto issue_o = [&](uint32_t g, bool first) -> bool {
                const int pb = g & 1;
                if (!mbar_wait(&p_ready[pb], (g >> 1) & 1, abort)) return false;
                tc_fence_after();
                const uint32_t st = sbase + (g % kStages) * kStageBytes;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = sdesc(pbase + pb * kPBytes + ks * 32, 16, 1024, kSwizzle128);
                    const uint64_t bd = sdesc(st + ks * 2048, kLatBox, 1024, kSwizzle128);
                    mma_ss(tmem + kColO, ad, bd, idO, (first && ks == 0) ? 0u : 1u);
                }
                mma_commit(&empty[g % kStages]);
                mma_commit(&p_free[pb]);
                return true;
            };
            while (ok && iter.next(item)) {
                if (!mbar_wait(&q_ready, n_items & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int T = item.t1 - item.t0;
                for (int k = 0; k < T && ok; ++k) {
                    const uint32_t g = it + k;
                    const int s = g % kStages;
                    if (!mbar_wait(&full[s], (g / kStages) & 1, abort)) { ok = false; break; }
                    if (g > 0 && !mbar_wait(&s_free, (g - 1) & 1, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = sbase + s * kStageBytes;
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks) {
                        const uint64_t bd = sdesc(st + (ks >> 2) * kLatBox + (ks & 3) * 32, 16, 1024, kSwizzle128);
                        mma_ts(tmem + kColS, tmem + kColQ + 8 * ks, bd, idS, ks ? 1u : 0u);
                    }
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const uint64_t bd = sdesc(st + 4 * kLatBox + ks * 32, 16, 512, kSwizzle64);
                        mma_ts(tmem + kColS, tmem + kColQ + 8 * (16 + ks), bd, idS, 1u);
                    }
                    mma_commit(&s_full);
                    if (k > 0 && !issue_o(g - 1, k == 1)) ok = false;
                }
                if (ok && T > 0 && !issue_o(it + T - 1, T == 1)) ok = false;
                it += T;
                ++n_items;
            }
            if (!ok) fail();
            mma_commit(&drain);
            mbar_wait(&drain, 0, nullptr);
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int h = q * 32 + lane;            // head == TMEM lane
        const int tid = threadIdx.x - 64;       // 0..127
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t sbase = smem_u32(smem);
        const uint32_t x_local = sbase + kOffX;
        const uint32_t x_peer = map_peer(x_local, peer);
        const uint32_t xbar_peer[2] = {map_peer(smem_u32(&x_full[0]), peer), map_peer(smem_u32(&x_full[1]), peer)};
        uint32_t o_seen[2] = {0, 0};            // completed O GEMMs observed per P buffer
        auto wait_o = [&](uint32_t g) -> bool { // O GEMM of global tile g has completed
            const int pb = g & 1;
            const uint32_t n = g >> 1;
            if (o_seen[pb] > n) return true;
            if (!mbar_wait(&p_free[pb], n & 1, abort)) return false;
            o_seen[pb] = n + 1;
            return true;
        };
        ItemIter iter;
        iter.init(a, pair);
        Item item;
        uint32_t it = 0;
        bool ok = true;
        while (ok && iter.next(item)) {
            // Q slice of this token into TMEM (A operand of the score GEMM)
            {
                const uint4* src = reinterpret_cast<const uint4*>(a.q_lat + ((int64_t)item.bj * 128 + h) * 576);
                uint32_t w[16];
#pragma unroll
                for (int c = 0; c < 8; ++c) {     // latent columns 256r + 32c .. +31 (16 words)
                    const uint4 v0 = src[(256 * rank + 32 * c) / 8 + 0];
                    const uint4 v1 = src[(256 * rank + 32 * c) / 8 + 1];
                    const uint4 v2 = src[(256 * rank + 32 * c) / 8 + 2];
                    const uint4 v3 = src[(256 * rank + 32 * c) / 8 + 3];
                    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
                    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
                    w[8] = v2.x; w[9] = v2.y; w[10] = v2.z; w[11] = v2.w;
                    w[12] = v3.x; w[13] = v3.y; w[14] = v3.z; w[15] = v3.w;
                    tmem_st16(tmem + lane_off + kColQ + 16 * c, w);
                }
                {
                    const uint4 v0 = src[(512 + 32 * rank) / 8 + 0];
                    const uint4 v1 = src[(512 + 32 * rank) / 8 + 1];
                    const uint4 v2 = src[(512 + 32 * rank) / 8 + 2];
                    const uint4 v3 = src[(512 + 32 * rank) / 8 + 3];
                    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
                    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
                    w[8] = v2.x; w[9] = v2.y; w[10] = v2.z; w[11] = v2.w;
                    w[12] = v3.x; w[13] = v3.y; w[14] = v3.z; w[15] = v3.w;
                    tmem_st16(tmem + lane_off + kColQ + 128, w);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&q_ready);
            }
            float m = -INFINITY, l = 0.f;
            const int T = item.t1 - item.t0;
            for (int k = 0; k < T && ok; ++k) {
                const uint32_t g = it + k;
                const int key0 = (item.t0 + k) * kAttnKeys;
                const int valid = min(kAttnKeys, item.n_vis - key0);
                if (!mbar_wait(&s_full, g & 1, abort)) { ok = false; break; }
                tc_fence_after();
                float sc[64];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[16];
                    tmem_ld16(tmem + lane_off + kColS + 16 * c, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) sc[16 * c + i] = __uint_as_float(r[i]);
                }
                tc_fence_before();
                mbar_arrive(&s_free);
                // partial scores to the peer, then the peer's partial for this row
                const uint32_t xb = (g & 1) * kXBytes + h * kXRow;
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    st_cluster_v4(x_peer + xb + 16 * c, sc[4 * c], sc[4 * c + 1], sc[4 * c + 2], sc[4 * c + 3]);
                mbar_arrive_peer(xbar_peer[g & 1]);
                if (!mbar_wait<true>(&x_full[g & 1], (g >> 1) & 1, abort)) { ok = false; break; }
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float4 v = ld_shared_v4(x_local + xb + 16 * c);
                    const float t4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = 4 * c + i;
                        const float s = (sc[n] + t4[i]) * a.scale_log2;
                        sc[n] = n < valid ? s : -INFINITY;
                        mx = fmaxf(mx, sc[n]);
                    }
                }
                const float m_new = fmaxf(m, mx);
                if (m_new > m + kRescaleThreshold) {
                    const float alpha = exp2f(m - m_new);
                    if (k > 0) {
                        if (!wait_o(g - 1)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < 16; ++c) {
                            uint32_t r[16];
                            tmem_ld16(tmem + lane_off + kColO + 16 * c, r);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                            tmem_st16(tmem + lane_off + kColO + 16 * c, r);
                        }
                        tmem_wait_st();
                    }
                    l *= alpha;
                    m = m_new;
                }
                // P buffer (g & 1) is free once the O GEMM of tile g - 2 completed
                if (g >= 2 && !wait_o(g - 2)) { ok = false; break; }
                if (valid < kAttnKeys) {
                    // rows past the visible keys may hold anything: zero them for the O GEMM
                    const uint32_t st = sbase + (g % kStages) * kStageBytes;
                    const int nchunks = (kAttnKeys - valid) * 32;
                    for (int i = tid; i < nchunks; i += 128) {
                        const int row = valid + (i >> 5), box = (i >> 3) & 3, ch = i & 7;
                        st_shared_v4(st + box * kLatBox + row * 128 + ch * 16, 0u, 0u, 0u, 0u);
                    }
                }
                const uint32_t prow = sbase + kOffP + (g & 1) * kPBytes + h * 128;
                float psum = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t pw[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __nv_bfloat162 p2 =
                            __floats2bfloat162_rn(exp2f(sc[8 * c + 2 * i] - m), exp2f(sc[8 * c + 2 * i + 1] - m));
                        const float2 f2 = __bfloat1622float2(p2);
                        psum += f2.x + f2.y;
                        pw[i] = *reinterpret_cast<const uint32_t*>(&p2);
                    }
                    st_shared_v4(prow + ((c ^ (h & 7)) << 4), pw[0], pw[1], pw[2], pw[3]);
                }
                l += psum;
                fence_async_smem();
                mbar_arrive(&p_ready[g & 1]);
            }
            if (!ok) break;
            // epilogue: normalised latent half (or partial + log2-sum-exp)
            const uint32_t g_last = it + T - 1;
            if (!wait_o(g_last)) { ok = false; break; }
            tc_fence_after();
            const float inv = 1.f / l;
            if (item.slot < 0) {
                uint4* dst = reinterpret_cast<uint4*>(a.o_lat + ((int64_t)item.bj * 128 + h) * 512 + 256 * rank);
#pragma unroll 1
                for (int c = 0; c < 16; ++c) {
                    uint32_t r[16];
                    tmem_ld16(tmem + lane_off + kColO + 16 * c, r);
                    tmem_wait_ld();
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        pk[i] = pack_bf16(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
                    dst[2 * c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[2 * c + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            } else {
                float4* dst = reinterpret_cast<float4*>(a.part_o + ((int64_t)item.slot * 128 + h) * 512 + 256 * rank);
#pragma unroll 1
                for (int c = 0; c < 16; ++c) {
                    uint32_t r[16];
                    tmem_ld16(tmem + lane_off + kColO + 16 * c, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[4 * c + i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                                     __uint_as_float(r[4 * i + 2]) * inv,
                                                     __uint_as_float(r[4 * i + 3]) * inv);
                }
                if (rank == 0) a.part_lse[item.slot * 128 + h] = m + log2f(l);
            }
            tc_fence_before();
            it += T;
        }
        if (!ok) fail();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    cluster_sync();          // no CTA leaves while its peer may still write to it
}

}  // namespace

int launch_attend(const DecodeCall& c, const __nv_bfloat16* q_lat, const int32_t* cum, __nv_bfloat16* o_lat,
                  float* part_o, float* part_lse, int pairs, int* launches) {
    CUtensorMap ml, mr;
    const uint64_t dims[3] = {576, (uint64_t)c.capacity, (uint64_t)c.batch};
    const uint64_t str[2] = {576 * 2, (uint64_t)c.capacity * 576 * 2};
    const uint32_t box_l[3] = {64, 64, 1}, box_r[3] = {32, 64, 1};
    if (!make_map(&ml, c.cache, 3, dims, str, box_l, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    if (!make_map(&mr, c.cache, 3, dims, str, box_r, CU_TENSOR_MAP_SWIZZLE_64B)) return MLA_ERR_CUDA;
    AttnArgs a{};
    a.q_lat = q_lat;
    a.cum = cum;
    a.seq_lens = c.seq_lens;
    a.BJ = c.batch * c.n_q;
    a.n_q = c.n_q;
    a.pairs = pairs;
    a.scale_log2 = c.d.softmax_scale * 1.4426950408889634f;
    a.o_lat = o_lat;
    a.part_o = part_o;
    a.part_lse = part_lse;
    a.status = c.status;
    const size_t smem = kSmemBytes + 1024;
    if (cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    prof_begin(c.stream, "sm100_attend");
    attend_kernel<<<2 * pairs, kThreads, smem, c.stream>>>(ml, mr, a);
    prof_end(c.stream);
    if (launches) ++*launches;
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla
