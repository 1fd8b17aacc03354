// Absorbed MLA attention against the latent cache on tcgen05 tensor cores.
//
// For one query token (b, j) and a range of 64-key tiles of its sequence,
// with q_lat = [W_uk q_nope || RoPE(q_rope)] (576 wide, all 128 heads):
//     S[h][n] = <q_lat[h], cache[b][n][0:576]>                    (score)
//     online softmax over n (base 2, scale folded in), fp32 state
//     O[h][0:512] += P[h][n] cache[b][n][0:512]                    (weighted latent)
// i.e. the score of "Understanding MLA (Multi-head Latent Attention)",
// section 4 (content part through the absorbed query, position part through
// the shared rope key), weighted over the cached latents as on aicassindra
// "Multi-head latent attention", "End-to-end flow".
//
// Work split.  All heads of a token share each cache row, so the 128 heads
// are the M dimension of both contractions.  A 128 x 512 fp32 accumulator
// would fill all of TMEM, so a cluster of two CTAs splits the latent: CTA r
// owns latent columns [256r, 256r+256) and rope columns [512+32r, +32).
// Each CTA loads only its 288 columns of every tile (each cache byte crosses
// HBM once, no multicast) and computes a partial score over them.  The
// exchange warps round their partial to fp16 and store it straight into the
// peer's shared memory (three buffers); each softmax thread adds its own
// fp32 partial to the peer's, then writes its P values over the very chunks
// it read, so the same buffer is the A operand of the O GEMM and returns to
// the peer when that GEMM completes.  The
// two CTAs' scores thus differ only by that fp16 rounding; each CTA keeps its
// own running max and sum and normalises its own half of O with them, so each
// half is self-consistent.  Each CTA accumulates its half of O from the same
// smem tile read as an MN-major operand.
//
// TMEM (512 columns): O [0,256), S double buffer [256,384), Q latent slice
// [384,512) (A operand of the score GEMM); the 32 rope columns of Q are an
// smem operand.
//
// Roles (480 threads): warp 0 TMA, warp 1 score-GEMM issue, warp 14
// latent-GEMM issue, warps 2-5 "exchange" (score tile -> fp16 -> peer smem,
// query loads; thread <-> head <-> TMEM lane), warps 6-13 "softmax" (P, O
// rescale, epilogue): two groups of four warps that take alternate tiles, one
// thread per head row.
//
// Work items.  The key tiles of all query tokens are concatenated and cut
// into one contiguous range per cluster.  A token whose tiles all fall in one
// cluster's range is finished there (normalised latent output, bf16); a token
// cut across clusters leaves fp32 partial outputs plus log2-sum-exp per piece
// for the combine step.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "profile.h"
#include "sm100_host.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

namespace {

constexpr int kKeys = 64;
constexpr int kStages = 4;
constexpr int kLatBox = 8192;                      // 64 keys x 64 columns x 2 B
constexpr int kRopeBox = 4096;                     // 64 keys x 32 columns x 2 B
constexpr int kStageBytes = 4 * kLatBox + kRopeBox;
constexpr int kTileBytes = 128 * 128;              // 128 rows x 64 x 2 B (exchange / P tiles)
constexpr int kXBufs = 3;                          // exchange buffers
constexpr int kOffXin = kStages * kStageBytes;     // the peer's partial scores, then P
constexpr int kOffQr = kOffXin + kXBufs * kTileBytes;  // 128 heads x 32 rope columns, SW64
constexpr int kSmemBytes = kOffQr + 128 * 64;
constexpr int kThreads = 480;
constexpr uint32_t kColO = 0, kColS = 256, kColQ = 384, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;          // log2 units

struct AttnArgs {
    const __nv_bfloat16* q_lat;   // [BJ][128][576]
    const int32_t* cum;           // [BJ + 1] tile prefix
    const int32_t* first_bj;      // [pairs] first query token of each cluster's range
    const int32_t* cut;           // [pairs + 1] first key tile of each cluster's range
    const int32_t* seq_lens;
    int BJ, n_q, pairs;
    float scale_log2;             // softmax_scale * log2(e)
    __nv_bfloat16* o_lat;         // [BJ][128][512]
    // split-KV pieces, normalised per piece, head-major and blocked by 64
    // latent columns: element (slot, head h, column c) at
    // ((h * 8 + c / 64) * 2 pairs + slot) * 64 + c % 64, so that one head's
    // pieces of a column block are contiguous
    __nv_bfloat16* part_o;
    float* part_lse;              // [128 heads][2 * pairs][2 latent halves], log2 domain
    int32_t* status;
    // sparse decode: the selected slots of each query token and their count
    const int32_t* sel;           // [BJ][max_sel]
    const int32_t* n_sel;         // [BJ] (nullptr: dense decode over keys 0..p)
    int max_sel;
    int64_t capacity;
};

struct Item {
    int bj, t0, t1, n_vis, slot;  // slot < 0: finished here; n_vis: keys this token attends
    int p;                        // the query's position
};

// Pieces of the concatenated tile range [s0, s1) of one cluster, in order.
struct ItemIter {
    const int32_t* cum;
    const int32_t* lens;
    const int32_t* n_sel;
    int BJ, n_q, bj, s0, s1, pair;
    __device__ void init(const AttnArgs& a, int p) {
        cum = a.cum;
        BJ = a.BJ;
        n_q = a.n_q;
        lens = a.seq_lens;
        n_sel = a.n_sel;
        pair = p;
        s0 = a.cut[p];
        s1 = a.cut[p + 1];
        bj = a.first_bj[p];           // first bj with cum[bj + 1] > s0 (from the plan)
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
            it.p = (int)query_pos(lens[b], n_q, j);
            it.n_vis = n_sel ? n_sel[cur] : it.p + 1;
            it.slot = (c0 >= s0 && c1 <= s1) ? -1 : (c0 < s0 ? 2 * pair : 2 * pair + 1);
            return true;
        }
        return false;
    }
};

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_shared_u4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Asynchronous 16-byte store into the peer CTA's shared memory; its bytes are
// counted (complete_tx) on the peer's mbarrier `bar` (both shared::cluster).
__device__ __forceinline__ void st_async_u4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                            uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     addr),
                 "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// a * b + c and a + b on two fp32 lanes at once (paired instructions), denormals flushed
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.ftz.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.ftz.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// kSparse: the key tiles are gathered rows (tile::gather4 from 2-D maps over
// [batch * capacity][576]); otherwise 64 consecutive keys (3-D maps).
template <bool kSparse>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attend_kernel(const __grid_constant__ CUtensorMap map_lat, const __grid_constant__ CUtensorMap map_rope,
              const __grid_constant__ CUtensorMap map_ql, const __grid_constant__ CUtensorMap map_qr, AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kStages], empty[kStages];
    // q0_full: the first item's query slice has landed (tensor copies into
    // stages 2-3 and the Q-rope area); q0_copied: its latent part is in TMEM
    // (tcgen05.cp), so stages 2-3 may take cache tiles
    __shared__ uint64_t s_full[2], s_free[2], o_done[2], q_ready, q0_full, q0_copied, drain, drain_o;
    __shared__ uint64_t p_ready[kXBufs], xin_full[kXBufs], rx_done[kXBufs];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    // per-warpgroup decisions, each written by the leader before a named barrier
    // and read after it; a barrier separates every read from the next write
    __shared__ int ex_stop;
    // softmax: the running row maximum after tile g (slot g & 1) and its
    // per-quarter barriers; per-item meeting of the two groups' row sums
    __shared__ uint64_t m_ready[2][4], ep_ready[4];
    // ep_done: both groups' warps of a lane quarter have read their half of O
    // (the next item's first value GEMM overwrites it); item_done: the item's
    // last value GEMM has completed (one completion per item)
    __shared__ uint64_t ep_done[4], item_done;
    __shared__ float m_pub[2][128];
    __shared__ float ep_m[2][2][128], ep_l[2][2][128];
    __shared__ __align__(16) uint32_t ep_scratch[8][32 * 16];   // per softmax warp: 32 rows x 64 bytes

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t peer = rank ^ 1u;
    const int pair = blockIdx.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 8);       // 4 exchange warps + the 4 warps of the tile's softmax group
        }
        for (int i = 0; i < kXBufs; ++i) {
            mbar_init(&xin_full[i], 1);     // my softmax leader's expect_tx + the peer's bytes
            mbar_init(&rx_done[i], 1);      // the peer's O GEMM has read the buffer (its commit)
            mbar_init(&p_ready[i], 4);      // P tile written over the exchange buffer (4 warps)
        }
        mbar_init(&o_done[0], 1);           // O GEMMs of even / odd global tiles
        mbar_init(&o_done[1], 1);
        mbar_init(&q_ready, 1);
        mbar_init(&q0_full, 1);
        mbar_init(&q0_copied, 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(&m_ready[0][i], 1);   // warp of lane quarter i in the group of an even tile
            mbar_init(&m_ready[1][i], 1);   // ... of an odd tile
            mbar_init(&ep_ready[i], 2);     // the two groups' warps of lane quarter i, once per item
            mbar_init(&ep_done[i], 2);      // ... after their epilogue reads of O, once per item
        }
        mbar_init(&item_done, 1);           // committed after each item's last O GEMM
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
    cluster_sync();          // the peer's barriers are initialised before any remote access
    tc_fence_after();
    grid_dep_wait();         // q_lat and the tile plan come from the previous kernel
    grid_dep_trigger();
    const uint32_t tmem = tmem_base;
    const uint32_t sbase = smem_u32(smem);
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
            const uint64_t stream_policy = l2_policy_evict_first();
            ItemIter iter;
            iter.init(a, pair);
            Item item;
            uint32_t it = 0;
            bool ok = true;
            {
                // The first item's query slice by tensor copies: this CTA's latent half
                // (four 64-column groups, 64 KB) into stages 2-3, its rope columns into
                // the Q-rope area.  (Later items' slices are loaded by the exchange
                // warps, after their predecessor's score GEMMs.)
                ItemIter peek = iter;
                Item first;
                if (peek.next(first)) {
                    mbar_expect_tx(&q0_full, 4 * 128 * 128 + 128 * 64);
                    tma_load_4d(smem + 2 * kStageBytes, &map_ql, &q0_full, 0, 0, 4 * (int)rank, first.bj);
                    tma_load_3d(smem + kOffQr, &map_qr, &q0_full, 512 + 32 * rank, 0, first.bj);
                }
            }
            while (ok && iter.next(item)) {
                const int b = item.bj / a.n_q;
                for (int t = item.t0; t < item.t1; ++t, ++it) {
                    const int s = it % kStages;
                    if (it >= kStages && !mbar_wait(&empty[s], ((it / kStages) - 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    // start-up: the first stage is requested alone, so every SM's first
                    // tile lands before the rest of the start-up burst
                    if (it == 1 && !mbar_wait(&full[0], 0, abort)) {
                        ok = false;
                        break;
                    }
                    // stages 2-3 hold the first query slice until it is copied to TMEM
                    if (it == 2 && !mbar_wait(&q0_copied, 0, abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * kStageBytes;
                    mbar_expect_tx(&full[s], kStageBytes);
                    const int key0 = t * kKeys;
                    if constexpr (kSparse) {
                        // the tile's 64 selected slots (padded with the first one past the
                        // count; those rows are masked and zeroed before the latent GEMM)
                        const int32_t* srow = a.sel + (int64_t)item.bj * a.max_sel + key0;
                        const int n = min(kKeys, item.n_vis - key0);
                        const int32_t rowbase = b * (int32_t)a.capacity;
                        int32_t rows[kKeys];
#pragma unroll
                        for (int i = 0; i < kKeys; ++i) rows[i] = srow[i < n ? i : 0];
                        bool bad = false;
#pragma unroll
                        for (int i = 0; i < kKeys; ++i) {
                            const bool ok_i = rows[i] >= 0 && rows[i] <= item.p;
                            bad |= !ok_i;
                            rows[i] = rowbase + (ok_i ? rows[i] : 0);
                        }
                        if (bad) set_status(a.status, MLA_ERR_INDEX);
#pragma unroll
                        for (int g4 = 0; g4 < kKeys / 4; ++g4) {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                tma_gather4(st + i * kLatBox + g4 * 512, &map_lat, &full[s], 256 * rank + 64 * i,
                                            rows[4 * g4], rows[4 * g4 + 1], rows[4 * g4 + 2], rows[4 * g4 + 3]);
                            tma_gather4(st + 4 * kLatBox + g4 * 256, &map_rope, &full[s], 512 + 32 * rank, rows[4 * g4],
                                        rows[4 * g4 + 1], rows[4 * g4 + 2], rows[4 * g4 + 3]);
                        }
                    } else {
                        // this CTA's four latent column groups in one copy (see launch_attend);
                        // each cache row is read once, so it leaves L2 first, ahead of the
                        // outputs the up-projection reads next
                        tma_load_4d_hint(st, &map_lat, &full[s], 0, key0, 4 * (int)rank, b, stream_policy);
                        tma_load_3d_hint(st + 4 * kLatBox, &map_rope, &full[s], 512 + 32 * rank, key0, b,
                                         stream_policy);
                    }
                }
            }
            if (!ok) fail();
            const uint32_t first = it > kStages ? it - kStages : 0;
            for (uint32_t i = first; i < it; ++i) mbar_wait(&full[i % kStages], (i / kStages) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ score GEMM issuer
        // Score GEMMs S(g) in tile order, each as soon as its stage has landed
        // and its score buffer is free (and, at an item's start, the item's
        // query slice is in TMEM).  The latent GEMMs O(g) come from warp 14: an
        // issuing thread stalls while the tensor pipe is full, so one issuer for
        // both streams held a ready O(g) behind the next score batch.  The tensor
        // pipe runs both warps' GEMMs in arrival order; each warp's commits track
        // its own.  The whole warp runs this loop (every decision is lane 0's
        // observation, broadcast) and one elected lane issues each instruction.
        constexpr uint32_t idS = idesc_bf16(128, 64, false, false);
        // descriptors of stage 0 / P buffer 0; other stages and steps are byte offsets
        const uint64_t dLatK = sdesc(sbase, 16, 1024, kSwizzle128);          // cache tile, K-major (score)
        const uint64_t dRope = sdesc(sbase + 4 * kLatBox, 16, 512, kSwizzle64);
        const uint64_t dQr = sdesc(sbase + kOffQr, 16, 512, kSwizzle64);
        ItemIter iterS;
        iterS.init(a, pair);
        Item itS;
        bool haveS = iterS.next(itS);
        int kS = 0;
        uint32_t gS = 0, nItemsS = 0;
        bool qS = false;                           // q_ready observed for the current S item
        uint32_t idle = 0;                         // consecutive passes without progress
        uint64_t t_idle = 0;                       // timer at the 256th of them
        bool ok = true;
        while (ok && haveS) {
            bool progressed = false;
            // score GEMM S(gS): 16 K-steps of latent (A = query slice in TMEM), 2 of rope
            {
                const int s = gS % kStages, sb = gS & 1;
                if (!qS && nItemsS == 0 && mbar_ready_w(&q0_full, 0)) {
                    // the first item's latent query slice: stages 2-3 -> TMEM (A operand
                    // of the score GEMM), 128 rows x 32 bytes per copy, ahead of the
                    // score GEMMs in this thread's order
                    tc_fence_after();
                    const uint64_t dq = sdesc(sbase + 2 * kStageBytes, 16, 1024, kSwizzle128);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tmem_cp_128x256b_w(tmem + kColQ + 32 * g + 8 * j, sdesc_add(dq, g * 16384 + j * 32));
                    mma_commit_w(&q0_copied);
                    qS = true;
                }
                if (!qS && nItemsS > 0) qS = mbar_ready_w(&q_ready, (nItemsS - 1) & 1);
                if (qS && mbar_ready_w(&full[s], (gS / kStages) & 1) &&
                    (gS < 2 || mbar_ready_w(&s_free[sb], ((gS >> 1) - 1) & 1))) {
                    tc_fence_after();
                    const uint32_t so = s * kStageBytes;
                    const uint32_t dS = tmem + kColS + 64 * sb;
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks)
                        mma_ts_w(dS, tmem + kColQ + 8 * ks, sdesc_add(dLatK, so + (ks >> 2) * kLatBox + (ks & 3) * 32),
                                 idS, ks ? 1u : 0u);
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
                        mma_ss_w(dS, sdesc_add(dQr, ks * 32), sdesc_add(dRope, so + ks * 32), idS, 1u);
                    mma_commit_w(&s_full[sb]);
                    ++gS;
                    if (++kS == itS.t1 - itS.t0) {
                        kS = 0;
                        qS = false;
                        ++nItemsS;
                        haveS = iterS.next(itS);
                    }
                    progressed = true;
                }
            }
            // bounded idle time: the timer is read once per 256 idle passes
            if (progressed) {
                idle = 0;
            } else if ((++idle & 255u) == 0) {
                const uint64_t now = globaltimer();
                if (idle == 256) t_idle = now;
                const int quit = (*abort || now - t_idle > kWaitLimitNs) ? 1 : 0;
                if (__shfl_sync(0xffffffffu, quit, 0)) ok = false;
            }
        }
        if (!ok && lane == 0) fail();
        mma_commit_w(&drain);
        mbar_wait(&drain, 0, nullptr);
    } else if (warp == 14) {
        // ------------------------------------------------------------ latent GEMM issuer
        // O(g) += P(g) V(g) in tile order, each as soon as its P tile is written
        // (P(g) implies S(g) was issued).  The commits release the cache stage,
        // tell the softmax O(g) is done, hand the exchange buffer back to the
        // peer and, after an item's last tile, signal item_done.
        constexpr uint32_t idO = idesc_bf16(128, 256, false, true);
        const uint64_t dLatN = sdesc(sbase, kLatBox, 1024, kSwizzle128);     // cache tile, MN-major (latent)
        const uint64_t dP = sdesc(sbase + kOffXin, 16, 1024, kSwizzle128);
        ItemIter iterO;
        iterO.init(a, pair);
        Item itO;
        bool haveO = iterO.next(itO);
        int kO = 0;
        uint32_t gO = 0;
        uint32_t idle = 0;                         // consecutive passes without progress
        uint64_t t_idle = 0;                       // timer at the 256th of them
        bool ok = true;
        while (ok && haveO) {
            bool progressed = false;
            if (mbar_ready_w(&p_ready[gO % kXBufs], (gO / kXBufs) & 1)) {
                tc_fence_after();
                const int s = gO % kStages;
                const uint32_t so = s * kStageBytes, po = (gO % kXBufs) * kTileBytes;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss_w(tmem + kColO, sdesc_add(dP, po + ks * 32), sdesc_add(dLatN, so + ks * 2048), idO,
                             (kO == 0 && ks == 0) ? 0u : 1u);
                mma_commit_w(&empty[s]);
                mma_commit_w(&o_done[gO & 1]);
                // P buffer gO % 3 is free again: the peer may send its tile gO + 3 into it
                mma_commit_mc_w(&rx_done[gO % kXBufs], (uint16_t)(1u << peer));
                ++gO;
                if (++kO == itO.t1 - itO.t0) {
                    mma_commit_w(&item_done);
                    kO = 0;
                    haveO = iterO.next(itO);
                }
                progressed = true;
            }
            // bounded idle time: the timer is read once per 256 idle passes
            if (progressed) {
                idle = 0;
            } else if ((++idle & 255u) == 0) {
                const uint64_t now = globaltimer();
                if (idle == 256) t_idle = now;
                const int quit = (*abort || now - t_idle > kWaitLimitNs) ? 1 : 0;
                if (__shfl_sync(0xffffffffu, quit, 0)) ok = false;
            }
        }
        if (!ok && lane == 0) fail();
        mma_commit_w(&drain_o);
        mbar_wait(&drain_o, 0, nullptr);
    } else if (warp < 6) {
        // ------------------------------------------------------------ exchange warpgroup
        // One leader does every mbarrier wait (bounded) and a named barrier
        // broadcasts the outcome, so the warpgroup never diverges on a timeout.
        const int q = warp & 3;
        const int h = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t xin_peer = map_peer(sbase + kOffXin, peer);
        uint32_t xbar_peer[kXBufs];
#pragma unroll
        for (int i = 0; i < kXBufs; ++i) xbar_peer[i] = map_peer(smem_u32(&xin_full[i]), peer);
        const bool leader = (warp == 2) && lane == 0;
        ItemIter iter;
        iter.init(a, pair);
        Item item;
        uint32_t it = 0;
        while (iter.next(item)) {
            if (leader) ex_stop = *abort;
            named_barrier(1, 128);
            if (ex_stop) break;
            // query slice of this token (the first item's comes by tensor copies):
            // latent part -> TMEM, rope part -> smem (SW64 rows).  Every score GEMM
            // of the previous item has completed: its last score tile was read
            // below before we got here.
            if (it > 0) {
                // loads in two batches of 16 (plus the rope chunks), each batch issued
                // before any TMEM store, so the slice costs two memory round trips
                const uint4* src = reinterpret_cast<const uint4*>(a.q_lat + ((int64_t)item.bj * 128 + h) * 576);
                uint4 rq[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) rq[c] = src[64 + 4 * rank + c];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint4 v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = src[32 * rank + 16 * half + i];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t w[16];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            w[4 * i] = v[4 * c + i].x; w[4 * i + 1] = v[4 * c + i].y;
                            w[4 * i + 2] = v[4 * c + i].z; w[4 * i + 3] = v[4 * c + i].w;
                        }
                        tmem_st16(tmem + lane_off + kColQ + 16 * (4 * half + c), w);
                    }
                }
                const uint32_t qrow = sbase + kOffQr + h * 64;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_shared_u4(qrow + ((c ^ ((h >> 1) & 3)) << 4), rq[c].x, rq[c].y, rq[c].z, rq[c].w);
                tmem_wait_st();
                fence_async_smem();
                tc_fence_before();
                named_barrier(1, 128);
                if (leader) mbar_arrive(&q_ready);
            }
            const int T = item.t1 - item.t0;
            bool stop = false;
            for (int k = 0; k < T; ++k) {
                const uint32_t g = it + k;
                const int sb = g & 1, xb = g % kXBufs;
                if (leader) {
                    // score tile g ready; the peer's buffer xb is free (its O GEMM of tile g - 3 is done)
                    bool ok = mbar_wait(&s_full[sb], (g >> 1) & 1, abort);
                    if (ok && g >= kXBufs) ok = mbar_wait<true>(&rx_done[xb], ((g / kXBufs) - 1) & 1, abort);
                    if (!ok) fail();
                    ex_stop = *abort;
                }
                named_barrier(1, 128);
                if (ex_stop) { stop = true; break; }
                tc_fence_after();
                // my raw partial scores rounded to fp16, stored straight into the peer's
                // buffer (the peer adds exactly these values; so do I)
                const uint32_t row = xin_peer + xb * kTileBytes + h * 128;
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_off + kColS + 64 * sb, r0);
                tmem_ld32(tmem + lane_off + kColS + 64 * sb + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int chunk = 0; chunk < 8; ++chunk) {
                    const uint32_t* r = chunk < 4 ? r0 + 8 * chunk : r1 + 8 * (chunk - 4);
                    uint32_t hw[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        __half2 v = __floats2half2_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        hw[i] = *reinterpret_cast<uint32_t*>(&v);
                    }
                    st_async_u4(row + ((chunk ^ (h & 7)) << 4), hw[0], hw[1], hw[2], hw[3], xbar_peer[xb]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[sb]);
            }
            if (stop) break;
            it += T;
        }
    } else {
        // ------------------------------------------------------------ softmax groups
        // Two groups of four warps take alternate global tiles (group 0 even g,
        // warps 6-9; group 1 odd g, warps 10-13).  One thread per head row (its
        // TMEM lane) handles all 64 score columns of its group's tiles.  The
        // running row maximum is handed from each tile to the next through m_pub
        // and a per-quarter mbarrier, so a group spends two tile periods on each
        // of its tiles while the other group works on the next one.  Each group
        // keeps its own part of the row sum, relative to the maximum it last
        // used; the two parts meet at the end of every item.
        const int grp = (warp - 6) >> 2;
        const int q = warp & 3;
        const int h = q * 32 + lane;
        const int gtid = (warp - 6 - 4 * grp) * 32 + lane;   // 0..127 within the group
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const bool xleader = (warp == 6 + 4 * grp) && lane == 0;   // the expect_tx of this group's tiles
        // O GEMM of global tile n = g - 1 has completed (the rescale before P of tile
        // g).  Completions alternate between two barriers, so the parity is exact
        // only if O(g - 3) is done and O(g + 1) is not: the peer's partial scores of
        // tile g (waited for above) are sent only after this CTA's O GEMM of tile
        // g - 3 released that exchange buffer, and O(g + 1) follows O(g), which
        // needs the P tile this thread has yet to write.
        // Exchange buffer g % 3 holds the peer's partial scores of tile g, then this
        // CTA's P tile g (each thread overwrites exactly the chunks it read); the
        // commit of O GEMM g hands it back to the peer (for its tile g + 3).
        auto wait_o = [&](uint32_t n) -> bool { return mbar_wait(&o_done[n & 1], (n >> 1) & 1, abort); };
        // lane 0 waits (bounded), the warp follows its outcome
        auto lane0 = [&](bool ok) -> bool { return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0; };
        ItemIter iter;
        iter.init(a, pair);
        Item item;
        uint32_t it = 0, n_item = 0;
        bool stop = false;
        while (!stop && iter.next(item)) {
            const int T = item.t1 - item.t0;
            float m_used = -INFINITY, l = 0.f;        // this group's part of the row sum, relative to m_used
            for (int k = 0; k < T && !stop; ++k) {
                const uint32_t g = it + k;
                if ((int)(g & 1) != grp) continue;
                const int sb = g & 1, xb = g % kXBufs;
                const int key0 = (item.t0 + k) * kKeys;
                const int valid = min(kKeys, item.n_vis - key0);
                bool ok = true;
                if (lane == 0) {
                    if (xleader) mbar_expect_tx(&xin_full[xb], kTileBytes);
                    ok = mbar_wait<true>(&xin_full[xb], (g / kXBufs) & 1, abort) &&
                         mbar_wait(&s_full[sb], (g >> 1) & 1, abort);
                }
                if (!lane0(ok)) { stop = true; break; }
                // own fp32 partial (TMEM) plus the peer's fp16 partial (smem)
                tc_fence_after();
                float x[64];
                {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tmem + lane_off + kColS + 64 * sb, r0);
                    tmem_ld32(tmem + lane_off + kColS + 64 * sb + 32, r1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        x[i] = __uint_as_float(r0[i]);
                        x[32 + i] = __uint_as_float(r1[i]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[sb]);      // this warp is done with score buffer sb
                const uint32_t prow = sbase + kOffXin + xb * kTileBytes + h * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = ld_shared_u4(prow + ((c ^ (h & 7)) << 4));
                    const uint32_t pw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 b2 = __half22float2(*reinterpret_cast<const __half2*>(&pw[i]));
                        const float2 s2 = fadd2(make_float2(x[8 * c + 2 * i], x[8 * c + 2 * i + 1]), b2);
                        x[8 * c + 2 * i] = s2.x;
                        x[8 * c + 2 * i + 1] = s2.y;
                    }
                }
                if (valid < kKeys) {
#pragma unroll
                    for (int n = 0; n < 64; ++n) x[n] = n < valid ? x[n] : -INFINITY;
                }
                float mx8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mx8[i] = fmaxf(fmaxf(fmaxf(x[i], x[i + 8]), fmaxf(x[i + 16], x[i + 24])),
                                   fmaxf(fmaxf(x[i + 32], x[i + 40]), fmaxf(x[i + 48], x[i + 56])));
#pragma unroll
                for (int i = 0; i < 4; ++i) mx8[i] = fmaxf(mx8[i], mx8[i + 4]);
                // softmax in base 2: scores scaled by scale * log2(e) (> 0, so the raw max serves)
                const float mx = fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])) * a.scale_log2;
                // the running maximum after tile g - 1 (ignored at an item's first tile)
                float m_prev = -INFINITY;
                if (g >= 1) {
                    const int pb = (g - 1) & 1;
                    if (lane == 0) ok = mbar_wait(&m_ready[pb][q], ((g - 1) >> 1) & 1, abort);
                    if (!lane0(ok)) { stop = true; break; }
                    if (k > 0) m_prev = m_pub[pb][h];
                }
                // Lazy rescaling: the maximum moves only when it grew by more than 2^8.
                const float m_cand = fmaxf(m_prev, mx);
                const float m = m_cand > m_prev + kRescaleThreshold ? m_cand : m_prev;
                m_pub[g & 1][h] = m;
                __syncwarp();
                if (lane == 0) mbar_arrive(&m_ready[g & 1][q]);
                // O holds the tiles before g relative to m_prev: rescale it when m moved.
                // TMEM accesses are warp-collective, so lanes that need none multiply by 1.
                const bool need = k > 0 && m > m_prev;
                if (__any_sync(0xffffffffu, need)) {
                    if (lane == 0) ok = wait_o(g - 1);
                    if (!lane0(ok)) { stop = true; break; }
                    tc_fence_after();
                    const float alpha = need ? ex2(m_prev - m) : 1.f;
#pragma unroll 1
                    for (int c = 0; c < 16; ++c) {
                        uint32_t r[16];
                        const uint32_t ta = tmem + lane_off + kColO + 16 * c;
                        tmem_ld16(ta, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st16(ta, r);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                }
                if (m > m_used) {
                    if (m_used != -INFINITY) l *= ex2(m_used - m);
                    m_used = m;
                }
                if (valid < kKeys) {
                    // rows past the visible keys may hold anything: zero them for the O GEMM
                    const uint32_t st = sbase + (g % kStages) * kStageBytes;
                    const int nchunks = (kKeys - valid) * 32;
                    for (int i = gtid; i < nchunks; i += 128) {
                        const int r = valid + (i >> 5), box = (i >> 3) & 3, c = i & 7;
                        st_shared_u4(st + box * kLatBox + r * 128 + c * 16, 0u, 0u, 0u, 0u);
                    }
                }
                float ps4[4] = {0.f, 0.f, 0.f, 0.f};
                const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m, -m);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t pw[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 y = ffma2(make_float2(x[8 * c + 2 * i], x[8 * c + 2 * i + 1]), sc2, nm2);
                        const float p0 = ex2(y.x);
                        const float p1 = ex2(y.y);
                        ps4[i] += p0 + p1;
                        pw[i] = pack_bf16(p0, p1);
                    }
                    // P over the chunk read above
                    st_shared_u4(prow + ((c ^ (h & 7)) << 4), pw[0], pw[1], pw[2], pw[3]);
                }
                l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_ready[xb]);
            }
            if (stop) break;
            // epilogue: both groups' sums meet; group c writes O columns [128c, 128c + 128)
            // of this CTA's latent half (normalised, or a partial plus log2-sum-exp)
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&item_done, n_item & 1, abort);
            if (!lane0(ok)) break;
            const int eb = n_item & 1;
            ep_m[eb][grp][h] = m_used;
            ep_l[eb][grp][h] = l;
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&ep_ready[q]);
                ok = mbar_wait(&ep_ready[q], eb, abort);
            }
            if (!lane0(ok)) break;
            const float m0 = ep_m[eb][0][h], m1 = ep_m[eb][1][h];
            const float mf = fmaxf(m0, m1);
            const float lsum = (m0 == -INFINITY ? 0.f : ep_l[eb][0][h] * ex2(m0 - mf)) +
                               (m1 == -INFINITY ? 0.f : ep_l[eb][1][h] * ex2(m1 - mf));
            tc_fence_after();
            const float inv = 1.f / lsum;
            // Rows leave TMEM one per thread; each 32-row x 64-byte block goes through
            // this warp's smem scratch so that a store instruction covers eight
            // contiguous 64-byte row segments instead of 32 scattered 16-byte pieces.
            const uint32_t scr = smem_u32(&ep_scratch[warp - 6][0]);
            auto put_rows = [&](const uint32_t (&w)[16], auto&& row_ptr) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    st_shared_u4(scr + lane * 64 + ((j ^ (lane & 3)) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int r = 8 * k + (lane >> 2), pc = lane & 3;
                    const uint4 v = ld_shared_u4(scr + r * 64 + ((pc ^ (r & 3)) << 4));
                    *reinterpret_cast<uint4*>(row_ptr(q * 32 + r) + 16 * pc) = v;
                }
                __syncwarp();
            };
            {
                // bf16, 32 columns (64 bytes) per row and block: the normalised output of a
                // token finished here, or this piece's normalised partial (plus its
                // log2-sum-exp) for the combine step
                char* base = reinterpret_cast<char*>(a.o_lat + (int64_t)item.bj * 128 * 512 + 256 * rank + 128 * grp);
                const int S2 = 2 * a.pairs;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + kColO + 128 * grp + 32 * c, r);
                    tmem_wait_ld();
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[i] = pack_bf16(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
                    if (item.slot < 0) {
                        put_rows(w, [&](int row) { return base + ((int64_t)row * 512 + 32 * c) * 2; });
                    } else {
                        const int kb = 4 * (int)rank + 2 * grp + (c >> 1);
                        put_rows(w, [&](int row) {
                            return reinterpret_cast<char*>(a.part_o + (((int64_t)row * 8 + kb) * S2 + item.slot) * 64 +
                                                           32 * (c & 1));
                        });
                    }
                }
                if (item.slot >= 0 && grp == 0) a.part_lse[(h * S2 + item.slot) * 2 + rank] = mf + __log2f(lsum);
            }
            // the next item's first O GEMM (accumulate = 0) may start only after both
            // groups' reads of this item's O
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&ep_done[q]);
                ok = mbar_wait(&ep_done[q], n_item & 1, abort);
            }
            if (!lane0(ok)) break;
            it += T;
            ++n_item;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    cluster_sync();          // no CTA leaves while its peer may still access it
}

}  // namespace

int launch_attend(const DecodeCall& c, const __nv_bfloat16* q_lat, const int32_t* cum, __nv_bfloat16* o_lat,
                  __nv_bfloat16* part_o, float* part_lse, const int32_t* first_bj, const int32_t* cut, int pairs,
                  int* launches) {
    const bool sparse = c.n_sel != nullptr;
    CUtensorMap ml, mr;
    if (sparse) {
        // 2-D view [batch * capacity][576], boxes one row high for tile::gather4
        const uint64_t dims[2] = {576, (uint64_t)c.capacity * (uint64_t)c.batch};
        const uint64_t str[1] = {576 * 2};
        const uint32_t box_l[2] = {64, 1}, box_r[2] = {32, 1};
        if (!make_map(&ml, c.cache, 2, dims, str, box_l, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
        if (!make_map(&mr, c.cache, 2, dims, str, box_r, CU_TENSOR_MAP_SWIZZLE_64B)) return MLA_ERR_CUDA;
    } else {
        // latent: rows viewed as 9 groups of 64 columns (group stride 128 bytes,
        // placed after the key dimension), one box = 64 keys x 4 groups landing
        // group-major: a whole latent half per tensor copy.  A single thread
        // issues about one tensor copy per 0.3 us whatever its size up to 16 KB,
        // so one copy instead of four keeps the loads at HBM speed.
        const uint64_t dl[4] = {64, (uint64_t)c.capacity, 9, (uint64_t)c.batch};
        const uint64_t sl[3] = {576 * 2, 64 * 2, (uint64_t)c.capacity * 576 * 2};
        const uint32_t box_l[4] = {64, 64, 4, 1};
        if (!make_map(&ml, c.cache, 4, dl, sl, box_l, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
        const uint64_t dims[3] = {576, (uint64_t)c.capacity, (uint64_t)c.batch};
        const uint64_t str[2] = {576 * 2, (uint64_t)c.capacity * 576 * 2};
        const uint32_t box_r[3] = {32, 64, 1};
        if (!make_map(&mr, c.cache, 3, dims, str, box_r, CU_TENSOR_MAP_SWIZZLE_64B)) return MLA_ERR_CUDA;
    }
    AttnArgs a{};
    a.q_lat = q_lat;
    a.cum = cum;
    a.first_bj = first_bj;
    a.cut = cut;
    a.seq_lens = c.seq_lens;
    a.BJ = c.batch * c.n_q;
    a.n_q = c.n_q;
    a.pairs = pairs;
    a.scale_log2 = c.d.softmax_scale * 1.4426950408889634f;
    a.o_lat = o_lat;
    a.part_o = part_o;
    a.part_lse = part_lse;
    a.status = c.status;
    a.sel = c.sel;
    a.n_sel = c.n_sel;
    a.max_sel = c.max_sel;
    a.capacity = c.capacity;
    const size_t smem = kSmemBytes + 1024;
    auto kernel = sparse ? attend_kernel<true> : attend_kernel<false>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    prof_begin(c.stream, "sm100_attend");
    // the first item's query slice: q_lat [BJ][128][576] as (column in group, head,
    // group of 64 columns, token), one box = all heads x four groups, landing
    // group-major; its rope columns as (column, head, token), SW64 rows
    CUtensorMap mql, mqr;
    const int64_t BJ = (int64_t)c.batch * c.n_q;
    {
        const uint64_t dims[4] = {64, 128, 9, (uint64_t)BJ};
        const uint64_t str[3] = {576 * 2, 64 * 2, 128 * 576 * 2};
        const uint32_t box[4] = {64, 128, 4, 1};
        if (!make_map(&mql, q_lat, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        const uint64_t dims[3] = {576, 128, (uint64_t)BJ};
        const uint64_t str[2] = {576 * 2, 128 * 576 * 2};
        const uint32_t box[3] = {32, 128, 1};
        if (!make_map(&mqr, q_lat, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B)) return MLA_ERR_CUDA;
    }
    const cudaError_t e =
        launch_pdl(kernel, dim3(2 * pairs), dim3(kThreads), smem, c.stream, ml, mr, mql, mqr, a);
    prof_end(c.stream);
    if (launches) ++*launches;
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla
