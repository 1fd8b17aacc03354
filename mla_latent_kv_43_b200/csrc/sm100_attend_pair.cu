// Absorbed MLA attention against the latent cache on a CTA pair
// (tcgen05 cta_group::2): the dense decode's core kernel.
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
// Work split.  A cluster of two CTAs on two SMs is one MMA unit.  All 128
// heads of a token are the M dimension of both contractions, split 64 / 64:
// CTA r holds the query rows and the softmax of heads [64r, 64r + 64).
//  * Score GEMM (M 128 heads, N 64 keys, K 576): CTA r stages keys
//    [32r, 32r + 32) of the tile, all 576 columns; each CTA's S holds its 64
//    heads against all 64 keys -- complete scores, no partial sums to
//    exchange.
//  * Value GEMM (M 128 heads, N 256 latent columns, twice, K 64 keys): CTA r
//    stages latent columns [128r, 128r + 128) and [256 + 128r, 256 + 128r +
//    128) of all 64 keys.  These are re-read from L2 (the score stage of the
//    same tile brought them there from HBM a tile period earlier), so each
//    cache byte crosses HBM once; no load is multicast.
// Each CTA keeps its 64 heads x 512 latent fp32 O in TMEM.
//
// TMEM per CTA (512 columns): O [0, 256), S double buffer [256, 288) and
// [288, 320).  In the pair layout (M = 128 over two CTAs) a CTA's 64 rows
// fill all 128 lanes: lane i and lane i + 64 both hold row i, the first and
// the second half of the N columns.
//
// Shared memory per CTA: the query rows (9 groups of 64 columns x 64 rows,
// 72 KB), two P buffers (64 heads x 64 keys bf16), a ring of two key tiles
// (this CTA's 32 keys x 9 column groups, 36 KB each) for the score GEMM and
// a ring of four value units (2 column groups x 64 keys, 16 KB; two per tile)
// for the value GEMM, so both rings hold two tiles.  Every staged unit
// arrives in ONE tensor copy: the maps view a cache row as 9 groups of
// 64 columns (a dimension of stride 128 bytes placed after the key
// dimension), so a box of several groups lands as consecutive 8 KB
// group-major blocks, the layout both GEMMs read.  (A single thread issues
// about one tensor copy per 0.3 us whatever its size up to 16 KB, so fewer,
// larger copies are what keeps the loads at HBM speed.)
//
// Roles (384 threads): warp 0 key / query loads, warp 1 MMA issue (even CTA;
// TMEM allocation in both), warp 2 value loads (and the zeroing of value rows
// past the visible keys), warps 4-11 softmax and epilogue: thread t of
// warps 4-7 and of warps 8-11 reads TMEM lane t (head 64r + t % 64, key /
// column half t / 64), the two warp sets splitting each lane's columns, so
// every tile's softmax runs on 256 threads of 16 scores each.
//
// Work items as in the single-CTA kernel: the 64-key tiles of all query
// tokens are concatenated and cut into one contiguous range per pair.  A
// token whose tiles all fall in one pair's range is finished there
// (normalised latent output, bf16); a token cut across pairs leaves partial
// outputs plus log2-sum-exp per piece for the merge before the up-projection.
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

constexpr int kKeys = 64;                    // keys per tile (the pair); 32 staged by each CTA for the score
constexpr int kBox = 8192;                   // one column group of 64 rows
constexpr int kQBoxes = 9;                   // 576 / 64 column groups
constexpr int kKTile = kQBoxes * 4096;       // one CTA's key tile: 9 groups x 32 keys
constexpr int kKS = 2;                       // key-tile ring slots
constexpr int kVS = 4;                       // value-unit ring slots
constexpr int kVUnits = 2;                   // value units per tile: 2 latent halves
constexpr int kOffQ = 0;
constexpr int kOffP = kOffQ + kQBoxes * kBox;         // 2 buffers of 64 heads x 64 keys
constexpr int kOffK = kOffP + 2 * kBox;
constexpr int kOffV = kOffK + kKS * kKTile;
constexpr int kSmemBytes = kOffV + kVS * 2 * kBox;
constexpr int kThreads = 384;
constexpr uint32_t kColO = 0, kColS = 256, kTmemCols = 512;
constexpr uint32_t kSCols = kKeys / 2;        // S columns per buffer (64 heads x 64 keys in the pair layout)
constexpr float kRescaleThreshold = 8.0f;    // log2 units
// value units of tile g may be fetched once the key tile g + 1 has been
// requested (tile g's latent columns are then in L2)
constexpr int kVLagTiles = 1;

struct PairArgs {
    const __nv_bfloat16* q_lat;   // [BJ][128][576]
    const int32_t* cum;           // [BJ + 1] 64-key tile prefix
    const int32_t* first_bj;      // [pairs] first query token of each pair's range
    const int32_t* cut;           // [pairs + 1] first key tile of each pair's range
    const int32_t* seq_lens;
    int BJ, n_q, pairs;
    float scale_log2;             // softmax_scale * log2(e)
    __nv_bfloat16* o_lat;         // [BJ][128][512]
    // split-KV pieces, normalised per piece: element (slot, head h, column c) at
    // ((h * 8 + c / 64) * 2 pairs + slot) * 64 + c % 64
    __nv_bfloat16* part_o;
    float* part_lse;              // [128 heads][2 * pairs][2 latent halves], log2 domain
    int32_t* status;
};

struct Item {
    int bj, t0, t1, n_vis, slot;  // slot < 0: finished here; n_vis: keys this token attends
};

// Pieces of the concatenated tile range [s0, s1) of one pair, in order.
struct ItemIter {
    const int32_t* cum;
    const int32_t* lens;
    int BJ, n_q, bj, s0, s1, pair;
    __device__ void init(const PairArgs& a, int p) {
        cum = a.cum;
        BJ = a.BJ;
        n_q = a.n_q;
        lens = a.seq_lens;
        pair = p;
        s0 = a.cut[p];
        s1 = a.cut[p + 1];
        bj = a.first_bj[p];
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
            it.n_vis = (int)query_pos(lens[b], n_q, j) + 1;
            it.slot = (c0 >= s0 && c1 <= s1) ? -1 : (c0 < s0 ? 2 * pair : 2 * pair + 1);
            return true;
        }
        return false;
    }
};

__device__ __forceinline__ void st_shared_u4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attend_pair_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, PairArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // waited on by the even CTA's MMA warp (arrivals and bytes from both CTAs)
    __shared__ uint64_t kfull[kKS], vready[kVS], qfull, sfree[2], pfull[2], ep_done;
    // completed by the pair's MMA commits in both CTAs, or local
    __shared__ uint64_t kempty[kKS], vempty[kVS], vland[kVS], qempty, sfull[2], pfree[2], o_done[2], item_done,
        drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ int k_issued;                  // key tiles this CTA has requested (value-load pacing)
    // the four threads of a head exchange tile maxima and row sums; every read
    // of one use precedes a group barrier that precedes the next write
    __shared__ float xch[256];
    __shared__ int group_ok[2];               // softmax group: outcome of the leader's bounded waits

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kKS; ++s) {
            mbar_init(&kfull[s], 1);          // the even CTA's expect_tx; bytes of both CTAs
            mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < kVS; ++s) {
            mbar_init(&vready[s], 2);         // each CTA's value loader, after landing (and zeroing)
            mbar_init(&vempty[s], 1);
            mbar_init(&vland[s], 1);
        }
        mbar_init(&qfull, 1);
        mbar_init(&qempty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sfree[i], 2);          // each CTA's softmax has read S
            mbar_init(&pfull[i], 2);          // each CTA's softmax has written P
            mbar_init(&sfull[i], 1);
            mbar_init(&pfree[i], 1);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(&ep_done, 2);               // each CTA's epilogue has read O
        mbar_init(&item_done, 1);
        mbar_init(&drain, 1);
        abort_flag = 0;
        k_issued = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();          // both CTAs' barriers are initialised before any remote access
    tc_fence_after();
    grid_dep_wait();         // q_lat and the tile plan come from the previous kernel
    grid_dep_trigger();
    const uint32_t tmem = tmem_base;
    const uint32_t sbase = smem_u32(smem);
    volatile int* abort = &abort_flag;
    volatile int* kiss = &k_issued;
    auto fail = [&]() {
        *abort = 1;
        set_status(a.status, MLA_ERR_TIMEOUT);
    };
    // barriers of the even CTA, as shared::cluster addresses
    auto lead = [&](uint64_t* bar) { return map_peer(smem_u32(bar), 0); };

    if (warp == 0) {
        // ------------------------------------------------------------ query and key loads
        if (elect_one()) {
            tma_prefetch(&map_q);
            tma_prefetch(&map_k);
            const uint64_t keep_l2 = l2_policy_evict_last();
            ItemIter iter;
            iter.init(a, pair);
            Item item;
            uint32_t kc = 0, n = 0;
            bool ok = true;
            while (ok && iter.next(item)) {
                const int b = item.bj / a.n_q;
                // the query rows of this item once every score GEMM of the previous one is done
                if (n > 0 && !mbar_wait(&qempty, (n - 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                if (rank == 0) mbar_expect_tx(&qfull, 2 * kQBoxes * kBox);
                tma_load_3d_pair(smem + kOffQ, &map_q, lead(&qfull), 0, item.bj * 128 + 64 * (int)rank, 0);
                for (int t = item.t0; t < item.t1; ++t, ++kc) {
                    const int key0 = t * kKeys + 32 * (int)rank;
                    const int s = kc % kKS;
                    if (kc >= (uint32_t)kKS && !mbar_wait(&kempty[s], ((kc / kKS) - 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_expect_tx(&kfull[s], 2 * kKTile);
                    // kept in L2 for the value re-read of the same tile
                    tma_load_4d_pair_hint(smem + kOffK + s * kKTile, &map_k, lead(&kfull[s]), 0, key0, 0, b, keep_l2);
                    *kiss = (int)kc + 1;
                }
                ++n;
            }
            *kiss = 0x7fffffff;               // no more key chunks: value loads need not wait
            if (!ok) fail();
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue (even CTA)
        // Two streams in tile order: score GEMMs S(g) (one key tile, 9 column
        // groups x 4 K-steps) and value GEMMs O(g) (2 value units, 4 K-steps
        // each), the latter advanced one unit at a time.  The whole warp runs the loop (decisions are
        // lane 0's observations, broadcast); one elected lane issues.
        if (rank == 0) {
            constexpr uint32_t idS = idesc_bf16(128, kKeys, false, false);      // pair: 32 keys from each CTA
            constexpr uint32_t idO = idesc_bf16(128, 256, false, true);
            const uint64_t dQ = sdesc(sbase + kOffQ, 16, 1024, kSwizzle128);     // query rows, K-major
            const uint64_t dK = sdesc(sbase + kOffK, 16, 1024, kSwizzle128);     // key tile, K-major
            const uint64_t dP = sdesc(sbase + kOffP, 16, 1024, kSwizzle128);     // P rows, K-major
            const uint64_t dV = sdesc(sbase + kOffV, kBox, 1024, kSwizzle128);   // value unit, MN-major
            ItemIter iterS, iterO;
            iterS.init(a, pair);
            iterO.init(a, pair);
            Item itS, itO;
            bool haveS = iterS.next(itS), haveO = iterO.next(itO);
            int kS = 0, kO = 0;                    // tile index within the current item
            uint32_t gS = 0, gO = 0;               // global tile counters
            uint32_t cO = 0;                       // value unit within the current tile
            uint32_t kc = 0, vc = 0;               // ring chunk counters
            uint32_t nS = 0, nO = 0;               // item counters
            bool qS = false;                       // query rows of the current S item landed
            uint32_t idle = 0;
            uint64_t t_idle = 0;
            bool ok = true;
            while (ok && haveO) {
                bool progressed = false;
                // value chunk of O(gO): needs P(gO) from both CTAs, its value chunk in both,
                // and (first tile of an item after the first) both epilogues done with O
                if (gO < gS) {
                    bool ready = true;
                    if (cO == 0) {
                        ready = mbar_ready_cluster_w(&pfull[gO & 1], (gO >> 1) & 1) &&
                                (kO != 0 || nO == 0 || mbar_ready_cluster_w(&ep_done, (nO - 1) & 1));
                    }
                    const int vs = vc % kVS;
                    if (ready && mbar_ready_cluster_w(&vready[vs], (vc / kVS) & 1)) {
                        tc_fence_after();
                        const int half = cO;                                 // latent half
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint32_t pa = (gO & 1) * kBox + ks * 32;
                            mma_pair_ss_w(tmem + kColO + 128 * half, sdesc_add(dP, pa),
                                          sdesc_add(dV, vs * 2 * kBox + ks * 2048), idO,
                                          (kO == 0 && ks == 0) ? 0u : 1u);
                        }
                        mma_commit_pair_w(&vempty[vs]);
                        ++vc;
                        if (++cO == kVUnits) {
                            cO = 0;
                            mma_commit_pair_w(&pfree[gO & 1]);
                            mma_commit_pair_w(&o_done[gO & 1]);
                            ++gO;
                            if (++kO == itO.t1 - itO.t0) {
                                mma_commit_pair_w(&item_done);
                                kO = 0;
                                ++nO;
                                haveO = iterO.next(itO);
                            }
                        }
                        progressed = true;
                    }
                }
                // S(gS): needs the item's query rows, a free S buffer and the key tile
                if (haveS) {
                    if (!qS) qS = mbar_ready_w(&qfull, nS & 1);
                    bool ready = qS;
                    if (ready && gS >= 2) ready = mbar_ready_cluster_w(&sfree[gS & 1], ((gS >> 1) - 1) & 1);
                    const int s = kc % kKS;
                    if (ready && mbar_ready_w(&kfull[s], (kc / kKS) & 1)) {
                        tc_fence_after();
#pragma unroll
                        for (int gi = 0; gi < kQBoxes; ++gi)
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_pair_ss_w(tmem + kColS + kSCols * (gS & 1), sdesc_add(dQ, gi * kBox + ks * 32),
                                              sdesc_add(dK, s * kKTile + gi * 4096 + ks * 32), idS,
                                              (gi == 0 && ks == 0) ? 0u : 1u);
                        mma_commit_pair_w(&kempty[s]);
                        mma_commit_pair_w(&sfull[gS & 1]);
                        ++kc;
                        ++gS;
                        if (++kS == itS.t1 - itS.t0) {
                            mma_commit_pair_w(&qempty);
                            kS = 0;
                            qS = false;
                            ++nS;
                            haveS = iterS.next(itS);
                        }
                        progressed = true;
                    }
                }
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
            mma_commit_pair_w(&drain);
            mbar_wait(&drain, 0, nullptr);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ value loads
        // Value unit (half h) of tile g: latent columns [256h + 128r, +128)
        // (column groups 4h + 2r and 4h + 2r + 1) of the tile's 64 keys, one
        // tensor copy.  A unit is requested once its slot is free and the key
        // tile g + 1 has been requested;
        // once it lands, rows past the visible keys (last tile of an item) are
        // zeroed, then the even CTA's MMA warp is told.
        // The warp runs one loop; lane 0 decides, every lane zeroes.
        const uint64_t last_use = l2_policy_evict_first();     // the cache rows' last read
        ItemIter it_req, it_rel;                 // the request and the relay side walk the same items
        it_req.init(a, pair);
        it_rel.init(a, pair);
        Item req, rel;
        bool have_req = it_req.next(req), have_rel = it_rel.next(rel);
        int tile_req = have_req ? req.t0 : 0, tile_rel = have_rel ? rel.t0 : 0;
        uint32_t c_req = 0, c_rel = 0;           // unit within the tile
        uint32_t g_req = 0;                      // global tile of the next request
        uint32_t vq = 0, vr = 0;                 // ring counters: requested, relayed
        uint32_t idle = 0;
        uint64_t t_idle = 0;
        bool ok = true;
        while (ok && have_rel) {
            bool progressed = false;
            if (have_req && vq < vr + kVS) {
                const int vs = vq % kVS;
                const bool lagged = *kiss >= (int)(g_req + 1 + kVLagTiles);
                const bool free_ = vq < (uint32_t)kVS || mbar_ready(&vempty[vs], ((vq / kVS) - 1) & 1);
                if (__shfl_sync(0xffffffffu, (lagged && free_) ? 1 : 0, 0)) {
                    if (lane == 0) {
                        const int b = req.bj / a.n_q;
                        const int half = c_req;
                        const int key0 = tile_req * kKeys;
                        mbar_expect_tx(&vland[vs], 2 * kBox);
                        tma_load_4d_hint(smem + kOffV + vs * 2 * kBox, &map_v, &vland[vs], 0, key0, 4 * half + 2 * (int)rank,
                                         b, last_use);
                    }
                    ++vq;
                    if (++c_req == kVUnits) {
                        c_req = 0;
                        ++g_req;
                        if (++tile_req == req.t1) {
                            have_req = it_req.next(req);
                            if (have_req) tile_req = req.t0;
                        }
                    }
                    progressed = true;
                }
            }
            if (vr < vq && mbar_ready_w(&vland[vr % kVS], (vr / kVS) & 1)) {
                const int vs = vr % kVS;
                // keys of this unit: [tile * 64, +64); rows of keys >= n_vis are zeroed
                const int first = tile_rel * kKeys;
                const int keep = max(0, min(64, rel.n_vis - first));
                if (keep < 64) {
                    const uint32_t base = sbase + kOffV + vs * 2 * kBox;
                    const int nrows = 64 - keep;           // rows keep..63 of both column groups
                    for (int i = lane; i < nrows * 16; i += 32) {
                        const int r = keep + (i >> 4), grp = (i >> 3) & 1, ch = i & 7;
                        st_shared_u4(base + grp * kBox + r * 128 + ch * 16, 0u, 0u, 0u, 0u);
                    }
                    fence_async_smem();
                    __syncwarp();
                }
                if (lane == 0) mbar_arrive_peer(lead(&vready[vs]));
                ++vr;
                if (++c_rel == kVUnits) {
                    c_rel = 0;
                    if (++tile_rel == rel.t1) {
                        have_rel = it_rel.next(rel);
                        if (have_rel) tile_rel = rel.t0;
                    }
                }
                progressed = true;
            }
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
        // every requested chunk has landed before the CTA may exit
        for (uint32_t i = vr; i < vq; ++i)
            if (lane == 0) mbar_wait(&vland[i % kVS], (i / kVS) & 1, nullptr);
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax and epilogue
        // st (0..255): TMEM lane t = st % 128 (head 64r + t % 64, key / column half
        // part = t / 64) and column half cv = st / 128 of that lane: keys
        // [32 part + 16 cv, +16) of each tile, O columns [128 cv, 128 cv + 128).
        // The four threads of a head meet through xch (tile maxima; row sums at the
        // end of an item).
        const int st = threadIdx.x - 128;
        const int t = st & 127, cv = st >> 7;
        const int q = warp & 3;
        const int hl = t & 63, part = t >> 6;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const bool leader = st == 0;
        auto group_sync = [&]() { named_barrier(1, 256); };
        // true when the predicate holds in any thread of the group (a group barrier)
        auto group_any = [&](bool v) -> bool {
            uint32_t r;
            asm volatile(
                "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, 256, p;\n\t"
                "selp.u32 %0, 1, 0, q;\n\t}"
                : "=r"(r)
                : "r"((uint32_t)v)
                : "memory");
            return r != 0;
        };
        // One thread waits (bounded) and the group barrier hands its outcome to all
        // eight warps, so they leave together on a timeout and no warp is left at a
        // group barrier.  Alternate flag slots: a thread reads use i before the
        // barrier of use i + 1, which precedes the leader's write of use i + 2.
        uint32_t n_wait = 0;
        auto group_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            const int slot = n_wait++ & 1;
            if (leader) group_ok[slot] = mbar_wait(bar, parity, abort) ? 1 : 0;
            group_sync();
            return group_ok[slot] != 0;
        };
        auto head_sum = [&](const float* v) { return (v[hl] + v[hl + 64]) + (v[hl + 128] + v[hl + 192]); };
        auto head_max = [&](const float* v) {
            return fmaxf(fmaxf(v[hl], v[hl + 64]), fmaxf(v[hl + 128], v[hl + 192]));
        };
        ItemIter iter;
        iter.init(a, pair);
        Item item;
        uint32_t g = 0, n_item = 0;
        bool stop = false;
        while (!stop && iter.next(item)) {
            const int T = item.t1 - item.t0;
            float m_used = -INFINITY, l = 0.f;     // this thread's part of the row sum, relative to m_used
            for (int k = 0; k < T && !stop; ++k, ++g) {
                const int sb = g & 1;
                if (!group_wait(&sfull[sb], (g >> 1) & 1)) { stop = true; break; }
                tc_fence_after();
                float x[16];
                {
                    uint32_t r[16];
                    tmem_ld16(tmem + lane_off + kColS + kSCols * sb + 16 * cv, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(r[i]);
                }
                tc_fence_before();
                // keys past the visible ones (last tile) take no weight, whatever they hold
                const int key0 = (item.t0 + k) * kKeys + 32 * part + 16 * cv;
                const int valid = min(16, item.n_vis - key0);
                if (valid < 16) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = i < valid ? x[i] : -INFINITY;
                }
                float mx4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) mx4[i] = fmaxf(fmaxf(x[i], x[i + 4]), fmaxf(x[i + 8], x[i + 12]));
                // base 2: scores scaled by scale * log2(e) (> 0, so the raw maximum serves)
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * a.scale_log2;
                xch[st] = mx;
                group_sync();                        // every S read of this tile is done, maxima published
                if (leader) mbar_arrive_peer(lead(&sfree[sb]));
                const float m_tile = head_max(xch);
                // Lazy rescaling: the maximum moves only when it grew by more than 2^8
                // (an item's first tile takes its maximum as it is).
                const float m_cand = fmaxf(m_used, m_tile);
                const float m = (k == 0 || m_cand > m_used + kRescaleThreshold) ? m_cand : m_used;
                // P buffer sb is free once O(g - 2) has completed
                if (g >= 2 && !group_wait(&pfree[sb], ((g >> 1) - 1) & 1)) { stop = true; break; }
                // O holds the item's tiles before g relative to m_used: rescale it when m
                // moved (after O(g - 1) completed).  Warp-collective TMEM access: lanes
                // that need none multiply by 1.  Whether any head of the group
                // rescales is itself a group decision (the barrier below is group-wide).
                const bool need = k > 0 && m > m_used;
                if (group_any(need)) {
                    if (!group_wait(&o_done[(g - 1) & 1], ((g - 1) >> 1) & 1)) { stop = true; break; }
                    tc_fence_after();
                    const float alpha = need ? ex2(m_used - m) : 1.f;
#pragma unroll 1
                    for (int c = 0; c < 8; ++c) {
                        uint32_t r[16];
                        const uint32_t ta = tmem + lane_off + kColO + 128 * cv + 16 * c;
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
                // P row: head hl, keys [32 part + 16 cv, +16) -> 16-byte chunks
                // 4 part + 2 cv and 4 part + 2 cv + 1 of row hl of buffer sb
                const uint32_t prow = sbase + kOffP + sb * kBox + hl * 128;
                float ps4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint32_t pw[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float p0 = ex2(fmaf(x[8 * cc + 2 * i], a.scale_log2, -m));
                        const float p1 = ex2(fmaf(x[8 * cc + 2 * i + 1], a.scale_log2, -m));
                        ps4[i] += p0 + p1;
                        pw[i] = pack_bf16(p0, p1);
                    }
                    st_shared_u4(prow + (((4 * part + 2 * cv + cc) ^ (hl & 7)) << 4), pw[0], pw[1], pw[2], pw[3]);
                }
                l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
                fence_async_smem();
                group_sync();
                if (leader) mbar_arrive_peer(lead(&pfull[sb]));
            }
            if (stop) break;
            // epilogue: the four parts of each head's row sum meet; every thread writes
            // its 128 latent columns (normalised, or a partial plus log2-sum-exp)
            if (!group_wait(&item_done, n_item & 1)) break;
            xch[st] = l;
            group_sync();
            const float lsum = head_sum(xch);
            tc_fence_after();
            const float inv = 1.f / lsum;
            const int head = 64 * (int)rank + hl;
            // each warp stages 32 rows x 64 bytes in its eighth of the P area so one
            // store instruction covers eight contiguous 64-byte row segments
            const uint32_t scr = sbase + kOffP + (warp - 4) * 2048;
#pragma unroll 1
            for (int sub = 0; sub < 4; ++sub) {                   // 32 columns per step
                uint32_t r[32];
                tmem_ld32(tmem + lane_off + kColO + 128 * cv + 32 * sub, r);
                tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    st_shared_u4(scr + lane * 64 + ((j ^ (lane & 3)) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2],
                                 w[4 * j + 3]);
                __syncwarp();
                // lane i of this warp holds TMEM lane 32 q + i: head 64 r + (32 q + i) % 64,
                // latent columns 256 cv + 128 part + 32 sub
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int rr = 8 * kk + (lane >> 2), pc = lane & 3;
                    const int tt = 32 * q + rr;
                    const int hh = 64 * (int)rank + (tt & 63);
                    const uint4 v = ld_shared_u4(scr + rr * 64 + ((pc ^ (rr & 3)) << 4));
                    const int col = 256 * cv + 128 * (tt >> 6) + 32 * sub + 8 * pc;
                    __nv_bfloat16* dst =
                        item.slot < 0 ? a.o_lat + ((int64_t)item.bj * 128 + hh) * 512 + col
                                      : a.part_o + (((int64_t)hh * 8 + (col >> 6)) * (2 * a.pairs) + item.slot) * 64 +
                                            (col & 63);
                    *reinterpret_cast<uint4*>(dst) = v;
                }
                __syncwarp();
            }
            if (item.slot >= 0 && part == 0 && cv == 0) {
                // the same log-sum-exp for both latent halves of the piece
                const float lse = m_used + __log2f(lsum);
                a.part_lse[(head * 2 * a.pairs + item.slot) * 2] = lse;
                a.part_lse[(head * 2 * a.pairs + item.slot) * 2 + 1] = lse;
            }
            // the next item's first value GEMM (accumulate = 0) may start only after
            // both CTAs' reads of this item's O
            tc_fence_before();
            group_sync();
            if (leader) mbar_arrive_peer(lead(&ep_done));
            ++n_item;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort) {
        // a wait expired: loads already requested may still be landing in this
        // CTA's shared memory; give them time before the CTA exits
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
    }
    cluster_sync();          // no CTA leaves while its peer may still access it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace

int launch_attend_pair(const DecodeCall& c, const __nv_bfloat16* q_lat, const int32_t* cum, __nv_bfloat16* o_lat,
                       __nv_bfloat16* part_o, float* part_lse, const int32_t* first_bj, const int32_t* cut, int pairs,
                       int* launches) {
    // Rows of 576 columns viewed as 9 groups of 64: (column in group, row,
    // group, ...) with the group dimension's stride 128 bytes, so one box of
    // several groups lands group-major (each group a 64-row x 128-byte block).
    CUtensorMap mq, mk, mv;
    {
        // query rows: [BJ * 128][576]; one box = 64 rows x all 9 groups
        const uint64_t dims[3] = {64, (uint64_t)c.batch * c.n_q * 128, 9};
        const uint64_t str[2] = {576 * 2, 64 * 2};
        const uint32_t box[3] = {64, 64, 9};
        if (!make_map(&mq, q_lat, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    {
        // cache [batch][capacity][576]; key tiles 32 keys x 9 groups, value units 64 keys x 2 groups
        const uint64_t dims[4] = {64, (uint64_t)c.capacity, 9, (uint64_t)c.batch};
        const uint64_t str[3] = {576 * 2, 64 * 2, (uint64_t)c.capacity * 576 * 2};
        const uint32_t box_k[4] = {64, 32, kQBoxes, 1}, box_v[4] = {64, 64, 2, 1};
        if (!make_map(&mk, c.cache, 4, dims, str, box_k, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
        if (!make_map(&mv, c.cache, 4, dims, str, box_v, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    }
    PairArgs a{};
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
    const size_t smem = kSmemBytes + 1024;
    if (cudaFuncSetAttribute(attend_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return MLA_ERR_CUDA;
    prof_begin(c.stream, "sm100_attend");
    const cudaError_t e = launch_pdl(attend_pair_kernel, dim3(2 * pairs), dim3(kThreads), smem, c.stream, mq, mk, mv, a);
    prof_end(c.stream);
    if (launches) ++*launches;
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla
