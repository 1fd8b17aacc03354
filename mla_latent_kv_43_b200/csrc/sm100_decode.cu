// Tensor-core decode path for the DeepSeek-V3 head geometry (bf16): workspace
// layout, the split-KV combine kernel and the launch sequence
//   absorb (+ q-RoPE + key-tile plan) -> attention -> combine -> up-projection.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "profile.h"
#include "sm100_host.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {
int launch_absorb(const DecodeCall& c, __nv_bfloat16* q_lat, int32_t* cum, int32_t* first_bj, int pairs,
                  int* launches);
int launch_upproj(const DecodeCall& c, const __nv_bfloat16* o_lat, int* launches);
int launch_attend(const DecodeCall& c, const __nv_bfloat16* q_lat, const int32_t* cum, __nv_bfloat16* o_lat,
                  __nv_bfloat16* part_o, float* part_lse, const int32_t* first_bj, int pairs, int* launches);

namespace {

constexpr int kHeads = 128, kDc = 512;

// Merge the pieces of query tokens whose key tiles were cut across clusters
// (log-sum-exp weighting, base 2), and zero the latent output of tokens with
// an invalid length.  Tokens finished inside one cluster are left untouched.
// grid (BJ, 128 / 4): 4 heads per block, 128 threads, 16 columns each.
__global__ void __launch_bounds__(128)
combine_kernel(const int32_t* __restrict__ cum, int BJ, int pairs, const __nv_bfloat16* __restrict__ part_o,
               const float* __restrict__ part_lse, __nv_bfloat16* __restrict__ o_lat) {
    grid_dep_wait();
    grid_dep_trigger();
    const int bj = blockIdx.x;
    const int T = cum[BJ];
    const int c0 = cum[bj], c1 = cum[bj + 1];
    const int h = blockIdx.y * 4 + (threadIdx.x >> 5);
    const int col = (threadIdx.x & 31) * 16;
    __nv_bfloat16* dst = o_lat + ((int64_t)bj * kHeads + h) * kDc + col;
    if (c1 == c0) {
        for (int i = 0; i < 16; ++i) dst[i] = __float2bfloat16_rn(0.f);
        return;
    }
    // cluster p covers key tiles [start(p), start(p + 1)); T * pairs fits 32 bits
    auto start = [&](int p) { return (int)(((uint32_t)p * (uint32_t)T) / (uint32_t)pairs); };
    auto pair_of = [&](int t) {      // largest p with start(p) <= t
        int lo = 0, hi = pairs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (start(mid) <= t) lo = mid; else hi = mid - 1;
        }
        return lo;
    };
    const int pf = pair_of(c0), pl = pair_of(c1 - 1);
    if (pf == pl) return;            // finished inside one cluster
    // clusters with an empty tile range between the first and the last piece hold nothing
    auto empty = [&](int p) { return start(p) == (p + 1 < pairs ? start(p + 1) : T); };
    // pieces in batches of kBatch: every load of a batch (log-sum-exps and partial
    // rows) is issued before any is used, so a batch costs one memory round trip
    // (two pieces per batch keep the registers low enough for ~1.5 waves)
    constexpr int kBatch = 2;
    float acc[16];
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    float wsum = 0.f;
    float M = -INFINITY;
    int p0 = pf;
    while (p0 <= pl) {
        int slots[kBatch] = {};
        int np = 0;
        for (; p0 <= pl && np < kBatch; ++p0) {
            if (p0 == pf || !empty(p0)) {
                const int sl = p0 == pf ? 2 * p0 + 1 : 2 * p0;
#pragma unroll
                for (int i = 0; i < kBatch; ++i)
                    if (i == np) slots[i] = sl;        // register-indexed, no local memory
                ++np;
            }
        }
        float lse[kBatch];
        uint4 v[kBatch][2];               // 16 bf16 columns per piece
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            if (i < np) {
                lse[i] = part_lse[slots[i] * kHeads + h];
                const uint4* src = reinterpret_cast<const uint4*>(part_o + ((int64_t)slots[i] * kHeads + h) * kDc + col);
                v[i][0] = src[0];
                v[i][1] = src[1];
            }
        }
        float Mb = M;
#pragma unroll
        for (int i = 0; i < kBatch; ++i)
            if (i < np) Mb = fmaxf(Mb, lse[i]);
        // rescale what was accumulated so far to the new maximum
        const float r = (M == -INFINITY) ? 0.f : exp2f(M - Mb);
        wsum *= r;
        for (int i = 0; i < 16; ++i) acc[i] *= r;
        M = Mb;
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            if (i < np) {
                const float w = exp2f(lse[i] - M);
                wsum += w;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint32_t pw[4] = {v[i][k].x, v[i][k].y, v[i][k].z, v[i][k].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[j]));
                        acc[8 * k + 2 * j] = fmaf(w, f.x, acc[8 * k + 2 * j]);
                        acc[8 * k + 2 * j + 1] = fmaf(w, f.y, acc[8 * k + 2 * j + 1]);
                    }
                }
            }
        }
    }
    const float inv = 1.f / wsum;
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * i] * inv, acc[2 * i + 1] * inv);
        pk[i] = *reinterpret_cast<uint32_t*>(&v);
    }
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

constexpr int kMaxPairs = 256;              // clusters per launch

// Clusters per launch.  splits > 0 asks for that many; 0 (auto) gives every
// cluster at least kMinTiles key tiles of the largest possible total
// (batch * n_q * ceil(max_len / 64)): fewer, longer pieces when there are few
// long sequences, all 74 clusters otherwise.
constexpr int64_t kMinTiles = 8;
int pairs_for(int splits, int64_t BJ, int64_t max_len) {
    const int max_pairs = std::max(1, std::min(sm_count() / 2, kMaxPairs));
    if (splits > 0) return std::min(splits, max_pairs);
    const int64_t tiles = BJ * ((max_len + 63) / 64);
    return (int)std::max<int64_t>(1, std::min<int64_t>(max_pairs, (tiles + kMinTiles - 1) / kMinTiles));
}

}  // namespace
}  // namespace sm100

bool sm100_decode_supported(const mla_dims& d) {
    return d.dtype == MLA_BF16 && d.heads == 128 && d.d_c == 512 && d.d_rope == 64 && d.qk_nope == 128 &&
           d.v_dim == 128;
}

void sm100_layout(const mla_dims& d, int batch, int n_q, int64_t max_len, int splits, mla_ws_layout* L) {
    const int64_t BJ = (int64_t)batch * n_q;
    const int P = sm100::pairs_for(splits, BJ, max_len);
    *L = mla_ws_layout{};
    size_t off = 0;
    auto take = [&](size_t bytes, size_t* o, size_t* sz) {
        *o = off;
        *sz = bytes;
        off = align_up(off + bytes, 256);
    };
    take(BJ * d.heads * (d.d_c + d.d_rope) * 2, &L->q_lat, &L->q_lat_bytes);
    take(BJ * d.heads * d.d_c * 2, &L->o_lat, &L->o_lat_bytes);
    take((size_t)2 * P * d.heads * d.d_c * 2, &L->part_o, &L->part_o_bytes);   // bf16
    take((size_t)2 * P * d.heads * 4, &L->part_lse, &L->part_lse_bytes);
    take((BJ + 1 + P) * 4, &L->sched, &L->sched_bytes);   // tile prefix, then each cluster's first token
    L->total = off;
    L->compute_dtype = MLA_BF16;
    L->splits = P;
}

int sm100_decode(const DecodeCall& c, int* launches) {
    // The tile ranges of the clusters are p * T / P in 32-bit arithmetic on the
    // device (T = total key tiles <= B * n_q * ceil(max_len / 64), or
    // ceil(max_sel / 64) per query for the sparse decode).
    const int64_t keys_bound = c.n_sel ? c.max_sel : c.max_len;
    if ((int64_t)c.batch * c.n_q * ((keys_bound + 63) / 64) * c.L.splits >= ((int64_t)1 << 31))
        return MLA_ERR_UNSUPPORTED;
    auto* q_lat = reinterpret_cast<__nv_bfloat16*>(c.ws + c.L.q_lat);
    auto* o_lat = reinterpret_cast<__nv_bfloat16*>(c.ws + c.L.o_lat);
    auto* part_o = reinterpret_cast<__nv_bfloat16*>(c.ws + c.L.part_o);
    auto* part_lse = reinterpret_cast<float*>(c.ws + c.L.part_lse);
    auto* cum = reinterpret_cast<int32_t*>(c.ws + c.L.sched);
    const int P = c.L.splits;
    const int BJ = c.batch * c.n_q;
    int rc;
    int32_t* first_bj = cum + BJ + 1;
    if ((rc = sm100::launch_absorb(c, q_lat, cum, first_bj, P, launches))) return rc;
    if ((rc = sm100::launch_attend(c, q_lat, cum, o_lat, part_o, part_lse, first_bj, P, launches))) return rc;
    prof_begin(c.stream, "sm100_combine");
    const cudaError_t e = sm100::launch_pdl(sm100::combine_kernel, dim3(BJ, 128 / 4), dim3(128), 0, c.stream,
                                            (const int32_t*)cum, BJ, P, (const __nv_bfloat16*)part_o,
                                            (const float*)part_lse, o_lat);
    prof_end(c.stream);
    if (launches) ++*launches;
    if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    return sm100::launch_upproj(c, o_lat, launches);
}


}  // namespace mla
