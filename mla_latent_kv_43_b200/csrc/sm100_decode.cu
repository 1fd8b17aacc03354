// Tensor-core decode path for the DeepSeek-V3 head geometry (bf16): workspace
// layout and the launch sequence
//   absorb (+ q-RoPE + key-tile plan) -> attention -> split-KV merge + up-projection.
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
int launch_upproj(const DecodeCall& c, __nv_bfloat16* o_lat, const __nv_bfloat16* part_o, const float* part_lse,
                  const int32_t* cum, int pairs, int* launches);
int launch_attend(const DecodeCall& c, const __nv_bfloat16* q_lat, const int32_t* cum, __nv_bfloat16* o_lat,
                  __nv_bfloat16* part_o, float* part_lse, const int32_t* first_bj, const int32_t* cut, int pairs,
                  int* launches);
int launch_attend_pair(const DecodeCall& c, const __nv_bfloat16* q_lat, const int32_t* cum, __nv_bfloat16* o_lat,
                       __nv_bfloat16* part_o, float* part_lse, const int32_t* first_bj, const int32_t* cut, int pairs,
                       int* launches);

namespace {

constexpr int kMaxPairs = 256;              // clusters per launch

// Clusters per launch.  splits > 0 asks for that many; 0 (auto) gives every
// cluster at least kMinTiles key tiles of the largest possible total
// (batch * n_q * ceil(max_len / 64)): fewer, longer pieces when there are few
// long sequences, all 74 clusters otherwise.
constexpr int64_t kMinTiles = 2;
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
    take((size_t)4 * P * d.heads * 4, &L->part_lse, &L->part_lse_bytes);   // [H][2P pieces][2 latent halves]
    // tile prefix, each cluster's first token, each piece slot's token, then
    // each cluster's first tile (and the total)
    take((BJ + 2 + 4 * P) * 4, &L->sched, &L->sched_bytes);
    L->total = off;
    L->compute_dtype = MLA_BF16;
    L->splits = P;
}

int sm100_decode(const DecodeCall& c, int* launches) {
    // Key-tile indices are int32 on the device (T = total key tiles <= B * n_q *
    // ceil(max_len / 64), or ceil(max_sel / 64) per query for the sparse decode,
    // plus the plan's per-token charge of 4 tiles).
    const int64_t keys_bound = c.n_sel ? c.max_sel : c.max_len;
    if ((int64_t)c.batch * c.n_q * ((keys_bound + 63) / 64 + 4) >= ((int64_t)1 << 31))
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
    const int32_t* cut = first_bj + 3 * P;
    if ((rc = sm100::launch_absorb(c, q_lat, cum, first_bj, P, launches))) return rc;
    // dense decode: the CTA-pair kernel or the latent-split kernel; decode over a
    // selection: the latent-split kernel gathering its rows (64-key tiles throughout).
    // The up-projection merges the split-KV pieces of each token.
    rc = (c.n_sel || !kDecodePairKernel)
             ? sm100::launch_attend(c, q_lat, cum, o_lat, part_o, part_lse, first_bj, cut, P, launches)
             : sm100::launch_attend_pair(c, q_lat, cum, o_lat, part_o, part_lse, first_bj, cut, P, launches);
    if (rc) return rc;
    return sm100::launch_upproj(c, o_lat, part_o, part_lse, cum, P, launches);
}


}  // namespace mla
