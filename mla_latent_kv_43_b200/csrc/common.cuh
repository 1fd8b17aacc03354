// Device helpers shared by every kernel of libmla: element conversion, the
// status word, and the rotary embedding of one interleaved pair.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mla.h"

namespace mla {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// First error wins: the word only changes while it still holds MLA_OK.
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
    if (status) atomicCAS(status, MLA_OK, code);
}

// Rotation of the interleaved pair (x0, x1) with index i of a d_rope-wide
// rope vector at position pos: angle = pos * base^(-2i/d_rope).  The angle and
// its sine/cosine are taken in double so that positions up to 2^31 keep the
// rotation exact to float rounding; the result is rounded to float once.
__device__ __forceinline__ void rope_pair(float x0, float x1, int64_t pos, int i, int d_rope,
                                          float base, float* y0, float* y1) {
    const double theta = pow((double)base, -2.0 * (double)i / (double)d_rope);
    const double ang = (double)pos * theta;
    double s, c;
    sincos(ang, &s, &c);
    *y0 = (float)((double)x0 * c - (double)x1 * s);
    *y1 = (float)((double)x0 * s + (double)x1 * c);
}

// Same rotation with the pair frequency given as a fraction of a turn in
// 64-bit fixed point, turn = round(theta / (2 pi) * 2^64) (rope_turn_table).
// pos * turn modulo 2^64 is frac(pos * theta / (2 pi)) exactly up to the
// table's rounding (< 2^-33 of a turn for pos < 2^31), so the angle reaches
// sincosf already reduced to [-pi, pi); only integer multiplies, no double.
__device__ __forceinline__ void rope_pair_turn(float x0, float x1, int64_t pos, uint64_t turn, float* y0,
                                               float* y1) {
    const uint64_t t = (uint64_t)pos * turn;
    const float ang = (float)(int32_t)(uint32_t)(t >> 32) * 1.46291807926715968e-9f;   // 2 pi / 2^32
    float s, c;
    sincosf(ang, &s, &c);
    *y0 = x0 * c - x1 * s;
    *y1 = x0 * s + x1 * c;
}

// The same rotation for results stored in bf16: the hardware sine / cosine
// (__sincosf, absolute error about 2^-21 on [-pi, pi), far below bf16's 2^-9
// relative rounding) instead of the correctly reduced sincosf, which costs
// microseconds per token in the absorb and prefill kernels.
// cos and sin of the angle pos * turn (turn: fractions of a full turn, 2^-64 units)
__device__ __forceinline__ void rope_cos_sin_turn(int64_t pos, uint64_t turn, float* c, float* s) {
    const uint64_t t = (uint64_t)pos * turn;
    const float ang = (float)(int32_t)(uint32_t)(t >> 32) * 1.46291807926715968e-9f;   // 2 pi / 2^32
    __sincosf(ang, s, c);
}

__device__ __forceinline__ void rope_pair_turn_bf16(float x0, float x1, int64_t pos, uint64_t turn, float* y0,
                                                    float* y1) {
    float s, c;
    rope_cos_sin_turn(pos, turn, &c, &s);
    *y0 = x0 * c - x1 * s;
    *y1 = x0 * s + x1 * c;
}

// Query position of token j of a sequence holding len keys (its queries'
// entries included): p = len - n_q + j.
__device__ __forceinline__ int64_t query_pos(int64_t len, int n_q, int j) { return len - n_q + j; }

__device__ __forceinline__ bool len_ok(int64_t len, int n_q, int64_t capacity, int64_t max_len) {
    return len >= n_q && len <= capacity && len <= max_len;
}

}  // namespace mla
