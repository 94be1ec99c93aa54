// prologue_math.cuh -- the elementwise maps of the layer's input prologue,
// shared by the prologue pass (prologue.cu) and the prefill kernel that
// applies the prologue while loading its inputs (chunk_pair_sm100.cu):
// SiLU after the width-4 convolution, beta = sigmoid(beta_raw) and
// g = -min(softplus(g_raw), 5) (Atomic-GDN2 model card, section 2.1: the bound
// 160 / bs2 with bs2 = 32).
#pragma once

#include <math.h>

#include "chunk_common.cuh"

namespace gdn {
namespace prologue_math {

__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2eP = 1.4426950408889634f;

// SiLU y / (1 + e^-y) with the hardware 2^x and a fast divide (relative
// error a few 1e-7, far below the bf16 rounding of the results).  The limits
// hold: e^-y overflows to inf for y < -88 (result -0), underflows to 0 for
// large y (result y).
__device__ __forceinline__ float act_fn(float y, bool silu) {
    return silu ? __fdividef(y, 1.f + ex2_fast(-y * kLog2eP)) : y;
}
__device__ __forceinline__ float sigmoid_fn(float x) { return 1.f / (1.f + expf(-x)); }

// log(1 + u) for u in [0, 1] from log(1 + u) = 2 atanh(s), s = u / (2 + u)
// in [0, 1/3], and the odd series atanh(s) = s + s^3/3 + s^5/5 + ...; eight
// terms leave a remainder below (1/3)^16 / 17 < 1.5e-9 of the sum.  Relative
// accuracy holds down to the smallest u (s ~ u/2), where log1p matters for
// a gate near 0.
__device__ __forceinline__ float log1p_unit(float u) {
    const float s = __fdividef(u, 2.f + u);
    const float z = s * s;
    float t = 1.f / 15.f;
    t = fmaf(t, z, 1.f / 13.f);
    t = fmaf(t, z, 1.f / 11.f);
    t = fmaf(t, z, 1.f / 9.f);
    t = fmaf(t, z, 1.f / 7.f);
    t = fmaf(t, z, 1.f / 5.f);
    t = fmaf(t, z, 1.f / 3.f);
    t = fmaf(t, z, 1.f);
    return 2.f * s * t;
}

// g = -min(softplus(x), 5) with softplus(x) = max(x, 0) + log1p(e^-|x|).
__device__ __forceinline__ float gate_fn(float x) {
    const float sp = fmaxf(x, 0.f) + log1p_unit(ex2_fast(-fabsf(x) * kLog2eP));
    return -fminf(sp, 5.f);
}

// The same two at a time, with paired fp32 (f32x2) arithmetic.  (Taking the
// reciprocals by Newton's iteration on the FMA pipe instead of the
// special-function unit measured slower: these maps are bound by instruction
// issue, not by the special-function unit.)
using chunk::add2;
using chunk::fma2;
using chunk::mul2;
__device__ __forceinline__ float2 gate_fn2(float2 x) {
    const float2 u = make_float2(ex2_fast(-fabsf(x.x) * kLog2eP), ex2_fast(-fabsf(x.y) * kLog2eP));
    const float2 s2 = make_float2(__fdividef(u.x, 2.f + u.x), __fdividef(u.y, 2.f + u.y));
    const float2 z = mul2(s2, s2);
    float2 t = make_float2(1.f / 15.f, 1.f / 15.f);
    t = fma2(t, z, make_float2(1.f / 13.f, 1.f / 13.f));
    t = fma2(t, z, make_float2(1.f / 11.f, 1.f / 11.f));
    t = fma2(t, z, make_float2(1.f / 9.f, 1.f / 9.f));
    t = fma2(t, z, make_float2(1.f / 7.f, 1.f / 7.f));
    t = fma2(t, z, make_float2(1.f / 5.f, 1.f / 5.f));
    t = fma2(t, z, make_float2(1.f / 3.f, 1.f / 3.f));
    t = fma2(t, z, make_float2(1.f, 1.f));
    const float2 l = mul2(mul2(s2, make_float2(2.f, 2.f)), t);
    return make_float2(-fminf(fmaxf(x.x, 0.f) + l.x, 5.f), -fminf(fmaxf(x.y, 0.f) + l.y, 5.f));
}
__device__ __forceinline__ float2 act_fn2(float2 y, bool silu) {
    if (!silu) return y;
    const float2 m = mul2(y, make_float2(-kLog2eP, -kLog2eP));
    const float2 d = add2(make_float2(ex2_fast(m.x), ex2_fast(m.y)), make_float2(1.f, 1.f));
    return mul2(y, make_float2(__fdividef(1.f, d.x), __fdividef(1.f, d.y)));
}

// Sums of 16 per-lane values (one per token) over the 32 lanes of a warp by
// a transposing butterfly: at each step a lane keeps half of its remaining
// tokens and adds its partner's partial for them, so that 8 + 4 + 2 + 1 + 1
// shuffles leave v[0] of lanes 2j and 2j + 1 with the warp's total for token
// butterfly_token(lane).
__device__ __forceinline__ void butterfly_sums16(float (&v)[16], int lane) {
#pragma unroll
    for (int half = 8, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
        }
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
}
__device__ __forceinline__ int butterfly_token(int lane) {
    return 8 * ((lane >> 4) & 1) + 4 * ((lane >> 3) & 1) + 2 * ((lane >> 2) & 1) + ((lane >> 1) & 1);
}

}  // namespace prologue_math
}  // namespace gdn
