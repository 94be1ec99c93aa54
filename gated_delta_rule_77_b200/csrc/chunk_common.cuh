// chunk_common.cuh -- device helpers shared by the chunkwise prefill kernels:
// split-precision tile stores, 128B-swizzled tile loads, and the 64x64 unit
// lower-triangular solve T = (I + A)^{-1} (chunk algebra of the Atomic-GDN2
// model card's recurrence, section 2.1, solved blockwise in fp32).
#pragma once

#include <stdint.h>

#include "sm100_util.cuh"

namespace gdn {
namespace chunk {

using namespace sm100;

// fp32 64x64 matrix in shared memory, float4 groups xor-swizzled by row so
// that row-parallel and column-parallel accesses both avoid bank conflicts.
__device__ __forceinline__ uint32_t fidx(int r, int m) {
    return static_cast<uint32_t>(r * 64 + ((((m >> 2) ^ r) & 15) << 2) + (m & 3));
}

// Eight fp32 values -> a 16-byte bf16 chunk (hi) and the bf16 rounding of the
// remainder (lo), so that hi + lo reproduces each value to ~2^-16.
__device__ __forceinline__ void store_split(uint8_t* hi_dst, uint8_t* lo_dst, const float* v) {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        hi[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        lo[e] = pack_bf16(v[2 * e] - bf16_lo(hi[e]), v[2 * e + 1] - bf16_hi(hi[e]));
    }
    *reinterpret_cast<uint4*>(hi_dst) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(lo_dst) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}

__device__ __forceinline__ void store_bf16x8(uint8_t* dst, const float* v) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
}

__device__ __forceinline__ void store_f16x8(uint8_t* dst, const float* v) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_f16(v[0], v[1]), pack_f16(v[2], v[3]),
                                                pack_f16(v[4], v[5]), pack_f16(v[6], v[7]));
}

__device__ __forceinline__ void load_bf16x8(const uint8_t* src, float* v) {
    const uint4 w = *reinterpret_cast<const uint4*>(src);
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        v[2 * e] = bf16_lo(x[e]);
        v[2 * e + 1] = bf16_hi(x[e]);
    }
}


// T = (I + A)^{-1} for a strictly lower triangular 64x64 fp32 A (layout fidx),
// written to T (plain row-major [64][64]; entries above the diagonal inside the
// 16x16 diagonal blocks are written as zero, other upper entries untouched).
// Y: 16 x 48 fp32 scratch.  Called by every thread of a CTA of at least 128
// threads (contains barriers).
//   (a) D_b = (I + A_bb)^{-1}, b = 0..3, by forward substitution: warp b,
//       lane = column;
//   (b) row blocks a = 1..3: T_{a,<a} = -D_a (A_{a,<a} T_{<a,<a}), both small
//       products register-blocked by four columns.
__device__ __forceinline__ void solve_unit_lower64(const float* sA, float* sT, float* sY, int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    if (warp < 4 && lane < 16) {
        const int o = warp * 16;
        float t[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            float a[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = *reinterpret_cast<const float4*>(&sA[fidx(o + rr, o + 4 * q)]);
                a[4 * q] = v.x; a[4 * q + 1] = v.y; a[4 * q + 2] = v.z; a[4 * q + 3] = v.w;
            }
            float acc[4] = {0.f, 0.f, 0.f, 0.f};     // short dependency chains
#pragma unroll
            for (int m = 0; m < rr; ++m) acc[m & 3] = fmaf(a[m], t[m], acc[m & 3]);
            t[rr] = (rr == lane) ? 1.f : -((acc[0] + acc[1]) + (acc[2] + acc[3]));
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) sT[(o + rr) * 64 + o + lane] = t[rr];
    }
    __syncthreads();
#pragma unroll 1
    for (int a = 1; a < 4; ++a) {
        // Thread tile: rows {rp, rp + 8} x four columns [4 c4, 4 c4 + 4).
        const int ncol4 = 4 * a;            // float4 column groups left of the diagonal block
        const int nitem = 8 * ncol4;
        const int rp = tid / ncol4, c4 = tid - (tid / ncol4) * ncol4;
        if (tid < nitem) {
            // Y[rr][4c4..] = sum_m A[16a+rr][m] T[m][4c4..]; T[m][c] = 0 for m < 4 c4.
            float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            for (int m4 = c4; m4 < 4 * a; ++m4) {
                const float4 a0 = *reinterpret_cast<const float4*>(&sA[fidx(16 * a + rp, 4 * m4)]);
                const float4 a1 = *reinterpret_cast<const float4*>(&sA[fidx(16 * a + rp + 8, 4 * m4)]);
                const float am[2][4] = {{a0.x, a0.y, a0.z, a0.w}, {a1.x, a1.y, a1.z, a1.w}};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 tv = *reinterpret_cast<const float4*>(&sT[(4 * m4 + e) * 64 + 4 * c4]);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        y[i][0] = fmaf(am[i][e], tv.x, y[i][0]);
                        y[i][1] = fmaf(am[i][e], tv.y, y[i][1]);
                        y[i][2] = fmaf(am[i][e], tv.z, y[i][2]);
                        y[i][3] = fmaf(am[i][e], tv.w, y[i][3]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
                *reinterpret_cast<float4*>(&sY[(rp + 8 * i) * 48 + 4 * c4]) =
                    make_float4(y[i][0], y[i][1], y[i][2], y[i][3]);
        }
        __syncthreads();
        if (tid < nitem) {
            // T[16a+rr][4c4..] = -sum_n D_a[rr][n] Y[n][4c4..]
            float t[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int n4 = 0; n4 < 4; ++n4) {
                const float4 d0 = *reinterpret_cast<const float4*>(&sT[(16 * a + rp) * 64 + 16 * a + 4 * n4]);
                const float4 d1 = *reinterpret_cast<const float4*>(&sT[(16 * a + rp + 8) * 64 + 16 * a + 4 * n4]);
                const float dn[2][4] = {{d0.x, d0.y, d0.z, d0.w}, {d1.x, d1.y, d1.z, d1.w}};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 yv = *reinterpret_cast<const float4*>(&sY[(4 * n4 + e) * 48 + 4 * c4]);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        t[i][0] = fmaf(dn[i][e], yv.x, t[i][0]);
                        t[i][1] = fmaf(dn[i][e], yv.y, t[i][1]);
                        t[i][2] = fmaf(dn[i][e], yv.z, t[i][2]);
                        t[i][3] = fmaf(dn[i][e], yv.w, t[i][3]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
                *reinterpret_cast<float4*>(&sT[(16 * a + rp + 8 * i) * 64 + 4 * c4]) =
                    make_float4(-t[i][0], -t[i][1], -t[i][2], -t[i][3]);
        }
        __syncthreads();
    }
}


}  // namespace chunk
}  // namespace gdn
