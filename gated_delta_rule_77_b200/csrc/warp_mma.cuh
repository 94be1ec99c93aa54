// warp_mma.cuh -- warp-level tensor-core products with mma.sync m16n8k16
// (bf16 in, fp32 accumulate) on fp32 operands split into bf16 hi + lo
// (hi*hi + hi*lo + lo*hi, about 2^-16 relative), shared by the backward
// kernels and the segment correction of the long-sequence prefill.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gdn {
namespace wmma16 {

// Products on the tensor cores with mma.sync m16n8k16 (bf16 in, fp32
// accumulate).  Every fp32 operand is split as x = hi + lo with hi, lo in
// bf16 (16 significant bits together) and a product is hi*hi + hi*lo + lo*hi,
// about 2^-16 relative: fp32-grade for these products.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 r = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc[j] += A[rb .. rb+15][0 .. K) * B[0 .. K)[cb + 8j .. cb + 8j + 7] for one
// warp, through element accessors a(r, k) and b(k, n).  Fragment layout of
// m16n8k16 (g = lane / 4, t = lane % 4): A rows g and g + 8, columns 2t, 2t+1
// and 2t+8, 2t+9; B columns n = g, rows 2t, 2t+1, 2t+8, 2t+9; the result
// acc[j][e] sits at row rb + g + 8 (e / 2), column cb + 8j + 2t + e % 2.
// With fp32 tiles of row stride 4 mod 32 the B reads of a row-major tile
// (bank 8t + g) are conflict-free and the others at most 2-way.
template <int NT, int K, typename FA, typename FB>
__device__ __forceinline__ void wmm(float (&acc)[NT][4], int rb, int cb, FA a, FB b) {
    const int l = threadIdx.x & 31, g = l >> 2, t = l & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t ah[4], al[4];
        split2(a(rb + g, k0 + 2 * t), a(rb + g, k0 + 2 * t + 1), ah[0], al[0]);
        split2(a(rb + g + 8, k0 + 2 * t), a(rb + g + 8, k0 + 2 * t + 1), ah[1], al[1]);
        split2(a(rb + g, k0 + 2 * t + 8), a(rb + g, k0 + 2 * t + 9), ah[2], al[2]);
        split2(a(rb + g + 8, k0 + 2 * t + 8), a(rb + g + 8, k0 + 2 * t + 9), ah[3], al[3]);
        uint32_t bh0[NT], bl0[NT], bh1[NT], bl1[NT];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int n = cb + 8 * j + g;
            split2(b(k0 + 2 * t, n), b(k0 + 2 * t + 1, n), bh0[j], bl0[j]);
            split2(b(k0 + 2 * t + 8, n), b(k0 + 2 * t + 9, n), bh1[j], bl1[j]);
        }
        // The three products of a tile accumulate in one register set: issue
        // them NT apart so that consecutive MMAs are independent.
#pragma unroll
        for (int j = 0; j < NT; ++j) mma16816(acc[j], ah, bh0[j], bh1[j]);
#pragma unroll
        for (int j = 0; j < NT; ++j) mma16816(acc[j], ah, bl0[j], bl1[j]);
#pragma unroll
        for (int j = 0; j < NT; ++j) mma16816(acc[j], al, bh0[j], bh1[j]);
    }
}

// ldmatrix of four 8 x 8 bf16 matrices (lane i gives the row address of
// matrix i / 8), plain or transposed.
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))) : "memory");
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))) : "memory");
}

// wmm with the B operand already split: bf16 tiles bh (hi) and bl (lo) of
// row length LD.  TRANS: B(k, n) = tile[k][n]; otherwise B(k, n) =
// tile[n][k].  Each ldmatrix.x4 brings both fragment registers of two
// 8-column tiles (NT even).  Rows must start on 16-byte boundaries.
template <int NT, int K, bool TRANS, int LD, typename FA>
__device__ __forceinline__ void wmm_sb(float (&acc)[NT][4], int rb, int cb, FA a,
                                       const __nv_bfloat16* bh, const __nv_bfloat16* bl) {
    static_assert(NT % 2 == 0, "pairs of 8-column tiles");
    const int l = threadIdx.x & 31, g = l >> 2, t = l & 3;
    const int mi = l >> 3, rr = l & 7;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t ah[4], al[4];
        split2(a(rb + g, k0 + 2 * t), a(rb + g, k0 + 2 * t + 1), ah[0], al[0]);
        split2(a(rb + g + 8, k0 + 2 * t), a(rb + g + 8, k0 + 2 * t + 1), ah[1], al[1]);
        split2(a(rb + g, k0 + 2 * t + 8), a(rb + g, k0 + 2 * t + 9), ah[2], al[2]);
        split2(a(rb + g + 8, k0 + 2 * t + 8), a(rb + g + 8, k0 + 2 * t + 9), ah[3], al[3]);
        uint32_t bhv[NT / 2][4], blv[NT / 2][4];
#pragma unroll
        for (int jp = 0; jp < NT / 2; ++jp) {
            const int n0 = cb + 16 * jp;
            long off;
            if (TRANS) off = (long)(k0 + rr + 8 * (mi & 1)) * LD + n0 + 8 * (mi >> 1);
            else off = (long)(n0 + rr + 8 * (mi >> 1)) * LD + k0 + 8 * (mi & 1);
            if (TRANS) { ldsm4t(bhv[jp], bh + off); ldsm4t(blv[jp], bl + off); }
            else { ldsm4(bhv[jp], bh + off); ldsm4(blv[jp], bl + off); }
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) mma16816(acc[j], ah, bhv[j / 2][2 * (j & 1)], bhv[j / 2][2 * (j & 1) + 1]);
#pragma unroll
        for (int j = 0; j < NT; ++j) mma16816(acc[j], ah, blv[j / 2][2 * (j & 1)], blv[j / 2][2 * (j & 1) + 1]);
#pragma unroll
        for (int j = 0; j < NT; ++j) mma16816(acc[j], al, bhv[j / 2][2 * (j & 1)], bhv[j / 2][2 * (j & 1) + 1]);
    }
}

// Single-pass fp16 variant (about 2^-11 relative per product), for terms
// whose error budget allows it: A from fp32 through an accessor, converted
// to fp16 pairs; B from an fp16 tile of row length LD via ldmatrix (TRANS:
// B(k, n) = tile[k][n], else tile[n][k]).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ void mma16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <int NT, int K, bool TRANS, int LD, typename FA>
__device__ __forceinline__ void wmm_f16(float (&acc)[NT][4], int rb, int cb, FA a, const __half* bt) {
    static_assert(NT % 2 == 0, "pairs of 8-column tiles");
    const int l = threadIdx.x & 31, g = l >> 2, t = l & 3;
    const int mi = l >> 3, rr = l & 7;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t af[4];
        af[0] = pack_f16x2(a(rb + g, k0 + 2 * t), a(rb + g, k0 + 2 * t + 1));
        af[1] = pack_f16x2(a(rb + g + 8, k0 + 2 * t), a(rb + g + 8, k0 + 2 * t + 1));
        af[2] = pack_f16x2(a(rb + g, k0 + 2 * t + 8), a(rb + g, k0 + 2 * t + 9));
        af[3] = pack_f16x2(a(rb + g + 8, k0 + 2 * t + 8), a(rb + g + 8, k0 + 2 * t + 9));
#pragma unroll
        for (int jp = 0; jp < NT / 2; ++jp) {
            const int n0 = cb + 16 * jp;
            long off;
            if (TRANS) off = (long)(k0 + rr + 8 * (mi & 1)) * LD + n0 + 8 * (mi >> 1);
            else off = (long)(n0 + rr + 8 * (mi >> 1)) * LD + k0 + 8 * (mi & 1);
            uint32_t bv[4];
            if (TRANS) ldsm4t(bv, bt + off); else ldsm4(bv, bt + off);
            mma16816_f16(acc[2 * jp], af, bv[0], bv[1]);
            mma16816_f16(acc[2 * jp + 1], af, bv[2], bv[3]);
        }
    }
}

// As wmm_f16, with A read as fp16 pairs straight from a row-major half
// array (leading dimension LDA) instead of through an accessor.
template <int NT, int K, bool TRANS, int LD, int LDA>
__device__ __forceinline__ void wmm_f16_ah(float (&acc)[NT][4], int rb, int cb, const __half* a,
                                           const __half* bt) {
    static_assert(NT % 2 == 0, "pairs of 8-column tiles");
    const int l = threadIdx.x & 31, g = l >> 2, t = l & 3;
    const int mi = l >> 3, rr = l & 7;
    auto a2 = [&](int r, int k) { return *reinterpret_cast<const uint32_t*>(a + (long)r * LDA + k); };
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t af[4];
        af[0] = a2(rb + g, k0 + 2 * t);
        af[1] = a2(rb + g + 8, k0 + 2 * t);
        af[2] = a2(rb + g, k0 + 2 * t + 8);
        af[3] = a2(rb + g + 8, k0 + 2 * t + 8);
#pragma unroll
        for (int jp = 0; jp < NT / 2; ++jp) {
            const int n0 = cb + 16 * jp;
            long off;
            if (TRANS) off = (long)(k0 + rr + 8 * (mi & 1)) * LD + n0 + 8 * (mi >> 1);
            else off = (long)(n0 + rr + 8 * (mi >> 1)) * LD + k0 + 8 * (mi & 1);
            uint32_t bv[4];
            if (TRANS) ldsm4t(bv, bt + off); else ldsm4(bv, bt + off);
            mma16816_f16(acc[2 * jp], af, bv[0], bv[1]);
            mma16816_f16(acc[2 * jp + 1], af, bv[2], bv[3]);
        }
    }
}

template <int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[NT][4]) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
}

// The 32 x N outputs of a chunk are split over the 8 warps as 2 x 4 blocks
// of 16 rows x N/4 columns (N/32 tiles of 8 columns per warp).
template <int N>
struct Tile32 {
    static constexpr int NT = N / 32;
    int rb, cb;
    __device__ Tile32() : rb(((threadIdx.x >> 5) >> 2) * 16), cb(((threadIdx.x >> 5) & 3) * (N / 4)) {}
    __device__ int row(int e) const { return rb + ((threadIdx.x & 31) >> 2) + 8 * (e >> 1); }
    __device__ int col(int j, int e) const { return cb + 8 * j + 2 * (threadIdx.x & 3) + (e & 1); }
};

}  // namespace wmma16
}  // namespace gdn
