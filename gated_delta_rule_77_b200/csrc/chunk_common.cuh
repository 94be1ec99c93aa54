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

// ---- paired fp32 arithmetic (sm_100 add/sub/mul .f32x2: one instruction for
// two lanes of a register pair) ------------------------------------------------
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\t"
        "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, c, d;\n\t"
        "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
        "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\t"
        "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\t"
        "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Eight fp32 values -> a 16-byte bf16 chunk (hi) and the bf16 rounding of the
// remainder (lo), so that hi + lo reproduces each value to ~2^-16.
__device__ __forceinline__ void store_split(uint8_t* hi_dst, uint8_t* lo_dst, const float* v) {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        hi[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        const float2 r = sub2(make_float2(v[2 * e], v[2 * e + 1]), make_float2(bf16_lo(hi[e]), bf16_hi(hi[e])));
        lo[e] = pack_bf16(r.x, r.y);
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

// 2^x on the special-function unit (approximate, denormals flushed).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// log2(e): exp(x) = 2^(x log2 e).
constexpr float kLog2e = 1.44269504088896340736f;

// Four pairs -> bf16 hi and bf16 rounding of the remainder (lo), as store_split.
__device__ __forceinline__ void store_split2(uint8_t* hi_dst, uint8_t* lo_dst, const float2* v) {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        hi[e] = pack_bf16(v[e].x, v[e].y);
        const float2 r = sub2(v[e], make_float2(bf16_lo(hi[e]), bf16_hi(hi[e])));
        lo[e] = pack_bf16(r.x, r.y);
    }
    *reinterpret_cast<uint4*>(hi_dst) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(lo_dst) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
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



// ---- T = (I + A)^{-1}: tf32 tensor-core helpers ------------------------------
// Products inside the triangular solve run on the warp-level tensor-core
// instruction mma.m16n8k8 with tf32 operands, each operand split as
// x = hi + lo (both tf32) and the product taken as hi*hi + hi*lo + lo*hi,
// which keeps fp32-class accuracy (error ~2^-22 relative per term).
//
// T layout: row-major [64][64] fp32 with the column index xor-ed by
// 8 * (row mod 4) (tidx), so that the fragment loads of four consecutive rows
// at one column fall in different banks; 4- and 8-aligned column groups stay
// contiguous.

__device__ __forceinline__ uint32_t tidx(int r, int c) {
    return static_cast<uint32_t>(r * 64 + (c ^ ((r & 3) << 3)));
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4],
                                                const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// d += A(16x8) B(8x8) with both operands split (three tf32 products).
// Three-term TF32 product with three independent accumulators (hi*hi,
// hi*lo, lo*hi), so that consecutive k-steps do not wait on each other.
struct Acc3 {
    float hh[4] = {0.f, 0.f, 0.f, 0.f};
    float hl[4] = {0.f, 0.f, 0.f, 0.f};
    float lh[4] = {0.f, 0.f, 0.f, 0.f};
    __device__ __forceinline__ void add(const float (&a)[4], const float (&b)[2]) {
        uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) split_tf32(a[i], ah[i], al[i]);
#pragma unroll
        for (int i = 0; i < 2; ++i) split_tf32(b[i], bh[i], bl[i]);
        mma_tf32_16x8x8(hh, ah, bh);
        mma_tf32_16x8x8(hl, ah, bl);
        mma_tf32_16x8x8(lh, al, bh);
    }
    __device__ __forceinline__ float sum(int i) const { return hh[i] + (hl[i] + lh[i]); }
};

// T = (I + A)^{-1} for a strictly lower triangular 64x64 fp32 A (fidx
// layout) by recursive doubling on 16-row blocks, with the inverse of a
// block lower triangular matrix [[P, 0], [R, Q]] written as
// [[P^-1, 0], [-Q^-1 R P^-1, Q^-1]]:
//   1. the four 16x16 diagonal blocks by forward substitution (fp32);
//   2. both 32x32 diagonal blocks: T_10 = -D_1 (A_10 D_0), T_32 = -D_3 (A_32 D_2);
//   3. the lower-left 32x32 block: -T_BB (A_BA T_AA).
// The part of Y = A_BA T_AA that needs only the diagonal blocks D_0, D_1 runs
// during stage 2 on warps 4-7; only the term with T_10 waits for it.  The
// products run on mma.m16n8k8 (tf32, hi/lo splits, fp32-class accuracy); the
// triangular operands' zero blocks are skipped.  T is written in the tidx
// layout (entries above the diagonal of the diagonal 16x16 blocks are zero,
// the rest of the upper triangle is not written).  Scratch sY: two [32][40]
// fp32 tiles (10 KB).  Works on warps 0-7 of a CTA of at least 8 warps (any
// further warps only take part in the barriers); ends with a barrier.
__device__ __forceinline__ void solve_unit_lower64_rd(const float* sA, float* sT, float* sY, int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    const int grp = lane >> 2, tig = lane & 3;
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
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m = 0; m < rr; ++m) acc[m & 3] = fmaf(a[m], t[m], acc[m & 3]);
            t[rr] = (rr == lane) ? 1.f : -((acc[0] + acc[1]) + (acc[2] + acc[3]));
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) sT[tidx(o + rr, o + lane)] = t[rr];
    }
    __syncthreads();

    float* sY3 = sY + 32 * 40;           // Y = A_BA T_AA, [32][40]
    // Stage 2, first product: Y_b = A[32b+16.., 32b..+16] D_{2b} (16x16 each),
    // warps 0-3: b = warp >> 1, output columns 8 nt.. with nt = warp & 1.
    // Warps 4-7: the D_0 / D_1 terms of Y = A_BA T_AA, row tile mt = (warp-4)>>1,
    // column tiles nt = 2((warp-4)&1) and +1.
    if (warp >= 4 && warp < 8) {
        const int w = warp - 4, mt = w >> 1;
        float* y = sY3 + (16 * mt) * 40;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int nt = 2 * (w & 1) + q;
            Acc3 acc;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int ks = 2 * (nt >> 1) + kk;       // 8-row group inside D_0 or D_1
                if (ks < nt) continue;
                const int k0 = 8 * ks + tig;
                const int r0 = 32 + 16 * mt + grp;
                const float af[4] = {sA[fidx(r0, k0)], sA[fidx(r0 + 8, k0)], sA[fidx(r0, k0 + 4)],
                                     sA[fidx(r0 + 8, k0 + 4)]};
                const float bf[2] = {sT[tidx(k0, 8 * nt + grp)], sT[tidx(k0 + 4, 8 * nt + grp)]};
                acc.add(af, bf);
            }
            const int c = 8 * nt + 2 * tig;
            *reinterpret_cast<float2*>(&y[grp * 40 + c]) = make_float2(acc.sum(0), acc.sum(1));
            *reinterpret_cast<float2*>(&y[(grp + 8) * 40 + c]) = make_float2(acc.sum(2), acc.sum(3));
        }
    } else if (warp < 4) {
        const int bb = warp >> 1, nt = warp & 1, base = 32 * bb;
        Acc3 acc;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            if (ks < nt) continue;                       // D rows above its columns are zero
            const int k0 = 8 * ks + tig;
            const float af[4] = {sA[fidx(base + 16 + grp, base + k0)], sA[fidx(base + 24 + grp, base + k0)],
                                 sA[fidx(base + 16 + grp, base + k0 + 4)], sA[fidx(base + 24 + grp, base + k0 + 4)]};
            const float bf[2] = {sT[tidx(base + k0, base + 8 * nt + grp)],
                                 sT[tidx(base + k0 + 4, base + 8 * nt + grp)]};
            acc.add(af, bf);
        }
        const int c = 8 * nt + 2 * tig;
        float* y = sY + (16 * bb) * 40;
        *reinterpret_cast<float2*>(&y[grp * 40 + c]) = make_float2(acc.sum(0), acc.sum(1));
        *reinterpret_cast<float2*>(&y[(grp + 8) * 40 + c]) = make_float2(acc.sum(2), acc.sum(3));
    }
    __syncthreads();
    // Stage 2, second product: T[32b+16.., 32b..] = -D_{2b+1} Y_b.
    if (warp < 4) {
        const int bb = warp >> 1, nt = warp & 1, base = 32 * bb;
        const float* y = sY + (16 * bb) * 40;
        Acc3 acc;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int k0 = 8 * ks + tig;
            const int r0 = base + 16 + grp;
            const float af[4] = {sT[tidx(r0, base + 16 + k0)], sT[tidx(r0 + 8, base + 16 + k0)],
                                 sT[tidx(r0, base + 16 + k0 + 4)], sT[tidx(r0 + 8, base + 16 + k0 + 4)]};
            const float bf[2] = {y[k0 * 40 + 8 * nt + grp], y[(k0 + 4) * 40 + 8 * nt + grp]};
            acc.add(af, bf);
        }
        const int c = base + 8 * nt + 2 * tig;
        const int r0 = base + 16 + grp, r1 = r0 + 8;
        sT[tidx(r0, c)] = -acc.sum(0);
        sT[tidx(r0, c + 1)] = -acc.sum(1);
        sT[tidx(r1, c)] = -acc.sum(2);
        sT[tidx(r1, c + 1)] = -acc.sum(3);
    }
    __syncthreads();

    // Stage 3: the T_10 term, Y[:, 0..16] += A[32.., 16..32] T_10 (warps 0-3:
    // mt = warp >> 1, nt = warp & 1), then T[32.., 0..32] = -T[32.., 32..] Y.
    if (warp < 4) {
        const int mt = warp >> 1, nt = warp & 1;
        Acc3 acc;
#pragma unroll
        for (int ks = 2; ks < 4; ++ks) {
            const int k0 = 8 * ks + tig;
            const int r0 = 32 + 16 * mt + grp;
            const float af[4] = {sA[fidx(r0, k0)], sA[fidx(r0 + 8, k0)], sA[fidx(r0, k0 + 4)],
                                 sA[fidx(r0 + 8, k0 + 4)]};
            const float bf[2] = {sT[tidx(k0, 8 * nt + grp)], sT[tidx(k0 + 4, 8 * nt + grp)]};
            acc.add(af, bf);
        }
        const int c = 8 * nt + 2 * tig;
        float* y = sY3 + (16 * mt) * 40;
        float2* y0 = reinterpret_cast<float2*>(&y[grp * 40 + c]);
        float2* y1 = reinterpret_cast<float2*>(&y[(grp + 8) * 40 + c]);
        *y0 = make_float2(y0->x + acc.sum(0), y0->y + acc.sum(1));
        *y1 = make_float2(y1->x + acc.sum(2), y1->y + acc.sum(3));
    }
    __syncthreads();
    const int mt = warp >> 2, nt = warp & 3;
    if (warp < 8) {
        Acc3 acc;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            if (ks > 2 * mt + 1) continue;               // T_BB is lower triangular
            const int k0 = 8 * ks + tig;
            const int r0 = 32 + 16 * mt + grp;
            const float af[4] = {sT[tidx(r0, 32 + k0)], sT[tidx(r0 + 8, 32 + k0)],
                                 sT[tidx(r0, 32 + k0 + 4)], sT[tidx(r0 + 8, 32 + k0 + 4)]};
            const float bf[2] = {sY3[k0 * 40 + 8 * nt + grp], sY3[(k0 + 4) * 40 + 8 * nt + grp]};
            acc.add(af, bf);
        }
        const int c = 8 * nt + 2 * tig;
        const int r0 = 32 + 16 * mt + grp, r1 = r0 + 8;
        sT[tidx(r0, c)] = -acc.sum(0);
        sT[tidx(r0, c + 1)] = -acc.sum(1);
        sT[tidx(r1, c)] = -acc.sum(2);
        sT[tidx(r1, c + 1)] = -acc.sum(3);
    }
    __syncthreads();
}

}  // namespace chunk
}  // namespace gdn
