// recurrent.cu -- token-serial fused recurrence (the decode mode).
//
// Method: Atomic-GDN2 model card, section 2.1 "Gated DeltaNet-2":
//     S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,  o_t = S_t^T q_t.
// The fused recurrent mode for decode ("Gated DeltaNet" entity trail, finding
// of 2026-07-29) processes one token at a time with the state resident.
//
// Per token, with S' = Diag(a) S:
//     x = S'^T k,  c = S'^T q   (column reductions over the key channels)
//     u = b (v - x)             (corrected value, delta rule)
//     S = S' + k u^T
//     o = S^T q = c + u (k . q)
// so the state is read once and written once per token (HBM-bound: 2 x 4 B
// per state element), and the output needs no second pass over S.
//
// Work split: one CTA per (batch, head, slice of COLS value columns).  Value
// columns are independent in the recurrence, so slices need no exchange.
// Each warp owns DK / NWARPS key rows of the slice and each lane VW = COLS/32
// adjacent columns (one vector load per row); the state stays in registers
// for all T tokens.  The two column reductions go through shared memory once
// per token; the rank-1 update and the output are then local.
//
// Decoupled erase and write gates (a reading of Gated DeltaNet-2, "Gated
// DeltaNet" entity trail, finding of 2026-05-22): with a write gate bw the
// update is S = S' - be k (k^T S') + bw k v^T, i.e. u = bw v - be x.
//
// Multi-token decode (speculative verification of T draft tokens): with a
// snapshot buffer every token's updated state slice is also stored, so that
// the caller can resume from the state after any accepted prefix.

#include "gdn_internal.cuh"

namespace gdn {
namespace {

template <int VW> struct VecF;
template <> struct VecF<1> { using T = float; };
template <> struct VecF<2> { using T = float2; };
template <> struct VecF<4> { using T = float4; };

template <int VW>
__device__ __forceinline__ void load_vec(float (&dst)[VW], const float* src) {
    if constexpr (VW == 4) {
        float4 t = *reinterpret_cast<const float4*>(src);
        dst[0] = t.x; dst[1] = t.y; dst[2] = t.z; dst[3] = t.w;
    } else if constexpr (VW == 2) {
        float2 t = *reinterpret_cast<const float2*>(src);
        dst[0] = t.x; dst[1] = t.y;
    } else {
        dst[0] = *src;
    }
}

template <int VW>
__device__ __forceinline__ void store_vec(float* dst, const float (&src)[VW]) {
    if constexpr (VW == 4) {
        *reinterpret_cast<float4*>(dst) = make_float4(src[0], src[1], src[2], src[3]);
    } else if constexpr (VW == 2) {
        *reinterpret_cast<float2*>(dst) = make_float2(src[0], src[1]);
    } else {
        *dst = src[0];
    }
}

__device__ __forceinline__ float ld_in(const float* p, long i) { return p[i]; }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p, long i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_out(float* p, long i, float x) { p[i] = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, long i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// EXT: the snapshot buffer and the separate write gate may be used (a
// separate instantiation, so that the plain decode step carries neither).
template <int DK, int COLS, int NWARPS, bool CHANNEL, typename TIN, typename TOUT, bool EXT>
__global__ void __launch_bounds__(NWARPS * 32)
recurrent_kernel(const TIN* __restrict__ q, const TIN* __restrict__ k,
                 const TIN* __restrict__ v, const float* __restrict__ g,
                 const float* __restrict__ beta, const float* state_in, float* state_out,
                 TOUT* __restrict__ out, float* __restrict__ snap, const float* __restrict__ beta_w,
                 int T, int H, int dv)
{
    constexpr int VW = COLS / 32;
    constexpr int R = DK / NWARPS;
    static_assert(COLS % 32 == 0 && VW <= 4 && DK % NWARPS == 0, "bad tiling");

    __shared__ float s_q[2][DK];
    __shared__ float s_k[2][DK];
    __shared__ float s_a[2][CHANNEL ? DK : 1];
    __shared__ float s_red[2][2][NWARPS][COLS];
    __shared__ float s_kq[2][NWARPS];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int nslices = dv / COLS;
    const int slice = blockIdx.x % nslices;
    const int h = (blockIdx.x / nslices) % H;
    const int b = blockIdx.x / nslices / H;
    const int col0 = slice * COLS + lane * VW;   // first value column of this lane
    const int row0 = warp * R;                        // first key row of this warp

    // Resident state slice: S[row0 + r][col0 + c].
    float s[R][VW];
    const long sbase = ((long)b * H + h) * DK * (long)dv;
    if (state_in != nullptr) {
#pragma unroll
        for (int r = 0; r < R; ++r) load_vec<VW>(s[r], state_in + sbase + (long)(row0 + r) * dv + col0);
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < VW; ++c) s[r][c] = 0.f;
    }

    for (int t = 0; t < T; ++t) {
        const int buf = t & 1;
        const long tok = ((long)b * T + t) * H + h;   // flat (b, t, h)
        // Stage q, k (and the per-channel decay) of this token.
        for (int i = threadIdx.x; i < DK; i += NWARPS * 32) {
            s_q[buf][i] = ld_in(q, tok * DK + i);
            s_k[buf][i] = ld_in(k, tok * DK + i);
            if constexpr (CHANNEL) s_a[buf][i] = expf(g[tok * DK + i]);
        }
        float vv[VW];
#pragma unroll
        for (int c = 0; c < VW; ++c) vv[c] = ld_in(v, tok * dv + col0 + c);
        const float bt = beta[tok];
        const float bw = (EXT && beta_w != nullptr) ? beta_w[tok] : bt;
        float a_scalar = 1.f;
        if constexpr (!CHANNEL) a_scalar = expf(g[tok]);
        __syncthreads();

        // S' = Diag(a) S; partial column reductions x = S'^T k and c = S'^T q.
        float px[VW], pc[VW];
#pragma unroll
        for (int c = 0; c < VW; ++c) { px[c] = 0.f; pc[c] = 0.f; }
        float kq = 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float ki = s_k[buf][row0 + r];
            const float qi = s_q[buf][row0 + r];
            const float ai = CHANNEL ? s_a[buf][row0 + r] : a_scalar;
            kq = fmaf(ki, qi, kq);
#pragma unroll
            for (int c = 0; c < VW; ++c) {
                s[r][c] *= ai;
                px[c] = fmaf(ki, s[r][c], px[c]);
                pc[c] = fmaf(qi, s[r][c], pc[c]);
            }
        }
#pragma unroll
        for (int c = 0; c < VW; ++c) {
            s_red[buf][0][warp][lane * VW + c] = px[c];
            s_red[buf][1][warp][lane * VW + c] = pc[c];
        }
        if (lane == 0) s_kq[buf][warp] = kq;
        __syncthreads();

        // Complete the reductions; u = b (v - x); S += k u^T; o = c + u (k.q).
        float kq_all = 0.f;
#pragma unroll
        for (int w = 0; w < NWARPS; ++w) kq_all += s_kq[buf][w];
        float u[VW];
#pragma unroll
        for (int c = 0; c < VW; ++c) {
            float x = 0.f, cc = 0.f;
#pragma unroll
            for (int w = 0; w < NWARPS; ++w) {
                x += s_red[buf][0][w][lane * VW + c];
                cc += s_red[buf][1][w][lane * VW + c];
            }
            u[c] = (EXT && beta_w != nullptr) ? fmaf(bw, vv[c], -bt * x) : bt * (vv[c] - x);
            if (warp == 0) st_out(out, tok * dv + col0 + c, fmaf(u[c], kq_all, cc));
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float ki = s_k[buf][row0 + r];
#pragma unroll
            for (int c = 0; c < VW; ++c) s[r][c] = fmaf(ki, u[c], s[r][c]);
        }
        if (EXT && snap != nullptr) {   // S after token t: snapshot [b, t, h]
            float* dst = snap + tok * DK * (long)dv;
#pragma unroll
            for (int r = 0; r < R; ++r) store_vec<VW>(dst + (long)(row0 + r) * dv + col0, s[r]);
        }
    }

    if (state_out != nullptr) {
#pragma unroll
        for (int r = 0; r < R; ++r) store_vec<VW>(state_out + sbase + (long)(row0 + r) * dv + col0, s[r]);
    }
}

template <int DK, int COLS, int NWARPS, bool CHANNEL, typename TIN, typename TOUT>
cudaError_t launch_typed(const Problem& p, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>(p.dv / COLS) * p.H * p.B;
    if (p.snapshots != nullptr || p.beta_write != nullptr) {
        recurrent_kernel<DK, COLS, NWARPS, CHANNEL, TIN, TOUT, true><<<grid, NWARPS * 32, 0, stream>>>(
            static_cast<const TIN*>(p.q), static_cast<const TIN*>(p.k), static_cast<const TIN*>(p.v),
            p.g, p.beta, p.state_in, p.state_out, static_cast<TOUT*>(p.out), p.snapshots, p.beta_write,
            p.T, p.H, p.dv);
        return cudaGetLastError();
    }
    recurrent_kernel<DK, COLS, NWARPS, CHANNEL, TIN, TOUT, false><<<grid, NWARPS * 32, 0, stream>>>(
        static_cast<const TIN*>(p.q), static_cast<const TIN*>(p.k), static_cast<const TIN*>(p.v),
        p.g, p.beta, p.state_in, p.state_out, static_cast<TOUT*>(p.out), p.snapshots, p.beta_write, p.T, p.H, p.dv);
    return cudaGetLastError();
}

template <int DK, bool CHANNEL, typename TIN, typename TOUT>
cudaError_t launch_dk(const Problem& p, cudaStream_t stream) {
    // Decode (one token): 64-column slices, 4 warps -> 32 rows x 2 columns of
    // state per thread (32 independent 8-byte loads in flight per thread);
    // measured fastest of 32/64/128-column slices x 4/8/16 warps on B200.
    // Long token loops (prefill) use 32-column slices for more CTAs per head.
    // A few tokens over many heads (multi-token decode) keep the decode tiling.
    const long ctas64 = (long)p.B * p.H * (p.dv / 64);
    if (p.T == 1 || (p.T <= 16 && ctas64 >= 2 * 148)) return launch_typed<DK, 64, 4, CHANNEL, TIN, TOUT>(p, stream);
    return launch_typed<DK, 32, DK / 16, CHANNEL, TIN, TOUT>(p, stream);
}

template <bool CHANNEL, typename TIN, typename TOUT>
cudaError_t launch_gate(const Problem& p, cudaStream_t stream) {
    if (p.dk == 128) return launch_dk<128, CHANNEL, TIN, TOUT>(p, stream);
    return launch_dk<64, CHANNEL, TIN, TOUT>(p, stream);
}

template <typename TIN, typename TOUT>
cudaError_t launch_io(const Problem& p, cudaStream_t stream) {
    return p.per_channel ? launch_gate<true, TIN, TOUT>(p, stream)
                         : launch_gate<false, TIN, TOUT>(p, stream);
}

// One CTA per (b, h): copies snapshot n_b - 1 of row b into the state.
__global__ void state_select_kernel(const float4* __restrict__ snap, const int* __restrict__ nacc,
                                    float4* __restrict__ state, int T, int H, long n4)
{
    const int h = blockIdx.x % H, b = blockIdx.x / H;
    const int n = nacc[b];
    if (n < 1 || n > T) return;
    const float4* src = snap + (((long)b * T + (n - 1)) * H + h) * n4;
    float4* dst = state + ((long)b * H + h) * n4;
    for (long i = threadIdx.x; i < n4; i += blockDim.x) dst[i] = src[i];
}

}  // namespace

cudaError_t launch_state_select(const float* snapshots, const int* num_accepted, float* state_out,
                                int B, int T, int H, int dk, int dv, cudaStream_t stream) {
    const long n4 = (long)dk * dv / 4;
    state_select_kernel<<<(unsigned)(B * H), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(snapshots), num_accepted, reinterpret_cast<float4*>(state_out),
        T, H, n4);
    return cudaGetLastError();
}

cudaError_t launch_recurrent(const Problem& p, cudaStream_t stream) {
    if (p.io_f32) {
        return p.out_f32 ? launch_io<float, float>(p, stream)
                         : launch_io<float, __nv_bfloat16>(p, stream);
    }
    return p.out_f32 ? launch_io<__nv_bfloat16, float>(p, stream)
                     : launch_io<__nv_bfloat16, __nv_bfloat16>(p, stream);
}

}  // namespace gdn
